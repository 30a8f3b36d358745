"""The seeded synthetic batches every measured number is quoted on (CPU).

bench.py, the profiles and the full-size parity tests describe their inputs by the sizes
below (for example the OPT-13B batch-64 step's 128 physical rows and 9196 packed tokens).
The batches come from a seeded generator; this test keeps the recipe from drifting under
those numbers.  Columns: prompts, prompt tokens, scored target tokens, shortest and longest
prompt, foreground rows, foreground tokens, physical tokens (both candidates of every prompt
plus the foreground rows)."""
import numpy as np
import pytest

from zeroth_order_fine_b200 import workload as wl

RECIPES = {
    "opt-13b-b64": (64, 4598, 64, 17, 128, 0, 0, 9196),
    "opt-13b-b16": (16, 1086, 16, 18, 103, 0, 0, 2172),
    "opt-6.7b-b64": (64, 8281, 294, 36, 255, 0, 0, 16562),
    "opt-1.3b-b16": (16, 1212, 16, 18, 114, 0, 0, 2424),
    "qwen3-8b-cobatch": (16, 4102, 16, 86, 387, 32, 7874, 16078),
    "tiny": (8, 256, 8, 32, 32, 0, 0, 512),
}


@pytest.mark.parametrize("name", sorted(RECIPES))
def test_seeded_batch_sizes(name):
    w = wl.WORKLOADS[name]
    b = wl.make_batch(w)
    F = len(b.fg_prompts)
    got = (len(b.prompts), int(b.seq_lens.sum()), int(b.target_lens.sum()),
           int(b.seq_lens.min()), int(b.seq_lens.max()), F,
           int(b.fg_seq_lens.sum()) if F else 0, int(b.n_tokens_physical))
    assert got == RECIPES[name]
    # physical rows: both candidates of each prompt, then the foreground rows
    assert b.n_tokens_physical == 2 * int(b.seq_lens.sum()) + (int(b.fg_seq_lens.sum()) if F else 0)
    # every target span lies inside its prompt and leaves at least one context token
    assert np.all(b.target_lens >= 1) and np.all(b.target_lens < b.seq_lens)


def test_batches_are_reproducible():
    for name in RECIPES:
        a, b = wl.make_batch(wl.WORKLOADS[name]), wl.make_batch(wl.WORKLOADS[name])
        assert all(np.array_equal(x, y) for x, y in zip(a.prompts, b.prompts))
