"""The Qwen3-8B co-batching configuration at its full size.

Qwen3-8B shape (36 layers, d = 4096, 32 query / 8 key-value heads, SwiGLU 12288, vocab
151936, bf16, random init on the device), MeZO-style factored direction r = 64 on all seven
matrices, physical batches of 32 probe rows (16 prompts x +-eps) and 32 foreground rows,
lengths 64-512.  Properties that fix the result at any size:

* the foreground rows of a mixed batch score bit for bit as the same rows alone, at every
  step ("Inference-Native Zeroth-Order Optimization", abstract: co-batched outputs and
  objectives show zero deviation);
* eps = 0 gives L+ == L- bit for bit;
* c is mean(L+ - L-) / (2 eps) of the returned objectives within their fp32 rounding.
"""
import numpy as np
import pytest
import torch

from zeroth_order_fine_b200 import workload as wl
from gpu_util import dev_fg_tokens, dev_tokens, needs_gpu

pytestmark = [pytest.mark.gpu, needs_gpu]

W = wl.WORKLOADS["qwen3-8b-cobatch"]


@pytest.fixture(scope="module")
def qwen():
    from zeroth_order_fine_b200 import zo
    batch = wl.make_batch(W)
    assert len(batch.prompts) == 16 and len(batch.fg_prompts) == 32
    model = zo.DeviceModel(W.shape, W.weight_seed)
    tg = zo.make_targets(W.shape.n_layers, W.matrices, W.scale_mode)
    h = zo.Handle(model, W.run_seed, W.nu, W.rank, tg,
                  max_tokens=batch.n_tokens_physical + 64, max_rows=2 * 16 + 32,
                  max_scored=2 * int(batch.target_lens.sum()) + int(batch.fg_target_lens.sum()),
                  max_slots=4)
    yield batch, h
    h.close()
    del model
    torch.cuda.empty_cache()


def test_cobatched_foreground_rows_are_bitwise_alone_at_every_step(qwen):
    batch, h = qwen
    toks, ftoks = dev_tokens(batch), dev_fg_tokens(batch)
    for t in range(2):
        h.zo_probe_plan(t, W.eps)
        Lp, Lm, _, flp = h.zo_score_cobatch(toks, batch.seq_lens, batch.target_lens, ftoks,
                                            batch.fg_seq_lens, batch.fg_target_lens)
        alone = h.zo_score_foreground(ftoks, batch.fg_seq_lens, batch.fg_target_lens)
        assert torch.equal(flp, alone), t
        assert torch.all(torch.isfinite(flp))
        Lp, Lm = Lp.cpu().numpy().astype(np.float64), Lm.cpu().numpy().astype(np.float64)
        c = h.zo_step(W.lr)
        c_host = float(np.mean(Lp - Lm) / (2.0 * np.float32(W.eps)))
        ulp = float(np.spacing(np.float32(max(np.abs(Lp).max(), np.abs(Lm).max()))))
        assert abs(c - c_host) <= 1.01 * ulp / (2.0 * np.float32(W.eps)) + 1e-12 * abs(c), (c, c_host)
    assert h.zo_stats()["last_error_code"] == 0


def test_eps_zero_rows_are_bitwise_equal(qwen):
    batch, h = qwen
    toks = dev_tokens(batch)
    step = h.zo_stats()["steps"]
    h.zo_probe_plan(step, 0.0)
    Lp, Lm, lp = h.zo_score(toks, batch.seq_lens, batch.target_lens, want_logprob=True)
    assert torch.equal(Lp, Lm)
    n = lp.numel() // 2
    assert torch.equal(lp[:n], lp[n:])
