"""Seeded random batch shapes against the oracle.

Each case draws a model family and precision, a batch of 1-12 prompts of 2-200 tokens with
target spans of 1-8 tokens, 0-4 foreground rows, a rank, the perturbed matrices and a lazy
window, and runs three steps across a window boundary.  L+- and the foreground rows'
per-token log-probs must match the oracle on the same state (fp32 at 1e-4; bf16 at the
same-state bound 2e-2, the oracle's bank loaded before each step), and c must follow the
oracle's within the fp32 bound.  The point is the shapes no hand-written case picked:
rows shorter than a tile, rows spanning several query tiles and key chunks, odd token
counts, spans next to the row start.
"""
import dataclasses

import numpy as np
import pytest

from zeroth_order_fine_b200 import workload as wl
from gpu_util import dev_fg_tokens, dev_tokens, gpu_handle, needs_gpu, oracle_run, oracle_state_blob

pytestmark = [pytest.mark.gpu, needs_gpu]

OPT_SMALL = wl.ModelShape("opt-small", wl.ARCH_OPT, 2, 256, 2, 2, 128, 512, 1000, 256, 1e-5, 0.0,
                          wl.DTYPE_FP32, True)
QWEN_SMALL = wl.ModelShape("qwen3-small", wl.ARCH_QWEN3, 2, 256, 4, 2, 128, 512, 1000, 4096,
                           1e-6, 1e6, wl.DTYPE_FP32, False)


def _case(seed):
    rng = np.random.default_rng(1000 + seed)
    arch = rng.integers(0, 2)
    dtype = wl.DTYPE_FP32 if rng.integers(0, 2) == 0 else wl.DTYPE_BF16
    base = OPT_SMALL if arch == 0 else QWEN_SMALL
    shape = dataclasses.replace(base, dtype=dtype)
    opt6 = (wl.MAT_Q, wl.MAT_K, wl.MAT_V, wl.MAT_O, wl.MAT_UP, wl.MAT_DOWN)
    mats = wl.QV if arch == 0 and rng.integers(0, 2) == 0 else (opt6 if arch == 0 else wl.ALL7)
    w = wl.Workload(f"random-{seed}", shape, int(rng.integers(1, 13)), 2, 200, 1, 8, True,
                    int(rng.choice([1, 2, 4])), mats,
                    wl.SCALE_LOZO if rng.integers(0, 2) == 0 else wl.SCALE_MEZO,
                    1e-2 if dtype == wl.DTYPE_BF16 else 1e-3, 1e-4, 2,
                    fg_rows=int(rng.integers(0, 5)), data_seed=int(rng.integers(1, 10**6)))
    return w


def _mean_lp(flp, tls):
    return np.array([x.mean() for x in np.split(flp, np.cumsum(tls)[:-1])])


@pytest.mark.parametrize("seed", range(24))
def test_random_batch_shapes_match_the_oracle(seed):
    w = _case(seed)
    fp32 = w.shape.dtype == wl.DTYPE_FP32
    batch = wl.make_batch(w)
    F = len(batch.fg_prompts)
    _, h = gpu_handle(w, fg=F, max_slots=4)
    orc = oracle_run(w)
    toks = dev_tokens(batch)
    ftoks = dev_fg_tokens(batch) if F else None
    tol = 1e-4 if fp32 else 2e-2
    for t in range(3):                                  # a window opens at steps 0 and 2
        if t > 0 and not fp32:
            h.zo_load_state(oracle_state_blob(orc, w))  # bf16: the same state each step
        h.zo_probe_plan(t, w.eps)
        orc.plan(t, w.eps)
        if F:
            Lp, Lm, _, flp = h.zo_score_cobatch(toks, batch.seq_lens, batch.target_lens, ftoks,
                                                batch.fg_seq_lens, batch.fg_target_lens)
            ref = orc.score(batch.prompts, batch.target_lens, batch.fg_prompts,
                            batch.fg_target_lens)
            got = _mean_lp(flp.cpu().numpy(), batch.fg_target_lens)
            want = np.array([np.asarray(x).mean() for x in ref.fg_logprob])
            assert np.max(np.abs(got - want)) <= tol, (seed, t)
        else:
            Lp, Lm, _ = h.zo_score(toks, batch.seq_lens, batch.target_lens)
            ref = orc.score(batch.prompts, batch.target_lens)
        assert np.max(np.abs(Lp.cpu().numpy() - ref.L_plus)) <= tol, (seed, t)
        assert np.max(np.abs(Lm.cpu().numpy() - ref.L_minus)) <= tol, (seed, t)
        c = h.zo_step(w.lr)
        c_ref = orc.step(w.lr)
        if fp32:
            assert abs(c - c_ref) <= 1e-2 * max(abs(c_ref), 1.0), (seed, t, c, c_ref)
    assert h.zo_stats()["last_error_code"] == 0
    h.close()


@pytest.mark.parametrize("seed", range(12))
def test_random_generation_shapes_match_the_oracle(seed):
    """Generation queries on random shapes: 1-6 prompts of 2-150 tokens, 1-6 new tokens,
    OPT or Qwen3 in fp32 or bf16.  Every generated token is a largest logit of the oracle
    teacher-forced on the GPU's own prefix (within the precision's bound, so near-ties may
    go either way), its log-prob matches, and so do L+-."""
    from oracle import model as om
    rng = np.random.default_rng(5000 + seed)
    w = _case(seed)
    w = dataclasses.replace(w, batch=int(rng.integers(1, 7)), len_hi=150, fg_rows=0)
    G = int(rng.integers(1, 7))
    fp32 = w.shape.dtype == wl.DTYPE_FP32
    logit_tol, lp_tol, L_tol = (1e-4, 1e-4, 1e-4) if fp32 else (5e-2, 3e-2, 2e-2)
    batch = wl.make_batch(w)
    B = len(batch.prompts)
    _, h = gpu_handle(w, max_new=G)
    h.zo_probe_plan(0, w.eps)
    Lp, Lm, gt, gl = h.zo_generate(dev_tokens(batch), batch.seq_lens, G)
    gt, gl = gt.cpu().numpy(), gl.cpu().numpy()
    orc = oracle_run(w)
    orc.plan(0, w.eps)
    rows = [np.concatenate([p, gt[r]]).astype(np.int64)
            for r, p in enumerate(list(batch.prompts) * 2)]
    hs = om.hidden_states(orc.w, rows, [1.0] * B + [-1.0] * B, orc.eps, orc.perturbation())
    logits = om.span_logits(orc.w, hs, rows, [G] * (2 * B))
    ref_lp = om.token_logprobs(orc.w, hs, rows, [G] * (2 * B))
    for r in range(2 * B):
        lg = logits[r].numpy()
        chosen = lg[np.arange(G), gt[r]]
        assert np.all(chosen >= lg.max(axis=1) - logit_tol), (seed, r)
        assert np.max(np.abs(gl[r] - ref_lp[r].numpy())) <= lp_tol, (seed, r)
    ref_L = np.array([-x.numpy().mean() for x in ref_lp])
    assert np.max(np.abs(Lp.cpu().numpy() - ref_L[:B])) <= L_tol
    assert np.max(np.abs(Lm.cpu().numpy() - ref_L[B:])) <= L_tol
    assert np.isfinite(h.zo_step(w.lr))
    h.close()
