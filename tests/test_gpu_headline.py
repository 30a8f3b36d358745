"""The headline configuration at its full size, through the calls bench.py times, and the
OPT-6.7B batch-64 configuration beside it.

OPT-13B shape (40 layers, d = 5120, vocab 50272, bf16, random init drawn on the device), the
seeded batch of 64 ragged prompts (128 physical rows, 9196 tokens), LoZO r = 2 on q and v;
OPT-6.7B shape (32 layers, d = 4096) on its batch of 64 prompts of 32-256 tokens, each scored
on a 1-8-token span, LoZO r = 4.  The float64 oracle cannot hold these models, so the
full-size checks are properties that fix the result at any size; the oracle itself checks
one full-width layer of each over the same batch (test_gpu_step.py):

* eps = 0 makes every + row and its - row the same computation: L+ == L- bit for bit;
* the step is deterministic: the same plan scored twice gives the same bits;
* c is the estimator of "Zeroth-Order Fine-Tuning Was an Inference Workload All Along"
  ("Why ZO Fine-Tuning Is Really Scoring"): mean(L+ - L-) / (2 eps), checked against the
  returned L+- within their fp32 rounding;
* the first update of the bank is A = -fp32(eta c) U_0 exactly, and the second adds
  -fp32(eta c_1) U_1 with one fused multiply-add, for sampled layers of q and v;
* foreground rows co-batched with the probe rows score bit for bit as alone.
"""
import numpy as np
import pytest
import torch

from zeroth_order_fine_b200 import workload as wl
from gpu_util import dev_fg_tokens, dev_tokens, needs_gpu

pytestmark = [pytest.mark.gpu, needs_gpu]

FG = 8


@pytest.fixture(scope="module", params=["opt-13b-b64", "opt-6.7b-b64"])
def headline(request):
    from zeroth_order_fine_b200 import zo
    W = wl.WORKLOADS[request.param]
    batch = wl.make_batch(W)
    assert batch.n_tokens_physical == sum(2 * len(p) for p in batch.prompts) > 9000
    model = zo.DeviceModel(W.shape, W.weight_seed)
    tg = zo.make_targets(W.shape.n_layers, W.matrices, W.scale_mode)
    B = len(batch.prompts)
    fg_tokens = int(sum(len(p) for p in batch.prompts[:FG]))
    h = zo.Handle(model, W.run_seed, W.nu, W.rank, tg,
                  max_tokens=batch.n_tokens_physical + fg_tokens + 64, max_rows=2 * B + FG,
                  max_scored=2 * int(batch.target_lens.sum()) + int(batch.target_lens[:FG].sum()),
                  max_slots=4)
    yield W, batch, h
    h.close()
    del model
    torch.cuda.empty_cache()


def test_eps_zero_rows_are_bitwise_equal_and_scoring_is_deterministic(headline):
    W, batch, h = headline
    toks = dev_tokens(batch)
    h.zo_probe_plan(0, 0.0)
    Lp, Lm, lp = h.zo_score(toks, batch.seq_lens, batch.target_lens, want_logprob=True)
    assert torch.equal(Lp, Lm)
    h.zo_probe_plan(0, W.eps)
    Lp1, Lm1, lp1 = h.zo_score(toks, batch.seq_lens, batch.target_lens, want_logprob=True)
    h.zo_probe_plan(0, W.eps)
    Lp2, Lm2, lp2 = h.zo_score(toks, batch.seq_lens, batch.target_lens, want_logprob=True)
    assert torch.equal(Lp1, Lp2) and torch.equal(Lm1, Lm2) and torch.equal(lp1, lp2)
    assert not torch.equal(Lp1, Lm1)                 # eps > 0 does move the objectives
    assert torch.all(torch.isfinite(Lp1)) and torch.all(torch.isfinite(Lm1))


def test_estimate_and_first_two_bank_updates_at_full_size(headline):
    W, batch, h = headline
    toks = dev_tokens(batch)
    state0 = h.zo_save_state()
    coefs = []
    A_prev = {}
    sample = [(0, wl.MAT_Q), (17, wl.MAT_V), (W.shape.n_layers - 1, wl.MAT_Q)]
    for t in range(2):
        h.zo_probe_plan(t, W.eps)
        Lp, Lm, _ = h.zo_score(toks, batch.seq_lens, batch.target_lens)
        Lp, Lm = Lp.cpu().numpy().astype(np.float64), Lm.cpu().numpy().astype(np.float64)
        U = {key: h.zo_read_factors(*key)[0] for key in sample}
        c = h.zo_step(W.lr)
        # c from the returned (fp32-rounded) objectives: each differs from the library's
        # float64 row objective by at most half an fp32 ulp
        c_host = float(np.mean(Lp - Lm) / (2.0 * np.float32(W.eps)))
        ulp = float(np.spacing(np.float32(max(np.abs(Lp).max(), np.abs(Lm).max()))))
        assert abs(c - c_host) <= 1.01 * ulp / (2.0 * np.float32(W.eps)) + 1e-12 * abs(c), (c, c_host)
        coef = np.float32(np.float64(np.float32(W.lr)) * c)
        coefs.append(coef)
        for key in sample:
            A = h.zo_read_bank(key[0], key[1], 0)
            if t == 0:
                expect = np.float32(-coef) * U[key]           # fma(-coef, u, 0): one rounding
            else:
                # fma(-coef_1, u_1, A_0) in float64 is exact before its single rounding
                expect = (np.float64(-coef) * U[key].astype(np.float64)
                          + A_prev[key].astype(np.float64)).astype(np.float32)
            assert np.array_equal(A, expect), (t, key)
            A_prev[key] = A
    assert h.zo_stats()["steps"] == 2 and h.zo_stats()["last_error_code"] == 0
    h.zo_load_state(state0)


def test_cobatched_foreground_rows_are_bitwise_alone_at_full_size(headline):
    W, batch, h = headline
    toks = dev_tokens(batch)
    fg = wl.Batch(batch.prompts, batch.target_lens, list(batch.prompts[:FG]),
                  np.asarray(batch.target_lens[:FG], dtype=np.int32))
    ftoks = dev_fg_tokens(fg)
    h.zo_probe_plan(0, W.eps)                      # the earlier tests leave the step at 0
    _, _, _, flp = h.zo_score_cobatch(toks, batch.seq_lens, batch.target_lens, ftoks,
                                      fg.fg_seq_lens, fg.fg_target_lens)
    alone = h.zo_score_foreground(ftoks, fg.fg_seq_lens, fg.fg_target_lens)
    assert torch.equal(flp, alone)
