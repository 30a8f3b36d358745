"""The data-parallel split of the step and the whole-step CUDA graph, against the oracle.

Data parallel: each replica scores its own prompts, writes {sum_i (L+_i - L-_i), n} into a
buffer of the caller's (zo_objective_sums), the caller sums those buffers over replicas
(the one all-reduce) and every replica applies c = sum / n / (2 eps) and the same bank
update (zo_step_from_sums) -- the estimator of "Zeroth-Order Fine-Tuning Was an Inference
Workload All Along" (section "Why ZO Fine-Tuning Is Really Scoring") over the union of the
replicas' prompts.  On one GPU the replicas are separate handles; their kernels never wait
on one another, and the sum of their buffers stands in for the all-reduce.

Whole-step graph: zo_step_graph (plan + score + step as one graph launch) scored on the
oracle's own state at every step -- the oracle's bank is loaded into the library before the
step (data flows oracle -> GPU only) -- across lazy-window boundaries.
"""
import dataclasses

import numpy as np
import pytest
import torch

from zeroth_order_fine_b200 import workload as wl
from gpu_util import dev_tokens, gpu_handle, needs_gpu, oracle_run, oracle_state_blob

pytestmark = [pytest.mark.gpu, needs_gpu]

TINY = wl.WORKLOADS["tiny"]
TINY_BF16 = dataclasses.replace(TINY, shape=wl.shrink_shape(wl.TINY, dtype=wl.DTYPE_BF16))
Q3_SMALL = wl.ModelShape("qwen3-small", wl.ARCH_QWEN3, 2, 256, 4, 2, 128, 512, 1000, 4096, 1e-6,
                         1e6, wl.DTYPE_BF16, False)
QWEN_SMALL = wl.Workload("qwen3-small", Q3_SMALL, 6, 20, 90, 1, 4, True, 8, wl.ALL7,
                         wl.SCALE_MEZO, 1e-3, 1e-4, 3, fg_rows=0, data_seed=11)


def test_replica_step_through_the_public_calls_matches_zo_step_and_oracle():
    """dp.dp_step (world of one: no process group) and zo_objective_sums -> caller buffer ->
    zo_step_from_sums give zo_step's c and bank bit for bit; c and L+- follow the oracle
    within the fp32 tolerances."""
    from zeroth_order_fine_b200 import dp
    w = TINY
    batch = wl.make_batch(w)
    toks = dev_tokens(batch)
    _, ha = gpu_handle(w, nu=3)
    _, hb = gpu_handle(w, nu=3)
    _, hc = gpu_handle(w, nu=3)
    orc = oracle_run(w, nu=3)
    sums_b = torch.zeros(2, dtype=torch.float64, device="cuda")
    for t in range(5):                                   # a window opens at step 3
        outs = []
        for h in (ha, hb, hc):
            h.zo_probe_plan(t, w.eps)
            Lp, Lm, _ = h.zo_score(toks, batch.seq_lens, batch.target_lens)
            outs.append((Lp.cpu().numpy(), Lm.cpu().numpy()))
        orc.plan(t, w.eps)
        ref = orc.score(batch.prompts, batch.target_lens)
        for Lp, Lm in outs:
            assert np.max(np.abs(Lp - ref.L_plus)) <= 1e-4
            assert np.max(np.abs(Lm - ref.L_minus)) <= 1e-4
        ca = ha.zo_step(w.lr)
        cb = dp.dp_step(hb, w.lr, sums_b, want_c=True)
        buf = torch.full((2,), float("nan"), dtype=torch.float64, device="cuda")
        hc.zo_objective_sums(buf)
        s = buf.cpu().numpy()
        assert s[1] == len(batch.prompts)
        assert abs(s[0] - np.sum(ref.L_plus - ref.L_minus)) <= 1e-4 * len(batch.prompts)
        cc = hc.zo_step_from_sums(w.lr, buf)
        c_ref = orc.step(w.lr)
        assert ca == cb == cc, (t, ca, cb, cc)
        assert abs(ca - c_ref) <= 1e-2 * max(abs(c_ref), 1.0), (t, ca, c_ref)
    assert ha.zo_save_state() == hb.zo_save_state() == hc.zo_save_state()


def test_two_replicas_on_prompt_shards_match_one_handle_on_the_batch():
    """Two replicas, each on its shard of an odd batch, summing their buffers: the same c on
    both (bit for bit), identical banks, and the c of one handle on the whole batch up to
    the order of the fp64 sum."""
    from zeroth_order_fine_b200 import dp
    w = TINY
    full = wl.make_batch(w, batch=7)
    shards = [dp.shard_batch(full, r, 2) for r in range(2)]
    toks = [dev_tokens(b) for b in shards]
    toks_full = dev_tokens(full)
    hs = [gpu_handle(w, batch=len(b.prompts))[1] for b in shards]
    _, hf = gpu_handle(w, batch=7)
    orc = oracle_run(w)
    for t in range(3):
        bufs = []
        for h, b, tk in zip(hs, shards, toks):
            h.zo_probe_plan(t, w.eps)
            h.zo_score(tk, b.seq_lens, b.target_lens)
            buf = torch.zeros(2, dtype=torch.float64, device="cuda")
            h.zo_objective_sums(buf)
            bufs.append(buf)
        total = bufs[0] + bufs[1]                          # the all-reduce's SUM
        cs = [h.zo_step_from_sums(w.lr, total) for h in hs]
        hf.zo_probe_plan(t, w.eps)
        hf.zo_score(toks_full, full.seq_lens, full.target_lens)
        cf = hf.zo_step(w.lr)
        orc.plan(t, w.eps)
        orc.score(full.prompts, full.target_lens)
        c_ref = orc.step(w.lr)
        assert cs[0] == cs[1]
        assert abs(cs[0] - cf) <= 1e-12 * max(abs(cf), 1.0), (cs[0], cf)
        assert abs(cs[0] - c_ref) <= 1e-2 * max(abs(c_ref), 1.0)
    assert hs[0].zo_save_state() == hs[1].zo_save_state()
    for (l, m) in orc.bank:
        A0 = hs[0].zo_read_bank(l, m, 0)
        Af = hf.zo_read_bank(l, m, 0)
        assert np.allclose(A0, Af, rtol=1e-6, atol=1e-12)


def _graph_case(name):
    if name == "tiny-fp32":
        return TINY, None, 1e-4
    if name == "tiny-bf16":
        return TINY_BF16, None, 2e-2
    return QWEN_SMALL, Q3_SMALL, 2e-2


@pytest.mark.parametrize("name", ["tiny-fp32", "tiny-bf16", "qwen3-bf16"])
def test_step_graph_matches_oracle_on_the_same_state(name):
    """Seven graph steps across three lazy windows (nu = 3): before each, the oracle's bank
    and step are loaded into the library; the graph's L+- must match the oracle's score of
    that state, and (fp32) the bank the graph leaves must match the oracle's update."""
    w, shape, tol = _graph_case(name)
    shape = shape or w.shape
    batch = wl.make_batch(w, fg_rows=0)
    toks = dev_tokens(batch)
    _, hg = gpu_handle(w, shape=shape, nu=3)
    orc = oracle_run(w, shape=shape, nu=3)
    for t in range(7):
        if t > 0:
            hg.zo_load_state(oracle_state_blob(orc, w, shape))
        Lp, Lm = hg.zo_step_graph(toks, batch.seq_lens, batch.target_lens, w.eps, w.lr)
        orc.plan(t, w.eps)
        ref = orc.score(batch.prompts, batch.target_lens)
        assert np.max(np.abs(Lp.cpu().numpy() - ref.L_plus)) <= tol, t
        assert np.max(np.abs(Lm.cpu().numpy() - ref.L_minus)) <= tol, t
        c_ref = orc.step(w.lr)
        if name == "tiny-fp32":
            # A_new - A_old = -lr c U: the graph's c within the fp32 bound of the oracle's
            for (l, m), slots in orc.bank.items():
                A = hg.zo_read_bank(l, m, len(slots) - 1)
                Ar = slots[-1][0].numpy()
                scale = w.lr * max(abs(c_ref), 1.0) * np.max(np.abs(orc.factors(l, m, t)[0]))
                assert np.max(np.abs(A - Ar)) <= 1e-2 * scale + 1e-9, (t, l, m)
    s = hg.zo_stats()
    assert s["steps"] == 7 and s["last_error_code"] == 0
    assert s["graph_replays"] == 7 and s["graph_captures"] >= 3
