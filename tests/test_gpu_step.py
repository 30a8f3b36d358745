"""End-to-end parity of the probe step through the C ABI against the oracle,
and the invariants the pages fix: eps = 0 gives L+ == L-, co-batched
foreground rows are bit-identical to the same rows scored alone, runs are
deterministic, a saved state resumes the same trajectory, non-finite
objectives are refused."""
import dataclasses

import numpy as np
import pytest
import torch

from zeroth_order_fine_b200 import workload as wl
from gpu_util import dev_fg_tokens, dev_tokens, gpu_handle, needs_gpu, oracle_run

pytestmark = [pytest.mark.gpu, needs_gpu]

TINY = wl.WORKLOADS["tiny"]
TINY_BF16 = dataclasses.replace(TINY, shape=wl.shrink_shape(wl.TINY, dtype=wl.DTYPE_BF16))
# A small Qwen3-family model (GQA, q/k RMSNorm, RoPE, SwiGLU) with the MeZO-style
# factorised direction on all seven matrices.
Q3_SMALL = wl.ModelShape("qwen3-small", wl.ARCH_QWEN3, 2, 256, 4, 2, 128, 512, 1000, 4096, 1e-6,
                         1e6, wl.DTYPE_FP32, False)
QWEN_SMALL = wl.Workload("qwen3-small", Q3_SMALL, 6, 20, 90, 1, 4, True, 8, wl.ALL7,
                         wl.SCALE_MEZO, 1e-3, 1e-4, 3, fg_rows=4, data_seed=11)


def _cat(xs):
    return np.concatenate([np.asarray(x) for x in xs])


@pytest.mark.parametrize("impl", [0, 1])
def test_tiny_fp32_steps_match_oracle(impl):
    """Config 1: one probe pair + update, then 10 more steps; fp32 tolerances."""
    w = TINY
    batch = wl.make_batch(w)
    model, h = gpu_handle(w, impl=impl)
    orc = oracle_run(w)
    toks = dev_tokens(batch)
    for t in range(11):
        h.zo_probe_plan(t, w.eps)
        orc.plan(t, w.eps)
        Lp, Lm, lp = h.zo_score(toks, batch.seq_lens, batch.target_lens,
                                target_ids=torch.from_numpy(batch.target_ids()).cuda(),
                                want_logprob=True)
        ref = orc.score(batch.prompts, batch.target_lens)
        ref_lp = _cat(ref.logprob_plus + ref.logprob_minus)
        assert np.max(np.abs(lp.cpu().numpy() - ref_lp)) <= 1e-4
        assert np.max(np.abs(Lp.cpu().numpy() - ref.L_plus)) <= 1e-4
        assert np.max(np.abs(Lm.cpu().numpy() - ref.L_minus)) <= 1e-4
        c = h.zo_step(w.lr)
        c_ref = orc.step(w.lr)
        assert abs(c - c_ref) <= 1e-2 * max(abs(c_ref), 1.0), (t, c, c_ref)
    for (l, m) in orc.bank:
        A = h.zo_read_bank(l, m, 0)
        Ar = orc.bank[(l, m)][0][0].numpy()
        assert np.max(np.abs(A - Ar)) <= 1e-2 * max(np.max(np.abs(Ar)), 1e-12) + 1e-9


def test_qwen3_mezo_fp32_matches_oracle():
    w = QWEN_SMALL
    batch = wl.make_batch(w)
    model, h = gpu_handle(w, fg=w.fg_rows, max_slots=4)
    orc = oracle_run(w)
    toks, ftoks = dev_tokens(batch), dev_fg_tokens(batch)
    for t in range(4):                        # crosses a window boundary (nu = 3)
        h.zo_probe_plan(t, w.eps)
        orc.plan(t, w.eps)
        Lp, Lm, lp, flp = h.zo_score_cobatch(toks, batch.seq_lens, batch.target_lens, ftoks,
                                             batch.fg_seq_lens, batch.fg_target_lens,
                                             want_logprob=True)
        ref = orc.score(batch.prompts, batch.target_lens, batch.fg_prompts, batch.fg_target_lens)
        assert np.max(np.abs(lp.cpu().numpy() - _cat(ref.logprob_plus + ref.logprob_minus))) <= 1e-4
        assert np.max(np.abs(flp.cpu().numpy() - _cat(ref.fg_logprob))) <= 1e-4
        c = h.zo_step(w.lr)
        c_ref = orc.step(w.lr)
        assert abs(c - c_ref) <= 1e-2 * max(abs(c_ref), 1.0)


def _bf16_same_state_parity(w, shape, batch, pre_steps, fp8=False):
    """L+- of the GPU and the oracle on the same state: step 0, then after the
    oracle's own pre_steps updates, its bank loaded into the library."""
    from gpu_util import oracle_state_blob
    model, h = gpu_handle(w, shape=shape, batch=len(batch.prompts), fp8=int(fp8))
    orc = oracle_run(w, shape=shape, fp8=fp8)
    toks = dev_tokens(batch)
    errs = []
    h.zo_probe_plan(0, w.eps)
    orc.plan(0, w.eps)
    Lp, Lm, _ = h.zo_score(toks, batch.seq_lens, batch.target_lens)
    ref = orc.score(batch.prompts, batch.target_lens)
    errs.append(max(np.max(np.abs(Lp.cpu().numpy() - ref.L_plus)),
                    np.max(np.abs(Lm.cpu().numpy() - ref.L_minus))))
    orc.step(w.lr)
    for t in range(1, pre_steps):
        orc.plan(t, w.eps)
        orc.score(batch.prompts, batch.target_lens)
        orc.step(w.lr)
    h.zo_load_state(oracle_state_blob(orc, w, shape))
    t = orc.t
    h.zo_probe_plan(t, w.eps)
    orc.plan(t, w.eps)
    Lp, Lm, _ = h.zo_score(toks, batch.seq_lens, batch.target_lens)
    ref = orc.score(batch.prompts, batch.target_lens)
    errs.append(max(np.max(np.abs(Lp.cpu().numpy() - ref.L_plus)),
                    np.max(np.abs(Lm.cpu().numpy() - ref.L_minus))))
    h.close()
    assert max(errs) <= 2e-2, errs
    return errs


def test_tiny_bf16_same_state_parity():
    w = TINY_BF16
    _bf16_same_state_parity(w, w.shape, wl.make_batch(w), pre_steps=3)


def test_opt_1_3b_width_slice_bf16_same_state_parity():
    """Two full-width OPT-1.3B layers (d=2048, vocab 50272) on the tensor-core path."""
    w = wl.WORKLOADS["opt-1.3b-b16"]
    shape = wl.shrink_shape(w.shape, n_layers=2)
    _bf16_same_state_parity(w, shape, wl.make_batch(w, batch=4, len_hi=64), pre_steps=2)


def test_opt_13b_width_layer_full_batch_64_bf16_same_state_parity():
    """One full-width OPT-13B layer (d = 5120, vocab 50272) over the whole seeded batch-64
    step: 128 physical rows, 9196 packed tokens, so every GEMM runs the SM-pair schedule of
    the headline step (36 row blocks in raster groups of 12, many tiles per pair) and the
    attention kernel its full tile list; L+- against the oracle at step 0 and after the
    oracle's first update (its bank loaded)."""
    w = wl.WORKLOADS["opt-13b-b64"]
    shape = wl.shrink_shape(w.shape, n_layers=1)
    batch = wl.make_batch(w)
    assert batch.n_tokens_physical > 12 * 256
    _bf16_same_state_parity(w, shape, batch, pre_steps=1)


def test_opt_6_7b_width_layer_full_batch_64_spans_bf16_same_state_parity():
    """One full-width OPT-6.7B layer (d = 4096, FFN 16384, vocab 50272) over the whole seeded
    batch of that workload: 64 prompts of 32-256 tokens, each scored on a 1-8-token span at
    its end, LoZO r = 4 on q and v; L+- against the oracle at step 0 and after the oracle's
    first update (its bank loaded)."""
    w = wl.WORKLOADS["opt-6.7b-b64"]
    shape = wl.shrink_shape(w.shape, n_layers=1)
    batch = wl.make_batch(w)
    assert batch.target_lens.max() > 1 and w.rank == 4
    _bf16_same_state_parity(w, shape, batch, pre_steps=1)


def test_qwen3_8b_width_layer_full_cobatch_step_bf16_same_state_parity():
    """One full-width Qwen3-8B layer (d = 4096, 32 / 8 heads, SwiGLU 12288, vocab 151936) over
    the whole seeded co-batching step: 16 prompts as 32 probe rows plus 32 foreground rows,
    64-512 tokens, MeZO r = 64 on all seven matrices.  L+- and the foreground rows' mean
    log-probs against the oracle at step 0 and after the oracle's first update (its bank
    loaded)."""
    from gpu_util import oracle_state_blob
    w = wl.WORKLOADS["qwen3-8b-cobatch"]
    shape = wl.shrink_shape(w.shape, n_layers=1)
    batch = wl.make_batch(w)
    assert len(batch.fg_prompts) == 32 and batch.n_tokens_physical > 12000
    _, h = gpu_handle(w, shape=shape, fg=len(batch.fg_prompts))
    orc = oracle_run(w, shape=shape)
    toks, ftoks = dev_tokens(batch), dev_fg_tokens(batch)
    fsplit = np.cumsum(batch.fg_target_lens)[:-1]

    def compare():
        Lp, Lm, _, flp = h.zo_score_cobatch(toks, batch.seq_lens, batch.target_lens, ftoks,
                                            batch.fg_seq_lens, batch.fg_target_lens)
        ref = orc.score(batch.prompts, batch.target_lens, batch.fg_prompts, batch.fg_target_lens)
        fg_mean = np.array([x.mean() for x in np.split(flp.cpu().numpy(), fsplit)])
        fg_ref = np.array([np.asarray(x).mean() for x in ref.fg_logprob])
        return max(np.max(np.abs(Lp.cpu().numpy() - ref.L_plus)),
                   np.max(np.abs(Lm.cpu().numpy() - ref.L_minus)),
                   np.max(np.abs(fg_mean - fg_ref)))

    errs = []
    h.zo_probe_plan(0, w.eps)
    orc.plan(0, w.eps)
    errs.append(compare())
    orc.step(w.lr)
    h.zo_load_state(oracle_state_blob(orc, w, shape))
    h.zo_probe_plan(orc.t, w.eps)
    orc.plan(orc.t, w.eps)
    errs.append(compare())
    h.close()
    assert max(errs) <= 2e-2, errs


def test_tiny_bf16_many_rows_parity_and_cobatching():
    """160 physical rows of ~62 tokens (~9900 tokens, more 128-row tiles than CTA pairs): the
    bank shrink's CTA pairs each take a second tile, handing the split halves over twice;
    L+- against the oracle, and co-batched foreground rows bit-identical to scored alone."""
    w = dataclasses.replace(TINY_BF16, batch=80, len_lo=60, len_hi=64, fg_rows=6)
    batch = wl.make_batch(w)
    assert batch.n_tokens_physical - int(batch.fg_seq_lens.sum()) > 74 * 128
    _bf16_same_state_parity(w, w.shape, wl.Batch(batch.prompts, batch.target_lens, [],
                                                 np.zeros(0, np.int32)), pre_steps=2)
    model, h = gpu_handle(w, fg=6)
    toks, ftoks = dev_tokens(batch), dev_fg_tokens(batch)
    for t in range(2):
        h.zo_probe_plan(t, w.eps)
        _, _, _, flp = h.zo_score_cobatch(toks, batch.seq_lens, batch.target_lens, ftoks,
                                          batch.fg_seq_lens, batch.fg_target_lens)
        alone = h.zo_score_foreground(ftoks, batch.fg_seq_lens, batch.fg_target_lens)
        assert torch.equal(flp, alone), t
        h.zo_step(w.lr)


@pytest.mark.parametrize("wk", ["tiny", "tiny-bf16"])
def test_foreground_scoring_between_score_and_step_leaves_the_step_alone(wk):
    """A serving-style zo_score_foreground between a plan's scoring and its zo_step must not
    touch the plan's objectives: c and the bank equal those of a handle that never served."""
    w = dataclasses.replace(TINY if wk == "tiny" else TINY_BF16, fg_rows=4)
    batch = wl.make_batch(w)
    toks, ftoks = dev_tokens(batch), dev_fg_tokens(batch)
    _, ha = gpu_handle(w, fg=4)
    _, hb = gpu_handle(w, fg=4)
    for t in range(3):
        cs = []
        for h, serve in ((ha, True), (hb, False)):
            h.zo_probe_plan(t, w.eps)
            h.zo_score_cobatch(toks, batch.seq_lens, batch.target_lens, ftoks,
                               batch.fg_seq_lens, batch.fg_target_lens)
            if serve:
                h.zo_score_foreground(ftoks, batch.fg_seq_lens, batch.fg_target_lens)
            cs.append(h.zo_step(w.lr))
        assert cs[0] == cs[1], (t, cs)
    assert ha.zo_save_state() == hb.zo_save_state()


def test_qwen3_head_dim_64_bf16_same_state_parity_and_cobatching():
    """A Qwen3-family model with 64-wide heads (8 query / 4 kv heads over d = 512): the q/k
    norm and rotary positions run as their own kernel (the fused epilogue takes 128-wide
    heads) and attention on the tensor cores' head_dim-64 form; L+- against the oracle on
    the same state, and co-batched foreground rows bit-identical to alone."""
    shape = wl.ModelShape("qwen3-hd64", wl.ARCH_QWEN3, 2, 512, 8, 4, 64, 1024, 1000, 4096, 1e-6,
                          1e6, wl.DTYPE_BF16, False)
    w = dataclasses.replace(QWEN_SMALL, shape=shape, fg_rows=0)
    _bf16_same_state_parity(w, shape, wl.make_batch(w, fg_rows=0), pre_steps=3)
    wf = dataclasses.replace(QWEN_SMALL, shape=shape, fg_rows=4)
    batch = wl.make_batch(wf)
    _, h = gpu_handle(wf, shape=shape, fg=4)
    toks, ftoks = dev_tokens(batch), dev_fg_tokens(batch)
    for t in range(2):
        h.zo_probe_plan(t, wf.eps)
        _, _, _, flp = h.zo_score_cobatch(toks, batch.seq_lens, batch.target_lens, ftoks,
                                          batch.fg_seq_lens, batch.fg_target_lens)
        assert torch.equal(flp, h.zo_score_foreground(ftoks, batch.fg_seq_lens,
                                                      batch.fg_target_lens))
        h.zo_step(wf.lr)
    assert h.zo_stats()["cuda_core_gemm_launches"] == 0


def test_qwen3_bf16_same_state_parity():
    shape = dataclasses.replace(Q3_SMALL, dtype=wl.DTYPE_BF16)
    w = dataclasses.replace(QWEN_SMALL, shape=shape, fg_rows=0)
    _bf16_same_state_parity(w, shape, wl.make_batch(w, fg_rows=0), pre_steps=4)


# The bf16 trajectory workloads: each side follows its own c for 100 steps, so the check
# is only meaningful when 100 steps move the loss far beyond the 2 % band.  The tiny model
# with the direction on q and v alone hardly moves (3.5 % at eta = 1e-4); with the direction
# on all six OPT matrices, eta = 2e-4, the oracle's loss falls by ~13 %.  eps = 1e-2: the
# difference L+ - L- = 2 eps c must stand well above the bf16 rounding of L (~1e-3), else
# each side's c carries that rounding and the two runs drift apart by several per cent.
TRAJ_TINY = wl.TRAJ_TINY_BF16


def _trajectory_vs_oracle(w, shape, batch, steps=100):
    """Mean objective (L+ + L-)/2 of every step, GPU and oracle each on its own c."""
    model, h = gpu_handle(w, shape=shape, batch=len(batch.prompts))
    orc = oracle_run(w, shape=shape)
    toks = dev_tokens(batch)
    traj, traj_ref = [], []
    for t in range(steps):
        h.zo_probe_plan(t, w.eps)
        orc.plan(t, w.eps)
        Lp, Lm, _ = h.zo_score(toks, batch.seq_lens, batch.target_lens)
        ref = orc.score(batch.prompts, batch.target_lens)
        traj.append(float((Lp.mean() + Lm.mean()).item()) / 2)
        traj_ref.append(float(ref.L_plus.mean() + ref.L_minus.mean()) / 2)
        h.zo_step(w.lr, want_c=False)
        orc.step(w.lr)
    h.close()
    return np.array(traj), np.array(traj_ref)


def _check_trajectory(traj, traj_ref):
    # the oracle's own movement is at least 5x the band, so an update of half (or twice)
    # the right strength cannot stay inside it
    move = abs(traj_ref[-1] - traj_ref[0]) / abs(traj_ref[0])
    assert move >= 0.10, move
    rel = np.abs(traj - traj_ref) / np.abs(traj_ref)
    assert np.max(rel) <= 0.02, (np.max(rel), int(np.argmax(rel)), traj[-1], traj_ref[-1])


def test_tiny_bf16_loss_trajectory_100_steps():
    """bf16 mode: the 100-step loss trajectory of the tiny model within 2 % of the oracle's."""
    w = TRAJ_TINY
    _check_trajectory(*_trajectory_vs_oracle(w, w.shape, wl.make_batch(w)))


def test_opt_1_3b_width_slice_bf16_loss_trajectory_100_steps():
    """bf16 mode: 100 steps of two full-width OPT-1.3B layers (d = 2048, vocab 50272,
    q and v targets, eta = 1e-4 as configured), trajectory within 2 % of the oracle's.
    eps = 1e-2, as for the tiny trajectory: on this slice an objective error of 1e-3 (the
    bf16 rounding of L) moves the oracle's own 100-step trajectory by up to 1.9 % at
    eps = 1e-3 but by 0.17 % at eps = 1e-2, where the oracle still falls by 20 %."""
    w = dataclasses.replace(wl.WORKLOADS["opt-1.3b-b16"], eps=1e-2)
    shape = wl.shrink_shape(w.shape, n_layers=2)
    _check_trajectory(*_trajectory_vs_oracle(w, shape, wl.make_batch(w, batch=4, len_hi=64)))


@pytest.mark.parametrize("wk", ["tiny", "tiny-bf16"])
def test_eps_zero_gives_bitwise_equal_objectives(wk):
    w = TINY if wk == "tiny" else TINY_BF16
    batch = wl.make_batch(w)
    model, h = gpu_handle(w)
    toks = dev_tokens(batch)
    h.zo_probe_plan(0, 0.0)
    Lp, Lm, lp = h.zo_score(toks, batch.seq_lens, batch.target_lens, want_logprob=True)
    assert torch.equal(Lp, Lm)
    n = lp.numel() // 2
    assert torch.equal(lp[:n], lp[n:])


def _cobatch_vs_alone(w, shape=None, steps=2):
    batch = wl.make_batch(w, fg_rows=5)
    model, h = gpu_handle(w, shape=shape, fg=5)
    toks, ftoks = dev_tokens(batch), dev_fg_tokens(batch)
    for t in range(steps):
        h.zo_probe_plan(t, w.eps)
        _, _, _, flp = h.zo_score_cobatch(toks, batch.seq_lens, batch.target_lens, ftoks,
                                          batch.fg_seq_lens, batch.fg_target_lens)
        alone = h.zo_score_foreground(ftoks, batch.fg_seq_lens, batch.fg_target_lens)
        assert torch.equal(flp, alone), t
        # the probe rows' results are not disturbed by the foreground rows either
        h.zo_score(toks, batch.seq_lens, batch.target_lens)
        h.zo_step(w.lr)


def test_cobatched_foreground_bit_identical_fp32():
    _cobatch_vs_alone(dataclasses.replace(TINY, fg_rows=5))


def test_cobatched_foreground_bit_identical_bf16():
    _cobatch_vs_alone(dataclasses.replace(TINY_BF16, fg_rows=5))


def test_cobatched_foreground_bit_identical_qwen3_bf16():
    shape = dataclasses.replace(Q3_SMALL, dtype=wl.DTYPE_BF16)
    _cobatch_vs_alone(dataclasses.replace(QWEN_SMALL, shape=shape), steps=4)


def test_deterministic_and_resumable():
    w = TINY_BF16
    batch = wl.make_batch(w)
    toks = dev_tokens(batch)

    def run(h, t0, t1):
        out = []
        for t in range(t0, t1):
            h.zo_probe_plan(t, w.eps)
            Lp, Lm, _ = h.zo_score(toks, batch.seq_lens, batch.target_lens)
            out.append((Lp.cpu().numpy().copy(), Lm.cpu().numpy().copy(), h.zo_step(w.lr)))
        return out

    _, h1 = gpu_handle(w, nu=3)
    a = run(h1, 0, 8)
    _, h2 = gpu_handle(w, nu=3)
    b = run(h2, 0, 4)
    state = h2.zo_save_state()
    h2.close()
    _, h3 = gpu_handle(w, nu=3)
    h3.zo_load_state(state)
    b += run(h3, 4, 8)
    for (x1, y1, c1), (x2, y2, c2) in zip(a, b):
        assert np.array_equal(x1, x2) and np.array_equal(y1, y2) and c1 == c2


def test_nonfinite_objective_refused_bank_unchanged():
    from zeroth_order_fine_b200 import zo
    w = TINY
    batch = wl.make_batch(w)
    model, h = gpu_handle(w)
    toks = dev_tokens(batch)
    h.zo_probe_plan(0, w.eps)
    h.zo_score(toks, batch.seq_lens, batch.target_lens)
    h.zo_step(w.lr)
    A0 = h.zo_read_bank(0, wl.MAT_Q, 0)
    h.zo_probe_plan(1, 0.0)                       # c = 0 / (2 * 0): not finite
    h.zo_score(toks, batch.seq_lens, batch.target_lens)
    with pytest.raises(zo.ZoError) as e:
        h.zo_step(w.lr)
    assert e.value.code == zo.ZO_ERR_NONFINITE
    assert np.array_equal(h.zo_read_bank(0, wl.MAT_Q, 0), A0)
    h.zo_probe_plan(1, w.eps)                     # the step counter did not advance
    h.zo_score(toks, batch.seq_lens, batch.target_lens)
    h.zo_step(w.lr)


def test_call_order_and_argument_errors():
    from zeroth_order_fine_b200 import zo
    w = TINY
    batch = wl.make_batch(w)
    model, h = gpu_handle(w)
    toks = dev_tokens(batch)
    with pytest.raises(zo.ZoError) as e:
        h.zo_probe_plan(3, w.eps)
    assert e.value.code == zo.ZO_ERR_STATE
    h.zo_probe_plan(0, w.eps)
    with pytest.raises(zo.ZoError) as e:
        h.zo_step(w.lr)
    assert e.value.code == zo.ZO_ERR_STATE
    bad = batch.target_lens.copy()
    bad[0] = batch.seq_lens[0]                    # no prefix left
    with pytest.raises(zo.ZoError) as e:
        h.zo_score(toks, batch.seq_lens, bad)
    assert e.value.code == zo.ZO_ERR_ARG
    wrong = torch.from_numpy(batch.target_ids()).cuda()
    wrong[0] += 1
    h.zo_score(toks, batch.seq_lens, batch.target_lens, target_ids=wrong)
    with pytest.raises(zo.ZoError) as e:
        h.zo_step(w.lr)
    assert e.value.code == zo.ZO_ERR_ARG


@pytest.mark.parametrize("dtype", [wl.DTYPE_FP32, wl.DTYPE_BF16])
def test_state_transition_bytes_counted(dtype):
    """The byte model of the state change: U written each step (fp32, or bf16 only for bf16
    models); the update writes the slot's accumulator (and its bf16 mirror) without reading
    it, rebuilding it from the window's coefficients (their history read, this step's
    written); a window writes V, its two copies in the extension operand and a zeroed slot."""
    w = dataclasses.replace(TINY, shape=wl.shrink_shape(wl.TINY, dtype=dtype))
    batch = wl.make_batch(w)
    model, h = gpu_handle(w, nu=4)
    toks = dev_tokens(batch)
    for t in range(6):
        h.zo_probe_plan(t, w.eps)
        h.zo_score(toks, batch.seq_lens, batch.target_lens)
        h.zo_step(w.lr)
    s = h.zo_stats()
    sh = w.shape
    es = 2 if dtype == wl.DTYPE_BF16 else 4
    mirror = 2 if dtype == wl.DTYPE_BF16 else 0
    u = sum(sh.matrix_dims(m)[0] * w.rank for m in w.matrices) * sh.n_layers
    v = sum(sh.matrix_dims(m)[1] * w.rank for m in w.matrices) * sh.n_layers
    per_step_u = (2 if dtype == wl.DTYPE_BF16 else 4) * u
    replay_lens = [1, 2, 3, 4, 1, 2]                   # steps since the slot opened (nu = 4)
    updates = sum((4 + mirror) * u + 4 * n for n in replay_lens)
    per_window = 4 * v + 2 * es * v + (4 + mirror) * u
    assert s["state_transition_bytes"] == 6 * per_step_u + updates + 2 * per_window
    assert s["dense_ref_bytes"] == 6 * 2 * es * sh.body_params()
    assert s["steps"] == 6 and s["bank_slots"] == 2


@pytest.mark.parametrize("shape", ["tiny-bf16", "qwen3-bf16"])
def test_bank_replay_equals_read_modify_write(shape, monkeypatch):
    """The update that rebuilds the slot from its coefficients and the one that reads it back
    give the same bank and the same objectives, bit for bit, across windows (nu = 3)."""
    if shape == "tiny-bf16":
        w = TINY_BF16
    else:
        w = dataclasses.replace(QWEN_SMALL, shape=dataclasses.replace(Q3_SMALL, dtype=wl.DTYPE_BF16),
                                fg_rows=0)
    batch = wl.make_batch(w, fg_rows=0)
    toks = dev_tokens(batch)
    runs = []
    for mode in ("1", "0"):
        monkeypatch.setenv("ZO_BANK_REPLAY", mode)
        _, h = gpu_handle(w, nu=3)
        out = []
        for t in range(8):
            h.zo_probe_plan(t, w.eps)
            Lp, Lm, _ = h.zo_score(toks, batch.seq_lens, batch.target_lens)
            out.append((Lp.cpu().numpy().copy(), Lm.cpu().numpy().copy(), h.zo_step(w.lr)))
        runs.append((out, h.zo_save_state(), h.zo_stats()["state_transition_bytes"]))
        h.close()
    (a, sa, ba), (b, sb, bb) = runs
    for (x1, y1, c1), (x2, y2, c2) in zip(a, b):
        assert np.array_equal(x1, x2) and np.array_equal(y1, y2) and c1 == c2
    assert sa == sb
    assert ba < bb                                     # the replay reads no accumulator


@pytest.mark.parametrize("shape", ["tiny-bf16", "qwen3-bf16"])
def test_bf16_models_never_leave_the_tensor_cores(shape):
    """Every GEMM of a bf16 model runs on tcgen05 whatever the bank width: a window
    opens every step (nu = 1), so the extension grows through widths of every residue."""
    if shape == "tiny-bf16":
        w = TINY_BF16
    else:
        w = dataclasses.replace(QWEN_SMALL, shape=dataclasses.replace(Q3_SMALL, dtype=wl.DTYPE_BF16),
                                fg_rows=0, rank=3)
    batch = wl.make_batch(w, fg_rows=0)
    model, h = gpu_handle(w, nu=1, max_slots=9)
    toks = dev_tokens(batch)
    for t in range(9):
        h.zo_probe_plan(t, w.eps)
        h.zo_score(toks, batch.seq_lens, batch.target_lens)
        h.zo_step(w.lr)
    s = h.zo_stats()
    assert s["bank_slots"] == 9
    assert s["cuda_core_gemm_launches"] == 0


def test_load_state_clears_slots_beyond_the_loaded_bank():
    """A shorter bank loaded into a handle that held a longer one scores like a fresh load."""
    w = TINY_BF16
    batch = wl.make_batch(w)
    toks = dev_tokens(batch)
    _, ha = gpu_handle(w, nu=1, max_slots=8)
    for t in range(2):
        ha.zo_probe_plan(t, w.eps)
        ha.zo_score(toks, batch.seq_lens, batch.target_lens)
        ha.zo_step(w.lr * 1000)
    short = ha.zo_save_state()
    for t in range(2, 6):
        ha.zo_probe_plan(t, w.eps)
        ha.zo_score(toks, batch.seq_lens, batch.target_lens)
        ha.zo_step(w.lr * 1000)
    ha.zo_load_state(short)
    _, hb = gpu_handle(w, nu=1, max_slots=8)
    hb.zo_load_state(short)
    outs = []
    for h in (ha, hb):
        h.zo_probe_plan(2, w.eps)
        Lp, Lm, _ = h.zo_score(toks, batch.seq_lens, batch.target_lens)
        outs.append((Lp.cpu().numpy(), Lm.cpu().numpy()))
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])


@pytest.mark.parametrize("dtype", [wl.DTYPE_FP32, wl.DTYPE_BF16])
def test_edge_rows_match_oracle(dtype):
    """The shortest rows (one prefix token), a row at the model's max_pos, a single
    prompt, and a target span covering all but the first token."""
    shape = wl.shrink_shape(wl.TINY, dtype=dtype)
    w = dataclasses.replace(TINY, shape=shape, tgt_hi=8)      # room for 8-token spans
    rng = np.random.default_rng(7)
    rows = [rng.integers(0, shape.vocab, size=L).astype(np.int32) for L in (2, shape.max_pos, 9)]
    tls = np.array([1, 3, 8], dtype=np.int32)
    batch = wl.Batch(rows, tls, [], np.zeros(0, np.int32))
    model, h = gpu_handle(w, batch=3)
    orc = oracle_run(w)
    tol = 1e-4 if dtype == wl.DTYPE_FP32 else 2e-2
    for sub in ([0], [0, 1, 2]):
        b = wl.Batch([rows[i] for i in sub], tls[sub], [], np.zeros(0, np.int32))
        h.zo_probe_plan(0, w.eps)
        orc.plan(0, w.eps)
        Lp, Lm, lp = h.zo_score(dev_tokens(b), b.seq_lens, b.target_lens, want_logprob=True)
        ref = orc.score(b.prompts, b.target_lens)
        assert np.max(np.abs(Lp.cpu().numpy() - ref.L_plus)) <= tol
        assert np.max(np.abs(Lm.cpu().numpy() - ref.L_minus)) <= tol
        if dtype == wl.DTYPE_FP32:
            assert np.max(np.abs(lp.cpu().numpy() - _cat(ref.logprob_plus + ref.logprob_minus))) <= 1e-4


def test_rows_beyond_max_pos_rejected():
    from zeroth_order_fine_b200 import zo
    w = TINY
    model, h = gpu_handle(w, batch=2)
    row = np.zeros(w.shape.max_pos + 1, dtype=np.int32)
    b = wl.Batch([row], np.array([1], np.int32), [], np.zeros(0, np.int32))
    h.zo_probe_plan(0, w.eps)
    with pytest.raises(zo.ZoError) as e:
        h.zo_score(dev_tokens(b), b.seq_lens, b.target_lens)
    assert e.value.code == zo.ZO_ERR_ARG


def _graph_workload(shape):
    if shape == "tiny-bf16":
        return TINY_BF16
    return dataclasses.replace(QWEN_SMALL, shape=dataclasses.replace(Q3_SMALL, dtype=wl.DTYPE_BF16),
                               fg_rows=0)


@pytest.mark.parametrize("shape", ["tiny-bf16", "qwen3-bf16"])
def test_step_graph_is_bit_identical_to_eager_steps(shape):
    """zo_step_graph replays one captured graph per window; L+/L- of every step and the
    final bank equal those of plan/score/step called one by one, across window
    boundaries (nu = 3) and with eager steps interleaved (the device step counter is
    re-seeded)."""
    w = _graph_workload(shape)
    batch = wl.make_batch(w, fg_rows=0)
    toks = dev_tokens(batch)
    _, he = gpu_handle(w, nu=3)
    _, hg = gpu_handle(w, nu=3)
    eager, graphed = [], []
    for t in range(8):
        he.zo_probe_plan(t, w.eps)
        Lp, Lm, _ = he.zo_score(toks, batch.seq_lens, batch.target_lens)
        eager.append((Lp.cpu().numpy().copy(), Lm.cpu().numpy().copy()))
        he.zo_step(w.lr, want_c=False)
        if t == 5:                                   # an eager step in the middle
            hg.zo_probe_plan(t, w.eps)
            Lp, Lm, _ = hg.zo_score(toks, batch.seq_lens, batch.target_lens)
            hg.zo_step(w.lr, want_c=False)
        else:
            Lp, Lm = hg.zo_step_graph(toks, batch.seq_lens, batch.target_lens, w.eps, w.lr)
        graphed.append((Lp.cpu().numpy().copy(), Lm.cpu().numpy().copy()))
    for (a, b), (c, d) in zip(eager, graphed):
        assert np.array_equal(a, c) and np.array_equal(b, d)
    assert he.zo_save_state() == hg.zo_save_state()
    s = hg.zo_stats()
    # windows open at steps 0, 3, 6: one capture each; the other graph steps replay
    assert s["graph_captures"] == 3 and s["graph_replays"] == 7
    assert s["steps"] == 8 and s["last_error_code"] == 0


def test_step_graph_follows_new_token_contents():
    """The graph reads the current contents of the token buffer: new prompts of the same
    layout give the same L+/L- as the eager path on those prompts."""
    w = TINY_BF16
    b0 = wl.make_batch(w)
    rng = np.random.default_rng(3)
    b1 = wl.Batch([rng.integers(0, w.shape.vocab, len(p)).astype(np.int32) for p in b0.prompts],
                  b0.target_lens, [], np.zeros(0, dtype=np.int32))
    toks = dev_tokens(b0)
    _, he = gpu_handle(w, nu=50)
    _, hg = gpu_handle(w, nu=50)
    for t, b in enumerate([b0, b1, b0]):
        toks.copy_(torch.from_numpy(b.packed()).cuda())
        he.zo_probe_plan(t, w.eps)
        Lp, Lm, _ = he.zo_score(toks, b.seq_lens, b.target_lens)
        he.zo_step(w.lr, want_c=False)
        Gp, Gm = hg.zo_step_graph(toks, b.seq_lens, b.target_lens, w.eps, w.lr)
        assert torch.equal(Lp, Gp) and torch.equal(Lm, Gm)
    assert hg.zo_stats()["graph_captures"] == 1


def test_step_graph_refuses_an_open_plan():
    from zeroth_order_fine_b200 import zo
    w = TINY_BF16
    batch = wl.make_batch(w)
    toks = dev_tokens(batch)
    _, h = gpu_handle(w)
    h.zo_probe_plan(0, w.eps)
    with pytest.raises(zo.ZoError) as e:
        h.zo_step_graph(toks, batch.seq_lens, batch.target_lens, w.eps, w.lr)
    assert e.value.code == zo.ZO_ERR_STATE
