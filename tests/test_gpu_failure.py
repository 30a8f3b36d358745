"""Failure paths on the GPU, made without faulting or hanging it.

* A bounded wait that runs out: every mbarrier wait of the tensor-core GEMM gives up after a
  bound (about 2 s by default), records bit 0 of the error word, drains what it issued,
  frees its tensor memory and returns.  Setting the bound to a few hundred cycles makes an
  ordinary, healthy launch give up at its first wait for data -- no barrier is broken,
  nothing traps -- and the next launch with the default bound must be clean and correct.
  Only the single-SM kernel is used here (N = 128).
* An allocation that fails: ZO_FAIL_ALLOC_AT=n makes the n-th device allocation of
  zo_create fail; the call returns ZO_ERR_OOM, says why, and frees everything it had taken.
"""
import os

import numpy as np

import pytest
import torch

from zeroth_order_fine_b200 import workload as wl
from gpu_util import needs_gpu

pytestmark = [pytest.mark.gpu, needs_gpu]


def _bf16_ulp(x):
    return torch.clamp(torch.abs(x), min=1e-30) * 2.0 ** -7


def test_expired_wait_reports_timeout_then_the_next_launch_is_clean():
    from zeroth_order_fine_b200 import zo
    g = torch.Generator().manual_seed(21)
    M, N, K = 256, 128, 4096                      # single-SM kernel, 64 K blocks per tile
    x = torch.randn(M, K, generator=g).to(torch.bfloat16)
    W = (torch.randn(N, K, generator=g) * 0.05).to(torch.bfloat16)
    ref = x.double() @ W.double().T
    xd, Wd = x.cuda(), W.cuda()
    y = torch.zeros(M, N, dtype=torch.bfloat16, device="cuda")
    zo.zo_op_linear(xd, Wd, out=y, impl=zo.IMPL_TENSOR_CORES)
    assert zo.zo_op_error_word() == 0
    model = zo.DeviceModel(wl.WORKLOADS["tiny"].shape)
    w = wl.WORKLOADS["tiny"]
    h = zo.Handle(model, w.run_seed, w.nu, w.rank, zo.make_targets(2, w.matrices, w.scale_mode),
                  max_tokens=64, max_rows=2, max_scored=2)
    old = zo.zo_op_set_wait_limit(300)
    try:
        zo.zo_op_linear(xd, Wd, out=y, impl=zo.IMPL_TENSOR_CORES)     # queued: returns ZO_OK
        torch.cuda.synchronize()
        # the handle reports the expired wait as ZO_ERR_TIMEOUT (and clears the word)
        assert h.zo_stats()["last_error_code"] == zo.ZO_ERR_TIMEOUT
        zo.zo_op_linear(xd, Wd, out=y, impl=zo.IMPL_TENSOR_CORES)
        assert zo.zo_op_error_word() & 1
    finally:
        restored = zo.zo_op_set_wait_limit(0)
    assert restored == 300 and old > 10 ** 9
    assert zo.zo_op_error_word() == 0
    # the same launch with the default bound: clean, correct, and the context still usable
    for _ in range(2):
        y2 = zo.zo_op_linear(xd, Wd, impl=zo.IMPL_TENSOR_CORES)
        assert zo.zo_op_error_word() == 0
        err = (y2.double().cpu() - ref).abs()
        assert torch.all(err <= _bf16_ulp(ref) + 1e-4 * (K ** 0.5) * 0.05), err.max()
    assert h.zo_stats()["last_error_code"] == 0
    h.close()


def _create(w, shape):
    from zeroth_order_fine_b200 import zo
    model = zo.DeviceModel(shape, w.weight_seed)
    h = zo.Handle(model, w.run_seed, w.nu, w.rank,
                  zo.make_targets(shape.n_layers, w.matrices, w.scale_mode),
                  max_tokens=512, max_rows=16, max_scored=16)
    return model, h


@pytest.mark.parametrize("wk", ["tiny", "tiny-bf16"])
def test_injected_allocation_failure_returns_oom_and_leaks_nothing(wk):
    """Every device allocation of zo_create in turn is made to fail (n = 1, 2, ... until a
    create goes through): each time the call returns ZO_ERR_OOM naming the allocation, and
    the device's free memory is back where it was."""
    from zeroth_order_fine_b200 import zo
    w = wl.WORKLOADS["tiny"]
    shape = w.shape if wk == "tiny" else wl.shrink_shape(w.shape, dtype=wl.DTYPE_BF16)
    model, h = _create(w, shape)                    # warm-up: modules loaded, then freed
    h.close()
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    tg = zo.make_targets(shape.n_layers, w.matrices, w.scale_mode)
    n = 0
    try:
        while True:
            n += 1
            assert n < 1000
            os.environ["ZO_FAIL_ALLOC_AT"] = str(n)
            try:
                h2 = zo.Handle(model, w.run_seed, w.nu, w.rank, tg, max_tokens=512,
                               max_rows=16, max_scored=16)
            except zo.ZoError as e:
                assert e.code == zo.ZO_ERR_OOM, (n, str(e))
                assert f"allocation {n} refused" in str(e), str(e)
                torch.cuda.synchronize()
                assert torch.cuda.mem_get_info()[0] == free0, n
                continue
            h2.close()                               # n is past the last allocation
            break
    finally:
        os.environ.pop("ZO_FAIL_ALLOC_AT", None)
    assert n > 20, n                                # every allocation point was visited
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0


@pytest.mark.parametrize("bad", ["vocab", "negative", "last-target"])
def test_out_of_range_token_ids_are_rejected_on_the_device(bad):
    """A token id outside [0, vocab) is never used as an index: build_tokens replaces it
    (its embedding row becomes NaN; a target's logit NaN), so only that prompt's L+- turn
    NaN, the other prompts score exactly as in a clean batch, zo_step reports ZO_ERR_ARG
    naming the id and leaves the bank as it was, and the next clean step goes through."""
    from zeroth_order_fine_b200 import zo
    from gpu_util import dev_tokens, gpu_handle
    w = wl.WORKLOADS["tiny"]
    batch = wl.make_batch(w)
    clean = batch.packed()
    _, h = gpu_handle(w)
    h.zo_probe_plan(0, w.eps)
    Lp0, Lm0, _ = h.zo_score(dev_tokens(batch), batch.seq_lens, batch.target_lens)
    Lp0, Lm0 = Lp0.cpu().numpy(), Lm0.cpu().numpy()
    state0 = h.zo_save_state()
    toks = clean.copy()
    starts = np.concatenate([[0], np.cumsum(batch.seq_lens)])
    i = 1                                                 # the prompt that gets the bad id
    pos = {"vocab": starts[i] + 1, "negative": starts[i] + 2,
           "last-target": starts[i + 1] - 1}[bad]
    toks[pos] = {"vocab": w.shape.vocab, "negative": -5, "last-target": w.shape.vocab + 7}[bad]
    h.zo_probe_plan(0, w.eps)
    Lp, Lm, _ = h.zo_score(torch.from_numpy(toks).cuda(), batch.seq_lens, batch.target_lens)
    Lp, Lm = Lp.cpu().numpy(), Lm.cpu().numpy()
    assert np.isnan(Lp[i]) and np.isnan(Lm[i])
    others = [j for j in range(len(batch.seq_lens)) if j != i]
    assert np.array_equal(Lp[others], Lp0[others]) and np.array_equal(Lm[others], Lm0[others])
    with pytest.raises(zo.ZoError) as e:
        h.zo_step(w.lr)
    assert e.value.code == zo.ZO_ERR_ARG and "token id" in str(e.value)
    assert h.zo_save_state() == state0                    # update refused, bank unchanged
    h.zo_probe_plan(0, w.eps)
    Lp1, Lm1, _ = h.zo_score(dev_tokens(batch), batch.seq_lens, batch.target_lens)
    assert np.array_equal(Lp1.cpu().numpy(), Lp0) and np.array_equal(Lm1.cpu().numpy(), Lm0)
    c = h.zo_step(w.lr)
    assert np.isfinite(c)
    h.close()


def test_capacity_limits_are_refused_and_leave_no_trace():
    """Batches past the handle's sizes (rows, tokens, scored positions), rows too short to
    score and an empty batch are refused with ZO_ERR_ARG before any launch; the handle then
    steps exactly like a fresh one."""
    from zeroth_order_fine_b200 import zo
    from gpu_util import dev_tokens, gpu_handle
    w = wl.WORKLOADS["tiny"]
    batch = wl.make_batch(w)
    B = len(batch.prompts)
    T = int(batch.seq_lens.sum())
    model = zo.DeviceModel(w.shape, w.weight_seed)
    tg = zo.make_targets(w.shape.n_layers, w.matrices, w.scale_mode)

    def handle():
        return zo.Handle(model, w.run_seed, w.nu, w.rank, tg, max_tokens=2 * T, max_rows=2 * B,
                         max_scored=2 * int(batch.target_lens.sum()))

    h, ref = handle(), handle()
    toks = dev_tokens(batch)
    h.zo_probe_plan(0, w.eps)
    rng = np.random.default_rng(3)
    cases = {
        "more rows than max_rows": list(batch.prompts) + [batch.prompts[0]],
        # rows of max_pos tokens: twice the physical tokens the handle was sized for
        "more tokens than max_tokens": [np.concatenate([p, p]) for p in batch.prompts],
    }
    for msg, prompts in cases.items():
        b = wl.Batch(prompts, np.ones(len(prompts), np.int32), [], np.zeros(0, np.int32))
        with pytest.raises(zo.ZoError) as e:
            h.zo_score(dev_tokens(b), b.seq_lens, b.target_lens)
        assert e.value.code == zo.ZO_ERR_ARG and msg in str(e.value), str(e.value)
    wide = batch.target_lens.copy() + 1                       # one more scored position each
    with pytest.raises(zo.ZoError) as e:
        h.zo_score(toks, batch.seq_lens, np.minimum(wide + 4, batch.seq_lens - 1))
    assert e.value.code == zo.ZO_ERR_ARG and "max_scored" in str(e.value)
    short = wl.Batch([rng.integers(0, w.shape.vocab, 1).astype(np.int32)], np.ones(1, np.int32),
                     [], np.zeros(0, np.int32))
    with pytest.raises(zo.ZoError) as e:
        h.zo_score(dev_tokens(short), short.seq_lens, short.target_lens)
    assert e.value.code == zo.ZO_ERR_ARG
    with pytest.raises(zo.ZoError) as e:
        h.zo_score(toks[:0], np.zeros(0, np.int32), np.zeros(0, np.int32))
    assert e.value.code == zo.ZO_ERR_ARG
    for hh in (h, ref):
        hh.zo_probe_plan(0, w.eps)
        hh.zo_score(toks, batch.seq_lens, batch.target_lens)
    assert h.zo_step(w.lr) == ref.zo_step(w.lr)
    assert h.zo_save_state() == ref.zo_save_state()
    h.close()
    ref.close()
