"""Pins of the oracle's estimator, perturbation and factored bank (CPU only).

* eps = 0 gives L+ == L- bit for bit;
* on a quadratic toy objective the central difference equals the exact
  directional derivative (the odd terms cancel), with no 1/r factor;
* c(eps) tends to the autograd directional derivative of the forward with an
  O(eps^2) error;
* the factored perturbation equals a brute-force forward with the dense
  W +/- eps U V^T (and the dense bank) materialised;
* the bank equals the dense sum of its updates, window by window;
* a non-finite objective leaves the bank and the step counter untouched.
"""
import numpy as np
import pytest
import torch

from oracle import generator as gen
from oracle import model as om
from oracle import zo
from zeroth_order_fine_b200 import workload as wl

from test_oracle_model import TINY_Q3


def _run(shape, nu=50, rank=2, mats=wl.QV, scale=wl.SCALE_LOZO, seed=5):
    w = om.init_weights(shape)
    return zo.OracleRun(w, seed, nu, rank, range(shape.n_layers), mats, scale)


def _batch(shape, B=3, lo=6, hi=14, seed=3):
    rng = np.random.default_rng(seed)
    rows = [rng.integers(0, shape.vocab, size=int(rng.integers(lo, hi + 1))).astype(np.int32)
            for _ in range(B)]
    tls = [1 + (i % 2) for i in range(B)]
    return rows, tls


def test_eps_zero_gives_identical_objectives():
    run = _run(wl.TINY)
    rows, tls = _batch(wl.TINY)
    run.plan(0, 0.0)
    res = run.score(rows, tls)
    assert np.array_equal(res.L_plus, res.L_minus)


@pytest.mark.parametrize("r", [1, 2, 4])
def test_quadratic_toy_central_difference_is_exact(r):
    rng = np.random.default_rng(r)
    di, do = 6, 5
    n = di * do
    M = rng.standard_normal((n, n))
    A = M @ M.T
    b = rng.standard_normal(n)
    theta = rng.standard_normal(n)
    U = gen.factor(1, 0, 50, 0, 0, 0, di, r, 0).astype(np.float64)
    V = gen.factor(1, 0, 50, 0, 0, 1, do, r, 0).astype(np.float64)
    z = (U @ V.T).reshape(-1)

    def f(x):
        return 0.5 * x @ A @ x + b @ x

    for eps in (1e-1, 1e-3):
        c = zo.estimate_c([f(theta + eps * z)], [f(theta - eps * z)], eps)
        exact = (A @ theta + b) @ z          # no 1/r: the directional derivative along U V^T
        assert abs(c - exact) <= 1e-7 * max(1.0, abs(exact))


@pytest.mark.parametrize("shape", [wl.TINY, TINY_Q3], ids=["opt", "qwen3"])
def test_c_tends_to_autograd_directional_derivative(shape):
    mats = wl.QV if shape.arch == wl.ARCH_OPT else wl.ALL7
    run = _run(shape, mats=mats)
    rows, tls = _batch(shape, B=2)
    run.plan(0, 1e-3)

    tau = torch.zeros((), dtype=torch.float64, requires_grad=True)
    hs = om.hidden_states(run.w, rows, [1.0] * len(rows), tau, run.perturbation())
    lps = om.token_logprobs(run.w, hs, rows, tls)
    D = torch.stack([-x.mean() for x in lps]).mean()
    (g,) = torch.autograd.grad(D, tau)
    errs = []
    # small eps: ReLU kinks crossed inside +/- eps make the error O(eps) at eps ~ 1e-3
    for eps in (1e-5, 1e-6):
        run.eps = eps
        res = run.score(rows, tls)
        c = zo.estimate_c(res.L_plus, res.L_minus, eps)
        errs.append(abs(c - float(g)))
    assert errs[1] < 1e-6 * max(1.0, abs(float(g)))
    assert errs[1] < errs[0] / 50          # O(eps^2): 10x smaller eps, ~100x smaller error


@pytest.mark.parametrize("shape,mats,scale", [(wl.TINY, wl.QV, wl.SCALE_LOZO),
                                              (TINY_Q3, wl.ALL7, wl.SCALE_MEZO)],
                         ids=["opt-lozo", "qwen3-mezo"])
def test_factored_equals_dense_brute_force(shape, mats, scale):
    run = _run(shape, nu=2, rank=4, mats=mats, scale=scale)
    rows, tls = _batch(shape)
    fg, fg_tls = _batch(shape, B=2, seed=9)
    for t in range(3):          # two windows -> two bank slots with non-zero A
        run.plan(t, 1e-2)
        run.score(rows, tls)
        run.step(1e-1)
    run.plan(3, 1e-2)
    a = run.score(rows, tls, fg, fg_tls)
    b = run.score(rows, tls, fg, fg_tls, dense=True)
    assert len(run.bank[(0, mats[0])]) == 2
    assert np.max(np.abs(a.L_plus - b.L_plus)) < 1e-12
    assert np.max(np.abs(a.L_minus - b.L_minus)) < 1e-12
    for x, y in zip(a.fg_logprob, b.fg_logprob):
        assert np.max(np.abs(x - y)) < 1e-12
    assert not np.allclose(a.L_plus, a.L_minus)


def test_foreground_rows_score_current_state():
    run = _run(wl.TINY, nu=3)
    rows, tls = _batch(wl.TINY)
    for t in range(2):
        run.plan(t, 1e-2)
        run.score(rows, tls)
        run.step(1.0)
    run.plan(2, 1e-2)
    res = run.score(rows, tls, rows, tls)
    # a foreground row scores theta_t: the mean of its + and - rows to first order, and
    # exactly the state without the direction
    hs = om.hidden_states(run.w, rows, [0.0] * len(rows), 0.0, run.perturbation(False))
    ref = om.token_logprobs(run.w, hs, rows, tls)
    for x, y in zip(res.fg_logprob, ref):
        assert np.max(np.abs(x - y.numpy())) < 1e-12


def test_bank_equals_dense_sum_of_updates():
    nu = 3
    run = _run(wl.TINY, nu=nu)
    rows, tls = _batch(wl.TINY)
    cs = []
    for t in range(7):
        run.plan(t, 1e-2)
        run.score(rows, tls)
        cs.append(run.step(1e-1))
    for (l, m) in run.bank:
        di, do = wl.TINY.matrix_dims(m)
        dense = torch.zeros(di, do, dtype=torch.float64)
        for t, c in enumerate(cs):
            U = torch.from_numpy(gen.factor(5, t, nu, l, m, 0, di, 2, 0).astype(np.float64))
            V = torch.from_numpy(gen.factor(5, t, nu, l, m, 1, do, 2, 0).astype(np.float64))
            dense = dense - 1e-1 * c * (U @ V.T)
        assert torch.allclose(run.dense_delta(l, m), dense, atol=1e-14, rtol=1e-12)
        assert len(run.bank[(l, m)]) == 3         # windows 0, 1, 2


def test_nonfinite_objective_refused():
    run = _run(wl.TINY)
    rows, tls = _batch(wl.TINY)
    run.plan(0, 1e-2)
    run.score(rows, tls)
    run.last.L_plus[1] = np.nan
    before = [s[0].clone() for s in run.bank[(0, wl.MAT_Q)]]
    c = run.step(1e-1)
    assert not np.isfinite(c)
    assert run.t == 0
    assert all(torch.equal(a, s[0]) for a, s in zip(before, run.bank[(0, wl.MAT_Q)]))


def test_bf16_mode_trajectory_close_to_fp32():
    """bf16 rounding points move L by far less than the 2e-2 parity bound."""
    sh16 = wl.shrink_shape(wl.TINY, dtype=wl.DTYPE_BF16)
    rows, tls = _batch(wl.TINY)
    r32, r16 = _run(wl.TINY), _run(sh16)
    for r in (r32, r16):
        r.plan(0, 1e-3)
    a, b = r32.score(rows, tls), r16.score(rows, tls)
    # different weights (bf16-rounded), same model: objectives agree to bf16 level
    assert np.max(np.abs(a.L_plus - b.L_plus)) < 2e-2


def test_trajectory_workload_discriminates_the_update_strength():
    """The bf16 100-step trajectory check (2 % band) can tell a wrong update strength: on its
    workload the oracle's loss moves by more than five times the band, and the oracle run
    with half (or twice) the learning rate leaves the band."""
    w = wl.TRAJ_TINY_BF16
    weights = om.init_weights(w.shape, w.weight_seed)
    batch = wl.make_batch(w)

    def trajectory(lr):
        run = zo.OracleRun(weights, w.run_seed, w.nu, w.rank, range(w.shape.n_layers),
                           w.matrices, w.scale_mode)
        out = []
        for t in range(100):
            run.plan(t, w.eps)
            res = run.score(batch.prompts, batch.target_lens)
            out.append(float(res.L_plus.mean() + res.L_minus.mean()) / 2)
            run.step(lr)
        return np.array(out)

    ref = trajectory(w.lr)
    assert abs(ref[-1] - ref[0]) / ref[0] >= 0.10
    for wrong in (w.lr / 2, w.lr * 2):
        assert np.max(np.abs(trajectory(wrong) - ref) / ref) > 0.025, wrong
