"""Pins of the oracle's E4M3 quantisation (oracle/fp8.py) against the format's
definition, and of its fp8 forward against its own invariants."""
import numpy as np
import pytest
import torch

from oracle import fp8
from zeroth_order_fine_b200 import workload as wl


def test_codebook_by_definition():
    v = fp8.e4m3_table()
    assert np.isnan(v[0x7F]) and np.isnan(v[0xFF])
    fin = v[np.isfinite(v)]
    assert len(fin) == 254
    assert fin.max() == 448.0 and fin.min() == -448.0
    pos = np.sort(fin[fin > 0])
    assert pos[0] == 2.0 ** -9                      # smallest subnormal
    assert 2.0 ** -6 in pos and 2.0 ** -6 - 2.0 ** -9 in pos   # smallest normal, largest subnormal
    assert len(pos) == 126 and v[0] == 0.0 and v[0x80] == 0.0


def _nearest_even(x: np.ndarray) -> np.ndarray:
    """Brute force: nearest finite E4M3 value; on a tie the one whose code is even."""
    v = fp8.e4m3_table()
    codes = np.array([c for c in range(256) if np.isfinite(v[c])])
    vals = v[codes]
    out = np.empty_like(x, dtype=np.float64)
    for i, xi in enumerate(np.clip(x.astype(np.float64), -448.0, 448.0)):
        d = np.abs(vals - xi)
        best = np.flatnonzero(d == d.min())
        cand = codes[best]
        if len(cand) > 1:
            cand = cand[(cand & 1) == 0]
        out[i] = v[cand[0]]
    return out


def test_cast_is_round_to_nearest_even_with_saturation():
    rng = np.random.default_rng(0)
    v = fp8.e4m3_table()
    fin = np.unique(v[np.isfinite(v)])
    mids = ((fin[1:] + fin[:-1]) / 2).astype(np.float32)       # every tie (exact in fp32)
    xs = np.concatenate([
        rng.standard_normal(3000).astype(np.float32) * np.float32(30.0),
        (rng.standard_normal(1000) * 0.01).astype(np.float32),  # subnormal range
        mids, fin.astype(np.float32),
        np.array([500.0, -1e6, 449.0, 464.0, 465.0, 0.0], dtype=np.float32)])
    got = fp8.round_e4m3(xs).astype(np.float64)
    want = _nearest_even(xs)
    assert np.array_equal(got, want)


def test_quantize_rows_bounds_and_equivariance():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((16, 300)).astype(np.float32)
    x[3] = 0.0
    codes, scale = fp8.quantize_rows(x)
    assert scale[3] == 1.0 and not codes[3].any()
    amax = np.abs(x).max(1)
    for r in range(16):
        if r == 3:
            continue
        assert np.max(np.abs(codes[r])) == 448.0              # the amax element saturates the range
        deq = codes[r].astype(np.float64) * scale[r]
        # half an E4M3 step: 2^-4 relative for normals, 2^-10 * scale absolute below them
        err = np.abs(deq - x[r])
        bound = np.maximum(np.abs(x[r]) * 2.0 ** -4, 2.0 ** -10 * scale[r]) * (1 + 1e-6)
        assert np.all(err <= bound + 2 * np.abs(x[r]) * 2.0 ** -23)
        assert np.isclose(scale[r], amax[r] / 448.0, rtol=1e-7)
    # scaling a row by a power of two keeps its codes and scales the scale
    c2, s2 = fp8.quantize_rows(x * np.float32(8.0))
    assert np.array_equal(c2, codes) and np.array_equal(s2[scale != 1], scale[scale != 1] * 8)


def test_fp8_forward_invariants():
    from oracle import model as om
    from oracle import zo as ozo
    w = wl.WORKLOADS["tiny"]
    sh = wl.shrink_shape(wl.TINY, dtype=wl.DTYPE_BF16)
    weights = om.init_weights(sh, w.weight_seed)
    batch = wl.make_batch(w, batch=3)
    base = ozo.OracleRun(weights, w.run_seed, w.nu, w.rank, range(sh.n_layers), w.matrices,
                         w.scale_mode)
    q = ozo.OracleRun(weights, w.run_seed, w.nu, w.rank, range(sh.n_layers), w.matrices,
                      w.scale_mode, fp8=True)
    for run in (base, q):
        run.plan(0, 0.0)
    r0 = q.score(batch.prompts, batch.target_lens)
    assert np.array_equal(r0.L_plus, r0.L_minus)               # eps = 0
    q2 = ozo.OracleRun(weights, w.run_seed, w.nu, w.rank, range(sh.n_layers), w.matrices,
                       w.scale_mode, fp8=True)
    q2.plan(0, w.eps)
    fac = q2.score(batch.prompts, batch.target_lens)
    den = q2.score(batch.prompts, batch.target_lens, dense=True)
    assert np.allclose(fac.L_plus, den.L_plus, atol=1e-10)     # factored == brute force
    assert np.allclose(fac.L_minus, den.L_minus, atol=1e-10)
    rb = base.score(batch.prompts, batch.target_lens)
    assert not np.array_equal(rb.L_plus, r0.L_plus)            # the quantiser is applied
    assert np.allclose(rb.L_plus, r0.L_plus, atol=5e-2)         # and only perturbs slightly
