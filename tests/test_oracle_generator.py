"""Pins of the oracle's counter-based direction stream (CPU only).

The stream is pinned to things other than itself: an independent pure-Python
integer splitmix64, the published first outputs of splitmix64 seeded with 0
(tests/golden/splitmix64_seed0.txt), libm for the own ln/sin/cos, and the
N(0,1) law for the Box-Muller output.
"""
import math
import os

import numpy as np
import pytest
from scipy import stats

from oracle import generator as g

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
MASK = (1 << 64) - 1


def py_splitmix64(seed, n):
    """Textbook splitmix64 on Python ints: state += gamma, then the finaliser."""
    out, state = [], seed & MASK
    for _ in range(n):
        state = (state + 0x9E3779B97F4A7C15) & MASK
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK
        out.append(z ^ (z >> 31))
    return out


def test_splitmix64_published_first_outputs():
    vals = []
    with open(os.path.join(GOLDEN, "splitmix64_seed0.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                vals.append(int(line, 16))
    assert [int(x) for x in g.stream(0, 0, len(vals))] == vals
    assert py_splitmix64(0, len(vals)) == vals


@pytest.mark.parametrize("key", [0, 1, 0xDEADBEEFCAFEF00D, MASK, g.factor_key(7, 3, 50, 2, 1, 0)])
def test_stream_matches_pure_python(key):
    ref = py_splitmix64(key, 300)
    assert [int(x) for x in g.stream(key, 0, 300)] == ref
    assert [int(x) for x in g.stream(key, 137, 50)] == ref[137:187]


def test_mix_int_matches_array_mix():
    zs = [0, 1, 12345, MASK, 0x8000000000000000]
    arr = g._mix_arr(np.array(zs, dtype=np.uint64))
    assert [int(a) for a in arr] == [g.mix_int(z) for z in zs]


def _ulp32(x):
    return np.spacing(np.abs(x).astype(np.float32)).astype(np.float64)


def test_own_ln_within_3ulp_of_libm_all_inputs():
    k = np.arange(1, (1 << 24) + 1, dtype=np.int64)
    u = k.astype(np.float32) * np.float32(2.0 ** -24)
    mine = g.ln_f32(u).astype(np.float64)
    ref = np.log(u.astype(np.float64))
    nz = ref != 0
    err = np.abs(mine[nz] - ref[nz]) / _ulp32(ref[nz])
    assert err.max() <= 3.0, err.max()
    assert mine[-1] == 0.0            # ln 1 = 0 exactly (u1 = 1 gives rho = 0)


def test_own_sincos_against_libm_all_inputs():
    k = np.arange(0, 1 << 24, dtype=np.int64)
    s, c = g.sincos_2pi_f32(k)
    ang = 2.0 * np.pi * k / float(1 << 24)
    assert np.max(np.abs(s - np.sin(ang))) < 2.5e-7
    assert np.max(np.abs(c - np.cos(ang))) < 2.5e-7
    # exact at the quarter turns (exact dyadic reduction)
    q = np.array([0, 1 << 22, 2 << 22, 3 << 22])
    s, c = g.sincos_2pi_f32(q)
    assert list(s) == [0.0, 1.0, 0.0, -1.0]
    assert list(np.abs(c)) == [1.0, 0.0, 1.0, 0.0]


def test_box_muller_pair_layout_and_odd_tail():
    key = g.factor_key(1, 0, 50, 0, 0, 0)
    z = g.normals(key, 11)
    z10 = g.normals(key, 10)
    assert np.array_equal(z[:10], z10)
    b = int(g.stream(key, 5, 1)[0])
    u1 = np.float32((b >> 40) + 1) * np.float32(2.0 ** -24)
    rho = np.sqrt(np.float32(-2.0) * g.ln_f32(np.array([u1], np.float32)))[0]
    s, c = g.sincos_2pi_f32(np.array([b & 0xFFFFFF]))
    assert z[10] == np.float32(rho * c[0])        # the last z1 is dropped
    # the same pair against libm in float64 (Box-Muller as published)
    assert abs(z[10] - math.sqrt(-2 * math.log(float(u1))) *
               math.cos(2 * math.pi * (b & 0xFFFFFF) / 2 ** 24)) < 1e-5


def test_normal_law():
    z = g.normals(g.factor_key(99, 5, 50, 1, 2, 1), 1 << 20).astype(np.float64)
    n = z.size
    assert abs(z.mean()) < 5 / math.sqrt(n)
    assert abs(z.var() - 1.0) < 5 * math.sqrt(2.0 / n)
    assert abs(stats.skew(z)) < 0.02
    assert abs(stats.kurtosis(z)) < 0.03
    assert stats.kstest(z, "norm").pvalue > 1e-3


def test_factor_keys_lazy_window():
    U0 = g.factor(1, 10, 5, 3, 0, 0, 64, 2, 0)
    U1 = g.factor(1, 11, 5, 3, 0, 0, 64, 2, 0)
    assert not np.array_equal(U0, U1)                              # U drawn every step
    V10 = g.factor(1, 10, 5, 3, 0, 1, 96, 2, 0)
    V14 = g.factor(1, 14, 5, 3, 0, 1, 96, 2, 0)
    V15 = g.factor(1, 15, 5, 3, 0, 1, 96, 2, 0)
    assert np.array_equal(V10, V14)                                # V held for the window
    assert not np.array_equal(V14, V15)                            # new window, new V
    assert not np.array_equal(g.factor(1, 10, 5, 3, 2, 0, 64, 2, 0), U0)   # matrix in key
    assert not np.array_equal(g.factor(1, 10, 5, 4, 0, 0, 64, 2, 0), U0)   # layer in key


def test_mezo_scale_is_one_over_sqrt_r():
    a = g.factor(3, 0, 50, 0, 4, 0, 40, 64, 0)
    b = g.factor(3, 0, 50, 0, 4, 0, 40, 64, 1)
    assert np.array_equal(b, (a * np.float32(0.125)).astype(np.float32))


def test_bf16_rounding_matches_torch():
    import torch
    x = (np.random.default_rng(0).standard_normal(100000) * 10).astype(np.float32)
    x[:4] = [1.00390625, 1.01171875, -1.00390625, 3.0e-39]        # ties and a subnormal
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(g.to_bf16(x), ref)


def test_weight_init_distribution():
    w = g.weight(0, 1, 0, 200000, 0.02, 0.0, False)
    assert abs(w.std() - 0.02) < 5e-4
    n = g.weight(0, 1, 14, 1000, 0.02, 1.0, False)
    assert abs(n.mean() - 1.0) < 5e-3
