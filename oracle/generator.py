"""Counter-based direction stream of the oracle (numpy, fp32 with one rounding per op).

The pages name a "random-direction stream" that the reorganised runtime keeps
unchanged ("Zeroth-Order Fine-Tuning Was an Inference Workload All Along",
section "The System Reorganization"), and LoZO's factors U, V of rank r
("Why ZO Fine-Tuning Is Really Scoring").  They do not say how the stream is
drawn; this library fixes one counter-based definition that the CUDA code
and this oracle implement independently and must agree on bit for bit:

* splitmix64 (Steele, Lea, Flood 2014; Vigna's public-domain finaliser):
  ``mix(z)`` and the j-th output of a generator seeded with ``key`` is
  ``mix(key + (j+1) * GAMMA) mod 2**64``.
* Keys chain ``mix`` over (run seed, step', layer, matrix*2 + factor),
  factor 0 = U, 1 = V; step' = t for U and nu*floor(t/nu) for V (V is held
  for the lazy window, section "The System Reorganization").
* Box-Muller on the 64-bit word b: u1 = ((b >> 40) + 1) * 2^-24 in (0, 1],
  u2 = (b & 0xFFFFFF) * 2^-24; z0 = sqrt(-2 ln u1) cos(2 pi u2),
  z1 = sqrt(-2 ln u1) sin(2 pi u2).
* ln, sin and cos are this library's own, written from their series so that
  both sides reproduce them exactly with +, -, *, / and sqrt alone (no fused
  multiply-add anywhere): ln m = 2 atanh((m-1)/(m+1)) on m in [sqrt(1/2),
  sqrt(2)); sin/cos by their Taylor series on [-pi/4, pi/4] after an exact
  quadrant reduction of the dyadic u2.
"""
from __future__ import annotations

import math

import numpy as np

MASK64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
M1 = 0xBF58476D1CE4E5B9
M2 = 0x94D049BB133111EB

# Weight tensors use a step' no direction ever has, so their keys never collide.
WEIGHT_TAG = MASK64

# Tensor ids of the initial weights are input keys, shared with the library's
# tests through the workload module (they hold no arithmetic of the method).
from zeroth_order_fine_b200.workload import (GLOBAL_LAYER, T_BIAS0, T_LN1_W, T_LN1_B,  # noqa: E402
                                             T_LN2_W, T_LN2_B, T_QNORM, T_KNORM, T_TOK_EMBED,
                                             T_POS_EMBED, T_FINAL_W, T_FINAL_B, T_LM_HEAD)

F32 = np.float32
_U64 = np.uint64


def mix_int(z: int) -> int:
    """splitmix64 finaliser on a Python int (the key chain is scalar)."""
    z &= MASK64
    z = ((z ^ (z >> 30)) * M1) & MASK64
    z = ((z ^ (z >> 27)) * M2) & MASK64
    return z ^ (z >> 31)


def _mix_arr(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> _U64(30))) * _U64(M1)
    z = (z ^ (z >> _U64(27))) * _U64(M2)
    return z ^ (z >> _U64(31))


def stream(key: int, j0: int, n: int) -> np.ndarray:
    """Outputs j0 .. j0+n-1 of splitmix64 seeded with key (uint64 array)."""
    with np.errstate(over="ignore"):
        j = np.arange(j0 + 1, j0 + n + 1, dtype=_U64)
        z = _U64(key) + j * _U64(GAMMA)
        return _mix_arr(z)


def factor_key(run_seed: int, step: int, nu: int, layer: int, matrix: int, factor: int) -> int:
    """Key of U (factor 0, keyed by t) or V (factor 1, keyed by its window start)."""
    step_p = step if factor == 0 else nu * (step // nu)
    k = mix_int(run_seed)
    k = mix_int(k ^ (step_p & MASK64))
    k = mix_int(k ^ layer)
    return mix_int(k ^ (matrix * 2 + factor))


def weight_key(weight_seed: int, layer: int, tensor: int) -> int:
    k = mix_int(weight_seed)
    k = mix_int(k ^ WEIGHT_TAG)
    k = mix_int(k ^ layer)
    return mix_int(k ^ tensor)


# ---- own fp32 ln / sin / cos (series; constants derived here from the mathematics) ----

def _f(x: float) -> np.float32:
    return F32(x)


_SQRT2 = _f(math.sqrt(2.0))
_ATANH = [_f(1.0 / k) for k in (3, 5, 7, 9, 11)]            # 1/3 .. 1/11
_LN2 = math.log(2.0)
_LN2_HI = np.array([_f(_LN2)], dtype=F32).view(np.uint32)
_LN2_HI = (_LN2_HI & np.uint32(0xFFFFFF00)).view(F32)[0]    # low 8 bits cleared: e*hi exact
_LN2_LO = _f(_LN2 - float(_LN2_HI))
_TWO_PI = _f(2.0 * math.pi)
_SIN = [_f(-1.0 / 6.0), _f(1.0 / 120.0), _f(-1.0 / 5040.0), _f(1.0 / 362880.0)]
_COS = [_f(-1.0 / 2.0), _f(1.0 / 24.0), _f(-1.0 / 720.0), _f(1.0 / 40320.0),
        _f(-1.0 / 3628800.0)]


def ln_f32(u: np.ndarray) -> np.ndarray:
    """ln(u) for fp32 u in [2^-24, 1], from ln m = 2 atanh(s), s = (m-1)/(m+1)."""
    u = np.asarray(u, dtype=F32)
    bits = u.view(np.uint32)
    e = (bits >> np.uint32(23)).astype(np.int32) - 127
    m = ((bits & np.uint32(0x7FFFFF)) | np.uint32(0x3F800000)).view(F32)
    big = m > _SQRT2
    m = np.where(big, m * F32(0.5), m).astype(F32)
    e = np.where(big, e + 1, e)
    s = (m - F32(1.0)) / (m + F32(1.0))
    s2 = s * s
    p = _ATANH[4]
    p = p * s2 + _ATANH[3]
    p = p * s2 + _ATANH[2]
    p = p * s2 + _ATANH[1]
    p = p * s2 + _ATANH[0]
    p = p * s2 + F32(1.0)
    ln_m = (s * p) * F32(2.0)
    ef = e.astype(F32)
    return (ef * _LN2_HI + (ef * _LN2_LO + ln_m)).astype(F32)


def sincos_2pi_f32(k24: np.ndarray):
    """(sin, cos) of 2*pi*k/2^24 for integer k in [0, 2^24), fp32 series after exact reduction."""
    k = np.asarray(k24, dtype=np.int64)
    qn = (k + (1 << 21)) >> 22                 # nearest quarter turn
    q = (qn & 3).astype(np.int64)
    f = (k - (qn << 22)).astype(F32) * F32(2.0 ** -24)   # in [-1/8, 1/8], exact
    th = f * _TWO_PI
    t2 = th * th
    ps = _SIN[3]
    ps = ps * t2 + _SIN[2]
    ps = ps * t2 + _SIN[1]
    ps = ps * t2 + _SIN[0]
    s = th + (th * t2) * ps
    pc = _COS[4]
    pc = pc * t2 + _COS[3]
    pc = pc * t2 + _COS[2]
    pc = pc * t2 + _COS[1]
    pc = pc * t2 + _COS[0]
    c = F32(1.0) + t2 * pc
    sin = np.select([q == 0, q == 1, q == 2], [s, c, -s], -c).astype(F32)
    cos = np.select([q == 0, q == 1, q == 2], [c, -s, -c], s).astype(F32)
    return sin, cos


def normals(key: int, n: int, chunk: int = 1 << 22) -> np.ndarray:
    """n N(0,1) fp32 values of the stream keyed by key: pair j -> elements 2j, 2j+1."""
    out = np.empty(n, dtype=F32)
    npairs = (n + 1) // 2
    for j0 in range(0, npairs, chunk):
        m = min(chunk, npairs - j0)
        b = stream(key, j0, m)
        k1 = (b >> _U64(40)).astype(np.int64) + 1
        u1 = k1.astype(F32) * F32(2.0 ** -24)
        k2 = (b & _U64(0xFFFFFF)).astype(np.int64)
        rho = np.sqrt(F32(-2.0) * ln_f32(u1)).astype(F32)
        sn, cs = sincos_2pi_f32(k2)
        z = np.empty(2 * m, dtype=F32)
        z[0::2] = rho * cs
        z[1::2] = rho * sn
        lo = 2 * j0
        hi = min(n, lo + 2 * m)
        out[lo:hi] = z[: hi - lo]
    return out


def mezo_scale(r: int) -> np.float32:
    return F32(1.0 / math.sqrt(r))


def factor(run_seed: int, step: int, nu: int, layer: int, matrix: int, which: int,
           dim: int, r: int, scale_mode: int) -> np.ndarray:
    """U_t (which=0, [d_in x r]) or V of the window holding t (which=1, [d_out x r]), fp32."""
    z = normals(factor_key(run_seed, step, nu, layer, matrix, which), dim * r).reshape(dim, r)
    if scale_mode == 1:
        z = (z * mezo_scale(r)).astype(F32)
    return z


def to_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (round to nearest even), returned as fp32 values."""
    b = np.asarray(x, dtype=F32).view(np.uint32).astype(np.uint64)
    b = (b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return (b.astype(np.uint32) << np.uint32(16)).view(F32)


def weight(weight_seed: int, layer: int, tensor: int, n: int, std: float, mean: float,
           bf16: bool) -> np.ndarray:
    """Initial weight tensor: fp32(z*std) (+ mean if mean != 0), optionally rounded to bf16."""
    w = normals(weight_key(weight_seed, layer, tensor), n) * F32(std)
    if mean != 0.0:
        w = (w + F32(mean)).astype(F32)
    return to_bf16(w) if bf16 else w
