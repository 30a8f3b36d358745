"""FP8 (E4M3) quantisation of the oracle: test infrastructure only.

The frozen base weights may be run in 8-bit floating point ("Inference-Native
Zeroth-Order Optimization", abstract: the probe queries run on an inference
runtime and inherit its quantisation).  The pages fix no format; the reading
taken here (and by the CUDA path) is:

* format E4M3 (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits,
  subnormals, no infinities; the all-ones exponent with all-ones mantissa is
  NaN, so the largest finite magnitude is 448);
* weights: one scale per output channel (row of W [d_out, d_in]);
  activations: one scale per token (row of x [T, d_in]);
* per row: amax = max |x|, inv = 448 / amax and scale = amax / 448, both
  fp32 quotients rounded to nearest; codes = E4M3(x * inv) with the fp32
  product rounded to nearest, then rounded to nearest-even E4M3 and clamped
  at +-448; an all-zero row has scale 1 and zero codes;
* the quantised product is dequant(x) dequant(W)^T = (codes_x * s_x)(codes_W * s_W)^T.

``e4m3_table`` decodes all 256 codes from the bit layout above; the tests pin
the library cast used by ``round_e4m3`` against it.
"""
from __future__ import annotations

from typing import Tuple

import numpy as np
import torch

E4M3_MAX = 448.0


def e4m3_table() -> np.ndarray:
    """Value of every code 0..255 (float64; NaN for the two NaN codes)."""
    vals = np.empty(256, dtype=np.float64)
    for c in range(256):
        s = -1.0 if c & 0x80 else 1.0
        e = (c >> 3) & 0xF
        m = c & 0x7
        if e == 0xF and m == 0x7:
            vals[c] = np.nan
        elif e == 0:
            vals[c] = s * (m / 8.0) * 2.0 ** (1 - 7)
        else:
            vals[c] = s * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


def round_e4m3(x: np.ndarray) -> np.ndarray:
    """fp32 values rounded to the nearest E4M3 value (ties to even), clamped at +-448."""
    x = np.clip(np.asarray(x, dtype=np.float32), -E4M3_MAX, E4M3_MAX)
    t = torch.from_numpy(np.ascontiguousarray(x)).to(torch.float8_e4m3fn)
    return t.to(torch.float32).numpy()


def quantize_rows(x: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Per-row E4M3 quantisation of an fp32 matrix: (values of the codes [R, K] fp32, scale [R] fp32)."""
    x = np.asarray(x, dtype=np.float32)
    amax = np.max(np.abs(x), axis=1).astype(np.float32)
    nz = amax > 0
    inv = np.ones_like(amax)
    inv[nz] = np.float32(E4M3_MAX) / amax[nz]
    scale = np.ones_like(amax)
    scale[nz] = amax[nz] / np.float32(E4M3_MAX)
    codes = round_e4m3((x * inv[:, None]).astype(np.float32))
    return codes, scale


def dequant_rows(x: np.ndarray) -> torch.Tensor:
    """dequant(quantize_rows(x)) as float64: codes times the row scale."""
    codes, scale = quantize_rows(x)
    return torch.from_numpy(codes.astype(np.float64) * scale.astype(np.float64)[:, None])
