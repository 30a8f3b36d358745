"""Decoder forward of the oracle: PyTorch CPU float64, written as the definitions.

Two families, both evaluated on the pages (OPT-1.3B..13B and Qwen3-8B; "LLM
Zeroth-Order Fine-Tuning is an Inference Workload", abstract, and
"Inference-Native Zeroth-Order Optimization", abstract):

* OPT: learned absolute positions (0-based, no offset), pre-LayerNorm blocks,
  multi-head attention with biases and 1/sqrt(d_h) scaling, ReLU FFN, final
  LayerNorm, lm_head tied to the token embedding.
* Qwen3: RMSNorm, per-head RMSNorm on q and k, rotary positions (rotate-half
  form, base rope_theta), grouped-query attention, SwiGLU FFN, no biases,
  untied lm_head.

Every row is its own causal sequence (packing is a physical layout only:
"Inference-Native Zeroth-Order Optimization", abstract, credits the
ragged-batch gain to padding elimination and variable-length packing, which
change speed, not results).  Token-wise layers run on the rows' tokens
concatenated; attention runs row by row.

Perturbed linears follow the factored definition.  With theta = W^T in
R^{d_in x d_out}, candidate sign s in {+1, -1, 0}, bank slots (A_j, V_j) and
the current direction U_t V_k^T:

    y = x theta + b + sum_j (x A_j) V_j^T + s * eps * (x U_t) V_k^T

which is x (theta + sum_j A_j V_j^T + s eps U_t V_k^T) + b without forming
the dense matrix (page 1, "The System Reorganization": accumulate on the U
factor, Delta W = U V^T).  ``dense=True`` forms the dense matrix instead;
the tests use it as the brute-force check.

bf16 mode (a reading: the pages name no precision): weights are bf16 values
and every activation entering a weight GEMM (normalised inputs, q/k/v,
attention output, FFN activation, final hidden state) is rounded to bf16;
everything else -- residual stream, norms, softmax, log-sum-exp, factors,
bank -- stays in float64 here.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np
import torch

from zeroth_order_fine_b200 import workload as wl
from . import fp8 as fp8q
from . import generator as gen

f64 = torch.float64


def bf16_round(x: torch.Tensor) -> torch.Tensor:
    """Round to bf16 (nearest even) through fp32, kept as float64 values."""
    return torch.from_numpy(gen.to_bf16(x.detach().to(torch.float32).numpy())).to(f64)


@dataclasses.dataclass
class Weights:
    shape: wl.ModelShape
    tok_embed: torch.Tensor                    # [V, d]
    pos_embed: Optional[torch.Tensor]          # [max_pos, d] (OPT)
    final_w: torch.Tensor
    final_b: Optional[torch.Tensor]
    lm_head: torch.Tensor                      # [V, d] (tok_embed when tied)
    layers: List[Dict[str, torch.Tensor]]      # keys: W0..W6 ([d_out, d_in]), b0..b6, ln1_w ...


def _t(a: np.ndarray, shape) -> torch.Tensor:
    return torch.from_numpy(a.astype(np.float64)).reshape(shape)


def init_weights(shape: wl.ModelShape, weight_seed: int = 0,
                 layers: Optional[Sequence[int]] = None) -> Weights:
    """The random-init model, drawn from the counter stream (generator.weight).

    Matrices and embeddings N(0, 0.02); biases N(0, 0.02); norm scales
    1 + N(0, 0.02); LayerNorm shifts N(0, 0.02).  Matrices and embeddings are
    bf16 in bf16 mode, 1-D parameters stay fp32.  ``layers`` restricts which
    layer indices are drawn (the others are left out of the list).
    """
    bf = shape.dtype == wl.DTYPE_BF16
    d, V = shape.d_model, shape.vocab
    G = gen.GLOBAL_LAYER
    tok = _t(gen.weight(weight_seed, G, gen.T_TOK_EMBED, V * d, 0.02, 0.0, bf), (V, d))
    pos = None
    fb = None
    if shape.arch == wl.ARCH_OPT:
        pos = _t(gen.weight(weight_seed, G, gen.T_POS_EMBED, shape.max_pos * d, 0.02, 0.0, bf),
                 (shape.max_pos, d))
        fb = _t(gen.weight(weight_seed, G, gen.T_FINAL_B, d, 0.02, 0.0, False), (d,))
    fw = _t(gen.weight(weight_seed, G, gen.T_FINAL_W, d, 0.02, 1.0, False), (d,))
    if shape.tie_lm_head:
        head = tok
    else:
        head = _t(gen.weight(weight_seed, G, gen.T_LM_HEAD, V * d, 0.02, 0.0, bf), (V, d))
    lay = []
    idx = range(shape.n_layers) if layers is None else layers
    for l in idx:
        p: Dict[str, torch.Tensor] = {}
        for m in shape.matrices():
            di, do = shape.matrix_dims(m)
            p[f"W{m}"] = _t(gen.weight(weight_seed, l, m, do * di, 0.02, 0.0, bf), (do, di))
            if shape.arch == wl.ARCH_OPT:
                p[f"b{m}"] = _t(gen.weight(weight_seed, l, gen.T_BIAS0 + m, do, 0.02, 0.0, False),
                                (do,))
        p["ln1_w"] = _t(gen.weight(weight_seed, l, gen.T_LN1_W, d, 0.02, 1.0, False), (d,))
        p["ln2_w"] = _t(gen.weight(weight_seed, l, gen.T_LN2_W, d, 0.02, 1.0, False), (d,))
        if shape.arch == wl.ARCH_OPT:
            p["ln1_b"] = _t(gen.weight(weight_seed, l, gen.T_LN1_B, d, 0.02, 0.0, False), (d,))
            p["ln2_b"] = _t(gen.weight(weight_seed, l, gen.T_LN2_B, d, 0.02, 0.0, False), (d,))
        else:
            hd = shape.head_dim
            p["q_norm"] = _t(gen.weight(weight_seed, l, gen.T_QNORM, hd, 0.02, 1.0, False), (hd,))
            p["k_norm"] = _t(gen.weight(weight_seed, l, gen.T_KNORM, hd, 0.02, 1.0, False), (hd,))
        lay.append(p)
    return Weights(shape, tok, pos, fw, fb, head, lay)


# ---- perturbation state handed to the forward ------------------------------------------

@dataclasses.dataclass
class MatrixPerturbation:
    """Per (layer, matrix): bank slots and the current direction."""
    bank: List[Tuple[torch.Tensor, torch.Tensor]]   # (A_j [d_in x r], V_j [d_out x r])
    U: Optional[torch.Tensor] = None                 # U_t [d_in x r]
    V: Optional[torch.Tensor] = None                 # V_k [d_out x r] of the current window


Perturb = Dict[Tuple[int, int], MatrixPerturbation]


# Matrices whose base product runs in FP8 in the fp8 mode: the ones fed by a norm
# (q, k, v and the FFN input projections), whose inputs have a per-token scale.
FP8_MATRICES = (wl.MAT_Q, wl.MAT_K, wl.MAT_V, wl.MAT_GATE, wl.MAT_UP)


def base_product(x: torch.Tensor, W: torch.Tensor, fp8: bool) -> torch.Tensor:
    """x W^T; with fp8, of the per-row E4M3 quantised x and W (oracle/fp8.py)."""
    if not fp8:
        return x @ W.T
    return (fp8q.dequant_rows(x.to(torch.float32).numpy()) @
            fp8q.dequant_rows(W.to(torch.float32).numpy()).T)


def perturbed_linear(x: torch.Tensor, W: torch.Tensor, b: Optional[torch.Tensor],
                     pert: Optional[MatrixPerturbation], sign_eps: torch.Tensor,
                     dense: bool, fp8: bool = False) -> torch.Tensor:
    """y = x (W^T + sum_j A_j V_j^T + s eps U V^T) + b, row-wise signs in sign_eps [T].

    With fp8 the base term x W^T is taken between the E4M3-quantised x and W; the
    bank and direction terms keep the exact x."""
    if pert is None:
        y = base_product(x, W, fp8)
    elif not dense:
        y = base_product(x, W, fp8)
        for A, Vj in pert.bank:
            y = y + (x @ A) @ Vj.T
        if pert.U is not None:
            y = y + sign_eps[:, None] * ((x @ pert.U) @ pert.V.T)
    else:
        # brute force: one dense theta per distinct sign value
        y = torch.empty(x.shape[0], W.shape[0], dtype=f64)
        base = torch.zeros_like(W.T) if fp8 else W.T.clone()
        for A, Vj in pert.bank:
            base = base + A @ Vj.T
        for se in torch.unique(sign_eps):
            theta = base.clone()
            if pert.U is not None:
                theta = theta + se * (pert.U @ pert.V.T)
            rows = sign_eps == se
            y[rows] = x[rows] @ theta
        if fp8:
            y = y + base_product(x, W, True)
    if b is not None:
        y = y + b
    return y


def layer_norm(x, w, b, eps):
    mu = x.mean(-1, keepdim=True)
    var = ((x - mu) ** 2).mean(-1, keepdim=True)
    return (x - mu) / torch.sqrt(var + eps) * w + b


def rms_norm(x, w, eps):
    return x / torch.sqrt((x * x).mean(-1, keepdim=True) + eps) * w


def rope(x: torch.Tensor, pos: torch.Tensor, theta: float) -> torch.Tensor:
    """Rotary positions, rotate-half pairing (i, i + hd/2); x [T, H, hd]."""
    hd = x.shape[-1]
    half = hd // 2
    inv = theta ** (-torch.arange(0, half, dtype=f64) * 2.0 / hd)
    ang = pos.to(f64)[:, None] * inv[None, :]
    cos = torch.cos(ang)[:, None, :]
    sin = torch.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return torch.cat([x1 * cos - x2 * sin, x2 * cos + x1 * sin], dim=-1)


def causal_attention(q, k, v, n_rep: int) -> torch.Tensor:
    """One row: q [L, H, hd], k/v [L, Hkv, hd] -> [L, H*hd]; softmax(q k^T / sqrt(hd) + causal) v."""
    L, H, hd = q.shape
    if n_rep > 1:
        k = k.repeat_interleave(n_rep, dim=1)
        v = v.repeat_interleave(n_rep, dim=1)
    s = torch.einsum("qhd,khd->hqk", q, k) / math.sqrt(hd)
    mask = torch.ones(L, L, dtype=torch.bool).tril()
    s = s.masked_fill(~mask, float("-inf"))
    p = torch.softmax(s, dim=-1)
    o = torch.einsum("hqk,khd->qhd", p, v)
    return o.reshape(L, H * hd)


def hidden_states(w: Weights, rows: Sequence[np.ndarray], signs: Sequence[float], eps,
                  perturb: Optional[Perturb], dense: bool = False,
                  layer_ids: Optional[Sequence[int]] = None, fp8: bool = False) -> torch.Tensor:
    """Final-norm hidden states [T, d] of the concatenated rows (float64).

    fp8: the base products of FP8_MATRICES use E4M3 inputs (oracle/fp8.py)."""
    sh = w.shape
    bf = sh.dtype == wl.DTYPE_BF16
    rnd = bf16_round if bf else (lambda t: t)
    lens = [len(r) for r in rows]
    tok = torch.from_numpy(np.concatenate(rows).astype(np.int64))
    pos = torch.cat([torch.arange(L) for L in lens])
    # eps may be a float or a 0-d tensor (the autograd pin differentiates through it)
    sign_eps = torch.cat([torch.full((L,), float(s), dtype=f64) * eps for L, s in zip(lens, signs)])
    h = w.tok_embed[tok].clone()
    if sh.arch == wl.ARCH_OPT:
        h = h + w.pos_embed[pos]
    bounds = np.cumsum([0] + lens)
    ids = range(len(w.layers)) if layer_ids is None else layer_ids
    H, Hkv, hd = sh.n_heads, sh.n_kv_heads, sh.head_dim

    for li, p in zip(ids, w.layers):
        def lin(x, m):
            pm = perturb.get((li, m)) if perturb else None
            return perturbed_linear(x, p[f"W{m}"], p.get(f"b{m}"), pm, sign_eps, dense,
                                    fp8 and m in FP8_MATRICES)

        if sh.arch == wl.ARCH_OPT:
            x = rnd(layer_norm(h, p["ln1_w"], p["ln1_b"], sh.norm_eps))
        else:
            x = rnd(rms_norm(h, p["ln1_w"], sh.norm_eps))
        q = rnd(lin(x, wl.MAT_Q)).reshape(-1, H, hd)
        k = rnd(lin(x, wl.MAT_K)).reshape(-1, Hkv, hd)
        v = rnd(lin(x, wl.MAT_V)).reshape(-1, Hkv, hd)
        if sh.arch == wl.ARCH_QWEN3:
            q = rope(rms_norm(q, p["q_norm"], sh.norm_eps), pos, sh.rope_theta)
            k = rope(rms_norm(k, p["k_norm"], sh.norm_eps), pos, sh.rope_theta)
        att = torch.cat([causal_attention(q[a:b], k[a:b], v[a:b], H // Hkv)
                         for a, b in zip(bounds[:-1], bounds[1:])])
        h = h + lin(rnd(att), wl.MAT_O)
        if sh.arch == wl.ARCH_OPT:
            x = rnd(layer_norm(h, p["ln2_w"], p["ln2_b"], sh.norm_eps))
            a = rnd(torch.relu(lin(x, wl.MAT_UP)))
        else:
            x = rnd(rms_norm(h, p["ln2_w"], sh.norm_eps))
            g = lin(x, wl.MAT_GATE)
            a = rnd(torch.nn.functional.silu(g) * lin(x, wl.MAT_UP))
        h = h + lin(a, wl.MAT_DOWN)

    if sh.arch == wl.ARCH_OPT:
        return layer_norm(h, w.final_w, w.final_b, sh.norm_eps)
    return rms_norm(h, w.final_w, sh.norm_eps)


def span_logits(w: Weights, hs: torch.Tensor, rows: Sequence[np.ndarray],
                target_lens: Sequence[int]) -> List[torch.Tensor]:
    """Per row, the full-vocabulary logits [tl, V] at the positions that predict its last
    tl tokens (positions L - tl - 1 .. L - 2)."""
    bf = w.shape.dtype == wl.DTYPE_BF16
    out = []
    off = 0
    for r, tl in zip(rows, target_lens):
        L = len(r)
        idx = torch.arange(off + L - tl - 1, off + L - 1)
        hsel = hs[idx]
        if bf:
            hsel = bf16_round(hsel)
        out.append(hsel @ w.lm_head.T)
        off += L
    return out


def token_logprobs(w: Weights, hs: torch.Tensor, rows: Sequence[np.ndarray],
                   target_lens: Sequence[int]) -> List[torch.Tensor]:
    """Per row, log p(target token | prefix) for each of its last target_lens tokens.

    The scored hidden state of target token j (position L - tl + j) is the
    one at the position before it; the log-probability is the full-vocabulary
    log-softmax of h W_lm^T there (the objective is token log-probabilities
    of the label tokens: page 1, "Why ZO Fine-Tuning Is Really Scoring" and
    "The System Reorganization").
    """
    out = []
    for r, tl, logits in zip(rows, target_lens, span_logits(w, hs, rows, target_lens)):
        L = len(r)
        lse = torch.logsumexp(logits, dim=-1)
        tgt = torch.from_numpy(np.asarray(r[L - tl:], dtype=np.int64))
        out.append(logits[torch.arange(tl), tgt] - lse)
    return out


def last_logits(w: Weights, hs: torch.Tensor, rows: Sequence[np.ndarray]) -> torch.Tensor:
    """Logits [rows, V] at each row's last position: the prediction of its next token."""
    bf = w.shape.dtype == wl.DTYPE_BF16
    ends = torch.from_numpy(np.cumsum([len(r) for r in rows]) - 1)
    hsel = hs[ends]
    if bf:
        hsel = bf16_round(hsel)
    return hsel @ w.lm_head.T
