"""Seeded synthetic workloads: model shapes and ragged prompt batches.

This module holds shapes and random inputs only -- no step of the ZO method.
Both the CUDA path (through the C-ABI) and the CPU oracle read the same
batches from here, so the two sides see identical tokens by construction.

Shapes follow the OPT and Qwen3 families the pages evaluate on ("LLM
Zeroth-Order Fine-Tuning is an Inference Workload", abstract: OPT-1.3B to
OPT-13B; "Inference-Native Zeroth-Order Optimization", abstract: Qwen3-8B
co-batching).  The pages' SST-2 prompts are replaced by synthetic ragged
prompts: token ids Zipf(1.1)-distributed over the vocabulary, lengths
uniform-integer in a range, and the scored span at each row's end.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import numpy as np

ARCH_OPT = 0
ARCH_QWEN3 = 1
DTYPE_FP32 = 0
DTYPE_BF16 = 1

# Matrix ids, in the order the direction keys use them.
MAT_Q, MAT_K, MAT_V, MAT_O, MAT_GATE, MAT_UP, MAT_DOWN = range(7)
MATRIX_NAMES = ("q", "k", "v", "o", "gate", "up", "down")

# Keys of the initial-weight tensors in the counter stream (weight_seed, layer, tensor):
# matrix ids 0..6 name the matrices themselves, 7 + id their biases.
T_BIAS0 = 7
T_LN1_W, T_LN1_B, T_LN2_W, T_LN2_B, T_QNORM, T_KNORM = 14, 15, 16, 17, 18, 19
T_TOK_EMBED, T_POS_EMBED, T_FINAL_W, T_FINAL_B, T_LM_HEAD = 32, 33, 34, 35, 36
GLOBAL_LAYER = 0xFFFF
# Initial distributions (a reading: the pages only say "random init"): matrices,
# embeddings and biases N(0, 0.02); norm scales 1 + N(0, 0.02); LayerNorm shifts N(0, 0.02).
INIT_STD = 0.02

SCALE_LOZO = 0       # factors unscaled
SCALE_MEZO = 1       # both factors multiplied by fp32(1/sqrt(r))


@dataclasses.dataclass(frozen=True)
class ModelShape:
    name: str
    arch: int
    n_layers: int
    d_model: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    d_ffn: int
    vocab: int
    max_pos: int
    norm_eps: float
    rope_theta: float
    dtype: int
    tie_lm_head: bool

    @property
    def q_dim(self) -> int:
        return self.n_heads * self.head_dim

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_dim

    def matrix_dims(self, m: int):
        """(d_in, d_out) of matrix m, with theta = W^T in R^{d_in x d_out}."""
        d, f = self.d_model, self.d_ffn
        return {
            MAT_Q: (d, self.q_dim), MAT_K: (d, self.kv_dim), MAT_V: (d, self.kv_dim),
            MAT_O: (self.q_dim, d), MAT_GATE: (d, f), MAT_UP: (d, f), MAT_DOWN: (f, d),
        }[m]

    def matrices(self):
        if self.arch == ARCH_OPT:
            return (MAT_Q, MAT_K, MAT_V, MAT_O, MAT_UP, MAT_DOWN)
        return (MAT_Q, MAT_K, MAT_V, MAT_O, MAT_GATE, MAT_UP, MAT_DOWN)

    def body_params(self) -> int:
        n = 0
        for m in self.matrices():
            di, do = self.matrix_dims(m)
            n += di * do
        return n * self.n_layers


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    shape: ModelShape
    batch: int                  # prompts (each scored as a + row and a - row)
    len_lo: int
    len_hi: int
    tgt_lo: int                 # target-span length range (tokens at row end)
    tgt_hi: int
    zipf: bool                  # Zipf(1.1) ids, else uniform
    rank: int
    matrices: tuple             # perturbed matrix ids
    scale_mode: int
    eps: float
    lr: float
    nu: int                     # lazy-V window
    fg_rows: int = 0            # co-batched foreground scoring rows
    fg_tgt_lo: int = 1
    fg_tgt_hi: int = 8
    data_seed: int = 1
    weight_seed: int = 0
    run_seed: int = 1234


def _opt(name, L, d, H, ffn, dtype, vocab=50272, max_pos=2048):
    return ModelShape(name, ARCH_OPT, L, d, H, H, d // H, ffn, vocab, max_pos,
                      1e-5, 0.0, dtype, True)


TINY = _opt("tiny-opt", 2, 128, 4, 512, DTYPE_FP32, vocab=1024, max_pos=64)
OPT_1_3B = _opt("opt-1.3b", 24, 2048, 32, 8192, DTYPE_BF16)
OPT_6_7B = _opt("opt-6.7b", 32, 4096, 32, 16384, DTYPE_BF16)
OPT_13B = _opt("opt-13b", 40, 5120, 40, 20480, DTYPE_BF16)
QWEN3_8B = ModelShape("qwen3-8b", ARCH_QWEN3, 36, 4096, 32, 8, 128, 12288, 151936,
                      4096, 1e-6, 1e6, DTYPE_BF16, False)

QV = (MAT_Q, MAT_V)
ALL7 = (MAT_Q, MAT_K, MAT_V, MAT_O, MAT_GATE, MAT_UP, MAT_DOWN)

WORKLOADS = {
    "tiny": Workload("tiny", TINY, 8, 32, 32, 1, 1, False, 2, QV, SCALE_LOZO,
                     1e-3, 1e-4, 50, data_seed=1),
    "opt-1.3b-b16": Workload("opt-1.3b-b16", OPT_1_3B, 16, 16, 128, 1, 1, True, 2, QV,
                             SCALE_LOZO, 1e-3, 1e-4, 50, data_seed=2),
    "opt-6.7b-b64": Workload("opt-6.7b-b64", OPT_6_7B, 64, 32, 256, 1, 8, True, 4, QV,
                             SCALE_LOZO, 1e-3, 1e-4, 50, data_seed=3),
    "opt-13b-b16": Workload("opt-13b-b16", OPT_13B, 16, 16, 128, 1, 1, True, 2, QV,
                            SCALE_LOZO, 1e-3, 1e-4, 50, data_seed=4),
    "opt-13b-b64": Workload("opt-13b-b64", OPT_13B, 64, 16, 128, 1, 1, True, 2, QV,
                            SCALE_LOZO, 1e-3, 1e-4, 50, data_seed=4),
    "qwen3-8b-cobatch": Workload("qwen3-8b-cobatch", QWEN3_8B, 16, 64, 512, 1, 1, True, 64,
                                 ALL7, SCALE_MEZO, 1e-3, 1e-4, 50, fg_rows=32,
                                 data_seed=5),
}


# bf16 100-step trajectory workload: the tiny model in bf16 with the direction on all six
# OPT matrices, eta = 2e-4 and eps = 1e-2.  100 steps move its loss by ~13 % (with q and v
# alone it moves 2.5-7 % at any eta), and at eps = 1e-3 the bf16 rounding of L is comparable
# to the paired difference 2 eps c, so two runs drift apart by several per cent.
TRAJ_TINY_BF16 = dataclasses.replace(
    WORKLOADS["tiny"], name="tiny-bf16-trajectory",
    shape=dataclasses.replace(TINY, name="tiny-opt-bf16", dtype=DTYPE_BF16),
    matrices=(MAT_Q, MAT_K, MAT_V, MAT_O, MAT_UP, MAT_DOWN), lr=2e-4, eps=1e-2)


def shrink_shape(shape: ModelShape, n_layers: Optional[int] = None, **kw) -> ModelShape:
    """The same family at another size (used for full-width layer slices)."""
    fields = dataclasses.asdict(shape)
    if n_layers is not None:
        fields["n_layers"] = n_layers
    fields.update(kw)
    return ModelShape(**fields)


@dataclasses.dataclass
class Batch:
    prompts: List[np.ndarray]        # per prompt, int32 tokens (target span included at the end)
    target_lens: np.ndarray          # int32 [B]
    fg_prompts: List[np.ndarray]
    fg_target_lens: np.ndarray

    @property
    def seq_lens(self) -> np.ndarray:
        return np.array([len(p) for p in self.prompts], dtype=np.int32)

    @property
    def fg_seq_lens(self) -> np.ndarray:
        return np.array([len(p) for p in self.fg_prompts], dtype=np.int32)

    def packed(self) -> np.ndarray:
        return np.concatenate(self.prompts).astype(np.int32) if self.prompts else np.zeros(0, np.int32)

    def fg_packed(self) -> np.ndarray:
        return (np.concatenate(self.fg_prompts).astype(np.int32) if self.fg_prompts
                else np.zeros(0, np.int32))

    def target_ids(self) -> np.ndarray:
        out = [p[len(p) - t:] for p, t in zip(self.prompts, self.target_lens)]
        return np.concatenate(out).astype(np.int32) if out else np.zeros(0, np.int32)

    def fg_target_ids(self) -> np.ndarray:
        out = [p[len(p) - t:] for p, t in zip(self.fg_prompts, self.fg_target_lens)]
        return np.concatenate(out).astype(np.int32) if out else np.zeros(0, np.int32)

    @property
    def n_tokens_physical(self) -> int:
        """Tokens of the physical batch: every prompt twice (+ and - row) plus foreground rows."""
        return 2 * int(self.seq_lens.sum()) + int(self.fg_seq_lens.sum())


def zipf_ids(rng: np.random.Generator, n: int, vocab: int, s: float = 1.1) -> np.ndarray:
    """Inverse-CDF draw with p(id) proportional to (id+1)^-s over [0, vocab)."""
    w = np.arange(1, vocab + 1, dtype=np.float64) ** (-s)
    cdf = np.cumsum(w)
    cdf /= cdf[-1]
    u = rng.random(n)
    return np.minimum(np.searchsorted(cdf, u, side="right"), vocab - 1).astype(np.int32)


def _draw_rows(rng, n, shape, len_lo, len_hi, tgt_lo, tgt_hi, zipf, labels):
    rows, tls = [], []
    for _ in range(n):
        L = int(rng.integers(len_lo, len_hi + 1))
        tl = int(rng.integers(tgt_lo, tgt_hi + 1))
        tl = max(1, min(tl, L - 1))
        if zipf:
            toks = zipf_ids(rng, L, shape.vocab)
        else:
            toks = rng.integers(0, shape.vocab, size=L).astype(np.int32)
        if tl == 1 and labels:
            # single label token drawn uniformly from two fixed ids
            toks[-1] = shape.vocab // 2 + int(rng.integers(0, 2))
        rows.append(toks.astype(np.int32))
        tls.append(tl)
    return rows, np.array(tls, dtype=np.int32)


def make_batch(w: Workload, batch: Optional[int] = None, fg_rows: Optional[int] = None,
               seed: Optional[int] = None, len_hi: Optional[int] = None) -> Batch:
    """The seeded ragged batch of workload w (optionally with fewer prompts or shorter rows)."""
    rng = np.random.default_rng(w.data_seed if seed is None else seed)
    B = w.batch if batch is None else batch
    F = w.fg_rows if fg_rows is None else fg_rows
    hi = w.len_hi if len_hi is None else len_hi
    lo = min(w.len_lo, hi)
    prompts, tls = _draw_rows(rng, B, w.shape, lo, hi, w.tgt_lo, w.tgt_hi, w.zipf, True)
    fg, fg_tls = _draw_rows(rng, F, w.shape, lo, hi, w.fg_tgt_lo, w.fg_tgt_hi, w.zipf, False)
    return Batch(prompts, tls, fg, fg_tls)
