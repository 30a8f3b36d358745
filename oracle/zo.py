"""Two-point ZO step of the oracle: probe plan, scoring, estimator, factored bank update.

Method ("Zeroth-Order Fine-Tuning Was an Inference Workload All Along"):

* two-point estimator (section "Why ZO Fine-Tuning Is Really Scoring"):
  L+ = L(theta + eps z), L- = L(theta - eps z), c = (L+ - L-) / (2 eps),
  update theta <- theta - eta c z;
* LoZO direction: per matrix z = U V^T of rank r; no 1/r factor in the
  estimator, matching the released LoZO code (section "The System
  Reorganization");
* lazy sampling: V held for a window of nu steps, U drawn every step; the
  update accumulates on the U side, U_{t+1} = U_t - eta c_t G_t with
  Delta W = U_{t+1} V^T, so over a window the change is
  (U_t - eta sum_s c_s G_s) V^T (same section, "Memory-write reduction").
  Here each window k owns a bank slot (A_k, V_k) with A_k starting at 0 and
  A_k <- A_k - eta c_t U_t; theta_t = theta_0 + sum_k A_k V_k^T.
* MeZO-style factorised mode multiplies both factors by 1/sqrt(r) (a
  reading of the multivariate central-limit remark in "Inference-Native
  Zeroth-Order Optimization", abstract: the product then has unit-variance
  entries as r grows).

Objective per prompt row (a reading of "token log-probabilities" / "option-
token losses"): the mean negative log-probability of the row's target span.
Over a batch of B prompts c = (1/B) sum_i (L+_i - L-_i) / (2 eps).
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np
import torch

from zeroth_order_fine_b200 import workload as wl
from . import generator as gen
from . import model as om

f64 = torch.float64


def estimate_c(L_plus: Sequence[float], L_minus: Sequence[float], eps: float) -> float:
    """c = mean_i (L+_i - L-_i) / (2 eps); no 1/r (page 1, "The System Reorganization")."""
    lp = np.asarray(L_plus, dtype=np.float64)
    lm = np.asarray(L_minus, dtype=np.float64)
    return float(np.mean(lp - lm) / (2.0 * eps))


def row_objective(logprobs: torch.Tensor) -> float:
    """L_row = mean over the target span of -log p."""
    return float(-logprobs.mean())


@dataclasses.dataclass
class ScoreResult:
    L_plus: np.ndarray           # [B]
    L_minus: np.ndarray          # [B]
    logprob_plus: List[np.ndarray]
    logprob_minus: List[np.ndarray]
    fg_logprob: List[np.ndarray]


class OracleRun:
    """Persistent-bank ZO run: plan(t) -> score -> step(lr), in the pages' order."""

    def __init__(self, weights: om.Weights, run_seed: int, nu: int, rank: int,
                 layers: Sequence[int], matrices: Sequence[int], scale_mode: int,
                 start_step: int = 0, fp8: bool = False):
        self.w = weights
        self.fp8 = fp8                  # E4M3 base products of the norm-fed matrices
        self.sh = weights.shape
        self.run_seed = run_seed
        self.nu = nu
        self.r = rank
        self.layers = list(layers)
        self.matrices = list(matrices)
        self.scale_mode = scale_mode
        self.t = start_step
        # bank[(layer, matrix)] = list of [A_k, V_k, window]
        self.bank: Dict[Tuple[int, int], List[list]] = {(l, m): [] for l in self.layers
                                                        for m in self.matrices}
        self.U: Dict[Tuple[int, int], torch.Tensor] = {}
        self.eps: Optional[float] = None
        self.last: Optional[ScoreResult] = None

    # -- plan ---------------------------------------------------------------------------
    def factors(self, layer: int, m: int, t: int):
        di, do = self.sh.matrix_dims(m)
        U = gen.factor(self.run_seed, t, self.nu, layer, m, 0, di, self.r, self.scale_mode)
        V = gen.factor(self.run_seed, t, self.nu, layer, m, 1, do, self.r, self.scale_mode)
        return U, V

    def plan(self, t: int, eps: float) -> None:
        """Draw U_t for every target; at a window start open a slot (A = 0, V = V_window)."""
        assert t == self.t
        self.eps = eps
        for (l, m), slots in self.bank.items():
            U, V = self.factors(l, m, t)
            self.U[(l, m)] = torch.from_numpy(U.astype(np.float64))
            window = t // self.nu
            if not slots or slots[-1][2] != window:
                di, _ = self.sh.matrix_dims(m)
                slots.append([torch.zeros(di, self.r, dtype=f64),
                              torch.from_numpy(V.astype(np.float64)), window])

    def perturbation(self, with_direction: bool = True) -> om.Perturb:
        out: om.Perturb = {}
        for (l, m), slots in self.bank.items():
            bank = [(A, V) for A, V, _ in slots]
            if with_direction and (l, m) in self.U:
                out[(l, m)] = om.MatrixPerturbation(bank, self.U[(l, m)], slots[-1][1])
            else:
                out[(l, m)] = om.MatrixPerturbation(bank)
        return out

    # -- score --------------------------------------------------------------------------
    def score(self, prompts: Sequence[np.ndarray], target_lens: Sequence[int],
              fg_prompts: Sequence[np.ndarray] = (), fg_target_lens: Sequence[int] = (),
              dense: bool = False, layer_ids: Optional[Sequence[int]] = None) -> ScoreResult:
        """Score every prompt under theta + eps z and theta - eps z (and fg rows under theta)."""
        B = len(prompts)
        rows = list(prompts) + list(prompts) + list(fg_prompts)
        signs = [1.0] * B + [-1.0] * B + [0.0] * len(fg_prompts)
        tls = list(target_lens) + list(target_lens) + list(fg_target_lens)
        hs = om.hidden_states(self.w, rows, signs, self.eps, self.perturbation(), dense,
                              layer_ids=layer_ids, fp8=self.fp8)
        lps = om.token_logprobs(self.w, hs, rows, tls)
        Lp = np.array([row_objective(x) for x in lps[:B]])
        Lm = np.array([row_objective(x) for x in lps[B:2 * B]])
        res = ScoreResult(Lp, Lm, [x.numpy() for x in lps[:B]],
                          [x.numpy() for x in lps[B:2 * B]], [x.numpy() for x in lps[2 * B:]])
        self.last = res
        return res

    # -- generation queries -------------------------------------------------------------
    def generate(self, prompts: Sequence[np.ndarray], n_new: int, dense: bool = False):
        """Greedy generation under theta + eps z (rows 0..B-1) and theta - eps z (rows
        B..2B-1): n_new tokens per row, each the largest logit of the full forward of the
        row so far (ties: lowest id); objective per row = mean -log p of its new tokens.

        A reading of "Inference-Native Zeroth-Order Optimization" (abstract: the same
        ProbePlan covers autoregressive generation); written as the plain definition, one
        full forward per new token, no cache.  Returns (L_plus, L_minus, tokens [2B, n_new],
        logprobs [2B, n_new]) and records the result for step()."""
        B = len(prompts)
        seqs = [list(np.asarray(prompts[r % B])) for r in range(2 * B)]   # one list per row
        signs = [1.0] * B + [-1.0] * B
        pert = self.perturbation()
        toks = np.zeros((2 * B, n_new), dtype=np.int64)
        lps = np.zeros((2 * B, n_new), dtype=np.float64)
        for g in range(n_new):
            rows = [np.asarray(x, dtype=np.int64) for x in seqs]
            hs = om.hidden_states(self.w, rows, signs, self.eps, pert, dense, fp8=self.fp8)
            logits = om.last_logits(self.w, hs, rows)
            lse = torch.logsumexp(logits, dim=-1)
            for r in range(2 * B):
                t = int(torch.argmax(logits[r]).item())
                toks[r, g] = t
                lps[r, g] = float(logits[r, t] - lse[r])
                seqs[r].append(t)
        L = -lps.mean(axis=1)
        res = ScoreResult(L[:B], L[B:], list(lps[:B]), list(lps[B:]), [])
        self.last = res
        return L[:B], L[B:], toks, lps

    # -- step ---------------------------------------------------------------------------
    def step(self, lr: float) -> float:
        """c from the last score; A_k <- A_k - lr c U_t for every target; t <- t + 1.

        A non-finite c is refused: the bank and the step counter stay as they were.
        """
        res = self.last
        c = estimate_c(res.L_plus, res.L_minus, self.eps)
        if not np.isfinite(c):
            return c          # refused: bank and step counter unchanged
        for key, slots in self.bank.items():
            slots[-1][0] = slots[-1][0] - lr * c * self.U[key]
        self.t += 1
        self.U = {}
        self.last = None
        return c

    def dense_delta(self, layer: int, m: int) -> torch.Tensor:
        """theta_t - theta_0 = sum_k A_k V_k^T for one matrix."""
        di, do = self.sh.matrix_dims(m)
        out = torch.zeros(di, do, dtype=f64)
        for A, V, _ in self.bank[(layer, m)]:
            out = out + A @ V.T
        return out


def run_steps(run: OracleRun, prompts, target_lens, eps: float, lr: float, n: int,
              fg_prompts=(), fg_target_lens=()) -> List[Tuple[float, float, float]]:
    """n consecutive plan/score/step rounds on one batch: [(mean L+, mean L-, c)]."""
    traj = []
    for _ in range(n):
        run.plan(run.t, eps)
        res = run.score(prompts, target_lens, fg_prompts, fg_target_lens)
        c = run.step(lr)
        traj.append((float(res.L_plus.mean()), float(res.L_minus.mean()), c))
    return traj
