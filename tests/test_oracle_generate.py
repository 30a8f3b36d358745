"""Pins of the oracle's generation queries (OracleRun.generate): greedy decoding by one
full forward per token, checked against teacher-forced scoring of the generated tokens, the
eps = 0 symmetry, the dense brute force, and the estimator on the generation objective."""
import dataclasses

import numpy as np
import torch

from oracle import model as om
from oracle import zo as ozo
from zeroth_order_fine_b200 import workload as wl


def _run(fp8=False, shape=None):
    w = wl.WORKLOADS["tiny"]
    sh = shape or w.shape
    weights = om.init_weights(sh, w.weight_seed)
    return w, ozo.OracleRun(weights, w.run_seed, w.nu, w.rank, range(sh.n_layers), w.matrices,
                            w.scale_mode, fp8=fp8)


def test_generated_logprobs_equal_teacher_forced_scoring():
    w, run = _run()
    batch = wl.make_batch(w, batch=3)
    run.plan(0, w.eps)
    Lp, Lm, toks, lps = run.generate(batch.prompts, 5)
    B = len(batch.prompts)
    rows = [np.concatenate([p, toks[r]]) for r, p in enumerate(list(batch.prompts) * 2)]
    tf = run.score(rows[:B], [5] * B)              # + rows, teacher forced
    # the - rows carry their own tokens: score them under the - candidate
    hs = om.hidden_states(run.w, rows, [1.0] * B + [-1.0] * B, run.eps, run.perturbation())
    ref = om.token_logprobs(run.w, hs, rows, [5] * (2 * B))
    for r in range(2 * B):
        assert np.allclose(ref[r].numpy(), lps[r], atol=1e-11, rtol=0)
    assert np.allclose(tf.L_plus, Lp, atol=1e-11)
    # every token is the argmax of its own prefix's logits
    logits = om.span_logits(run.w, hs, rows, [5] * (2 * B))
    for r in range(2 * B):
        assert np.array_equal(torch.argmax(logits[r], dim=-1).numpy(), toks[r])
    assert np.allclose(Lp, -lps[:B].mean(1)) and np.allclose(Lm, -lps[B:].mean(1))


def test_eps_zero_generates_identical_candidates():
    w, run = _run()
    batch = wl.make_batch(w, batch=2)
    run.plan(0, 0.0)
    Lp, Lm, toks, _ = run.generate(batch.prompts, 4)
    assert np.array_equal(toks[:2], toks[2:]) and np.array_equal(Lp, Lm)


def test_generation_factored_equals_dense_and_feeds_the_estimator():
    w, run = _run()
    batch = wl.make_batch(w, batch=2)
    run.plan(0, w.eps)
    a = run.generate(batch.prompts, 3)
    b = run.generate(batch.prompts, 3, dense=True)
    assert np.array_equal(a[2], b[2])
    assert np.allclose(a[0], b[0], atol=1e-10) and np.allclose(a[1], b[1], atol=1e-10)
    run.generate(batch.prompts, 3)
    c = run.step(w.lr)
    assert np.isclose(c, ozo.estimate_c(a[0], a[1], w.eps))
    assert run.t == 1
