"""Generation queries through the C ABI (zo_generate): greedy decoding of both candidates
with the KV cache, checked against the oracle teacher-forced on the GPU's own tokens (each
token must be a largest logit there, within the mode's tolerance, and its log-probability
must match), the eps = 0 symmetry, the GPU's own prefill scoring of the generated rows, and
the update that follows."""
import dataclasses

import numpy as np
import pytest
import torch

from zeroth_order_fine_b200 import workload as wl
from gpu_util import dev_tokens, gpu_handle, needs_gpu, oracle_run

pytestmark = [pytest.mark.gpu, needs_gpu]

TINY = wl.WORKLOADS["tiny"]
TINY_BF16 = dataclasses.replace(TINY, shape=wl.shrink_shape(wl.TINY, dtype=wl.DTYPE_BF16))
Q3_SMALL_BF16 = wl.ModelShape("qwen3-small", wl.ARCH_QWEN3, 2, 256, 4, 2, 128, 512, 1000, 4096,
                              1e-6, 1e6, wl.DTYPE_BF16, False)
QWEN_SMALL = wl.Workload("qwen3-small", Q3_SMALL_BF16, 6, 20, 90, 1, 4, True, 8, wl.ALL7,
                         wl.SCALE_MEZO, 1e-3, 1e-4, 3, fg_rows=0, data_seed=11)
G = 6


def _check_against_oracle(w, fp8, logit_tol, lp_tol, L_tol, impl=0):
    from oracle import model as om
    batch = wl.make_batch(w, fg_rows=0)
    B = len(batch.prompts)
    _, h = gpu_handle(w, max_new=G, fp8=int(fp8), impl=impl)
    toks = dev_tokens(batch)
    h.zo_probe_plan(0, w.eps)
    Lp, Lm, gt, gl = h.zo_generate(toks, batch.seq_lens, G)
    gt, gl = gt.cpu().numpy(), gl.cpu().numpy()
    orc = oracle_run(w, fp8=fp8)
    orc.plan(0, w.eps)
    rows = [np.concatenate([p, gt[r]]).astype(np.int64)
            for r, p in enumerate(list(batch.prompts) * 2)]
    hs = om.hidden_states(orc.w, rows, [1.0] * B + [-1.0] * B, orc.eps, orc.perturbation(),
                          fp8=fp8)
    logits = om.span_logits(orc.w, hs, rows, [G] * (2 * B))
    ref_lp = om.token_logprobs(orc.w, hs, rows, [G] * (2 * B))
    for r in range(2 * B):
        lg = logits[r].numpy()
        chosen = lg[np.arange(G), gt[r]]
        assert np.all(chosen >= lg.max(axis=1) - logit_tol), (r, lg.max(axis=1) - chosen)
        assert np.max(np.abs(gl[r] - ref_lp[r].numpy())) <= lp_tol, r
    ref_L = np.array([-x.numpy().mean() for x in ref_lp])
    assert np.max(np.abs(Lp.cpu().numpy() - ref_L[:B])) <= L_tol
    assert np.max(np.abs(Lm.cpu().numpy() - ref_L[B:])) <= L_tol
    c = h.zo_step(w.lr)
    assert np.isfinite(c) and h.zo_stats()["steps"] == 1
    return h, batch, gt


@pytest.mark.parametrize("impl", [0, 1])
def test_tiny_fp32_generation_matches_oracle(impl):
    _check_against_oracle(TINY, False, 1e-4, 1e-4, 1e-4, impl=impl)


def test_opt_width_bf16_generation_matches_oracle():
    """Two full-width OPT-1.3B layers (d = 2048, vocab 50272): the decode GEMMs stream the
    weights for their 8 rows on the swapped single-SM kernel with K split over the SMs."""
    w = wl.WORKLOADS["opt-1.3b-b16"]
    w = dataclasses.replace(w, shape=wl.shrink_shape(w.shape, n_layers=2), batch=4, len_hi=48)
    _check_against_oracle(w, False, 5e-2, 3e-2, 2e-2)


def test_tiny_bf16_generation_matches_oracle():
    _check_against_oracle(TINY_BF16, False, 5e-2, 3e-2, 2e-2)


def test_qwen3_bf16_generation_matches_oracle():
    _check_against_oracle(QWEN_SMALL, False, 5e-2, 3e-2, 2e-2)


Q3_WIDE = wl.ModelShape("qwen3-wide", wl.ARCH_QWEN3, 2, 1024, 8, 2, 128, 2048, 4096, 4096, 1e-6,
                        1e6, wl.DTYPE_BF16, False)
QWEN_WIDE = dataclasses.replace(QWEN_SMALL, shape=Q3_WIDE)


def test_qwen3_wide_bf16_generation_matches_oracle():
    """d = 1024: every decode GEMM splits K, including the q/k-norm + RoPE and SwiGLU forms
    whose epilogues then run in the split reduction."""
    _check_against_oracle(QWEN_WIDE, False, 5e-2, 3e-2, 2e-2)


def test_qwen3_fp8_generation_matches_oracle():
    _check_against_oracle(QWEN_SMALL, True, 5e-2, 3e-2, 2e-2)


def test_opt_width_fp8_generation_matches_oracle():
    """E4M3 q|k|v and fc1 at OPT-1.3B width: the decode steps run them on the swapped
    single-SM kernel with kind::f8f6f4 main blocks and the bf16 bank extension.  The prefill's
    attention (head_dim 64) runs on the tensor cores with P rounded to bf16; where that moves
    a value of the next layer's input across an E4M3 code boundary (codes 12.5 % apart) a
    token's log-prob moves by a few 1e-2, so the log-prob bound is the logit bound, 5e-2."""
    w = wl.WORKLOADS["opt-1.3b-b16"]
    w = dataclasses.replace(w, shape=wl.shrink_shape(w.shape, n_layers=2), batch=4, len_hi=48)
    _check_against_oracle(w, True, 5e-2, 5e-2, 2e-2)


@pytest.mark.parametrize("heads,kv_heads", [(6, 2), (8, 1)], ids=["group3", "group8"])
def test_qwen3_query_group_sizes_generation_matches_oracle(heads, kv_heads):
    """Query-head groups of 3 (the decode attention pads them to 4 with zero queries) and of
    8 per kv head."""
    shape = dataclasses.replace(Q3_SMALL_BF16, name=f"qwen3-group{heads // kv_heads}",
                                n_heads=heads, n_kv_heads=kv_heads)
    _check_against_oracle(dataclasses.replace(QWEN_SMALL, shape=shape), False, 5e-2, 3e-2, 2e-2)


def test_qwen3_long_prompts_generation_matches_oracle():
    """Prompts of 150-300 tokens: with few (row, kv head) pairs the decode attention splits
    each row's keys over several CTAs and merges the partial softmaxes in order."""
    w = dataclasses.replace(QWEN_SMALL, len_lo=150, len_hi=300)
    _check_against_oracle(w, False, 5e-2, 3e-2, 2e-2)


@pytest.mark.parametrize("w", [TINY, TINY_BF16, QWEN_SMALL], ids=["fp32", "bf16", "qwen3-bf16"])
def test_generation_eps_zero_is_symmetric(w):
    batch = wl.make_batch(w, fg_rows=0)
    B = len(batch.prompts)
    _, h = gpu_handle(w, max_new=G)
    h.zo_probe_plan(0, 0.0)
    Lp, Lm, gt, gl = h.zo_generate(dev_tokens(batch), batch.seq_lens, G)
    assert torch.equal(gt[:B], gt[B:]) and torch.equal(gl[:B], gl[B:]) and torch.equal(Lp, Lm)


OPT_WIDTH = dataclasses.replace(wl.WORKLOADS["opt-1.3b-b16"],
                                shape=wl.shrink_shape(wl.WORKLOADS["opt-1.3b-b16"].shape, n_layers=2),
                                batch=4, len_hi=48)


@pytest.mark.parametrize("w,tol", [(TINY, 1e-4), (QWEN_SMALL, 2e-2), (OPT_WIDTH, 2e-2),
                                   (QWEN_WIDE, 2e-2)],
                         ids=["fp32", "qwen3-bf16", "opt-width-bf16", "qwen3-wide-bf16"])
def test_decode_agrees_with_prefill_scoring_of_the_generated_rows(w, tol):
    """The KV-cache decode path and the packed prefill path give the same log-probs for the
    generated tokens (the + rows scored under the + candidate as target spans)."""
    batch = wl.make_batch(w, fg_rows=0)
    B = len(batch.prompts)
    _, h = gpu_handle(w, max_new=G)
    h.zo_probe_plan(0, w.eps)
    _, _, gt, gl = h.zo_generate(dev_tokens(batch), batch.seq_lens, G)
    gt_h = gt.cpu().numpy()
    rows = [np.concatenate([p, gt_h[r]]).astype(np.int32) for r, p in enumerate(batch.prompts)]
    full = wl.Batch(rows, np.full(B, G, dtype=np.int32), [], np.zeros(0, dtype=np.int32))
    _, h2 = gpu_handle(dataclasses.replace(w, len_hi=w.len_hi + G, tgt_hi=G), max_new=0, batch=B)
    h2.zo_probe_plan(0, w.eps)
    _, _, lp = h2.zo_score(dev_tokens(full), full.seq_lens, full.target_lens, want_logprob=True)
    plus = lp[:B * G].cpu().numpy().reshape(B, G)
    assert np.max(np.abs(plus - gl[:B].cpu().numpy())) <= tol


def test_generation_argument_checks():
    from zeroth_order_fine_b200 import zo
    w = TINY
    batch = wl.make_batch(w, fg_rows=0)
    toks = dev_tokens(batch)
    _, h0 = gpu_handle(w)
    h0.zo_probe_plan(0, w.eps)
    with pytest.raises(zo.ZoError) as e:
        h0.zo_generate(toks, batch.seq_lens, 2)
    assert e.value.code == zo.ZO_ERR_UNSUPPORTED
    _, h = gpu_handle(w, max_new=4)
    h.zo_probe_plan(0, w.eps)
    with pytest.raises(zo.ZoError) as e:
        h.zo_generate(toks, batch.seq_lens, 5)
    assert e.value.code == zo.ZO_ERR_ARG
