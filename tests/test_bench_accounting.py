"""The benchmark's algorithmic work accounting (host logic, CPU): the FLOPs and bytes the
roofline fractions divide by.

The counts follow the definition of the step: every decoder linear layer over every token of
both candidates, the lm_head only at the scored positions, causal attention, and the shrink /
expand of the perturbation and the bank; the dense lm_head over all tokens and a dense
W +- eps U V^T are work the method avoids and are not counted."""
import numpy as np
import pytest

import bench
from zeroth_order_fine_b200 import workload as wl


def test_body_parameters_match_the_published_model_sizes():
    # OPT-13B: 40 layers of d = 5120, FFN 20480 -> 12.58 B matrix parameters (the published
    # 12.85 B less the 50272 x 5120 embedding and the learned positions); Qwen3-8B: 6.95 B
    # non-embedding parameters (36 layers, d = 4096, 8 kv heads of 128, FFN 12288)
    opt = wl.WORKLOADS["opt-13b-b64"].shape
    qwen = wl.WORKLOADS["qwen3-8b-cobatch"].shape
    assert abs(opt.body_params() - 12.58e9) / 12.58e9 < 0.002
    assert abs(qwen.body_params() - 6.95e9) / 6.95e9 < 0.002


def _brute_force_flops(w, batch, n_slots):
    """The same work counted GEMM by GEMM and attention pair by pair on a small batch."""
    sh = w.shape
    rows = list(batch.prompts) * 2 + list(batch.fg_prompts)
    spans = list(batch.target_lens) * 2 + list(batch.fg_target_lens)
    fl = 0
    for row, span in zip(rows, spans):
        L = len(row)
        for _ in range(sh.n_layers):
            for m in sh.matrices():
                di, do = sh.matrix_dims(m)
                fl += 2 * L * di * do                          # x W^T for this row
            for m in w.matrices:
                di, do = sh.matrix_dims(m)
                fl += 2 * L * di * w.rank * (1 + n_slots)      # shrink x [U | A_0..]
                fl += 2 * L * do * w.rank * (1 + n_slots)      # expand S [V | V_0..]^T
            pairs = sum(1 for i in range(L) for j in range(L) if j <= i)
            fl += 2 * 2 * pairs * sh.q_dim                     # q.k and p.v per causal pair
        fl += 2 * int(span) * sh.vocab * sh.d_model            # lm_head at the scored positions
    return fl


@pytest.mark.parametrize("name,n_slots", [("tiny", 1), ("tiny", 3), ("qwen3-8b-cobatch", 2)])
def test_step_flops_equal_a_gemm_by_gemm_count(name, n_slots):
    w = wl.WORKLOADS[name]
    batch = wl.make_batch(w, batch=3, fg_rows=min(w.fg_rows, 2), len_hi=24)
    flops, _, T, S = bench.step_work(w, [batch], n_slots)
    assert T == batch.n_tokens_physical
    assert S == int(2 * batch.target_lens.sum() + batch.fg_target_lens.sum())
    ref = _brute_force_flops(w, batch, n_slots)
    assert abs(flops - ref) <= 1e-9 * ref


def test_weights_are_counted_once_per_rank_and_work_scales_with_batches():
    w = wl.WORKLOADS["opt-13b-b64"]
    b1 = wl.make_batch(w, batch=4, fg_rows=0, seed=1)
    b2 = wl.make_batch(w, batch=4, fg_rows=0, seed=2)
    f1, by1, _, _ = bench.step_work(w, [b1], 1)
    f2, by2, _, _ = bench.step_work(w, [b2], 1)
    f12, by12, _, _ = bench.step_work(w, [b1, b2], 1)
    assert abs(f12 - (f1 + f2)) <= 1e-9 * f12
    weights = (w.shape.body_params() + w.shape.vocab * w.shape.d_model) * 2
    assert abs(by12 - (by1 + by2 - weights)) <= 1e-6 * by12


def test_fp8_share_is_the_norm_fed_base_products():
    for name in ("opt-13b-b64", "qwen3-8b-cobatch"):
        w = wl.WORKLOADS[name]
        sh = w.shape
        batch = wl.make_batch(w, batch=2, fg_rows=0, len_hi=32)
        total, _, T, _ = bench.step_work(w, [batch], 1)
        f8 = bench.fp8_flops(w, [batch])
        # q|k|v and the FFN input(s) of every layer, every token
        n_in = 2 if sh.arch == wl.ARCH_QWEN3 else 1
        ref = 2.0 * T * sh.n_layers * sh.d_model * (sh.q_dim + 2 * sh.kv_dim + n_in * sh.d_ffn)
        assert abs(f8 - ref) <= 1e-9 * ref
        assert 0.3 < f8 / total < 0.8


@pytest.mark.parametrize("name,G", [("tiny", 5), ("qwen3-8b-cobatch", 8)])
def test_generation_work_counts_weights_and_cache_per_decode_step(name, G):
    w = wl.WORKLOADS[name]
    sh = w.shape
    batch = wl.make_batch(w, batch=3, fg_rows=0, len_hi=20)
    flops, decode_bytes = bench.generate_work(w, batch, G)
    assert flops == bench.step_work(w, [batch], 1)[0]          # the prefill is a scoring step
    es = 2 if sh.dtype == wl.DTYPE_BF16 else 4
    ref = 0
    for s in range(1, G):              # token s + 1 of each row: the prefill gave the first
        ref += (sh.body_params() + sh.vocab * sh.d_model) * es
        for p in list(batch.prompts) * 2:
            ref += (len(p) + s) * 2 * sh.kv_dim * sh.n_layers * es    # k and v of every key
    assert abs(decode_bytes - ref) <= 1e-9 * ref
