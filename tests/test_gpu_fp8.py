"""The E4M3 option (zo_options.fp8) through the C ABI: the row quantiser bit for bit
against the oracle's, the E4M3 tensor-core GEMM against its dequantised float64
product, and the probe step against the oracle's fp8 mode with the invariants the
pages fix (eps = 0, co-batched rows, the whole-step graph)."""
import dataclasses

import numpy as np
import pytest
import torch

from zeroth_order_fine_b200 import workload as wl
from gpu_util import dev_fg_tokens, dev_tokens, gpu_handle, needs_gpu

pytestmark = [pytest.mark.gpu, needs_gpu]

TINY_BF16 = dataclasses.replace(wl.WORKLOADS["tiny"],
                                shape=wl.shrink_shape(wl.TINY, dtype=wl.DTYPE_BF16))
Q3_SMALL_BF16 = wl.ModelShape("qwen3-small", wl.ARCH_QWEN3, 2, 256, 4, 2, 128, 512, 1000, 4096,
                              1e-6, 1e6, wl.DTYPE_BF16, False)
QWEN_SMALL = wl.Workload("qwen3-small", Q3_SMALL_BF16, 6, 20, 90, 1, 4, True, 8, wl.ALL7,
                         wl.SCALE_MEZO, 1e-3, 1e-4, 3, fg_rows=0, data_seed=11)


def _codes_to_values(q: torch.Tensor) -> np.ndarray:
    from oracle import fp8
    return fp8.e4m3_table()[q.cpu().numpy().astype(np.int64)]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("rows,cols", [(7, 1000), (33, 5121), (5, 3)])
def test_quantizer_bit_exact_with_oracle(dtype, rows, cols):
    from oracle import fp8
    from zeroth_order_fine_b200 import zo
    g = torch.Generator().manual_seed(rows * cols)
    x = torch.randn(rows, cols, generator=g) * torch.logspace(-6, 3, rows)[:, None]
    x[1] = 0.0
    x = x.to(dtype)
    q, sc = zo.zo_op_quantize_rows_e4m3(x.cuda())
    codes, scale = fp8.quantize_rows(x.float().numpy())
    assert np.array_equal(_codes_to_values(q), codes.astype(np.float64))
    assert np.array_equal(sc.cpu().numpy().view(np.uint32), scale.view(np.uint32))


@pytest.mark.parametrize("M,N,K,act", [(300, 640, 512, 0), (257, 320, 208, 1), (1000, 384, 1024, 0),
                                       (1, 256, 16, 1)])
def test_fp8_linear_matches_dequantized_product(M, N, K, act):
    from zeroth_order_fine_b200 import zo
    g = torch.Generator().manual_seed(M + N + K)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16).cuda()
    W = (torch.randn(N, K, generator=g) * 0.05).to(torch.bfloat16).cuda()
    b = torch.randn(N, generator=g).cuda()
    xq, sx = zo.zo_op_quantize_rows_e4m3(x)
    wq, sw = zo.zo_op_quantize_rows_e4m3(W)
    y = zo.zo_op_linear_fp8(xq, sx, wq, sw, b, act=act)
    assert zo.zo_op_error_word() == 0
    xd = torch.from_numpy(_codes_to_values(xq)) * sx.double().cpu()[:, None]
    wd = torch.from_numpy(_codes_to_values(wq)) * sw.double().cpu()[:, None]
    ref = xd @ wd.T + b.double().cpu()
    if act:
        ref = torch.relu(ref)
    err = (y.double().cpu() - ref).abs()
    # exact E4M3 products summed in fp32, two scale multiplies, one bf16 rounding
    bound = ref.abs() * 2.0 ** -8 + 1e-5 * (xd.abs() @ wd.abs().T + b.abs().double().cpu())
    assert torch.all(err <= bound), (err - bound).max()


def test_fp8_option_refused_where_it_does_not_apply():
    from zeroth_order_fine_b200 import zo
    w = wl.WORKLOADS["tiny"]                        # fp32 model
    with pytest.raises(zo.ZoError) as e:
        gpu_handle(w, fp8=1)
    assert e.value.code == zo.ZO_ERR_UNSUPPORTED


def test_tiny_fp8_same_state_parity():
    from test_gpu_step import _bf16_same_state_parity
    w = TINY_BF16
    _bf16_same_state_parity(w, w.shape, wl.make_batch(w), pre_steps=3, fp8=True)


def test_qwen3_fp8_same_state_parity():
    from test_gpu_step import _bf16_same_state_parity
    w = QWEN_SMALL
    _bf16_same_state_parity(w, w.shape, wl.make_batch(w, fg_rows=0), pre_steps=4, fp8=True)


def test_fp8_eps_zero_and_quantisation_applied():
    w = TINY_BF16
    batch = wl.make_batch(w)
    toks = dev_tokens(batch)
    _, h8 = gpu_handle(w, fp8=1)
    _, hb = gpu_handle(w)
    out = []
    for h in (h8, hb):
        h.zo_probe_plan(0, 0.0)
        Lp, Lm, _ = h.zo_score(toks, batch.seq_lens, batch.target_lens)
        assert torch.equal(Lp, Lm)
        out.append(Lp.cpu().numpy())
    assert not np.array_equal(out[0], out[1])           # the E4M3 path ran
    assert np.max(np.abs(out[0] - out[1])) < 5e-2


def test_fp8_cobatched_foreground_bit_identical():
    w = dataclasses.replace(QWEN_SMALL, fg_rows=4)
    batch = wl.make_batch(w, fg_rows=5)
    _, h = gpu_handle(w, fg=5, fp8=1)
    toks, ftoks = dev_tokens(batch), dev_fg_tokens(batch)
    for t in range(4):
        h.zo_probe_plan(t, w.eps)
        _, _, _, flp = h.zo_score_cobatch(toks, batch.seq_lens, batch.target_lens, ftoks,
                                          batch.fg_seq_lens, batch.fg_target_lens)
        alone = h.zo_score_foreground(ftoks, batch.fg_seq_lens, batch.fg_target_lens)
        assert torch.equal(flp, alone), t
        h.zo_score(toks, batch.seq_lens, batch.target_lens)
        h.zo_step(w.lr)
    assert h.zo_stats()["cuda_core_gemm_launches"] == 0


def test_fp8_step_graph_bit_identical_to_eager():
    w = QWEN_SMALL
    batch = wl.make_batch(w, fg_rows=0)
    toks = dev_tokens(batch)
    _, he = gpu_handle(w, nu=3, fp8=1)
    _, hg = gpu_handle(w, nu=3, fp8=1)
    for t in range(5):
        he.zo_probe_plan(t, w.eps)
        Lp, Lm, _ = he.zo_score(toks, batch.seq_lens, batch.target_lens)
        he.zo_step(w.lr, want_c=False)
        Gp, Gm = hg.zo_step_graph(toks, batch.seq_lens, batch.target_lens, w.eps, w.lr)
        assert torch.equal(Lp, Gp) and torch.equal(Lm, Gm), t
    assert he.zo_save_state() == hg.zo_save_state()
