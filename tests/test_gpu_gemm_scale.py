"""The tensor-core GEMM at the sizes of the OPT-13B batch-64 probe step, through the C ABI.

The batched forward of both candidates is the step's dominant cost ("Zeroth-Order
Fine-Tuning Was an Inference Workload All Along", section "Why ZO Fine-Tuning Is Really
Scoring"), and at 9196 packed token rows the SM-pair kernel runs a schedule that small
shapes never reach: 36 row blocks of 256 walked in raster groups of 12, 20-80 column blocks,
so every SM pair computes many tiles in turn, alternating its two TMEM accumulators and
wrapping its 6-stage operand ring across tiles.  Each case draws seeded inputs, runs one
fused group of the step (base GEMM + the extension K blocks that carry the perturbation
and the bank, then the group's epilogue) and compares against a float64 product of the
same operands on a sample of rows: six rows of every 128-row half of every row block, plus
the ragged last block whole, with every column -- so every tile of every pair is checked.
"""
import numpy as np
import pytest
import torch

from gpu_util import needs_gpu

pytestmark = [pytest.mark.gpu, needs_gpu]

M_STEP = 9196                 # packed rows of the seeded OPT-13B batch-64 step


def _bf16_ulp(x):
    return torch.clamp(torch.abs(x), min=1e-30) * 2.0 ** -7


def _sample_rows(M):
    rows = [b + o for b in range(0, M, 128) for o in (0, 1, 45, 64, 126, 127) if b + o < M]
    rows += list(range(max(0, M - 150), M))
    return torch.tensor(sorted(set(rows)), dtype=torch.long)


def _operands(M, N, K, K2, seed, bias=True):
    """x ~ N(0,1), W ~ N(0, 0.05^2) (bf16), the extension as the step builds it: x2 the
    shrink output (a few units), W2 the expand factors; bias N(0,1) (fp32)."""
    g = torch.Generator(device="cuda").manual_seed(seed)
    x = torch.randn(M, K, device="cuda", generator=g).to(torch.bfloat16)
    W = (torch.randn(N, K, device="cuda", generator=g) * 0.05).to(torch.bfloat16)
    x2 = W2 = None
    if K2:
        x2 = (torch.randn(M, K2, device="cuda", generator=g) * 0.5).to(torch.bfloat16)
        W2 = (torch.randn(N, K2, device="cuda", generator=g) * 0.5).to(torch.bfloat16)
    b = torch.randn(N, device="cuda", generator=g) if bias else None
    return x, W, x2, W2, b


def _ref(x, W, x2, W2, b, rows):
    """float64 x W^T + x2 W2^T + b on the sampled rows."""
    xs = x[rows.cuda()].double().cpu()
    acc = xs @ W.double().cpu().T
    if x2 is not None:
        acc += x2[rows.cuda()].double().cpu() @ W2.double().cpu().T
    if b is not None:
        acc += b.double().cpu()
    return acc


def _acc_tol(K, K2):
    # fp32 accumulation of K products of size ~0.05 and K2 of size ~0.25
    return 1e-4 * (K ** 0.5) * 0.05 + 1e-4 * (max(K2, 1) ** 0.5) * 0.25


@pytest.mark.parametrize("N,K,K2,act", [(15360, 5120, 16, 0),     # q|k|v with the bank extension
                                        (20480, 5120, 0, 1)])      # fc1 + ReLU
def test_pair_gemm_store_at_step_size(N, K, K2, act):
    from zeroth_order_fine_b200 import zo
    M = M_STEP
    x, W, x2, W2, b = _operands(M, N, K, K2, seed=N + K)
    y = zo.zo_op_linear_ext(x, W, b, x2, W2, epi=zo.EPI_RELU if act else zo.EPI_STORE)
    assert zo.zo_op_error_word() == 0
    rows = _sample_rows(M)
    ref = _ref(x, W, x2, W2, b, rows)
    if act:
        ref = torch.relu(ref)
    got = y[rows.cuda()].double().cpu()
    err = (got - ref).abs()
    bad = err > _bf16_ulp(ref) + _acc_tol(K, K2)
    assert not bool(bad.any()), (int(bad.sum()), float(err.max()))
    # the persistent schedule does not leak into a row's bits: the same rows computed in a
    # small call (one tile per pair) are bit-identical
    sub = slice(5000, 5300)
    y_sub = zo.zo_op_linear_ext(x[sub].contiguous(), W, b,
                                None if x2 is None else x2[sub].contiguous(), W2,
                                epi=zo.EPI_RELU if act else zo.EPI_STORE)
    assert torch.equal(y_sub, y[sub])


@pytest.mark.parametrize("N,K,K2", [(5120, 5120, 8),          # o projection + bank, residual add
                                    (5120, 20480, 0)])        # fc2, K = 20480
def test_pair_gemm_residual_at_step_size(N, K, K2):
    from zeroth_order_fine_b200 import zo
    M = M_STEP
    x, W, x2, W2, b = _operands(M, N, K, K2, seed=3 * N + K)
    g = torch.Generator(device="cuda").manual_seed(99)
    y0 = torch.randn(M, N, device="cuda", generator=g)
    y = y0.clone()
    zo.zo_op_linear_ext(x, W, b, x2, W2, epi=zo.EPI_RESID, out=y)
    assert zo.zo_op_error_word() == 0
    rows = _sample_rows(M)
    ref = y0[rows.cuda()].double().cpu() + _ref(x, W, x2, W2, b, rows)
    got = y[rows.cuda()].double().cpu()
    err = (got - ref).abs()
    tol = 1e-6 * (K ** 0.5) * torch.clamp(ref.abs(), min=1.0) * 10
    bad = err > tol
    assert not bool(bad.any()), (int(bad.sum()), float(err.max()))


def test_pair_gemm_swiglu_at_qwen3_8b_width():
    """Qwen3-8B's FFN input: [gate|up] interleaved in 128-row blocks (N = 2 x 12288), the
    MeZO-style r = 64 bank extension, silu(gate) * up written by the epilogue."""
    from zeroth_order_fine_b200 import zo
    M, F, K, K2 = M_STEP, 12288, 4096, 256
    N = 2 * F
    x, W, x2, W2, _ = _operands(M, N, K, K2, seed=77, bias=False)
    y = zo.zo_op_linear_ext(x, W, None, x2, W2, epi=zo.EPI_SWIGLU)
    assert zo.zo_op_error_word() == 0
    assert y.shape == (M, F)
    rows = _sample_rows(M)
    acc = _ref(x, W, x2, W2, None, rows)                      # [rows x N], interleaved
    blk = acc.reshape(len(rows), F // 128, 2, 128)
    gate = blk[:, :, 0, :].reshape(len(rows), F)
    up = blk[:, :, 1, :].reshape(len(rows), F)
    silu = gate / (1.0 + torch.exp(-gate))
    ref = silu * up
    got = y[rows.cuda()].double().cpu()
    d = _acc_tol(K, K2)
    # first-order error of silu(g) u from accumulator errors d in g and u (|silu'| <= 1.1)
    tol = _bf16_ulp(ref) + d * (1.1 * up.abs() + silu.abs()) + 1e-6
    err = (got - ref).abs()
    bad = err > tol
    assert not bool(bad.any()), (int(bad.sum()), float(err.max()))


def test_pair_gemm_qk_norm_rope_at_qwen3_8b_width():
    """Qwen3-8B's q|k|v (32 query heads, 8 key/value heads, head_dim 128) with the r = 64
    extension; the fused epilogue's per-head RMSNorm and rotary positions against the same
    GEMM stored plainly, then normalised and rotated in float64."""
    from zeroth_order_fine_b200 import zo
    M, K, K2 = M_STEP, 4096, 192
    Hq, Hkv, hd = 32, 8, 128
    N = (Hq + 2 * Hkv) * hd
    x, W, x2, W2, _ = _operands(M, N, K, K2, seed=55, bias=False)
    rng = np.random.default_rng(4)
    lens, tot = [], 0
    while tot < M:                                             # ragged rows of 64..512 tokens
        L = int(min(rng.integers(64, 513), M - tot))
        lens.append(L)
        tot += L
    pos = torch.from_numpy(np.concatenate([np.arange(L) for L in lens]).astype(np.int32))
    g = torch.Generator().manual_seed(6)
    qn = 1.0 + 0.02 * torch.randn(hd, generator=g)
    kn = 1.0 + 0.02 * torch.randn(hd, generator=g)
    theta, max_pos = 1e6, 4096
    cos_t, sin_t = zo.zo_op_rope_table(max_pos, hd, theta)
    qk = {"tok_pos": pos.cuda(), "q_norm": qn.cuda(), "k_norm": kn.cuda(), "rope_cos": cos_t,
          "rope_sin": sin_t, "eps": 1e-6, "n_q_heads": Hq, "n_kv_heads": Hkv}
    y = zo.zo_op_linear_ext(x, W, None, x2, W2, epi=zo.EPI_QK_NORM_ROPE, qk=qk)
    plain = zo.zo_op_linear_ext(x, W, None, x2, W2, epi=zo.EPI_STORE)
    assert zo.zo_op_error_word() == 0
    # the plain store against float64 on the sampled rows
    rows = _sample_rows(M)
    ref = _ref(x, W, x2, W2, None, rows)
    err = (plain[rows.cuda()].double().cpu() - ref).abs()
    assert not bool((err > _bf16_ulp(ref) + _acc_tol(K, K2)).any()), float(err.max())
    # value heads pass through as stored
    assert torch.equal(y[:, (Hq + Hkv) * hd:], plain[:, (Hq + Hkv) * hd:])
    # q and k heads: RMSNorm of the stored bf16 head, then the rotate-half rotation
    a = plain[:, :(Hq + Hkv) * hd].double().cpu().reshape(M, Hq + Hkv, hd)
    w = torch.cat([qn.double().expand(Hq, hd), kn.double().expand(Hkv, hd)]).unsqueeze(0)
    an = a / torch.sqrt((a * a).mean(-1, keepdim=True) + 1e-6) * w
    i = torch.arange(hd // 2, dtype=torch.float64)
    ang = pos.double().unsqueeze(1) * theta ** (-2.0 * i / hd)          # [M x 64]
    c, s = torch.cos(ang).unsqueeze(1), torch.sin(ang).unsqueeze(1)
    lo, hi = an[..., :hd // 2], an[..., hd // 2:]
    ref_qk = torch.cat([lo * c - hi * s, hi * c + lo * s], dim=-1)
    got = y[:, :(Hq + Hkv) * hd].double().cpu().reshape(M, Hq + Hkv, hd)
    tol = _bf16_ulp(ref_qk) + 1e-5 * (torch.cat([lo.abs() + hi.abs()] * 2, dim=-1)) + 1e-6
    err = (got - ref_qk).abs()
    bad = err > tol
    assert not bool(bad.any()), (int(bad.sum()), float(err.max()))


def test_linear_ext_checks_its_arguments():
    from zeroth_order_fine_b200 import zo
    x = torch.zeros(300, 256, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(512, 256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(zo.ZoError) as e:                       # SwiGLU needs N % 256 == 0
        zo.zo_op_linear_ext(x, W[:384].contiguous(), epi=zo.EPI_SWIGLU)
    assert e.value.code == zo.ZO_ERR_UNSUPPORTED
    with pytest.raises(zo.ZoError) as e:                       # unknown epilogue
        zo.zo_op_linear_ext(x, W, epi=3)
    assert e.value.code == zo.ZO_ERR_ARG
    with pytest.raises(zo.ZoError) as e:                       # the q/k norm needs its tables
        zo.zo_op_linear_ext(x, W, epi=zo.EPI_QK_NORM_ROPE,
                            out=torch.empty(300, 512, dtype=torch.bfloat16, device="cuda"))
    assert e.value.code == zo.ZO_ERR_ARG
