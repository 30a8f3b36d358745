"""Kernel-level parity through the C ABI: the tensor-core and CUDA-core GEMMs,
the lm_head log-sum-exp and the packed attention, against float64 CPU
references computed from the same inputs (ragged shapes, tails, tiny cases)."""
import numpy as np
import pytest
import torch

from gpu_util import needs_gpu

pytestmark = [pytest.mark.gpu, needs_gpu]


def _rand(shape, dtype, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(dtype)


def _bf16_ulp(x):
    return torch.clamp(torch.abs(x), min=1e-30) * 2.0 ** -7


@pytest.mark.parametrize("M,N,K", [(1, 256, 64), (127, 320, 200), (129, 512, 512),
                                   (300, 1000, 1024), (1000, 768, 5120), (257, 256, 8),
                                   (33, 40, 72), (130, 64, 320), (300, 104, 1000),
                                   (65, 128, 2048)])
@pytest.mark.parametrize("impl", [1, 2])
def test_linear_store_bf16(M, N, K, impl):
    from zeroth_order_fine_b200 import zo
    x = _rand((M, K), torch.bfloat16, 1)
    W = _rand((N, K), torch.bfloat16, 2, 0.05)
    b = _rand((N,), torch.float32, 3)
    ref = x.double() @ W.double().T + b.double()
    for act in (0, 1):
        y = zo.zo_op_linear(x.cuda(), W.cuda(), b.cuda(), act=act, impl=impl)
        assert zo.zo_op_error_word() == 0
        r = torch.relu(ref) if act else ref
        err = (y.double().cpu() - r).abs()
        # fp32 accumulation, then one bf16 rounding of the output
        assert torch.all(err <= _bf16_ulp(r) + 1e-4 * (K ** 0.5) * 0.05), err.max()


@pytest.mark.parametrize("M,N,K", [(5, 256, 64), (200, 640, 520), (513, 5120, 2048),
                                   (200, 96, 520), (77, 64, 136)])
@pytest.mark.parametrize("impl", [1, 2])
def test_linear_residual_accumulate(M, N, K, impl):
    from zeroth_order_fine_b200 import zo
    x = _rand((M, K), torch.bfloat16, 4)
    W = _rand((N, K), torch.bfloat16, 5, 0.05)
    b = _rand((N,), torch.float32, 6)
    y0 = _rand((M, N), torch.float32, 7)
    y = y0.cuda().clone()
    zo.zo_op_linear(x.cuda(), W.cuda(), b.cuda(), out=y, accumulate=True, impl=impl)
    ref = y0.double() + x.double() @ W.double().T + b.double()
    assert zo.zo_op_error_word() == 0
    assert torch.max((y.double().cpu() - ref).abs()) < 2e-4


# decode-step GEMMs: swapped single-SM tiles for M <= 128 (N tile 32 / 64 / 128, ragged
# weight-row tiles, K not a multiple of the 64-wide block, 1..16 K splits), the SM-pair split
# for M > 128; the slices are summed in split order
@pytest.mark.parametrize("M,N,K", [(1, 256, 512), (17, 392, 1000), (32, 5120, 5120),
                                   (40, 1280, 2048), (64, 640, 776), (100, 4096, 4096),
                                   (128, 15360, 5120), (32, 5120, 20480), (160, 2048, 1024),
                                   (0, 256, 64)])
def test_linear_decode(M, N, K):
    from zeroth_order_fine_b200 import zo
    x = _rand((M, K), torch.bfloat16, 31)
    W = _rand((N, K), torch.bfloat16, 32, 0.05)
    b = _rand((N,), torch.float32, 33)
    ref = x.double() @ W.double().T + b.double()
    for act in (0, 1):
        y = zo.zo_op_linear_decode(x.cuda(), W.cuda(), b.cuda(), act=act)
        assert zo.zo_op_error_word() == 0
        r = torch.relu(ref) if act else ref
        err = (y.double().cpu() - r).abs()
        assert torch.all(err <= _bf16_ulp(r) + 1e-4 * (K ** 0.5) * 0.05), err.max()
    y0 = _rand((M, N), torch.float32, 34)
    y = y0.cuda().clone()
    zo.zo_op_linear_decode(x.cuda(), W.cuda(), b.cuda(), out=y, accumulate=True)
    assert zo.zo_op_error_word() == 0
    if M:
        # fp32 accumulation over K products and the split slices: rounding grows like sqrt(K)
        # ulps of the running sum
        r = y0.double() + ref
        err = (y.double().cpu() - r).abs()
        assert torch.all(err <= 1e-6 * (K ** 0.5) * torch.clamp(r.abs(), min=1.0)), err.max()


def test_linear_decode_is_deterministic_and_checks_its_workspace():
    from zeroth_order_fine_b200 import zo
    x = _rand((32, 5120), torch.bfloat16, 35).cuda()
    W = _rand((5120, 5120), torch.bfloat16, 36, 0.05).cuda()
    y1 = zo.zo_op_linear_decode(x, W)
    y2 = zo.zo_op_linear_decode(x, W)
    assert torch.equal(y1, y2)
    # a single-slice workspace forces one split: the same values up to the fp32 summation
    # order, so both sit within the bound against the float64 product
    y3 = zo.zo_op_linear_decode(x, W, ws=torch.empty(32 * 5120, device="cuda"))
    ref = x.double().cpu() @ W.double().cpu().T
    for y in (y1, y3):
        err = (y.double().cpu() - ref).abs()
        assert torch.all(err <= _bf16_ulp(ref) + 1e-4 * (5120 ** 0.5) * 0.05), err.max()
    with pytest.raises(RuntimeError):
        zo.zo_op_linear_decode(x, W, ws=torch.empty(100, device="cuda"))


def test_tensor_cores_match_cuda_cores_closely():
    from zeroth_order_fine_b200 import zo
    x = _rand((700, 2048), torch.bfloat16, 8)
    W = _rand((1536, 2048), torch.bfloat16, 9, 0.05)
    y0 = torch.zeros(700, 1536, device="cuda")
    y1 = torch.zeros(700, 1536, device="cuda")
    zo.zo_op_linear(x.cuda(), W.cuda(), out=y0, accumulate=True, impl=2)
    zo.zo_op_linear(x.cuda(), W.cuda(), out=y1, accumulate=True, impl=1)
    assert torch.max((y0 - y1).abs()).item() < 1e-3


def test_linear_fp32_cuda_cores():
    from zeroth_order_fine_b200 import zo
    x = _rand((77, 130), torch.float32, 10)
    W = _rand((90, 130), torch.float32, 11)
    y = zo.zo_op_linear(x.cuda(), W.cuda(), impl=1)
    ref = x.double() @ W.double().T
    assert torch.max((y.double().cpu() - ref).abs()) < 1e-4


def test_tensor_core_rows_are_position_independent():
    """A row's output bits do not depend on where it sits in the batch."""
    from zeroth_order_fine_b200 import zo
    x = _rand((300, 1024), torch.bfloat16, 12).cuda()
    W = _rand((512, 1024), torch.bfloat16, 13, 0.05).cuda()
    y = zo.zo_op_linear(x, W, impl=2)
    perm = torch.randperm(300, generator=torch.Generator().manual_seed(0)).cuda()
    yp = zo.zo_op_linear(x[perm].contiguous(), W, impl=2)
    assert torch.equal(yp, y[perm])
    y1 = zo.zo_op_linear(x[17:18].contiguous(), W, impl=2)
    assert torch.equal(y1, y[17:18])


@pytest.mark.parametrize("S,V,d,dtype", [(1, 1000, 128, torch.float32),
                                         (40, 50272, 256, torch.bfloat16),
                                         (130, 4099, 512, torch.bfloat16),
                                         (128, 50272, 5120, torch.bfloat16)])
@pytest.mark.parametrize("impl", [1, 2])
def test_lm_head_logprob(S, V, d, dtype, impl):
    from zeroth_order_fine_b200 import zo
    if dtype == torch.float32 and impl == 2:
        pytest.skip("tensor cores take bf16")
    h = _rand((S, d), dtype, 14)
    E = _rand((V, d), dtype, 15, 0.02)
    tg = torch.randint(0, V, (S,), generator=torch.Generator().manual_seed(1), dtype=torch.int32)
    tg[0] = V - 1
    got = zo.zo_op_lm_head_logprob(h.cuda(), E.cuda(), tg.cuda(), impl=impl)
    logits = h.double() @ E.double().T
    ref = logits[torch.arange(S), tg.long()] - torch.logsumexp(logits, dim=-1)
    assert zo.zo_op_error_word() == 0
    assert torch.max((got.double().cpu() - ref).abs()) < 2e-4


@pytest.mark.parametrize("lens,H,Hkv,hd,dtype,impl", [
    ([1, 5, 64, 65, 130], 4, 4, 128, torch.float32, 1),
    ([16, 128, 77, 3], 40, 40, 128, torch.bfloat16, 1),
    ([16, 128, 77, 3], 40, 40, 128, torch.bfloat16, 2),
    ([1, 129, 300, 256, 512], 4, 2, 128, torch.bfloat16, 2),
    # several items per persistent CTA, 1-5 key chunks each, in mixed order
    ([int(x) for x in np.random.default_rng(5).integers(1, 600, 40)], 8, 2, 128,
     torch.bfloat16, 2),
    ([200, 1, 64], 8, 2, 64, torch.float32, 1),
    # head_dim 64 on the tensor cores (OPT-1.3B's heads): one 64-column atom per tile
    ([1, 5, 64, 65, 130, 300], 32, 32, 64, torch.bfloat16, 2),
    ([int(x) for x in np.random.default_rng(6).integers(1, 400, 30)], 8, 2, 64,
     torch.bfloat16, 2),
    # rows at OPT's longest position (2048 tokens: 16 query tiles of up to 16 key chunks)
    ([2048, 1, 1500], 4, 2, 128, torch.bfloat16, 2),
    ([2048, 700], 4, 4, 64, torch.bfloat16, 2)])
def test_attention_matches_oracle(lens, H, Hkv, hd, dtype, impl):
    from oracle import model as om
    from zeroth_order_fine_b200 import zo
    T = sum(lens)
    qkv = _rand((T, (H + 2 * Hkv) * hd), dtype, 16)
    out = zo.zo_op_attention(qkv.cuda(), lens, H, Hkv, hd, impl=impl).double().cpu()
    assert zo.zo_op_error_word() == 0
    q = qkv.double()[:, :H * hd].reshape(T, H, hd)
    k = qkv.double()[:, H * hd:(H + Hkv) * hd].reshape(T, Hkv, hd)
    v = qkv.double()[:, (H + Hkv) * hd:].reshape(T, Hkv, hd)
    off = 0
    tol = 1e-4 if dtype == torch.float32 else 2e-2
    for L in lens:
        ref = om.causal_attention(q[off:off + L], k[off:off + L], v[off:off + L], H // Hkv)
        assert torch.max((out[off:off + L] - ref).abs()) < tol
        off += L


@pytest.mark.parametrize("out_offset", [0, 8])
def test_attention_many_items_per_cta_and_output_alignment(out_offset):
    """220 short rows x 32 heads = 7040 (query tile, head) items, more than 40 per persistent
    CTA on 148 SMs: each role then decodes its items from the tile list instead of the
    shared-memory item table.  With out_offset = 8 the output starts 16 bytes past a 32-byte
    boundary, so its rows are written with 16-byte stores instead of 32-byte ones."""
    from oracle import model as om
    from zeroth_order_fine_b200 import zo
    lens = [int(x) for x in np.random.default_rng(7).integers(1, 25, 220)]
    H, Hkv, hd = 32, 8, 64
    T = sum(lens)
    qkv = _rand((T, (H + 2 * Hkv) * hd), torch.bfloat16, 17)
    buf = torch.empty(out_offset + T * H * hd, dtype=torch.bfloat16, device="cuda")
    out = buf[out_offset:].view(T, H * hd)
    zo.zo_op_attention(qkv.cuda(), lens, H, Hkv, hd, impl=2, out=out)
    assert zo.zo_op_error_word() == 0
    got = out.double().cpu()
    q = qkv.double()[:, :H * hd].reshape(T, H, hd)
    k = qkv.double()[:, H * hd:(H + Hkv) * hd].reshape(T, Hkv, hd)
    v = qkv.double()[:, (H + Hkv) * hd:].reshape(T, Hkv, hd)
    off = 0
    for L in lens:
        ref = om.causal_attention(q[off:off + L], k[off:off + L], v[off:off + L], H // Hkv)
        assert torch.max((got[off:off + L] - ref).abs()) < 2e-2
        off += L
