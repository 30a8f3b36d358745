"""The allocation-free lm_head entry point agrees with the workspace one.

zo_op_lm_head_logprob_noalloc serves callers that may not allocate device
memory at call time and have no workspace to lend (their device memory is
owned by another runtime's pool, or they must not touch the allocator once
running).  It keeps its scratch in a fixed array inside the library; this
test calls it through the C ABI twice in a row -- the second call reuses the
array with the first call's values still in it -- and compares each result
with zo_op_lm_head_logprob on the same inputs.  The file sorts last so a
stop-at-first-failure run has executed everything else first; it also
passes alone in a fresh process.
"""
import pytest
import torch

from gpu_util import needs_gpu

pytestmark = [pytest.mark.gpu, needs_gpu]


@pytest.mark.parametrize("impl", [1, 2])
def test_noalloc_matches_workspace_entry_point_twice(impl):
    from zeroth_order_fine_b200 import zo
    gen = torch.Generator().manual_seed(5)
    S, V, d = 96, 50272, 1024
    E = (torch.randn(V, d, generator=gen) * 0.02).to(torch.bfloat16).cuda()
    out = torch.empty(S, dtype=torch.float32, device="cuda")
    for call in range(2):
        h = torch.randn(S, d, generator=gen).to(torch.bfloat16).cuda()
        tg = torch.randint(0, V, (S,), generator=gen, dtype=torch.int32).cuda()
        ref = zo.zo_op_lm_head_logprob(h, E, tg, impl=impl)
        got = zo.zo_op_lm_head_logprob_noalloc(h, E, tg, out, impl=impl)
        assert zo.zo_op_error_word() == 0
        # the same kernels in the same order on the same inputs: the same bits
        assert torch.equal(got, ref), (call, torch.max(torch.abs(got - ref)).item())


@pytest.mark.parametrize("impl", [1, 2])
def test_noalloc_out_of_range_targets_read_nan_not_the_last_call(impl):
    """The array keeps the previous call's values: a row whose target lies outside
    [0, vocab) must come out NaN, not the target logit a previous call left behind -- also
    for target == vocab when vocab is not a multiple of the 32-column epilogue chunk."""
    from zeroth_order_fine_b200 import zo
    gen = torch.Generator().manual_seed(8)
    S, V, d = 40, 4099, 256
    E = (torch.randn(V, d, generator=gen) * 0.02).to(torch.bfloat16).cuda()
    h = torch.randn(S, d, generator=gen).to(torch.bfloat16).cuda()
    tg = torch.randint(0, V, (S,), generator=gen, dtype=torch.int32)
    tg[:4] = torch.tensor([V - 1, V - 2, 0, 5], dtype=torch.int32)
    out = torch.empty(S, dtype=torch.float32, device="cuda")
    first = zo.zo_op_lm_head_logprob_noalloc(h, E, tg.cuda(), out, impl=impl).clone()
    assert bool(torch.isfinite(first).all())
    bad = tg.clone()
    bad[0], bad[1], bad[2] = V, -1, V + 4000
    second = zo.zo_op_lm_head_logprob_noalloc(h, E, bad.cuda(), out, impl=impl)
    assert zo.zo_op_error_word() == 0
    assert bool(torch.isnan(second[:3]).all()), second[:3]
    assert torch.equal(second[3:], first[3:])


def test_noalloc_rejects_requests_beyond_its_array():
    from zeroth_order_fine_b200 import zo
    cap = zo.lib().zo_op_lm_head_noalloc_capacity()
    V, d = 151936, 128
    S = cap // (2 * ((V + 63) // 64)) + 1            # one row more than fits on CUDA cores
    h = torch.zeros(S, d, dtype=torch.float32, device="cuda")
    E = torch.zeros(V, d, dtype=torch.float32, device="cuda")
    tg = torch.zeros(S, dtype=torch.int32, device="cuda")
    out = torch.empty(S, dtype=torch.float32, device="cuda")
    with pytest.raises(zo.ZoError) as e:
        zo.zo_op_lm_head_logprob_noalloc(h, E, tg, out, impl=1)
    assert e.value.code == zo.ZO_ERR_UNSUPPORTED
