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
        assert torch.max(torch.abs(got - ref)).item() <= 2e-4, call


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
