"""Direction and weight streams: the CUDA generator against the oracle, bit for bit."""
import numpy as np
import pytest
import torch

from zeroth_order_fine_b200 import workload as wl
from gpu_util import gpu_handle, needs_gpu

pytestmark = [pytest.mark.gpu, needs_gpu]


@pytest.mark.parametrize("n,dtype,mean", [(1, torch.float32, 0.0), (1001, torch.float32, 0.0),
                                          (4096, torch.bfloat16, 0.0), (777, torch.float32, 1.0),
                                          (3_000_001, torch.bfloat16, 0.0)])
def test_init_tensor_bit_exact(n, dtype, mean):
    from oracle import generator as g
    from zeroth_order_fine_b200 import zo
    t = torch.empty(n, dtype=dtype, device="cuda")
    zo.zo_init_tensor(t, 7, 3, 5, 0.02, mean)
    torch.cuda.synchronize()
    ref = g.weight(7, 3, 5, n, 0.02, mean, dtype == torch.bfloat16)
    got = t.float().cpu().numpy()
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("scale", [wl.SCALE_LOZO, wl.SCALE_MEZO])
def test_factors_bit_exact_across_windows(scale):
    from oracle import generator as g
    w = wl.WORKLOADS["tiny"]
    import dataclasses
    w = dataclasses.replace(w, scale_mode=scale, rank=3, matrices=(wl.MAT_Q, wl.MAT_V, wl.MAT_UP,
                                                                    wl.MAT_DOWN))
    nu = 3
    model, h = gpu_handle(w, nu=nu, max_slots=4)
    batch = wl.make_batch(w, batch=2)
    toks = torch.from_numpy(batch.packed()).cuda()
    for t in range(7):
        h.zo_probe_plan(t, w.eps)
        for layer in range(w.shape.n_layers):
            for m in w.matrices:
                di, do = w.shape.matrix_dims(m)
                U, V = h.zo_read_factors(layer, m)
                Ur = g.factor(w.run_seed, t, nu, layer, m, 0, di, w.rank, scale)
                Vr = g.factor(w.run_seed, t, nu, layer, m, 1, do, w.rank, scale)
                assert np.array_equal(U.view(np.uint32), Ur.view(np.uint32)), (t, layer, m)
                assert np.array_equal(V.view(np.uint32), Vr.view(np.uint32)), (t, layer, m)
        h.zo_score(toks, batch.seq_lens, batch.target_lens)
        h.zo_step(w.lr)
    assert h.zo_stats()["bank_slots"] == 3
    h.close()
