"""Shared set-up of the GPU tests: the same workload on the CUDA path (through the
C ABI) and in the oracle."""
import numpy as np
import pytest
import torch

from zeroth_order_fine_b200 import workload as wl

needs_gpu = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


def gpu_handle(w: wl.Workload, shape=None, batch=None, max_slots=8, impl=0, nu=None,
               layers=None, start_step=0, fg=0, fp8=0, max_new=0):
    from zeroth_order_fine_b200 import zo
    shape = shape or w.shape
    model = zo.DeviceModel(shape, w.weight_seed)
    tg = zo.make_targets(shape.n_layers, w.matrices, w.scale_mode, layers)
    B = batch or w.batch
    max_len = w.len_hi
    h = zo.Handle(model, w.run_seed, nu or w.nu, w.rank, tg,
                  max_tokens=(2 * B + fg) * max_len + 64, max_rows=2 * B + fg,
                  max_scored=(2 * B + fg) * max(w.tgt_hi, w.fg_tgt_hi if fg else 1),
                  max_slots=max_slots, start_step=start_step, impl=impl, fp8=fp8,
                  max_new=max_new)
    return model, h


def oracle_run(w: wl.Workload, shape=None, nu=None, layers=None, start_step=0, fp8=False):
    from oracle import model as om
    from oracle import zo as ozo
    shape = shape or w.shape
    weights = om.init_weights(shape, w.weight_seed)
    ls = range(shape.n_layers) if layers is None else layers
    return ozo.OracleRun(weights, w.run_seed, nu or w.nu, w.rank, ls, w.matrices, w.scale_mode,
                         start_step, fp8=fp8)


def dev_tokens(batch: wl.Batch):
    return torch.from_numpy(batch.packed()).cuda()


def dev_fg_tokens(batch: wl.Batch):
    return torch.from_numpy(batch.fg_packed()).cuda()


def oracle_state_blob(orc, w: wl.Workload, shape=None) -> bytes:
    """The oracle's bank in the library's state layout (zo.h, zo_save_state)."""
    import struct
    shape = shape or w.shape
    r = w.rank
    groups = ([wl.MAT_Q, wl.MAT_K, wl.MAT_V], [wl.MAT_O],
              [wl.MAT_UP] if shape.arch == wl.ARCH_OPT else [wl.MAT_GATE, wl.MAT_UP],
              [wl.MAT_DOWN])
    n_slots = len(next(iter(orc.bank.values())))
    payload = []
    for l in range(shape.n_layers):
        for g in groups:
            tg = [m for m in g if m in w.matrices and (l, m) in orc.bank]
            for j in range(n_slots):
                for m in tg:
                    A = orc.bank[(l, m)][j][0].numpy()          # [d_in x r]
                    payload.append(np.ascontiguousarray(A.T.astype(np.float32)))
    data = b"".join(a.tobytes() for a in payload)
    lo = hi = 0
    for l in range(shape.n_layers):
        if l < 64:
            lo |= 1 << l
        else:
            hi |= 1 << (l - 64)
    mm = sum(1 << m for m in w.matrices)
    start_window = orc.bank[next(iter(orc.bank))][0][2]
    head = struct.pack("<5Q4i2I3Q", 0x5A4F42414E4B3031, 1, w.run_seed, orc.t, start_window,
                       orc.nu, r, n_slots, w.scale_mode, mm, 0, lo, hi, len(data) // 4)
    return head + data
