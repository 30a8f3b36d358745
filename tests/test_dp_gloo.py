"""Data-parallel host logic with two CPU ranks over gloo.

Each rank scores its shard of the prompts with the oracle, all-reduces its
{sum of paired differences, prompt count} through zeroth_order_fine_b200.dp,
and must obtain the c that one process computes over the whole batch; the
bank update that follows is then identical on both ranks.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from zeroth_order_fine_b200 import workload as wl


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        from oracle import model as om
        from oracle import zo as ozo
        from zeroth_order_fine_b200 import dp
        w = wl.WORKLOADS["tiny"]
        full = wl.make_batch(w, batch=5)                   # odd count: uneven shards
        mine = dp.shard_batch(full, rank, world)
        run = ozo.OracleRun(om.init_weights(w.shape), w.run_seed, w.nu, w.rank,
                            range(w.shape.n_layers), w.matrices, w.scale_mode)
        cs = []
        for t in range(2):
            run.plan(t, w.eps)
            res = run.score(mine.prompts, mine.target_lens)
            sums = torch.tensor([float(np.sum(res.L_plus - res.L_minus)), float(len(mine.prompts))],
                                dtype=torch.float64)
            dp.allreduce_sums(sums)
            c = float(sums[0] / sums[1] / (2 * w.eps))
            for key, slots in run.bank.items():            # the same update on every rank
                slots[-1][0] = slots[-1][0] - w.lr * c * run.U[key]
            run.t += 1
            cs.append(c)
        A = run.bank[(0, wl.MAT_Q)][0][0].numpy().copy()
        out_q.put((rank, len(mine.prompts), cs, A))
    finally:
        dist.destroy_process_group()


def test_two_rank_objective_allreduce_matches_single_process():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=300) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    results.sort(key=lambda x: x[0])
    assert [r[1] for r in results] == [3, 2]

    from oracle import model as om
    from oracle import zo as ozo
    w = wl.WORKLOADS["tiny"]
    full = wl.make_batch(w, batch=5)
    run = ozo.OracleRun(om.init_weights(w.shape), w.run_seed, w.nu, w.rank,
                        range(w.shape.n_layers), w.matrices, w.scale_mode)
    ref = []
    for t in range(2):
        run.plan(t, w.eps)
        run.score(full.prompts, full.target_lens)
        ref.append(run.step(w.lr))
    for _, _, cs, A in results:
        assert np.allclose(cs, ref, rtol=1e-12, atol=0)
        assert np.allclose(A, run.bank[(0, wl.MAT_Q)][0][0].numpy(), rtol=1e-12, atol=1e-18)
    assert np.array_equal(results[0][3], results[1][3])     # replicas stay identical


def test_shards_cover_the_batch_once():
    from zeroth_order_fine_b200 import dp
    w = wl.WORKLOADS["tiny"]
    b = wl.make_batch(w, batch=7, fg_rows=3)
    parts = [dp.shard_batch(b, r, 3) for r in range(3)]
    assert sum(len(p.prompts) for p in parts) == 7
    assert sum(len(p.fg_prompts) for p in parts) == 3
    assert np.array_equal(np.concatenate([p.packed() for p in parts]), b.packed())


def test_allreduce_rejects_wrong_shape():
    from zeroth_order_fine_b200 import dp
    with pytest.raises(ValueError):
        dp.allreduce_sums(torch.zeros(3, dtype=torch.float64))
