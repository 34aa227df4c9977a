"""Multi-rank host logic of bench.py on CPU with world_size-2 gloo ranks: each
rank runs its own copy of the workload (different seeds, no data exchange) and
the job time is the maximum over ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from gated_delta_rule_130_b200 import inputs as I
        ms_local = 100.0 + 50.0 * rank              # rank 1 is the slow one
        value, ms_step = bench.weak_scaling_value(ms_local, 10, 4096, world, torch.device("cpu"))
        w = I.workload("tiny_f32")
        q = I.chunk_inputs(w, seed=w.seed + rank)["q"]
        gathered = [torch.zeros_like(q) for _ in range(world)]
        dist.all_gather(gathered, q)                # test-only: compare the ranks' inputs
        out[rank] = (value, ms_step, bool(torch.equal(gathered[0], gathered[1])))
    finally:
        dist.destroy_process_group()


def test_weak_scaling_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    (v0, ms0, same0), (v1, ms1, same1) = out[0], out[1]
    # both ranks report the slowest rank's time, and the job's tokens/s counts both ranks
    assert ms0 == ms1 == pytest.approx(150.0 / 10)
    assert v0 == v1 == pytest.approx(2 * 4096 / (15.0e-3))
    assert not same0 and not same1              # each rank has its own batch
