"""The N > 1 bench path on CPU with the gloo backend (world size 2): every rank draws its
own inputs, the job's step time is the slowest rank's, and the job's work is the sum."""
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
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import synth
        ms = bench._max_over_ranks(10.0 + 5.0 * rank, world, device="cpu")
        tok = bench._sum_over_ranks(64.0, world, device="cpu")
        seed = bench.rank_seed(2, rank, 1)
        pos = synth.uniform_positions(8, 8192, 131072, bench.rank_seed(2, rank, 0))
        bench._barrier(world)
        out[rank] = (ms, tok, seed, pos.tolist())
    finally:
        dist.destroy_process_group()


def test_two_ranks_time_is_max_work_is_sum_inputs_differ():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    r0, r1 = out[0], out[1]
    assert r0[0] == r1[0] == 15.0
    assert r0[1] == r1[1] == 128.0
    assert r0[2] != r1[2]
    assert r0[3] != r1[3]
