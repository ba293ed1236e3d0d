"""The multi-rank host logic on the CPU with world-size-2 gloo ranks.

The layer shards by (batch, head) with no exchange step, so N GPUs run N
independent shards.  These tests check, on the CPU, that (1) sharding the
batch over ranks and gathering the results reproduces the single-process
result exactly (the heads are independent), and (2) the benchmark's
whole-job rate uses the slowest rank's time.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from kalman_filter_linear_b200 import synth
from oracle import kdn_ref


def _free_port():
    with socket.socket() as s:
        s.bind(('127.0.0.1', 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ['MASTER_ADDR'] = '127.0.0.1'
    os.environ['MASTER_PORT'] = str(port)
    dist.init_process_group('gloo', rank=rank, world_size=world)
    try:
        B, T, H, d = 4, 40, 2, 16
        x = synth.layer_inputs(B, T, H, d, d, 'diag', seed=5, dtype='bf16')
        shard = slice(rank * B // world, (rank + 1) * B // world)
        o, S, p = kdn_ref.diag_forward(*(x[n][shard].double().numpy() for n in 'qkvawr'))
        got = [torch.zeros(B // world, T, H, d, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(got, torch.from_numpy(o))
        # slowest rank decides the step time
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, dist, torch.device('cpu'))
        if rank == 0:
            q.put((torch.cat(got).numpy(), ms))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_sharded_ranks_reproduce_single_process_and_time_is_max():
    world = 2
    ctx = mp.get_context('spawn')
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    o_sharded, ms = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    B, T, H, d = 4, 40, 2, 16
    x = synth.layer_inputs(B, T, H, d, d, 'diag', seed=5, dtype='bf16')
    o, _, _ = kdn_ref.diag_forward(*(x[n].double().numpy() for n in 'qkvawr'))
    np.testing.assert_array_equal(o_sharded, o)
    assert ms == 15.0
    assert bench.whole_job_rate(1000, world, ms) == pytest.approx(2 * 1000 / 0.015)
