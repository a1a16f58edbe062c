"""The multi-GPU path of bench.py is one independent replica per rank (weak scaling):
seeds per rank, max-over-ranks timing and whole-job throughput, checked with two gloo
ranks on CPU."""

import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from paged_kv_cache_399_b200 import workloads
        w = workloads.make("tiny", seed=bench.rank_seed("tiny", rank))
        fake_ms = 10.0 + 5.0 * rank               # rank 1 is the slow one
        max_ms = bench.reduce_over_ranks(fake_ms, "max", dist)
        total_blocks = bench.reduce_over_ranks(float(w.blocks_used.sum()), "sum", dist)
        bytes_step = bench.decode_bytes(w) + bench.cache_write_bytes(w)
        out[rank] = (w.seed, tuple(w.query.shape), max_ms, total_blocks, bytes_step,
                     float(w.query.float().sum()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_run_independent_replicas():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    r0, r1 = out[0], out[1]
    assert r0[0] != r1[0]                      # each rank has its own seed ...
    assert r0[1] == r1[1]                      # ... and the same shapes
    assert r0[5] != r1[5]                      # ... hence different data
    assert r0[2] == r1[2] == 15.0              # max over ranks of the device time
    assert r0[3] == r1[3] > 0                  # a sum all ranks agree on
    job = bench.aggregate_throughput(r0[4], 100, r0[2], world)
    assert job == pytest.approx(world * r0[4] * 100 / 15e-3 / 1e9)
