"""Context parallelism (one long sequence's blocks over the GPUs of a group): the ranges the
ranks take, and the exchange of their pieces, checked with gloo ranks on CPU. Each rank's
pieces here come from an fp64 evaluation over its range (the kernels need a GPU; their
parity is tests/test_gpu_context_parallel.py); the gathered pieces, merged by the log-sum-exp
rule, must give the oracle's decode."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from paged_kv_cache_399_b200.context_parallel import gather_partials, rank_block_range


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("max_blocks", [1, 5, 16, 257])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_rank_ranges_cover_each_table_once(max_blocks, world):
    ranges = [rank_block_range(max_blocks, r, world) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == max_blocks
    for (lo, hi), (lo2, _) in zip(ranges, ranges[1:]):
        assert lo <= hi == lo2
    with pytest.raises(ValueError):
        rank_block_range(max_blocks, world, world)


def _f64(bits):
    return (np.asarray(bits).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _pieces(w, kc, vc, lo, hi):
    """fp64 pieces of every row over table entries [lo, hi): o = sum 2^(s-m) v, m, l."""
    B, QS, HQ, D = w.query.shape
    g = HQ // w.num_kv_heads
    q = _f64(w.query.view(torch.int16).numpy().view(np.uint16))
    K, V = _f64(kc), _f64(vc)
    o = np.zeros((B, QS, HQ, D))
    ml = np.zeros((B, QS, HQ, 2))
    ml[..., 0] = -np.inf
    for b in range(B):
        ctx = int(w.context_lens[b])
        for i in range(QS):
            pos = ctx - QS + i
            keys = [t for t in range(lo * 16, min(hi * 16, ctx)) if t <= pos]
            if not keys:
                continue
            blk = [int(w.block_tables[b, t // 16]) for t in keys]
            for h in range(HQ):
                kv = h // g
                kk = np.stack([K[pb, t % 16, kv] for pb, t in zip(blk, keys)])
                vv = np.stack([V[pb, t % 16, kv] for pb, t in zip(blk, keys)])
                s = (kk @ q[b, i, h]) * w.scale * np.log2(np.e)
                m = s.max()
                p = np.exp2(s - m)
                o[b, i, h] = p @ vv
                ml[b, i, h] = (m, p.sum())
    return o, ml


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import Oracle
        from paged_kv_cache_399_b200 import workloads
        w = workloads.build_workload("cp", 6100, [300, 45, 170, 16], 2, 8, 2, 16)  # ragged, q = 2, GQA 4
        orc = Oracle()
        kc, vc = orc.reshape_and_cache(w.key, w.value, w.key_cache, w.value_cache, w.slot_mapping)
        lo, hi = rank_block_range(w.block_tables.shape[1], rank, world)
        o, ml = _pieces(w, kc, vc, lo, hi)
        all_o, all_ml = gather_partials(torch.from_numpy(o), torch.from_numpy(ml))
        out[rank] = (all_o.numpy(), all_ml.numpy(),
                     orc.decode(w.query, kc, vc, w.block_tables, w.context_lens, w.q_per_seq, w.scale))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gathered_pieces_merge_to_the_oracle_decode(world):
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    all_o, all_ml, ref = out[0]
    for r in range(1, world):  # every rank holds the same gathered pieces, in rank order
        assert np.array_equal(out[r][0], all_o) and np.array_equal(out[r][1], all_ml)
    m = all_ml[..., 0]
    M = m.max(axis=0)
    wgt = np.where(np.isneginf(m), 0.0, np.exp2(m - M))
    merged = (wgt[..., None] * all_o).sum(0) / (wgt * all_ml[..., 1]).sum(0)[..., None]
    np.testing.assert_allclose(merged, ref, rtol=1e-10, atol=1e-12)
