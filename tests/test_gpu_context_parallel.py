"""Context parallelism on one GPU: pa_decode_partial over the table ranges that the ranks of a
group would take, merged by pa_merge_partials (directly, or after pa_combine_partials turned each
rank's pieces into one record per row), against the fp64 oracle's decode. The ranks are
emulated one after another on this device (no rank waits for another): the pieces of each range
go to their slice of one part-major buffer, as the all-gather leaves them. Table entries outside
a range are poisoned, and in the pools of the separate-pool case every block of another range
holds NaN, so a kernel that read outside its range would fail the comparison."""

import math

import numpy as np
import pytest
import torch

from gpu_util import DeviceWorkload, assert_close, oracle_pools
from paged_kv_cache_399_b200 import pa, workloads
from paged_kv_cache_399_b200.context_parallel import partial_pieces, rank_block_range

pytestmark = pytest.mark.gpu

# name, context lengths, q_per_seq, H_q, H_kv, head_dim
CASES = [
    ("long_q1", [3000, 1200, 777, 16], 1, 8, 1, 128),   # 8 rows: mma.sync tiles
    ("spec6", [900, 2049, 33], 6, 32, 8, 128),          # 24 rows, causal rows in the last range
    ("mha_d64", [500, 129, 64], 1, 4, 4, 64),           # 1 row: CUDA cores
    ("rows64", [700, 300], 16, 16, 4, 128),             # 64 rows: two row chunks
]
WORLDS = [1, 2, 3, 7]


def _workload(case, seed):
    name, ctxs, q, hq, hkv, d = case
    return workloads.build_workload(name, seed, ctxs, q, hq, hkv, d, scale=1.0 / math.sqrt(d))


@pytest.fixture(scope="module")
def prepared(oracle_lib):
    out = {}
    for k, case in enumerate(CASES):
        w = _workload(case, 6200 + k)
        kc, vc = oracle_pools(oracle_lib, w)
        ref = oracle_lib.decode(w.query, kc, vc, w.block_tables, w.context_lens, w.q_per_seq, w.scale)
        out[case[0]] = (w, ref)
    return out


def _pieces(dw, world, pools=None):
    """Part-major pieces of every range; each range reads a table whose other entries name a
    block past the pool (zero-filled by TMA if read), from its own pools when given."""
    w = dw.w
    B, QS, HQ, D = w.query.shape
    mb = w.block_tables.shape[1]
    S = partial_pieces(dw.query, dw.key_cache, mb, world)
    part_o = torch.empty((world, S, B, QS, HQ, D), dtype=torch.float32, device="cuda")
    part_ml = torch.empty((world, S, B, QS, HQ, 2), dtype=torch.float32, device="cuda")
    for r in range(world):
        lo, hi = rank_block_range(mb, r, world)
        tables = dw.tables.clone()
        tables[:, :lo] = w.num_blocks + 7
        tables[:, hi:] = w.num_blocks + 7
        kc, vc = pools[r] if pools else (dw.key_cache, dw.value_cache)
        pa.pa_decode_partial(part_o[r], part_ml[r], dw.query, kc, vc, tables, dw.ctx, w.q_per_seq, w.scale, lo, hi)
    return part_o.flatten(0, 1), part_ml.flatten(0, 1)


def _write(dw):
    pa.pa_reshape_and_cache(dw.key, dw.value, dw.key_cache, dw.value_cache, dw.slots)


@pytest.mark.parametrize("world", WORLDS)
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_partial_pieces_merge_to_the_decode(case, world, prepared):
    w, ref = prepared[case[0]]
    dw = DeviceWorkload(w)
    _write(dw)
    part_o, part_ml = _pieces(dw, world)
    out = torch.full_like(dw.query, float("nan"))
    pa.pa_merge_partials(out, part_o, part_ml)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error(reset=True) == 0
    assert_close(out, ref, f"{case[0]}/world {world}")
    # the merge does not depend on the order of the pieces
    perm = torch.randperm(part_o.shape[0], generator=torch.Generator().manual_seed(world)).cuda()
    out2 = torch.empty_like(out)
    pa.pa_merge_partials(out2, part_o[perm].contiguous(), part_ml[perm].contiguous())
    torch.cuda.synchronize()
    assert_close(out2, ref, f"{case[0]}/world {world}, pieces reordered")
    # each rank combines its own pieces into one record per row; the records merge to the same
    B, QS, HQ, D = w.query.shape
    S = part_o.shape[0] // world
    rec_o = torch.empty((world, B, QS, HQ, D), dtype=torch.float32, device="cuda")
    rec_ml = torch.empty((world, B, QS, HQ, 2), dtype=torch.float32, device="cuda")
    for r in range(world):
        pa.pa_combine_partials(rec_o[r], rec_ml[r], part_o[r * S:(r + 1) * S].contiguous(),
                               part_ml[r * S:(r + 1) * S].contiguous())
    out3 = torch.empty_like(out)
    pa.pa_merge_partials(out3, rec_o, rec_ml)
    torch.cuda.synchronize()
    assert_close(out3, ref, f"{case[0]}/world {world}, records combined per rank")


@pytest.mark.parametrize("case", CASES[:2], ids=[c[0] for c in CASES[:2]])
def test_each_range_reads_only_its_own_pool(case, prepared):
    """Three ranks with pools of their own: every block that another range's entries name holds
    NaN in this rank's pool (K and V)."""
    w, ref = prepared[case[0]]
    dw = DeviceWorkload(w)
    _write(dw)
    world, mb = 3, w.block_tables.shape[1]
    pools = []
    for r in range(world):
        lo, hi = rank_block_range(mb, r, world)
        mine = set()
        for b in range(w.num_seqs):
            nb = -(-int(w.context_lens[b]) // 16)
            mine.update(int(x) for x in w.block_tables[b, lo:min(hi, nb)])
        others = [blk for blk in range(w.num_blocks) if blk not in mine]
        kc, vc = dw.key_cache.clone(), dw.value_cache.clone()
        idx = torch.tensor(others, device="cuda")
        kc[idx] = float("nan")
        vc[idx] = float("nan")
        pools.append((kc, vc))
    part_o, part_ml = _pieces(dw, world, pools)
    out = torch.empty_like(dw.query)
    pa.pa_merge_partials(out, part_o, part_ml)
    torch.cuda.synchronize()
    assert bool(torch.isfinite(out.float()).all())
    assert_close(out, ref, f"{case[0]}/separate pools")


def test_an_empty_range_gives_empty_pieces(prepared):
    """A range past every context, in three pieces: m = -inf, l = 0 and o = 0 for every row."""
    w, _ = prepared["long_q1"]
    dw = DeviceWorkload(w)
    mb = w.block_tables.shape[1]
    B, QS, HQ, D = w.query.shape
    part_o = torch.full((3, B, QS, HQ, D), 1.0, device="cuda")
    part_ml = torch.full((3, B, QS, HQ, 2), 1.0, device="cuda")
    pa.pa_decode_partial(part_o, part_ml, dw.query, dw.key_cache, dw.value_cache, dw.tables, dw.ctx,
                         w.q_per_seq, w.scale, mb, mb)
    torch.cuda.synchronize()
    assert bool((part_o == 0).all()) and bool((part_ml[..., 1] == 0).all())
    assert bool(torch.isneginf(part_ml[..., 0]).all())
