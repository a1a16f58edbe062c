"""pa_decode with a sliding window against the fp64 oracle: the mma.sync and CUDA-core grid
paths and the tcgen05 kernel, windows around block and split boundaries, speculative rows,
and the null block
(table entries wholly before the window point at block 0, which holds NaN, and the slots
before the window in its first block hold NaN as well)."""

import math

import numpy as np
import pytest
import torch

from gpu_util import DeviceWorkload, assert_close, oracle_pools, run_step
from paged_kv_cache_399_b200 import workloads

pytestmark = pytest.mark.gpu

# name, context lengths, q_per_seq, H_q, H_kv, head_dim
CASES = [
    ("w_ragged", [17, 49, 200, 255, 1000], 1, 8, 2, 128),   # 4 rows: mma.sync tiles
    ("w_spec3", [9, 40, 129, 517], 3, 8, 2, 128),           # 12 rows, causal inside the window
    ("w_d64", [5, 77, 160, 333], 1, 8, 2, 64),
    ("w_rows1", [40, 97, 300], 1, 4, 4, 128),               # 1 row: CUDA cores
    ("w_rows32", [33, 700], 4, 32, 4, 128),                  # 32 rows: the widest tile core
]
WINDOWS = [1, 15, 16, 17, 100, 1000]
PLANS = [
    ("auto", {}),
    ("single_grid", dict(path=1, schedule=1)),
    ("tile_grid", dict(path=2, schedule=1)),
    ("tile_split1", dict(path=2, split_blocks=1)),
    ("tile_split3", dict(path=2, split_blocks=3)),
    ("tcgen05", dict(path=3)),
    ("tcgen05_ctas5", dict(path=3, num_ctas=5)),   # units cut into many pieces
]


def _workload(case, seed):
    name, ctxs, q, hq, hkv, d = case
    return workloads.build_workload(name, seed, ctxs, q, hq, hkv, d, scale=1.0 / math.sqrt(d),
                                    pool_factor=1.5)


@pytest.fixture(scope="module")
def prepared(oracle_lib):
    out = {}
    for k, case in enumerate(CASES):
        w = _workload(case, 3000 + k)
        kc, vc = oracle_pools(oracle_lib, w)
        for W in WINDOWS:
            out[(case[0], W)] = (w, oracle_lib.decode(w.query, kc, vc, w.block_tables, w.context_lens,
                                                      w.q_per_seq, w.scale, window=W))
    return out


def _plan(w, spec, W):
    from paged_kv_cache_399_b200 import pa
    spec = dict(spec)
    num_ctas = spec.pop("num_ctas", None)
    if spec.get("path") == pa.PA_PATH_TCGEN05 and w.head_dim != 128:
        pytest.skip("the tcgen05 path runs head_dim 128")
    plan = pa.pa_decode_plan(w.num_seqs, w.q_per_seq, w.num_q_heads, w.num_kv_heads, w.head_dim,
                             w.max_blocks_per_seq, sliding_window=W, **spec)
    assert plan.sliding_window == W
    if plan.path == pa.PA_PATH_TCGEN05:
        assert plan.schedule == pa.PA_SCHEDULE_PERSISTENT
        if num_ctas is not None:
            plan.num_ctas = num_ctas
        return plan
    assert plan.schedule == pa.PA_SCHEDULE_GRID
    span = min(w.max_blocks_per_seq, -(-(W + w.q_per_seq - 1) // 16) + 1)
    assert plan.num_splits == -(-span // plan.split_blocks)
    return plan


@pytest.mark.parametrize("plan_spec", PLANS, ids=[p[0] for p in PLANS])
@pytest.mark.parametrize("W", WINDOWS)
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_window_matches_oracle(case, W, plan_spec, prepared):
    w, ref = prepared[(case[0], W)]
    plan = _plan(w, plan_spec[1], W)
    out = run_step(DeviceWorkload(w), plan)
    assert_close(out, ref, f"{case[0]}/W={W}/{plan_spec[0]}")


@pytest.mark.parametrize("plan_spec", PLANS, ids=[p[0] for p in PLANS])
@pytest.mark.parametrize("W", [15, 17, 100])
def test_window_never_reads_before_the_window(W, plan_spec, oracle_lib):
    """Entries wholly before a sequence's window name the null block 0 (NaN in K and V);
    the slots of its first window block below every row's window hold NaN too."""
    w = _workload(("w_null", [70, 300, 513, 999], 2, 8, 2, 128), 3100)
    bs = 16
    tables = w.block_tables.copy()
    kc, vc = w.key_cache.clone(), w.value_cache.clone()
    used = set()
    for b in range(w.num_seqs):
        used.update(int(x) for x in tables[b, :-(-int(w.context_lens[b]) // bs)])
    if 0 in used:   # make block 0 unused: swap it with a free block, contents and names
        free = next(x for x in range(w.num_blocks) if x not in used)
        kc[[0, free]] = kc[[free, 0]]
        vc[[0, free]] = vc[[free, 0]]
        tables = np.where(tables == 0, free, tables).astype(np.int32)
    w.block_tables, w.key_cache, w.value_cache = tables, kc, vc
    w.slot_mapping = w.slot_mapping.copy()   # the step's slots follow the new block names
    for t in range(w.num_tokens):
        b, i = divmod(t, w.q_per_seq)
        p = int(w.context_lens[b]) - w.q_per_seq + i
        w.slot_mapping[t] = int(tables[b, p // bs]) * bs + p % bs
    pk, pv = oracle_pools(oracle_lib, w)
    ref = oracle_lib.decode(w.query, pk, pv, tables, w.context_lens, w.q_per_seq, w.scale, window=W)

    null_tables = tables.copy()
    dw = DeviceWorkload(w)
    dw.key_cache[0] = float("nan")
    dw.value_cache[0] = float("nan")
    poisoned = 0
    for b in range(w.num_seqs):
        lo = max(0, int(w.context_lens[b]) - w.q_per_seq - W + 1)   # row 0's window start
        null_tables[b, :lo // bs] = 0
        first = int(null_tables[b, lo // bs])
        for off in range(lo % bs):
            dw.key_cache[first, off] = float("nan")
            dw.value_cache[first, off] = float("inf") if off % 2 else float("nan")
            poisoned += 1
    assert poisoned > 0 and (null_tables == 0).any()
    dw.tables = torch.from_numpy(null_tables).to(dw.tables.device)
    out = run_step(dw, _plan(w, plan_spec[1], W))
    assert_close(out, ref, f"null block W={W}/{plan_spec[0]}")


def test_window_rejected_with_sharing_or_the_mma_sync_persistent_schedule():
    from paged_kv_cache_399_b200 import pa
    for hints in (dict(path=2, schedule=2), dict(path=1, schedule=2), dict(path=2, share_prefix=True),
                  dict(path=3, share_prefix=True)):
        with pytest.raises(pa.PAError) as err:
            pa.pa_decode_plan(4, 1, 32, 8, 128, 64, sliding_window=64, **hints)
        assert err.value.status == pa.PA_ERR_UNSUPPORTED


def test_sliding_window_workload_full_size(oracle_lib):
    """The benchmark's sliding-window workload in the plan bench.py times, every output row
    against the oracle."""
    from paged_kv_cache_399_b200 import pa
    w = workloads.make("sliding_window")
    plan = pa.pa_decode_plan(w.num_seqs, w.q_per_seq, w.num_q_heads, w.num_kv_heads, w.head_dim,
                             w.max_blocks_per_seq, sliding_window=w.window)
    out = run_step(DeviceWorkload(w), plan).clone()
    kc, vc = oracle_pools(oracle_lib, w)
    ref = oracle_lib.decode(w.query, kc, vc, w.block_tables, w.context_lens, w.q_per_seq, w.scale,
                            window=w.window)
    assert_close(out, ref, "sliding_window full size")
