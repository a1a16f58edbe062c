"""pa_decode against the fp64 oracle on small shapes that span several blocks,
ragged tails, every kernel and forced context splits, plus the degenerate cases."""

import math

import numpy as np
import pytest
import torch

from gpu_util import DeviceWorkload, assert_close, oracle_pools, run_step
from paged_kv_cache_399_b200 import workloads

pytestmark = pytest.mark.gpu

# name, context lengths, q_per_seq, H_q, H_kv, head_dim, scale, shared-prefix groups
# [(first sequence, members, prefix tokens)]
CASES = [
    ("ctx1", [1, 1, 1], 1, 4, 2, 64, None, []),
    ("mult16", [16, 32, 64, 128], 1, 8, 2, 128, None, []),
    ("ragged", [17, 49, 33, 200, 255], 1, 8, 2, 128, None, []),
    ("mha", [40, 97, 300], 1, 4, 4, 128, None, []),
    ("mqa", [40, 97, 300], 1, 8, 1, 128, None, []),
    ("d64_gqa4", [5, 77, 160, 333], 1, 8, 2, 64, None, []),
    ("spec2", [9, 40, 129], 2, 8, 2, 128, None, []),
    ("spec6", [6, 16, 22, 300, 517], 6, 32, 8, 128, None, []),
    ("spec6_d64", [7, 100, 64], 6, 4, 1, 64, None, []),
    ("rows64", [33, 70], 16, 16, 4, 128, None, []),        # G*q = 64: two 32-row chunks
    ("single_rows16", [50, 81], 2, 8, 1, 128, None, []),  # 16 rows on the CUDA-core path
    ("zero_scale", [25, 66], 3, 4, 2, 128, 0.0, []),
    ("long_ragged", [1000, 2049, 3001], 1, 8, 1, 128, None, []),
    # prefix sharing: groups of adjacent sequences over the same physical prefix blocks
    ("shared3", [70, 49, 95, 33, 300], 1, 8, 2, 128, None, [(0, 3, 48)]),
    ("shared9", [260 + 7 * k for k in range(9)] + [40], 1, 8, 2, 128, None, [(0, 9, 256)]),
    ("shared_spec2", [64, 70, 81, 66], 2, 4, 2, 128, None, [(0, 4, 64)]),
    ("shared_short", [20, 16, 300, 310], 1, 4, 1, 64, None, [(0, 2, 16), (2, 2, 288)]),
    ("many_seqs", [1 + (37 * k) % 40 for k in range(1500)], 1, 4, 2, 64, None, []),
    # more sequences than the tcgen05 kernel stages in shared memory for its scan (2048 at N = 16)
    ("many_seqs_d128", [1 + (53 * k) % 47 for k in range(2100)], 1, 8, 2, 128, None, []),
    # GQA groups that do not divide the tcgen05 MMA's N (16 / 32): Q rows by plain loads
    ("g3", [40, 97, 300, 17], 1, 24, 8, 128, None, []),
    ("g6_spec3", [30, 200, 77], 3, 12, 2, 128, None, []),
    # sharing with G = 3: windows of 10 sequences hold 30 of the 32 rows
    ("shared_g3", [64 + 9 * k for k in range(10)] + [50, 90], 1, 24, 8, 128, None, [(0, 10, 64)]),
]

PLANS = [
    ("auto", {}),
    ("single_grid", dict(path=1, schedule=1)),
    ("tile_grid", dict(path=2, schedule=1)),
    ("single_persist", dict(path=1, schedule=2)),
    ("tile_persist", dict(path=2, schedule=2)),
    ("share", dict(path=2, share_prefix=True)),
    ("share_persist", dict(path=2, schedule=2, share_prefix=True)),
    ("share_split2", dict(path=2, split_blocks=2, share_prefix=True)),
    ("single_split1", dict(path=1, split_blocks=1)),
    ("tile_split1", dict(path=2, split_blocks=1)),
    ("tile_split3", dict(path=2, split_blocks=3)),
    ("tcgen05", dict(path=3)),
    # fewer / more CTAs than usual: units cut into many pieces, CTAs without work
    ("tcgen05_ctas3", dict(path=3, num_ctas=3)),
    ("tcgen05_ctas1000", dict(path=3, num_ctas=1000)),
    ("tcgen05_share", dict(path=3, share_prefix=True)),
    ("tcgen05_share_ctas5", dict(path=3, share_prefix=True, num_ctas=5)),
]


def _workload(case, seed):
    name, ctxs, q, hq, hkv, d, scale, groups = case
    share = [(list(range(first, first + n)), tokens) for first, n, tokens in groups]
    return workloads.build_workload(name, seed, ctxs, q, hq, hkv, d,
                                    scale=(1.0 / math.sqrt(d)) if scale is None else scale,
                                    pool_factor=1.5, share_groups=share)


@pytest.fixture(scope="module")
def prepared(oracle_lib):
    out = {}
    for k, case in enumerate(CASES):
        w = _workload(case, 2000 + k)
        kc, vc = oracle_pools(oracle_lib, w)
        ref = oracle_lib.decode(w.query, kc, vc, w.block_tables, w.context_lens, w.q_per_seq, w.scale)
        out[case[0]] = (w, ref)
    return out


def _plan(w, plan_spec):
    from paged_kv_cache_399_b200 import pa
    if not plan_spec[1]:
        return None
    hints = dict(plan_spec[1])
    num_ctas = hints.pop("num_ctas", None)
    try:
        plan = pa.pa_decode_plan(w.num_seqs, w.q_per_seq, w.num_q_heads, w.num_kv_heads,
                                 w.head_dim, w.max_blocks_per_seq, **hints)
    except pa.PAError as exc:
        assert exc.status == pa.PA_ERR_UNSUPPORTED
        if hints.get("path") == pa.PA_PATH_TCGEN05 and w.head_dim != 128:
            pytest.skip("the tcgen05 path runs head_dim 128")
        assert hints.get("share_prefix")
        pytest.skip("prefix sharing needs G*q <= 16 rows")
    if plan.path == pa.PA_PATH_TCGEN05:
        assert plan.schedule == pa.PA_SCHEDULE_PERSISTENT and plan.rows_per_cta in (16, 32)
        assert plan.share_cap == (32 // (w.num_q_heads // w.num_kv_heads * w.q_per_seq)
                                  if hints.get("share_prefix") else 0)
    if num_ctas is not None:
        plan.num_ctas = num_ctas
    return plan


@pytest.mark.parametrize("plan_spec", PLANS, ids=[p[0] for p in PLANS])
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_decode_matches_oracle(case, plan_spec, prepared):
    w, ref = prepared[case[0]]
    plan = _plan(w, plan_spec)
    dw = DeviceWorkload(w)
    out = run_step(dw, plan)
    assert_close(out, ref, f"{case[0]}/{plan_spec[0]}")


def _poison_unwritten(dw, w):
    """Fill the slots of each sequence's last block that lie past its context (and that no
    other sequence sees) with NaN in K and NaN / +Inf in V; returns how many slots."""
    bs = 16
    live = set()
    for b in range(w.num_seqs):
        for t in range(int(w.context_lens[b])):
            live.add((int(w.block_tables[b, t // bs]), t % bs))
    dead = set()
    for b in range(w.num_seqs):
        ctx = int(w.context_lens[b])
        if ctx % bs:
            phys = int(w.block_tables[b, (ctx - 1) // bs])
            dead.update((phys, off) for off in range(ctx % bs, bs) if (phys, off) not in live)
    dead = sorted(dead)
    if not dead:
        return 0
    blk = torch.tensor([d[0] for d in dead], device=dw.key_cache.device)
    off = torch.tensor([d[1] for d in dead], device=dw.key_cache.device)
    dw.key_cache[blk, off] = float("nan")
    dw.value_cache[blk, off] = float("nan")
    dw.value_cache[blk[::2], off[::2]] = float("inf")
    return len(dead)


POISON_CASES = ["ragged", "spec6", "spec6_d64", "rows64", "long_ragged", "shared9", "shared_spec2", "g6_spec3",
                "shared_g3"]


@pytest.mark.parametrize("plan_spec", PLANS, ids=[p[0] for p in PLANS])
@pytest.mark.parametrize("name", POISON_CASES)
def test_unwritten_slots_do_not_leak(name, plan_spec, prepared):
    """Slots past a sequence's context hold whatever the pool memory held. Their softmax
    weight is exactly zero, so NaN or Inf there must leave the output unchanged (the oracle
    reads only visible tokens, so its reference is the un-poisoned one)."""
    w, ref = prepared[name]
    plan = _plan(w, plan_spec)
    dw = DeviceWorkload(w)
    assert _poison_unwritten(dw, w) > 0
    out = run_step(dw, plan)
    assert_close(out, ref, f"{name}/{plan_spec[0]} poisoned")


def test_tiny_workload_every_path(oracle_lib):
    from paged_kv_cache_399_b200 import pa
    w = workloads.tiny()
    kc, vc = oracle_pools(oracle_lib, w)
    ref = oracle_lib.decode(w.query, kc, vc, w.block_tables, w.context_lens, 1, w.scale)
    outs = []
    for path in (pa.PA_PATH_SINGLE, pa.PA_PATH_TILE):
        for split in (0, 1, 2):  # 0: persistent schedule, else grid with that split
            plan = pa.pa_decode_plan(w.num_seqs, 1, 4, 2, 64, w.max_blocks_per_seq, path, split)
            out = run_step(DeviceWorkload(w), plan)
            assert_close(out, ref, f"tiny path={path} split={split}")
            outs.append(out.float().cpu())
    # cross-path agreement: every kernel / split within rounding of each other
    for o in outs[1:]:
        assert float((o - outs[0]).abs().max()) <= 2e-2


def test_ctx1_returns_v0_exactly(oracle_lib):
    """Closed form: one visible key gives out == v_0 (bf16 round trip is exact)."""
    w = _workload(CASES[0], 2000)
    dw = DeviceWorkload(w)
    out = run_step(dw)
    kc, vc = oracle_pools(oracle_lib, w)
    g = w.num_q_heads // w.num_kv_heads
    for b in range(w.num_seqs):
        blk = int(w.block_tables[b, 0])
        v0 = torch.from_numpy(vc[blk, 0].view(np.int16)).view(torch.bfloat16)
        for h in range(w.num_q_heads):
            assert torch.equal(out[b, 0, h].cpu(), v0[h // g])


def test_block_permutation_invariance():
    """Moving physical blocks (with a matching table) leaves the output unchanged."""
    from paged_kv_cache_399_b200 import pa
    w = _workload(CASES[2], 2002)
    base = run_step(DeviceWorkload(w)).clone()
    dw = DeviceWorkload(w)
    pa.pa_reshape_and_cache(dw.key, dw.value, dw.key_cache, dw.value_cache, dw.slots)
    sigma = torch.randperm(w.num_blocks, generator=torch.Generator().manual_seed(5))
    inv = torch.empty_like(sigma)
    inv[sigma] = torch.arange(w.num_blocks)
    kc = torch.empty_like(dw.key_cache)
    vc = torch.empty_like(dw.value_cache)
    kc[sigma.cuda()] = dw.key_cache
    vc[sigma.cuda()] = dw.value_cache
    dw.key_cache, dw.value_cache = kc, vc
    dw.tables = sigma.cuda()[dw.tables.long()].to(torch.int32)
    out = run_step(dw, write=False)
    assert torch.equal(out, base)


def test_validate_reports_bad_entries():
    from paged_kv_cache_399_b200 import pa
    w = _workload(CASES[2], 2002)
    dw = DeviceWorkload(w)
    assert pa.pa_validate(dw.tables, dw.ctx, dw.slots, w.q_per_seq, w.num_blocks) == 0
    bad_tables = dw.tables.clone()
    bad_tables[1, 0] = w.num_blocks + 3
    bad_tables[2, 1] = -1
    bad_ctx = dw.ctx.clone()
    bad_ctx[0] = w.max_blocks_per_seq * 16 + 1
    bad_slots = dw.slots.clone()
    bad_slots[0] = w.num_blocks * 16
    assert pa.pa_validate(bad_tables, bad_ctx, bad_slots, w.q_per_seq, w.num_blocks) == 4


@pytest.mark.parametrize("plan_spec", PLANS, ids=[p[0] for p in PLANS])
def test_empty_sequences_give_zero_rows(plan_spec, oracle_lib):
    """Sequences with context length 0 (nothing to attend to, no slot written) between
    ordinary ones: their rows are 0, the others match the oracle."""
    w = _workload(("with_empty", [5, 37, 9, 300, 12], 1, 8, 2, 128, None, []), 2990)
    empty = [0, 2, 4]
    w.context_lens = w.context_lens.copy()
    w.slot_mapping = w.slot_mapping.copy()
    for b in empty:
        w.context_lens[b] = 0
        w.slot_mapping[b * w.q_per_seq:(b + 1) * w.q_per_seq] = -1
    kc, vc = oracle_pools(oracle_lib, w)
    ref = oracle_lib.decode(w.query, kc, vc, w.block_tables, w.context_lens, w.q_per_seq, w.scale)
    assert all(float(np.abs(ref[b]).max()) == 0.0 for b in empty)
    plan = _plan(w, plan_spec)
    out = run_step(DeviceWorkload(w), plan)
    assert_close(out, ref, f"with_empty/{plan_spec[0]}")
    for b in empty:
        assert float(out[b].float().abs().max()) == 0.0
