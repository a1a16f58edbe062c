"""pa_decode_fp8 against the fp64 oracle over FP8 (E4M3) pools: every decode case of
test_gpu_decode.py, the FP8 plans (grid and persistent schedules, forced splits, prefix
sharing, sliding windows), NaN codes in slots outside every context, and the full-size
llama8b_fp8 workload. The step's new K/V go through pa_reshape_and_cache_fp8 on the GPU and
oracle_reshape_and_cache_fp8 on the host; the attention tolerance is the bf16 path's."""

import math

import numpy as np
import pytest
import torch

from gpu_util import MAX_ABS_TOL, MEAN_ABS_TOL, assert_close
from paged_kv_cache_399_b200 import workloads
from test_gpu_decode import CASES, _workload

pytestmark = pytest.mark.gpu

KS, VS = 0.01, 0.013   # pool scales: different, so a swapped scale cannot pass

PLANS = [
    ("auto", {}),
    ("tile_grid", dict(path=2, schedule=1)),
    ("tile_persist", dict(path=2, schedule=2)),
    ("share", dict(path=2, share_prefix=True)),
    ("share_persist", dict(path=2, schedule=2, share_prefix=True)),
    ("tile_split1", dict(path=2, split_blocks=1)),
    ("tile_split3", dict(path=2, split_blocks=3)),
]


def _fp8(w):
    return workloads.with_fp8_pools(w, KS, VS)


def _oracle(orc, w, window=0):
    kc, vc = orc.reshape_and_cache_fp8(w.key, w.value, w.key_cache.numpy(), w.value_cache.numpy(),
                                       w.slot_mapping, w.k_scale, w.v_scale)
    ref = orc.decode_fp8(w.query, kc, vc, w.block_tables, w.context_lens, w.q_per_seq, w.scale,
                         w.k_scale, w.v_scale, window=window)
    return ref


class DeviceFp8:
    def __init__(self, w):
        self.w = w
        self.query = w.query.cuda()
        self.key = w.key.cuda()
        self.value = w.value.cuda()
        self.slots = torch.from_numpy(w.slot_mapping).cuda()
        self.tables = torch.from_numpy(w.block_tables).cuda()
        self.ctx = torch.from_numpy(w.context_lens).cuda()
        self.key_cache = w.key_cache.cuda()
        self.value_cache = w.value_cache.cuda()
        self.out = torch.empty_like(self.query)

    def step(self, plan=None, write=True):
        from paged_kv_cache_399_b200 import pa
        w = self.w
        if write:
            pa.pa_reshape_and_cache_fp8(self.key, self.value, self.key_cache, self.value_cache, self.slots,
                                        w.k_scale, w.v_scale)
        need = pa.pa_decode_workspace_size(plan, w.num_seqs, w.q_per_seq, w.num_q_heads, w.num_kv_heads,
                                           w.head_dim, w.max_blocks_per_seq)
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda") if need else None
        pa.pa_decode_fp8(self.out, self.query, self.key_cache, self.value_cache, self.tables, self.ctx,
                         w.q_per_seq, w.scale, w.k_scale, w.v_scale, plan=plan, workspace=ws)
        torch.cuda.synchronize()
        assert pa.pa_get_device_error(reset=True) == 0
        return self.out


def _plan(w, spec, **extra):
    from paged_kv_cache_399_b200 import pa
    hints = dict(spec[1], **extra)
    if not hints:
        return None
    try:
        return pa.pa_decode_plan(w.num_seqs, w.q_per_seq, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                 w.max_blocks_per_seq, kv_cache_dtype=pa.PA_KV_FP8_E4M3, **hints)
    except pa.PAError as exc:
        assert exc.status == pa.PA_ERR_UNSUPPORTED and hints.get("share_prefix")
        pytest.skip("prefix sharing needs G*q <= 16 rows")


@pytest.fixture(scope="module")
def prepared(oracle_lib):
    out = {}
    for k, case in enumerate(CASES):
        w = _fp8(_workload(case, 4000 + k))
        out[case[0]] = (w, _oracle(oracle_lib, w))
    return out


@pytest.mark.parametrize("plan_spec", PLANS, ids=[p[0] for p in PLANS])
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_fp8_decode_matches_oracle(case, plan_spec, prepared):
    w, ref = prepared[case[0]]
    out = DeviceFp8(w).step(_plan(w, plan_spec))
    assert_close(out, ref, f"fp8 {case[0]}/{plan_spec[0]}")


@pytest.mark.parametrize("plan_spec", PLANS[:3], ids=[p[0] for p in PLANS[:3]])
@pytest.mark.parametrize("name", ["ragged", "spec6", "spec6_d64", "rows64", "shared9"])
def test_fp8_nan_codes_outside_every_context_do_not_leak(name, plan_spec, prepared):
    """E4M3 has no infinity; its NaN codes (0x7F, 0xFF) in slots past each sequence's
    context (which no sequence sees) leave the output unchanged."""
    w, ref = prepared[name]
    dw = DeviceFp8(w)
    bs = 16
    live = {(int(w.block_tables[b, t // bs]), t % bs) for b in range(w.num_seqs)
            for t in range(int(w.context_lens[b]))}
    dead = set()
    for b in range(w.num_seqs):
        ctx = int(w.context_lens[b])
        if ctx % bs:
            phys = int(w.block_tables[b, (ctx - 1) // bs])
            dead.update((phys, o) for o in range(ctx % bs, bs) if (phys, o) not in live)
    assert dead
    blk = torch.tensor([d[0] for d in sorted(dead)], device="cuda")
    off = torch.tensor([d[1] for d in sorted(dead)], device="cuda")
    dw.key_cache[blk, off] = 0x7F
    dw.value_cache[blk, off] = 0xFF
    out = dw.step(_plan(w, plan_spec))
    assert_close(out, ref, f"fp8 {name}/{plan_spec[0]} NaN codes")


@pytest.mark.parametrize("window", [1, 16, 37, 100])
@pytest.mark.parametrize("name", ["long_ragged", "spec6", "d64_gqa4"])
def test_fp8_sliding_window(name, window, oracle_lib):
    case = next(c for c in CASES if c[0] == name)
    w = _fp8(_workload(case, 4100 + window))
    ref = _oracle(oracle_lib, w, window=window)
    out = DeviceFp8(w).step(_plan(w, ("window", dict(path=2)), sliding_window=window))
    assert_close(out, ref, f"fp8 {name} window {window}")


def test_fp8_scale_is_applied_to_keys_and_values(oracle_lib):
    """The same codes at other pool scales: k_scale changes the softmax temperature and
    v_scale multiplies the output; both against the oracle."""
    case = next(c for c in CASES if c[0] == "ragged")
    base = _workload(case, 4200)
    for ks, vs in ((0.002, 0.05), (0.05, 0.002)):
        w = workloads.with_fp8_pools(base, ks, vs)
        ref = _oracle(oracle_lib, w)
        out = DeviceFp8(w).step()
        assert_close(out, ref, f"fp8 scales {ks} {vs}")


def test_fp8_large_and_small_queries(oracle_lib):
    """bf16 queries beyond f16's range (and far below it) still match: each row is scaled by
    a power of two before its f16 conversion."""
    case = next(c for c in CASES if c[0] == "spec2")
    w = _fp8(_workload(case, 4300))
    q = w.query.float()
    q[0] *= 2.0 ** 20          # |q| ~ 1e6: beyond f16's 65504
    q[1] *= 2.0 ** -30         # |q| ~ 1e-9: below f16's normal range
    w.query = q.to(torch.bfloat16)
    w.scale = 2.0 ** -22       # keep the first sequence's scores moderate
    ref = _oracle(oracle_lib, w)
    out = DeviceFp8(w).step()
    assert_close(out, ref, "fp8 large/small queries")


def test_fp8_plans_and_pools_must_agree():
    from paged_kv_cache_399_b200 import pa
    case = next(c for c in CASES if c[0] == "ragged")
    w = _fp8(_workload(case, 4400))
    dw = DeviceFp8(w)
    bf16_plan = pa.pa_decode_plan(w.num_seqs, w.q_per_seq, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                  w.max_blocks_per_seq, pa.PA_PATH_TILE)
    with pytest.raises(pa.PAError) as exc:
        dw.step(bf16_plan)
    assert exc.value.status == pa.PA_ERR_INVALID_ARG
    for k_scale in (0.0, -1.0, float("nan"), float("inf")):
        with pytest.raises(pa.PAError) as exc:
            pa.pa_decode_fp8(dw.out, dw.query, dw.key_cache, dw.value_cache, dw.tables, dw.ctx, w.q_per_seq,
                             w.scale, k_scale, 1.0)
        assert exc.value.status == pa.PA_ERR_INVALID_ARG


def test_fp8_full_size_llama8b(oracle_lib):
    """The benchmark's FP8 workload at full size, in its launch configuration (the
    heuristic plan), on every output row; a second call gives the same bits."""
    w = workloads.make("llama8b_fp8")
    dw = DeviceFp8(w)
    out = dw.step().clone()
    ref = _oracle(oracle_lib, w)
    mx, mean = assert_close(out, ref, "llama8b_fp8")
    print(f"llama8b_fp8: max |err| {mx:.3e}, mean |err| {mean:.3e}")
    assert torch.equal(dw.step(write=False), out)
    del dw
    torch.cuda.empty_cache()
