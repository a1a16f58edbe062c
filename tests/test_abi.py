"""The C-ABI library: loads, exports every declared symbol, and rejects bad
arguments on the host before any launch (none of these calls touch a GPU)."""

import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pa.h")


def declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"PA_API\s+[\w\s\*]+?\b(pa_\w+)\s*\(", text)


@pytest.fixture(scope="module")
def pa():
    from paged_kv_cache_399_b200 import build
    build.build()
    from paged_kv_cache_399_b200 import pa as mod
    return mod


def test_header_declares_the_hot_path_calls():
    syms = declared_symbols()
    for name in ["pa_reshape_and_cache", "pa_decode", "pa_decode_workspace_size", "pa_decode_plan",
                 "pa_validate", "pa_get_device_error", "pa_copy_blocks", "pa_status_string",
                 "pa_version"]:
        assert name in syms


def test_library_exports_every_declared_symbol(pa):
    out = subprocess.run(["nm", "-D", "--defined-only", pa.library_path()], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in declared_symbols():
        assert name in exported, name
        assert hasattr(pa.raw_library(), name)
    assert set(pa.EXPORTED) == set(declared_symbols())
    # only the C ABI is visible
    assert all(s.startswith("pa_") or not s[0].isalpha() or s.startswith("_") for s in exported
               if not s.startswith(("_init", "_fini"))), sorted(exported)[:20]


def test_status_strings_and_version(pa):
    for code in range(7):
        assert pa.pa_status_string(code).startswith("PA_")
    assert pa.pa_version() == 10200


def _decode_raw(lib, **kw):
    args = dict(out=8 * 1024, query=16 * 1024, kc=32 * 1024, vc=48 * 1024, bt=64 * 1024, cl=80 * 1024,
                B=2, q=1, hq=4, hkv=2, d=64, bs=16, mb=4, nb=8, scale=0.125, plan=None, ws=None,
                ws_bytes=0)
    args.update(kw)
    return lib.pa_decode(args["out"], args["query"], args["kc"], args["vc"], args["bt"], args["cl"],
                         args["B"], args["q"], args["hq"], args["hkv"], args["d"], args["bs"],
                         args["mb"], args["nb"], args["scale"], args["plan"], args["ws"],
                         args["ws_bytes"], None)


def test_decode_rejects_bad_arguments_before_launch(pa):
    lib = pa.raw_library()
    assert _decode_raw(lib, out=None) == pa.PA_ERR_INVALID_ARG
    assert _decode_raw(lib, query=16 * 1024 + 2) == pa.PA_ERR_INVALID_ARG      # misaligned
    assert _decode_raw(lib, hq=3) == pa.PA_ERR_INVALID_ARG                     # H_q % H_kv
    assert _decode_raw(lib, d=96) == pa.PA_ERR_UNSUPPORTED
    assert _decode_raw(lib, bs=32) == pa.PA_ERR_UNSUPPORTED
    assert _decode_raw(lib, q=17) == pa.PA_ERR_UNSUPPORTED
    assert _decode_raw(lib, q=0) == pa.PA_ERR_INVALID_ARG
    assert _decode_raw(lib, scale=float("nan")) == pa.PA_ERR_INVALID_ARG
    assert _decode_raw(lib, B=0) == pa.PA_OK                                    # no-op
    # a split plan needs a workspace
    plan = pa.pa_decode_plan(2, 1, 4, 2, 64, 4, pa.PA_PATH_TILE, 1)
    assert plan.num_splits == 4
    assert _decode_raw(lib, plan=ctypes.byref(plan)) == pa.PA_ERR_WORKSPACE
    need = pa.pa_decode_workspace_size(plan, 2, 1, 4, 2, 64, 4)
    assert need == 2 * 4 * 1 * 4 * (64 + 2) * 4
    assert _decode_raw(lib, plan=ctypes.byref(plan), ws=96 * 1024, ws_bytes=need - 1) == pa.PA_ERR_WORKSPACE
    bad = pa.pa_plan_t.from_buffer_copy(plan)
    bad.num_splits += 1
    assert _decode_raw(lib, plan=ctypes.byref(bad), ws=96 * 1024, ws_bytes=need) == pa.PA_ERR_INVALID_ARG
    # the persistent schedule always needs its pre-pass tables
    pplan = pa.pa_decode_plan(2, 1, 4, 2, 64, 4, pa.PA_PATH_TILE, schedule=pa.PA_SCHEDULE_PERSISTENT)
    pneed = pa.pa_decode_workspace_size(pplan, 2, 1, 4, 2, 64, 4)
    assert pneed > 0
    assert _decode_raw(lib, plan=ctypes.byref(pplan)) == pa.PA_ERR_WORKSPACE


def test_cache_write_rejects_bad_arguments_before_launch(pa):
    lib = pa.raw_library()

    def call(**kw):
        a = dict(k=1024, v=2048, ks=128, vs=128, kc=4096, vc=8192, slots=16384, T=4, hkv=2, d=64,
                 nb=8, bs=16)
        a.update(kw)
        return lib.pa_reshape_and_cache(a["k"], a["v"], a["ks"], a["vs"], a["kc"], a["vc"], a["slots"],
                                        a["T"], a["hkv"], a["d"], a["nb"], a["bs"], None)
    assert call(k=None) == pa.PA_ERR_INVALID_ARG
    assert call(kc=4096 + 8) == pa.PA_ERR_INVALID_ARG
    assert call(ks=100) == pa.PA_ERR_INVALID_ARG          # stride below a row
    assert call(ks=132) == pa.PA_ERR_INVALID_ARG          # stride*2 not a multiple of 16
    assert call(slots=16384 + 4) == pa.PA_ERR_INVALID_ARG
    assert call(bs=8) == pa.PA_ERR_UNSUPPORTED
    assert call(T=0, k=None) == pa.PA_OK                  # no-op


def test_copy_blocks_rejects_bad_mappings_before_launch(pa):
    """Every check of pa_copy_blocks runs on the host before any CUDA call (the pools
    are never touched here, so fake aligned addresses stand in for them)."""
    import numpy as np
    lib = pa.raw_library()

    def call(pairs, **kw):
        a = dict(kc=4096, vc=8192, nb=10, hkv=2, d=64, bs=16)
        a.update(kw)
        m = np.ascontiguousarray(np.asarray(pairs, dtype=np.int64).reshape(-1, 2))
        return lib.pa_copy_blocks(a["kc"], a["vc"], a["nb"], a["hkv"], a["d"], a["bs"],
                                  m.ctypes.data if m.shape[0] else None, m.shape[0], None)
    assert call([]) == pa.PA_OK                                   # no-op
    assert call([[1, 2]], kc=None) == pa.PA_ERR_INVALID_ARG
    assert call([[1, 2]], vc=8192 + 4) == pa.PA_ERR_INVALID_ARG
    assert call([[1, 2]], bs=32) == pa.PA_ERR_UNSUPPORTED
    assert call([[1, 2]], d=96) == pa.PA_ERR_UNSUPPORTED
    assert call([[1, 10]]) == pa.PA_ERR_OUT_OF_RANGE              # past the pool
    assert call([[10, 1]]) == pa.PA_ERR_OUT_OF_RANGE
    assert call([[1, 3], [2, 3]]) == pa.PA_ERR_INVALID_ARG        # a destination twice
    assert call([[1, 3], [3, 4]]) == pa.PA_ERR_INVALID_ARG        # a destination also a source
    assert lib.pa_copy_blocks(4096, 8192, 10, 2, 64, 16, None, -1, None) == pa.PA_ERR_INVALID_ARG


def test_plan_heuristic_host_logic(pa):
    # rows = G*q <= 2 -> CUDA-core kernel; more rows -> tensor-core tiles
    assert pa.pa_decode_plan(4, 1, 4, 2, 64, 5).path == pa.PA_PATH_SINGLE
    p = pa.pa_decode_plan(32, 6, 32, 8, 64, 1024)      # 24 rows, head_dim 64: mma.sync tiles
    assert p.path == pa.PA_PATH_TILE and p.rows_per_cta == 24
    p = pa.pa_decode_plan(32, 6, 32, 8, 128, 1024)     # 24 rows, head_dim 128: tcgen05
    assert (p.path, p.schedule, p.rows_per_cta) == (pa.PA_PATH_TCGEN05, pa.PA_SCHEDULE_PERSISTENT, 32)
    p = pa.pa_decode_plan(64, 1, 32, 8, 128, 256)      # 4 rows: mma.sync tiles, grid schedule
    assert (p.path, p.schedule, p.rows_per_cta) == (pa.PA_PATH_TILE, pa.PA_SCHEDULE_GRID, 8)
    p = pa.pa_decode_plan(32, 6, 32, 8, 128, 1024, split_blocks=16)   # a forced split: grid tiles
    assert (p.path, p.schedule) == (pa.PA_PATH_TILE, pa.PA_SCHEDULE_GRID)
    p = pa.pa_decode_plan(4, 1, 64, 8, 128, 8192, schedule=pa.PA_SCHEDULE_PERSISTENT)
    assert p.schedule == pa.PA_SCHEDULE_PERSISTENT and p.num_ctas >= 1 and p.share_cap == 0
    p = pa.pa_decode_plan(4, 1, 64, 8, 128, 8192, schedule=pa.PA_SCHEDULE_GRID)
    assert p.num_splits > 1 and p.split_blocks * p.num_splits >= 8192
    # prefix sharing: a shared unit holds 32 rows = 8 sequences of 4 rows; automatic choice:
    # tcgen05 windows; mma.sync grid or persistent sharing on request
    p = pa.pa_decode_plan(128, 1, 32, 8, 128, 144, share_prefix=True)
    assert (p.path, p.schedule, p.rows_per_cta, p.share_cap) == (3, 2, 32, 8)
    assert pa.pa_decode_workspace_size(p, 128, 1, 32, 8, 128, 144) > 0
    p = pa.pa_decode_plan(128, 1, 32, 8, 128, 144, pa.PA_PATH_TILE, share_prefix=True)
    assert (p.path, p.schedule, p.rows_per_cta, p.share_cap) == (2, 1, 32, 8)
    assert pa.pa_decode_workspace_size(p, 128, 1, 32, 8, 128, 144) > 0
    p = pa.pa_decode_plan(128, 1, 32, 8, 128, 144, pa.PA_PATH_TILE, share_prefix=True,
                          schedule=pa.PA_SCHEDULE_PERSISTENT)
    assert (p.path, p.schedule, p.rows_per_cta, p.share_cap) == (2, 2, 32, 8)
    with pytest.raises(pa.PAError) as exc:   # 24 rows per sequence: two do not fit 32 rows
        pa.pa_decode_plan(32, 6, 32, 8, 128, 1024, share_prefix=True)
    assert exc.value.status == pa.PA_ERR_UNSUPPORTED
    # tcgen05: N = 16 or 32 rows per unit, its own persistent equal-tile schedule
    p = pa.pa_decode_plan(32, 6, 32, 8, 128, 1024, pa.PA_PATH_TCGEN05)
    assert (p.path, p.schedule, p.rows_per_cta, p.num_splits) == (3, 2, 32, 1) and p.num_ctas >= 1
    p = pa.pa_decode_plan(64, 1, 32, 8, 128, 256, pa.PA_PATH_TCGEN05)
    assert (p.path, p.schedule, p.rows_per_cta) == (3, 2, 16)
    assert pa.pa_decode_workspace_size(p, 64, 1, 32, 8, 128, 256) >= 2 * p.num_ctas * (16 * 128 + 32) * 4
    with pytest.raises(pa.PAError):          # no grid schedule on the tcgen05 path
        pa.pa_decode_plan(32, 6, 32, 8, 128, 1024, pa.PA_PATH_TCGEN05, schedule=pa.PA_SCHEDULE_GRID)
    with pytest.raises(pa.PAError):          # head_dim 128 only
        pa.pa_decode_plan(32, 6, 32, 8, 64, 1024, pa.PA_PATH_TCGEN05)
    # prefix sharing on the tcgen05 path: windows of 8 sequences x 4 rows = N 32
    p = pa.pa_decode_plan(8, 1, 32, 8, 128, 64, pa.PA_PATH_TCGEN05, share_prefix=True)
    assert (p.path, p.schedule, p.rows_per_cta, p.share_cap) == (3, 2, 32, 8)
    forced = pa.pa_decode_plan(4, 1, 64, 8, 128, 8192, pa.PA_PATH_SINGLE, 64)
    assert (forced.path, forced.split_blocks, forced.num_splits, forced.rows_per_cta) == (1, 64, 128, 8)
    # rows beyond one CTA are split into row chunks
    assert pa.pa_decode_plan(2, 16, 16, 1, 128, 8).rows_per_cta == 32
    with pytest.raises(pa.PAError):
        pa.pa_decode_plan(2, 1, 4, 2, 80, 8)


@pytest.mark.parametrize("hints", [
    {}, {"path": 1}, {"path": 2}, {"path": 3}, {"schedule": 2}, {"path": 1, "schedule": 2},
    {"share_prefix": True}, {"share_prefix": True, "schedule": 2}, {"split_blocks": 3},
    {"path": 3, "split_blocks": 2}, {"share_prefix": True, "split_blocks": 5},
    {"path": 3, "share_prefix": True},
    {"sliding_window": 64}, {"sliding_window": 64, "path": 1}, {"sliding_window": 17, "split_blocks": 2},
    {"sliding_window": 5000},
])
def test_every_plan_passes_decode_validation(pa, hints):
    """A plan from pa_decode_plan is accepted by pa_decode's own checks (on a machine
    without a GPU the call then stops at the first CUDA call, never at validation)."""
    lib = pa.raw_library()
    B, q, hq, hkv, d, mb = 8, 1, 8, 2, 128, 40
    plan = pa.pa_decode_plan(B, q, hq, hkv, d, mb, **hints)
    need = pa.pa_decode_workspace_size(plan, B, q, hq, hkv, d, mb)
    st = _decode_raw(lib, B=B, q=q, hq=hq, hkv=hkv, d=d, mb=mb, nb=400, plan=ctypes.byref(plan),
                     ws=1 << 20, ws_bytes=need)
    assert st not in (pa.PA_ERR_INVALID_ARG, pa.PA_ERR_UNSUPPORTED, pa.PA_ERR_WORKSPACE), (plan, st)


def test_window_plans_on_the_host(pa):
    """Sliding-window plans: the grid schedule (splits over the window's span of blocks) or
    the tcgen05 kernel; prefix sharing and the mma.sync persistent schedule are refused
    before any device query."""
    lib = pa.raw_library()
    plan = pa.pa_plan_t()
    for hints in ((2, 2, 0, 0, 64), (0, 2, 0, 0, 64), (2, 0, 0, 1, 64), (3, 0, 0, 1, 64)):
        h = pa.pa_plan_hints_t(*hints)
        assert lib.pa_decode_plan(4, 1, 32, 8, 128, 64, ctypes.byref(h), ctypes.byref(plan)) == \
            pa.PA_ERR_UNSUPPORTED, hints
    h = pa.pa_plan_hints_t(0, 0, 0, 0, -1)
    assert lib.pa_decode_plan(4, 1, 32, 8, 128, 64, ctypes.byref(h), ctypes.byref(plan)) == pa.PA_ERR_INVALID_ARG
    # 24 rows at head_dim 128: the tcgen05 kernel, window or not
    p = pa.pa_decode_plan(32, 6, 32, 8, 128, 1024, sliding_window=4096)
    assert (p.path, p.schedule, p.sliding_window) == (pa.PA_PATH_TCGEN05, pa.PA_SCHEDULE_PERSISTENT, 4096)
    # 4 rows: the mma.sync tiles on the grid, splits over the window's span
    p = pa.pa_decode_plan(32, 1, 32, 8, 128, 1024, sliding_window=4096)
    assert (p.path, p.schedule, p.sliding_window) == (pa.PA_PATH_TILE, pa.PA_SCHEDULE_GRID, 4096)
    span = -(-(4096 + 1 - 1) // 16) + 1
    assert p.split_blocks <= span and p.num_splits == -(-span // p.split_blocks)
    p = pa.pa_decode_plan(4, 1, 32, 8, 128, 64, sliding_window=100000)   # wider than the table
    assert p.num_splits == -(-64 // p.split_blocks)


def test_window_plan_covers_every_visible_block(pa):
    """The grid kernel walks a sequence's blocks from the window's first block,
    floor(max(0, ctx - q - W + 1) / 16), in num_splits pieces of split_blocks: the plan must
    leave room for every block up to ceil(ctx / 16) at every context the table allows."""
    for W in (1, 5, 15, 16, 17, 31, 100, 1000, 4096):
        for q in (1, 2, 6, 16):
            for mb in (1, 3, 64, 257, 2048):
                for forced in (0, 1, 3):
                    p = pa.pa_decode_plan(4, q, 8, 2, 128, mb, split_blocks=forced, sliding_window=W)
                    ctx = np.arange(q, mb * 16 + 1)
                    need = -(-ctx // 16) - np.maximum(0, ctx - q - W + 1) // 16
                    assert int(need.max()) <= p.num_splits * p.split_blocks, (W, q, mb, forced, p)


def test_fp8_cache_write_rejects_bad_arguments_before_launch(pa):
    lib = pa.raw_library()

    def call(**kw):
        a = dict(k=1024, v=2048, ks=128, vs=128, kc=4096, vc=8192, slots=16384, T=4, hkv=2, d=64,
                 nb=8, bs=16, kscale=0.5, vscale=0.5)
        a.update(kw)
        return lib.pa_reshape_and_cache_fp8(a["k"], a["v"], a["ks"], a["vs"], a["kc"], a["vc"], a["slots"],
                                            a["T"], a["hkv"], a["d"], a["nb"], a["bs"], a["kscale"], a["vscale"],
                                            None)
    assert call(k=None) == pa.PA_ERR_INVALID_ARG
    assert call(kc=4096 + 8) == pa.PA_ERR_INVALID_ARG
    assert call(ks=100) == pa.PA_ERR_INVALID_ARG
    assert call(kscale=0.0) == pa.PA_ERR_INVALID_ARG
    assert call(vscale=float("nan")) == pa.PA_ERR_INVALID_ARG
    assert call(kscale=float("inf")) == pa.PA_ERR_INVALID_ARG
    assert call(bs=8) == pa.PA_ERR_UNSUPPORTED
    assert call(hkv=1, d=8) == pa.PA_ERR_UNSUPPORTED   # a row of 8 elements: not a multiple of 16
    assert call(T=0, k=None) == pa.PA_OK


def test_size_query_and_static_scratch_check_before_sizing(pa):
    """The workspace size of a caller plan divides by plan and shape fields: both the size
    query and pa_decode_static_scratch run pa_decode's checks first (no SIGFPE, and the same
    status pa_decode returns)."""
    lib = pa.raw_library()
    size = lib.pa_decode_workspace_size
    plan = pa.pa_decode_plan(2, 1, 4, 2, 64, 4, pa.PA_PATH_TILE, schedule=pa.PA_SCHEDULE_PERSISTENT)
    assert size(ctypes.byref(plan), 2, 1, 4, 2, 64, 4) > 0
    assert size(ctypes.byref(plan), 2, 1, 4, 0, 64, 4) == 0            # num_kv_heads = 0
    assert size(ctypes.byref(plan), -3, 1, 4, 2, 64, 4) == 0           # negative num_seqs
    zeroed = pa.pa_plan_t()
    zeroed.path, zeroed.schedule = pa.PA_PATH_TILE, pa.PA_SCHEDULE_PERSISTENT
    assert size(ctypes.byref(zeroed), 2, 1, 4, 2, 64, 4) == 0
    zeroed.num_ctas = 4                                                # rows_per_cta still 0
    assert size(ctypes.byref(zeroed), 2, 1, 4, 2, 64, 4) == 0

    def static(plan_ref, B=2, hkv=2):
        return lib.pa_decode_static_scratch(8 * 1024, 16 * 1024, 32 * 1024, 48 * 1024, 64 * 1024, 80 * 1024,
                                            B, 1, 4, hkv, 64, 16, 4, 8, 0.125, plan_ref, None)
    assert static(ctypes.byref(plan), hkv=0) == pa.PA_ERR_INVALID_ARG
    assert static(ctypes.byref(plan), B=-3) == pa.PA_ERR_INVALID_ARG
    assert static(ctypes.byref(zeroed)) == pa.PA_ERR_INVALID_ARG
    assert _decode_raw(lib, plan=ctypes.byref(zeroed), ws=96 * 1024, ws_bytes=1 << 20) == pa.PA_ERR_INVALID_ARG


def _decode_fp8_raw(lib, ks=0.01, vs=0.01, **kw):
    args = dict(out=8 * 1024, query=16 * 1024, kc=32 * 1024, vc=48 * 1024, bt=64 * 1024, cl=80 * 1024,
                B=2, q=1, hq=4, hkv=2, d=64, bs=16, mb=4, nb=8, scale=0.125, plan=None, ws=None,
                ws_bytes=0)
    args.update(kw)
    return lib.pa_decode_fp8(args["out"], args["query"], args["kc"], args["vc"], args["bt"], args["cl"],
                             args["B"], args["q"], args["hq"], args["hkv"], args["d"], args["bs"],
                             args["mb"], args["nb"], args["scale"], ks, vs, args["plan"], args["ws"],
                             args["ws_bytes"], None)


def test_fp8_plans_on_the_host(pa):
    """FP8 pools are read by the mma.sync tiles: the automatic FP8 plan takes them, the
    CUDA-core and tcgen05 kernels are refused, and a plan only decodes the pools it was made
    for (before any device work)."""
    lib = pa.raw_library()
    fp8 = pa.PA_KV_FP8_E4M3
    p = pa.pa_decode_plan(32, 6, 32, 8, 128, 1024, kv_cache_dtype=fp8)   # 24 rows: tcgen05 for bf16
    assert (p.path, p.kv_cache_dtype) == (pa.PA_PATH_TILE, fp8)
    p = pa.pa_decode_plan(4, 1, 4, 2, 64, 8, kv_cache_dtype=fp8)          # 2 rows: CUDA cores for bf16
    assert p.path == pa.PA_PATH_TILE
    for path in (pa.PA_PATH_SINGLE, pa.PA_PATH_TCGEN05):
        with pytest.raises(pa.PAError) as exc:
            pa.pa_decode_plan(4, 1, 32, 8, 128, 64, path, kv_cache_dtype=fp8)
        assert exc.value.status == pa.PA_ERR_UNSUPPORTED
    h = pa.pa_plan_hints_t(0, 0, 0, 0, 0, 2)
    plan = pa.pa_plan_t()
    assert lib.pa_decode_plan(4, 1, 32, 8, 128, 64, ctypes.byref(h), ctypes.byref(plan)) == pa.PA_ERR_INVALID_ARG
    for hints in ({}, {"schedule": pa.PA_SCHEDULE_PERSISTENT}, {"share_prefix": True}, {"split_blocks": 3},
                  {"sliding_window": 40}):
        p = pa.pa_decode_plan(2, 1, 4, 2, 64, 4, kv_cache_dtype=fp8, **hints)
        need = pa.pa_decode_workspace_size(p, 2, 1, 4, 2, 64, 4)
        # a plan for FP8 pools is refused by pa_decode, accepted by pa_decode_fp8's checks
        assert _decode_raw(lib, plan=ctypes.byref(p), ws=96 * 1024, ws_bytes=need) == pa.PA_ERR_INVALID_ARG
        st = _decode_fp8_raw(lib, plan=ctypes.byref(p), ws=96 * 1024, ws_bytes=need)
        assert st not in (pa.PA_ERR_INVALID_ARG, pa.PA_ERR_UNSUPPORTED, pa.PA_ERR_WORKSPACE), (hints, st)
    bf16_plan = pa.pa_decode_plan(2, 1, 4, 2, 64, 4, pa.PA_PATH_TILE)
    assert _decode_fp8_raw(lib, plan=ctypes.byref(bf16_plan)) == pa.PA_ERR_INVALID_ARG
    forged = pa.pa_plan_t.from_buffer_copy(pa.pa_decode_plan(2, 1, 4, 2, 64, 4, kv_cache_dtype=fp8))
    forged.path = pa.PA_PATH_SINGLE
    forged.rows_per_cta = 2
    assert _decode_fp8_raw(lib, plan=ctypes.byref(forged)) == pa.PA_ERR_INVALID_ARG
    for ks, vs in ((0.0, 1.0), (1.0, -2.0), (float("nan"), 1.0), (1.0, float("inf"))):
        assert _decode_fp8_raw(lib, ks=ks, vs=vs) == pa.PA_ERR_INVALID_ARG


def test_prefill_rejects_bad_arguments_before_launch(pa):
    lib = pa.raw_library()

    def call(**kw):
        a = dict(out=8192, q=16384, kc=32768, vc=49152, bt=65536, cl=81920, qs=98304, B=2, T=10, mq=8, hq=32,
                 hkv=8, d=128, bs=16, mb=8, nb=64, scale=0.088)
        a.update(kw)
        return lib.pa_prefill(a["out"], a["q"], a["kc"], a["vc"], a["bt"], a["cl"], a["qs"], a["B"], a["T"], a["mq"],
                              a["hq"], a["hkv"], a["d"], a["bs"], a["mb"], a["nb"], a["scale"], None)
    assert call(d=64) == pa.PA_ERR_UNSUPPORTED             # head_dim 128 only
    assert call(hq=24, hkv=8) == pa.PA_ERR_UNSUPPORTED     # G = 3 does not divide 128
    assert call(bs=32) == pa.PA_ERR_UNSUPPORTED
    assert call(hq=30, hkv=8) == pa.PA_ERR_INVALID_ARG     # H_q % H_kv
    assert call(qs=None) == pa.PA_ERR_INVALID_ARG
    assert call(out=8192 + 8) == pa.PA_ERR_INVALID_ARG     # misaligned
    assert call(cl=81920 + 2) == pa.PA_ERR_INVALID_ARG
    assert call(scale=float("inf")) == pa.PA_ERR_INVALID_ARG
    assert call(scale=-0.5) == pa.PA_ERR_INVALID_ARG        # the row maximum is taken on raw scores
    assert call(B=-1) == pa.PA_ERR_INVALID_ARG
    assert call(B=0) == pa.PA_OK and call(T=0) == pa.PA_OK and call(mq=0) == pa.PA_OK   # no-ops
    assert call(mq=3_000_000) == pa.PA_ERR_UNSUPPORTED     # more tiles than the grid holds


def test_partial_decode_and_merge_reject_bad_arguments_before_launch(pa):
    """Context parallelism's entry points: host checks that return before any launch (fake
    device addresses are never dereferenced)."""
    lib = pa.raw_library()

    def partial(**kw):
        a = dict(po=8192, pml=16384, q=24576, kc=32768, vc=49152, bt=65536, cl=81920, B=2, qs=1, hq=8, hkv=2,
                 d=128, bs=16, mb=8, nb=64, scale=0.088, lo=0, hi=8, S=2)
        a.update(kw)
        return lib.pa_decode_partial(a["po"], a["pml"], a["q"], a["kc"], a["vc"], a["bt"], a["cl"], a["B"], a["qs"],
                                     a["hq"], a["hkv"], a["d"], a["bs"], a["mb"], a["nb"], a["scale"], a["lo"],
                                     a["hi"], a["S"], None)
    assert partial(lo=-1) == pa.PA_ERR_INVALID_ARG
    assert partial(S=0) == pa.PA_ERR_INVALID_ARG
    assert partial(lo=5, hi=4) == pa.PA_ERR_INVALID_ARG      # an inverted range
    assert partial(hi=9) == pa.PA_ERR_INVALID_ARG            # past the table
    assert partial(po=None) == pa.PA_ERR_INVALID_ARG
    assert partial(pml=16384 + 8) == pa.PA_ERR_INVALID_ARG   # misaligned
    assert partial(hq=7) == pa.PA_ERR_INVALID_ARG            # H_q % H_kv
    assert partial(d=96) == pa.PA_ERR_UNSUPPORTED
    assert partial(qs=17) == pa.PA_ERR_UNSUPPORTED
    assert partial(B=0, po=None, pml=None) == pa.PA_OK       # nothing to do

    def merge(**kw):
        a = dict(out=8192, po=16384, pml=32768, P=3, B=2, qs=1, hq=8, d=128)
        a.update(kw)
        return lib.pa_merge_partials(a["out"], a["po"], a["pml"], a["P"], a["B"], a["qs"], a["hq"], a["d"], None)
    assert merge(P=0) == pa.PA_ERR_INVALID_ARG
    assert merge(B=-1) == pa.PA_ERR_INVALID_ARG
    assert merge(out=None) == pa.PA_ERR_INVALID_ARG
    assert merge(po=16384 + 4) == pa.PA_ERR_INVALID_ARG
    assert merge(d=96) == pa.PA_ERR_UNSUPPORTED
    assert merge(B=0, out=None) == pa.PA_OK
    def combine(**kw):
        a = dict(ro=8192, rml=16384, po=32768, pml=49152, P=3, B=2, qs=1, hq=8, d=128)
        a.update(kw)
        return lib.pa_combine_partials(a["ro"], a["rml"], a["po"], a["pml"], a["P"], a["B"], a["qs"], a["hq"],
                                       a["d"], None)
    assert combine(P=0) == pa.PA_ERR_INVALID_ARG
    assert combine(ro=None) == pa.PA_ERR_INVALID_ARG
    assert combine(rml=16384 + 8) == pa.PA_ERR_INVALID_ARG
    assert combine(d=32) == pa.PA_ERR_UNSUPPORTED
    assert combine(B=0, ro=None) == pa.PA_OK
    # pieces of a range: at least one for good shapes, 0 for bad ones
    assert pa.pa_decode_partial_pieces(4, 1, 64, 8, 128, 1024) >= 1
    assert pa.pa_decode_partial_pieces(4, 1, 64, 8, 96, 1024) == 0
    assert pa.pa_decode_partial_pieces(4, 1, 64, 8, 128, -1) == 0


def test_prepared_calls_check_their_tensors_once_on_the_host(pa):
    """PreparedDecode / PreparedCacheWrite build their C arguments at construction (host only,
    stream given as a handle): wrong dtypes, layouts or scale arguments are refused there."""
    import torch
    B, q, HQ, HKV, D, NB, MB = 2, 1, 8, 2, 128, 8, 4
    out = torch.zeros(B, q, HQ, D, dtype=torch.bfloat16)
    query = torch.zeros(B, q, HQ, D, dtype=torch.bfloat16)
    kc = torch.zeros(NB, 16, HKV, D, dtype=torch.bfloat16)
    vc = torch.zeros_like(kc)
    tables = torch.zeros(B, MB, dtype=torch.int32)
    ctx = torch.ones(B, dtype=torch.int32)
    call = pa.PreparedDecode(out, query, kc, vc, tables, ctx, q, 0.1, stream=0)
    assert call._args[6:14] == (B, q, HQ, HKV, D, 16, MB, NB)
    with pytest.raises(TypeError):
        pa.PreparedDecode(out, query, kc, vc, tables.long(), ctx, q, 0.1, stream=0)
    with pytest.raises(ValueError):
        pa.PreparedDecode(out, query, kc, vc, tables.t().contiguous().t(), ctx, q, 0.1, stream=0)
    with pytest.raises(ValueError):   # scales belong to E4M3 pools
        pa.PreparedDecode(out, query, kc, vc, tables, ctx, q, 0.1, stream=0, k_scale=1.0, v_scale=1.0)
    with pytest.raises(ValueError):   # q_per_seq disagrees with the query
        pa.PreparedDecode(out, query, kc, vc, tables, ctx, 2, 0.1, stream=0)
    k8 = torch.zeros(NB, 16, HKV, D, dtype=torch.uint8)
    with pytest.raises(ValueError):   # E4M3 pools need both scales
        pa.PreparedDecode(out, query, k8, k8.clone(), tables, ctx, q, 0.1, stream=0)
    pa.PreparedDecode(out, query, k8, k8.clone(), tables, ctx, q, 0.1, stream=0, k_scale=0.5, v_scale=0.5)
    key = torch.zeros(3, HKV, D, dtype=torch.bfloat16)
    slots = torch.zeros(3, dtype=torch.int64)
    pa.PreparedCacheWrite(key, key.clone(), kc, vc, slots, stream=0)
    with pytest.raises(TypeError):
        pa.PreparedCacheWrite(key, key.clone(), kc, vc, slots.int(), stream=0)
    with pytest.raises(ValueError):
        pa.PreparedCacheWrite(key, key.clone(), k8, k8.clone(), slots, stream=0)


def test_tcgen05_decode_refuses_shapes_past_its_scan_range(pa):
    """The tcgen05 kernel's range scan packs (tiles, units) sums in 64 bits: a decode whose
    units (sequence x kv head x row chunk) reach 2^28, or whose tiles reach 2^35, is refused
    on the host (PA_ERR_UNSUPPORTED) before the workspace check and before any launch."""
    fake = 1 << 12   # aligned non-null pointers: nothing is read before the refusal
    for B, hq, hkv, mb in [(65535, 8192, 8192, 4), (65535, 64, 64, 65536)]:
        plan = pa.pa_decode_plan(B, 1, hq, hkv, 128, mb, path=3)
        assert plan.path == 3
        st = pa._lib.pa_decode(fake, fake, fake, fake, fake, fake, B, 1, hq, hkv, 128, 16, mb, 1000, 0.1,
                               ctypes.byref(plan), None, 0, None)
        assert st == pa.PA_ERR_UNSUPPORTED, (B, hq, hkv, mb, st)
