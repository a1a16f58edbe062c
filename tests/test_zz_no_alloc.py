"""pa_decode_static_scratch -- the decode entry point for callers that cannot
allocate device memory where they decode -- against pa_decode with a caller
workspace. Collected last on purpose (file name) so that, under -x, every other
test has run before it; it also passes alone in a fresh process.
"""

import math

import numpy as np
import pytest
import torch

from gpu_util import MAX_ABS_TOL, MEAN_ABS_TOL, DeviceWorkload
from paged_kv_cache_399_b200 import workloads

pytestmark = pytest.mark.gpu


def _close(a: torch.Tensor, b: torch.Tensor, what: str):
    err = (a.double() - b.double()).abs()
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL, f"{what}: max {mx:.3e} mean {mean:.3e}"


def _workload():
    rng = np.random.default_rng(3101)
    ctx = rng.integers(500, 4000, size=16, endpoint=True)
    return workloads.build_workload("noalloc", 3100, ctx, 2, 32, 8, 128, scale=1.0 / math.sqrt(128))


def _spec_workload():
    """q_per_seq 6 at 32/8 heads: 24 rows per kv head, the tcgen05 kernel's shape."""
    rng = np.random.default_rng(3103)
    ctx = rng.integers(6, 3000, size=12, endpoint=True)
    return workloads.build_workload("noalloc_spec", 3102, ctx, 6, 32, 8, 128, scale=1.0 / math.sqrt(128))


def _shared_workload():
    """Two groups of adjacent sequences over common prefix blocks (parallel sampling)."""
    rng = np.random.default_rng(3105)
    ctx = [512 + int(t) for t in rng.integers(1, 200, size=16)]
    groups = [(list(range(0, 8)), 512), (list(range(8, 16)), 512)]
    return workloads.build_workload("noalloc_shared", 3104, ctx, 1, 32, 8, 128, scale=1.0 / math.sqrt(128),
                                    pool_factor=1.5, share_groups=groups)


def _plans(w, pa):
    def plan(**hints):
        return pa.pa_decode_plan(w.num_seqs, w.q_per_seq, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                 w.max_blocks_per_seq, **hints)
    return plan


def test_static_scratch_matches_pa_decode_on_two_calls_in_a_row():
    """Every schedule whose workspace holds state between its kernels (split records, the
    persistent schedule's counters and lists, the tcgen05 descriptors and prefix lengths)
    goes through the array right after a call of another shape or plan, so the array holds
    that call's contents when the next one starts."""
    from paged_kv_cache_399_b200 import pa
    cases = []
    w = _workload()
    mk = _plans(w, pa)
    cases += [(w, None), (w, mk(path=pa.PA_PATH_TILE, split_blocks=16)),
              (w, mk(path=pa.PA_PATH_SINGLE, split_blocks=48)),
              (w, mk(path=pa.PA_PATH_TILE, schedule=pa.PA_SCHEDULE_PERSISTENT))]
    ws_ = _spec_workload()
    cases += [(ws_, _plans(ws_, pa)(path=pa.PA_PATH_TCGEN05))]
    wsh = _shared_workload()
    mk = _plans(wsh, pa)
    cases += [(wsh, mk(path=pa.PA_PATH_TILE, schedule=pa.PA_SCHEDULE_PERSISTENT, share_prefix=True)),
              (ws_, _plans(ws_, pa)(path=pa.PA_PATH_TILE, schedule=pa.PA_SCHEDULE_PERSISTENT)),
              (wsh, mk(path=pa.PA_PATH_TCGEN05, share_prefix=True)),
              (w, _plans(w, pa)(path=pa.PA_PATH_TCGEN05))]
    devs = {}
    for w, plan in cases:
        if id(w) not in devs:
            dw = DeviceWorkload(w)
            pa.pa_reshape_and_cache(dw.key, dw.value, dw.key_cache, dw.value_cache, dw.slots)
            devs[id(w)] = dw
        dw = devs[id(w)]
        need = pa.pa_decode_workspace_size(plan, w.num_seqs, w.q_per_seq, w.num_q_heads,
                                           w.num_kv_heads, w.head_dim, w.max_blocks_per_seq)
        assert need <= pa.PA_STATIC_SCRATCH_BYTES
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
        ref = torch.empty_like(dw.query)
        pa.pa_decode(ref, dw.query, dw.key_cache, dw.value_cache, dw.tables, dw.ctx, w.q_per_seq,
                     w.scale, plan=plan, workspace=ws)
        outs = []
        for _ in range(2):  # the array keeps the previous call's contents
            out = torch.full_like(dw.query, float("nan"))
            pa.pa_decode_static_scratch(out, dw.query, dw.key_cache, dw.value_cache, dw.tables, dw.ctx,
                                        w.q_per_seq, w.scale, plan=plan)
            outs.append(out)
        torch.cuda.synchronize()
        assert pa.pa_get_device_error(reset=True) == 0
        for k, out in enumerate(outs):
            assert bool(torch.isfinite(out.float()).all())
            _close(out, ref, f"{w.name} plan {plan} call {k}")


def test_static_scratch_rejects_plans_beyond_its_size():
    from paged_kv_cache_399_b200 import pa
    w = _workload()
    dw = DeviceWorkload(w)
    plan = pa.pa_decode_plan(w.num_seqs, w.q_per_seq, w.num_q_heads, w.num_kv_heads, w.head_dim,
                             w.max_blocks_per_seq, pa.PA_PATH_TILE, 1)
    need = pa.pa_decode_workspace_size(plan, w.num_seqs, w.q_per_seq, w.num_q_heads, w.num_kv_heads,
                                       w.head_dim, w.max_blocks_per_seq)
    assert need > pa.PA_STATIC_SCRATCH_BYTES
    sentinel = torch.full_like(dw.query, 7.0)
    out = sentinel.clone()
    with pytest.raises(pa.PAError) as exc:
        pa.pa_decode_static_scratch(out, dw.query, dw.key_cache, dw.value_cache, dw.tables, dw.ctx,
                                    w.q_per_seq, w.scale, plan=plan)
    assert exc.value.status == pa.PA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.equal(out, sentinel)  # nothing was launched
