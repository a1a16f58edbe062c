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


def test_static_scratch_matches_pa_decode_on_two_calls_in_a_row():
    from paged_kv_cache_399_b200 import pa
    w = _workload()
    dw = DeviceWorkload(w)
    pa.pa_reshape_and_cache(dw.key, dw.value, dw.key_cache, dw.value_cache, dw.slots)
    plans = [None,  # heuristic
             pa.pa_decode_plan(w.num_seqs, w.q_per_seq, w.num_q_heads, w.num_kv_heads, w.head_dim,
                               w.max_blocks_per_seq, pa.PA_PATH_TILE, 16),
             pa.pa_decode_plan(w.num_seqs, w.q_per_seq, w.num_q_heads, w.num_kv_heads, w.head_dim,
                               w.max_blocks_per_seq, pa.PA_PATH_SINGLE, 48)]
    for plan in plans:
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
            _close(out, ref, f"plan {plan} call {k}")


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
