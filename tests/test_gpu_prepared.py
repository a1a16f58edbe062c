"""PreparedCacheWrite / PreparedDecode: the step's calls with their arguments built once. Each
call must leave exactly what the per-call entry points leave (same kernels, same plan): the
pools bit for bit, the outputs bit for bit, on bf16 and E4M3 pools, across repeated calls
and after the buffers' contents change in place."""

import math

import pytest
import torch

from gpu_util import DeviceWorkload, assert_close, oracle_pools
from paged_kv_cache_399_b200 import pa, workloads

pytestmark = pytest.mark.gpu

KS, VS = 0.01, 0.013

CASES = [
    ("spec", [900, 33, 2049], 6, 32, 8, 128),    # tcgen05 plan (24 rows)
    ("llama", [700, 300, 45, 1], 1, 32, 8, 128),  # mma.sync tiles, splits
    ("mha64", [129, 64, 17], 1, 4, 4, 64),       # CUDA cores
]


def _ws(plan, w):
    n = pa.pa_decode_workspace_size(plan, w.num_seqs, w.q_per_seq, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                    w.max_blocks_per_seq)
    return torch.empty(max(n, 16), dtype=torch.uint8, device="cuda") if n else None


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_prepared_bf16_step_equals_the_per_call_entry_points(case, oracle_lib):
    name, ctxs, q, hq, hkv, d = case
    w = workloads.build_workload(name, 7100, ctxs, q, hq, hkv, d, scale=1.0 / math.sqrt(d))
    a, b = DeviceWorkload(w), DeviceWorkload(w)
    plan = pa.pa_decode_plan(w.num_seqs, q, hq, hkv, d, w.max_blocks_per_seq)
    ws_a, ws_b = _ws(plan, w), _ws(plan, w)
    pa.pa_reshape_and_cache(a.key, a.value, a.key_cache, a.value_cache, a.slots)
    pa.pa_decode(a.out, a.query, a.key_cache, a.value_cache, a.tables, a.ctx, q, w.scale, plan=plan, workspace=ws_a)
    write = pa.PreparedCacheWrite(b.key, b.value, b.key_cache, b.value_cache, b.slots)
    decode = pa.PreparedDecode(b.out, b.query, b.key_cache, b.value_cache, b.tables, b.ctx, q, w.scale, plan=plan,
                               workspace=ws_b)
    for _ in range(3):   # repeated calls on the same buffers
        write()
        decode()
    torch.cuda.synchronize()
    assert pa.pa_get_device_error(reset=True) == 0
    assert torch.equal(a.key_cache, b.key_cache) and torch.equal(a.value_cache, b.value_cache)
    assert torch.equal(a.out, b.out)
    kc, vc = oracle_pools(oracle_lib, w)
    ref = oracle_lib.decode(w.query, kc, vc, w.block_tables, w.context_lens, q, w.scale)
    assert_close(b.out, ref, f"{name}: prepared")
    # new queries written in place are what the next call reads
    b.query.copy_(b.query.flip(0))
    a.query.copy_(a.query.flip(0))
    decode()
    pa.pa_decode(a.out, a.query, a.key_cache, a.value_cache, a.tables, a.ctx, q, w.scale, plan=plan, workspace=ws_a)
    torch.cuda.synchronize()
    assert torch.equal(a.out, b.out)


def test_prepared_fp8_step_equals_the_per_call_entry_points():
    w = workloads.build_workload("fp8", 7200, [700, 64, 1500], 1, 32, 8, 128, scale=1.0 / math.sqrt(128))
    a, b = DeviceWorkload(w), DeviceWorkload(w)
    for dw in (a, b):
        dw.key_cache = torch.zeros(dw.key_cache.shape, dtype=torch.uint8, device="cuda")
        dw.value_cache = torch.zeros(dw.value_cache.shape, dtype=torch.uint8, device="cuda")
    plan = pa.pa_decode_plan(w.num_seqs, 1, 32, 8, 128, w.max_blocks_per_seq, kv_cache_dtype=pa.PA_KV_FP8_E4M3)
    ws_a, ws_b = _ws(plan, w), _ws(plan, w)
    pa.pa_reshape_and_cache_fp8(a.key, a.value, a.key_cache, a.value_cache, a.slots, KS, VS)
    pa.pa_decode_fp8(a.out, a.query, a.key_cache, a.value_cache, a.tables, a.ctx, 1, w.scale, KS, VS, plan=plan,
                     workspace=ws_a)
    pa.PreparedCacheWrite(b.key, b.value, b.key_cache, b.value_cache, b.slots, k_scale=KS, v_scale=VS)()
    pa.PreparedDecode(b.out, b.query, b.key_cache, b.value_cache, b.tables, b.ctx, 1, w.scale, plan=plan,
                      workspace=ws_b, k_scale=KS, v_scale=VS)()
    torch.cuda.synchronize()
    assert pa.pa_get_device_error(reset=True) == 0
    assert torch.equal(a.key_cache, b.key_cache) and torch.equal(a.value_cache, b.value_cache)
    assert torch.equal(a.out, b.out)


def test_prepared_decode_reports_the_entry_points_errors():
    w = workloads.build_workload("err", 7300, [100, 50], 1, 8, 2, 128, scale=0.1)
    dw = DeviceWorkload(w)
    plan = pa.pa_decode_plan(w.num_seqs, 1, 8, 2, 128, w.max_blocks_per_seq, split_blocks=1)
    need = pa.pa_decode_workspace_size(plan, w.num_seqs, 1, 8, 2, 128, w.max_blocks_per_seq)
    assert need > 0
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    call = pa.PreparedDecode(dw.out, dw.query, dw.key_cache, dw.value_cache, dw.tables, dw.ctx, 1, w.scale,
                             plan=plan, workspace=small)
    with pytest.raises(pa.PAError):
        call()


@pytest.mark.parametrize("case", CASES[:2], ids=[c[0] for c in CASES[:2]])
def test_prepared_decode_in_a_cuda_graph(case):
    """A prepared decode made on the capture stream is captured like the per-call one; the
    replays read the buffers' current contents."""
    name, ctxs, q, hq, hkv, d = case
    w = workloads.build_workload(name, 7400, ctxs, q, hq, hkv, d, scale=1.0 / math.sqrt(d))
    dw = DeviceWorkload(w)
    pa.pa_reshape_and_cache(dw.key, dw.value, dw.key_cache, dw.value_cache, dw.slots)
    plan = pa.pa_decode_plan(w.num_seqs, q, hq, hkv, d, w.max_blocks_per_seq)
    ws = _ws(plan, w)
    ref = torch.empty_like(dw.out)
    pa.pa_decode(ref, dw.query, dw.key_cache, dw.value_cache, dw.tables, dw.ctx, q, w.scale, plan=plan, workspace=ws)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call = pa.PreparedDecode(dw.out, dw.query, dw.key_cache, dw.value_cache, dw.tables, dw.ctx, q, w.scale,
                                 plan=plan, workspace=ws)
        call()
    dw.out.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert pa.pa_get_device_error(reset=True) == 0
    assert torch.equal(dw.out, ref)
    dw.query.mul_(-1.0)   # new contents, same buffer
    graph.replay()
    pa.pa_decode(ref, dw.query, dw.key_cache, dw.value_cache, dw.tables, dw.ctx, q, w.scale, plan=plan, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(dw.out, ref)
    del graph
