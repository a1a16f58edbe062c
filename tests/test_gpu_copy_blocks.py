"""pa_copy_blocks (copy-on-write block copy) against the oracle: bit-exact over the whole
pools, the copy-on-write fork followed by the cache write and the decode, the argument
checks, and the benchmark's workloads at full size."""

import math

import numpy as np
import pytest
import torch

from paged_kv_cache_399_b200 import workloads

pytestmark = pytest.mark.gpu


def _u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _pools(nb, hkv, d, seed):
    g = torch.Generator().manual_seed(seed)
    shape = (nb, 16, hkv, d)
    mk = lambda: torch.randint(-32768, 32768, shape, generator=g, dtype=torch.int32).to(
        torch.int16).view(torch.bfloat16)
    return mk(), mk()


def _mapping(rng, nb, n, pad=0):
    """n pairs: sources with repeats, destinations distinct and never a source."""
    perm = rng.permutation(nb)
    half = nb // 2
    src = rng.choice(perm[:half], size=n, replace=True)
    dst = perm[half:half + n]
    m = np.stack([src, dst], axis=1).astype(np.int64)
    if pad:
        m = np.concatenate([m, np.array([[-1, 0]] * pad, dtype=np.int64)])
        m = m[rng.permutation(len(m))]
    return m


@pytest.mark.parametrize("hkv,d,n,nb", [(1, 64, 1, 8), (2, 128, 7, 64), (8, 128, 112, 400),
                                        (4, 64, 129, 600), (2, 128, 3000, 8192)],
                         ids=["one", "seven", "fork112", "over-small-cap", "multi-launch"])
def test_copy_blocks_bit_exact(hkv, d, n, nb, oracle_lib):
    from paged_kv_cache_399_b200 import pa
    rng = np.random.default_rng(n * 31 + hkv)
    kc0, vc0 = _pools(nb, hkv, d, seed=n + d)
    m = _mapping(rng, nb, n, pad=3)
    dk, dv = kc0.cuda(), vc0.cuda()
    pa.pa_copy_blocks(dk, dv, m)
    torch.cuda.synchronize()
    ek, ev = oracle_lib.copy_blocks(kc0, vc0, m)
    assert np.array_equal(_u16(dk), ek)
    assert np.array_equal(_u16(dv), ev)


def test_copy_blocks_padding_and_empty_are_noops():
    from paged_kv_cache_399_b200 import pa
    kc0, vc0 = _pools(16, 2, 64, seed=3)
    dk, dv = kc0.cuda(), vc0.cuda()
    pa.pa_copy_blocks(dk, dv, np.array([[-1, 4], [3, -1]], dtype=np.int64))
    pa.pa_copy_blocks(dk, dv, np.zeros((0, 2), dtype=np.int64))
    torch.cuda.synchronize()
    assert np.array_equal(_u16(dk), _u16(kc0)) and np.array_equal(_u16(dv), _u16(vc0))


@pytest.mark.parametrize("bad,code", [([[1, 3], [2, 3]], "PA_ERR_INVALID_ARG"),
                                      ([[1, 3], [3, 5]], "PA_ERR_INVALID_ARG"),
                                      ([[1, 16]], "PA_ERR_OUT_OF_RANGE")])
def test_copy_blocks_rejects_and_leaves_pools(bad, code):
    from paged_kv_cache_399_b200 import pa
    kc0, vc0 = _pools(16, 2, 64, seed=5)
    dk, dv = kc0.cuda(), vc0.cuda()
    with pytest.raises(pa.PAError) as err:
        pa.pa_copy_blocks(dk, dv, np.asarray(bad, dtype=np.int64))
    assert err.value.status == getattr(pa, code)
    torch.cuda.synchronize()
    assert np.array_equal(_u16(dk), _u16(kc0)) and np.array_equal(_u16(dv), _u16(vc0))


def test_copy_on_write_fork_then_decode(oracle_lib):
    """A parallel-sampling fork on the device: the samples share the prompt's blocks; each
    sample but the first copies the partly filled last block, writes its next token into the
    copy, and decodes. Pools bit-exact and attention within tolerance of the oracle run of
    the same steps."""
    from paged_kv_cache_399_b200 import pa
    rng = np.random.default_rng(7)
    g = torch.Generator().manual_seed(7)
    samples, L, hq, hkv, d, nb = 4, 37, 8, 2, 128, 24
    kc0 = torch.randn(nb, 16, hkv, d, generator=g).to(torch.bfloat16)
    vc0 = torch.randn(nb, 16, hkv, d, generator=g).to(torch.bfloat16)
    perm = rng.permutation(nb)
    prompt = perm[:3]
    tables = np.zeros((samples, 3), dtype=np.int32)
    tables[:] = prompt
    mapping = []
    for s in range(1, samples):
        dst = int(perm[3 + s])
        mapping.append([int(prompt[2]), dst])
        tables[s, 2] = dst
    mapping = np.asarray(mapping, dtype=np.int64)
    key = torch.randn(samples, hkv, d, generator=g).to(torch.bfloat16)
    value = torch.randn(samples, hkv, d, generator=g).to(torch.bfloat16)
    slots = np.array([int(tables[s, 2]) * 16 + L % 16 for s in range(samples)], dtype=np.int64)
    slots[0] = -1   # the first sample keeps the original block and does not write here
    ctx = np.array([L] + [L + 1] * (samples - 1), dtype=np.int32)
    query = torch.randn(samples, 1, hq, d, generator=g).to(torch.bfloat16)
    scale = 1.0 / math.sqrt(d)

    dk, dv = kc0.cuda(), vc0.cuda()
    pa.pa_copy_blocks(dk, dv, mapping)
    pa.pa_reshape_and_cache(key.cuda(), value.cuda(), dk, dv, torch.from_numpy(slots).cuda())
    out = torch.empty_like(query).cuda()
    plan = pa.pa_decode_plan(samples, 1, hq, hkv, d, tables.shape[1])
    ws_bytes = pa.pa_decode_workspace_size(plan, samples, 1, hq, hkv, d, tables.shape[1])
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    pa.pa_decode(out, query.cuda(), dk, dv, torch.from_numpy(tables).cuda(), torch.from_numpy(ctx).cuda(),
                 1, scale, plan=plan, workspace=ws)
    torch.cuda.synchronize()

    ek, ev = oracle_lib.copy_blocks(kc0, vc0, mapping)
    ek, ev = oracle_lib.reshape_and_cache(key, value, ek, ev, slots)
    assert np.array_equal(_u16(dk), ek) and np.array_equal(_u16(dv), ev)
    ref = oracle_lib.decode(query, ek, ev, tables, ctx, 1, scale)
    err = np.abs(out.float().cpu().numpy() - ref)
    assert err.max() <= 2e-2 and err.mean() <= 2e-3, (err.max(), err.mean())


@pytest.mark.parametrize("name", ["cow_fork", "cow_bulk"])
def test_benchmark_copy_workloads_full_size(name, oracle_lib):
    """The benchmark's copy workloads, in the launches bench.py times: the whole pools
    bit-exact against the oracle's copy."""
    from paged_kv_cache_399_b200 import pa
    w = workloads.make_copy(name)
    dk, dv = w.key_cache.cuda(), w.value_cache.cuda()
    pa.pa_copy_blocks(dk, dv, w.mapping)
    torch.cuda.synchronize()
    ek, ev = oracle_lib.copy_blocks(w.key_cache, w.value_cache, w.mapping)
    assert np.array_equal(_u16(dk), ek)
    assert np.array_equal(_u16(dv), ev)
