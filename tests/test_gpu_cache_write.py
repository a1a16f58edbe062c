"""pa_reshape_and_cache against the oracle: bit-exact over the whole pool."""

import numpy as np
import pytest
import torch

from gpu_util import DeviceWorkload
from paged_kv_cache_399_b200 import workloads

pytestmark = pytest.mark.gpu


def _u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("name", ["tiny", "llama8b", "prefix_sharing", "spec_verify"])
def test_cache_write_bit_exact(name, oracle_lib):
    from paged_kv_cache_399_b200 import pa
    w = workloads.make(name)
    dw = DeviceWorkload(w)
    pa.pa_reshape_and_cache(dw.key, dw.value, dw.key_cache, dw.value_cache, dw.slots)
    torch.cuda.synchronize()
    kc, vc = oracle_lib.reshape_and_cache(w.key, w.value, w.key_cache, w.value_cache, w.slot_mapping)
    assert np.array_equal(_u16(dw.key_cache), kc)
    assert np.array_equal(_u16(dw.value_cache), vc)


def test_cache_write_skips_negative_slots_and_strided_rows(oracle_lib):
    from paged_kv_cache_399_b200 import pa
    g = torch.Generator().manual_seed(7)
    T, H, D, NB = 37, 4, 128, 20
    fused = torch.randn(T, 3 * H * D, generator=g).to(torch.bfloat16)  # [T, q|k|v] rows
    key = fused[:, H * D:2 * H * D].view(T, H, D)
    value = fused[:, 2 * H * D:].view(T, H, D)
    slots = torch.randperm(NB * 16, generator=g)[:T].to(torch.int64)
    slots[::5] = -1
    kc0 = torch.randn(NB, 16, H, D, generator=g).to(torch.bfloat16)
    vc0 = torch.randn(NB, 16, H, D, generator=g).to(torch.bfloat16)
    dk, dv = kc0.cuda(), vc0.cuda()
    fused_d = fused.cuda()
    pa.pa_reshape_and_cache(fused_d[:, H * D:2 * H * D].view(T, H, D), fused_d[:, 2 * H * D:].view(T, H, D),
                            dk, dv, slots.cuda())
    torch.cuda.synchronize()
    kc, vc = oracle_lib.reshape_and_cache(key.contiguous(), value.contiguous(), kc0, vc0, slots.numpy())
    assert np.array_equal(_u16(dk), kc)
    assert np.array_equal(_u16(dv), vc)


def test_cache_write_zero_tokens_is_a_noop():
    from paged_kv_cache_399_b200 import pa
    kc = torch.zeros(4, 16, 2, 64, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(0, 2, 64, dtype=torch.bfloat16, device="cuda")
    pa.pa_reshape_and_cache(k, k, kc, kc.clone(), torch.zeros(0, dtype=torch.int64, device="cuda"))
    torch.cuda.synchronize()
    assert int(kc.abs().sum()) == 0
