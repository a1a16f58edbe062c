"""pa_reshape_and_cache_fp8 against the oracle: the E4M3 codes of the fp32 quotients,
bit-exact over the whole pools, for scales that keep the codes normal, saturate them, or make
them subnormal, with strided (fused-QKV) rows and padding slots."""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("hkv,d", [(2, 64), (8, 128)])
@pytest.mark.parametrize("k_scale,v_scale", [(0.05, 0.02), (0.001, 0.004), (300.0, 1000.0)],
                         ids=["normal", "saturating", "subnormal"])
def test_fp8_cache_write_bit_exact(hkv, d, k_scale, v_scale, oracle_lib):
    from paged_kv_cache_399_b200 import pa
    g = torch.Generator().manual_seed(hkv * 1000 + d)
    T, NB = 41, 24
    fused = (torch.randn(T, 3 * hkv * d, generator=g) * 3).to(torch.bfloat16)   # [T, q|k|v]
    key = fused[:, hkv * d:2 * hkv * d].view(T, hkv, d)
    value = fused[:, 2 * hkv * d:].view(T, hkv, d)
    slots = torch.randperm(NB * 16, generator=g)[:T].to(torch.int64)
    slots[::7] = -1
    kc0 = torch.randint(0, 256, (NB, 16, hkv, d), generator=g, dtype=torch.int32).to(torch.uint8)
    vc0 = torch.randint(0, 256, (NB, 16, hkv, d), generator=g, dtype=torch.int32).to(torch.uint8)
    dk, dv = kc0.cuda(), vc0.cuda()
    fd = fused.cuda()
    pa.pa_reshape_and_cache_fp8(fd[:, hkv * d:2 * hkv * d].view(T, hkv, d), fd[:, 2 * hkv * d:].view(T, hkv, d),
                                dk, dv, slots.cuda(), k_scale, v_scale)
    torch.cuda.synchronize()
    ek, ev = oracle_lib.reshape_and_cache_fp8(key.contiguous(), value.contiguous(), kc0.numpy(), vc0.numpy(),
                                              slots.numpy(), k_scale, v_scale)
    assert np.array_equal(dk.cpu().numpy(), ek)
    assert np.array_equal(dv.cpu().numpy(), ev)


def test_fp8_cache_write_rejects_bad_scales():
    from paged_kv_cache_399_b200 import pa
    k = torch.zeros(1, 2, 64, dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros(4, 16, 2, 64, dtype=torch.uint8, device="cuda")
    s = torch.zeros(1, dtype=torch.int64, device="cuda")
    for ks, vs in ((0.0, 1.0), (1.0, float("nan")), (-1.0, 1.0), (1.0, float("inf"))):
        with pytest.raises(pa.PAError) as err:
            pa.pa_reshape_and_cache_fp8(k, k, kc, kc.clone(), s, ks, vs)
        assert err.value.status == pa.PA_ERR_INVALID_ARG
