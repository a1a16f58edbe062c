"""The failure path on a GPU without a fault: a bounded wait that nothing completes
gives up after its limit, the kernel records its code and returns, and the context
stays usable."""

import time

import pytest
import torch

from gpu_util import DeviceWorkload, assert_close, oracle_pools, run_step
from paged_kv_cache_399_b200 import workloads

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_reports(oracle_lib):
    from paged_kv_cache_399_b200 import pa
    assert pa.pa_get_device_error(reset=True) == 0
    t0 = time.monotonic()
    pa.pa_selftest_bounded_wait()
    code = pa.pa_get_device_error(reset=True)   # synchronous
    waited = time.monotonic() - t0
    assert code == 0x600
    assert 0.5 < waited < 30.0, waited        # about one wait limit (1 s)
    assert pa.pa_get_device_error(reset=True) == 0
    # the context is still usable: a decode right after matches the oracle
    w = workloads.tiny()
    kc, vc = oracle_pools(oracle_lib, w)
    ref = oracle_lib.decode(w.query, kc, vc, w.block_tables, w.context_lens, 1, w.scale)
    out = run_step(DeviceWorkload(w))
    assert_close(out, ref, "decode after the self-test")
    torch.cuda.synchronize()
