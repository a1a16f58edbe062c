"""Helpers shared by the GPU tests: move a workload to the device, run the hot
path through the C ABI binding, and compare with the fp64 oracle."""

from __future__ import annotations

import numpy as np
import torch

# Tolerances of the decode output (bf16) against the fp64 oracle.
MAX_ABS_TOL = 2e-2
MEAN_ABS_TOL = 2e-3


class DeviceWorkload:
    def __init__(self, w, device="cuda"):
        self.w = w
        self.query = w.query.to(device)
        self.key = w.key.to(device)
        self.value = w.value.to(device)
        self.slots = torch.from_numpy(w.slot_mapping).to(device)
        self.tables = torch.from_numpy(w.block_tables).to(device)
        self.ctx = torch.from_numpy(w.context_lens).to(device)
        self.key_cache = w.key_cache.to(device)
        self.value_cache = w.value_cache.to(device)
        self.out = torch.empty_like(self.query)


def run_step(dw: DeviceWorkload, plan=None, write=True):
    from paged_kv_cache_399_b200 import pa
    w = dw.w
    if write:
        pa.pa_reshape_and_cache(dw.key, dw.value, dw.key_cache, dw.value_cache, dw.slots)
    ws_bytes = pa.pa_decode_workspace_size(plan, w.num_seqs, w.q_per_seq, w.num_q_heads,
                                           w.num_kv_heads, w.head_dim, w.max_blocks_per_seq)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dw.query.device) if ws_bytes else None
    pa.pa_decode(dw.out, dw.query, dw.key_cache, dw.value_cache, dw.tables, dw.ctx, w.q_per_seq,
                 w.scale, plan=plan, workspace=ws)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error(reset=True) == 0
    return dw.out


def oracle_pools(orc, w):
    """Pool after the step's cache write, computed by the oracle on the host."""
    kc, vc = orc.reshape_and_cache(w.key, w.value, w.key_cache, w.value_cache, w.slot_mapping)
    return kc, vc


def errors(got: torch.Tensor, ref: np.ndarray):
    g = got.detach().float().cpu().double().numpy()
    err = np.abs(g - ref)
    assert np.all(np.isfinite(g)), "non-finite output"
    return float(err.max()), float(err.mean())


def assert_close(got: torch.Tensor, ref: np.ndarray, what: str = ""):
    mx, mean = errors(got, ref)
    assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL, f"{what}: max {mx:.3e} mean {mean:.3e}"
    return mx, mean
