"""pa_prefill (chunked-prefill attention) against the fp64 oracle: ragged chunk lengths that
cross the kernel's 128-row tiles, several GQA group sizes, chunks that are whole prompts,
chunks of one token, NaN / Inf in slots past each context, and the full-size chunked_prefill
workload on sampled rows. The oracle's reference for sequence b is its decode with
q_per_seq = the chunk length (the same definition: the chunk's tokens are the last positions
of the context, causal among themselves)."""

import numpy as np
import pytest
import torch

from gpu_util import assert_close
from paged_kv_cache_399_b200 import workloads

pytestmark = pytest.mark.gpu

# name, context lengths, chunk lengths, H_q, H_kv
CASES = [
    ("g4_ragged", [300, 130, 1000, 64, 45], [200, 130, 37, 1, 33], 32, 8),
    ("g1_mha", [257, 129, 700], [129, 128, 300], 4, 4),
    ("g8", [520, 96, 2049], [17, 96, 250], 16, 2),
    ("g16_mqa", [333, 17], [33, 17], 16, 1),
    ("whole_prompts", [128, 256, 160], [128, 256, 160], 8, 2),
    ("decode_like", [900, 33, 4000, 16], [1, 1, 1, 1], 32, 8),
    ("empty_chunk", [100, 200, 50], [0, 77, 0], 8, 2),
]


def _oracle(orc, w):
    kc, vc = orc.reshape_and_cache(w.key, w.value, w.key_cache, w.value_cache, w.slot_mapping)
    out = np.zeros((w.num_tokens, w.num_q_heads, w.head_dim))
    for b in range(w.num_seqs):
        s0, s1 = int(w.query_start[b]), int(w.query_start[b + 1])
        if s1 == s0:
            continue
        q = w.query[s0:s1].unsqueeze(0)
        out[s0:s1] = orc.decode(q, kc, vc, w.block_tables[b:b + 1], w.context_lens[b:b + 1], s1 - s0, w.scale)[0]
    return kc, vc, out


class DevicePrefill:
    def __init__(self, w):
        self.w = w
        self.query = w.query.cuda()
        self.key = w.key.cuda()
        self.value = w.value.cuda()
        self.slots = torch.from_numpy(w.slot_mapping).cuda()
        self.tables = torch.from_numpy(w.block_tables).cuda()
        self.ctx = torch.from_numpy(w.context_lens).cuda()
        self.qstart = torch.from_numpy(w.query_start).cuda()
        self.key_cache = w.key_cache.cuda()
        self.value_cache = w.value_cache.cuda()
        self.out = torch.full_like(self.query, float("nan"))

    def step(self, write=True):
        from paged_kv_cache_399_b200 import pa
        if write:
            pa.pa_reshape_and_cache(self.key, self.value, self.key_cache, self.value_cache, self.slots)
        pa.pa_prefill(self.out, self.query, self.key_cache, self.value_cache, self.tables, self.ctx, self.qstart,
                      self.w.max_query_len, self.w.scale)
        torch.cuda.synchronize()
        assert pa.pa_get_device_error(reset=True) == 0
        return self.out


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_prefill_matches_oracle(case, oracle_lib):
    name, ctx, ql, hq, hkv = case
    w = workloads.build_prefill(name, 5000 + len(name), ctx, ql, hq, hkv, 128)
    _, _, ref = _oracle(oracle_lib, w)
    out = DevicePrefill(w).step()
    if w.num_tokens:
        assert_close(out, ref, name)


def test_prefill_unwritten_slots_do_not_leak(oracle_lib):
    """NaN in K and NaN / Inf in V in the slots of each sequence's last block past its
    context: their weight is zero and they must not reach any row."""
    w = workloads.build_prefill("poison", 5100, [300, 130, 1000, 70], [200, 5, 37, 70], 32, 8, 128)
    _, _, ref = _oracle(oracle_lib, w)
    dw = DevicePrefill(w)
    bs = 16
    for b in range(w.num_seqs):
        ctx = int(w.context_lens[b])
        if ctx % bs:
            phys = int(w.block_tables[b, (ctx - 1) // bs])
            dw.key_cache[phys, ctx % bs:] = float("nan")
            dw.value_cache[phys, ctx % bs:] = float("inf")
            dw.value_cache[phys, bs - 1] = float("nan")
    out = dw.step()
    assert_close(out, ref, "poisoned")


def test_prefill_chunks_compose_to_the_whole_prompt(oracle_lib):
    """A 400-token prompt attended as chunks of 150, 150 and 100 (three steps, each writing
    its own K/V first) gives the rows of one 400-token chunk (within the tolerance)."""
    from paged_kv_cache_399_b200 import pa
    whole = workloads.build_prefill("whole", 5200, [400], [400], 32, 8, 128)
    dwh = DevicePrefill(whole)
    ref_whole = dwh.step().clone()
    got = torch.empty_like(ref_whole)
    done = 0
    for n in (150, 150, 100):
        dw = DevicePrefill(whole)
        dw.key_cache, dw.value_cache = dwh.key_cache, dwh.value_cache   # the pool already holds the prompt
        sub = slice(done, done + n)
        q = dw.query[sub].contiguous()
        out = torch.empty_like(q)
        pa.pa_prefill(out, q, dw.key_cache, dw.value_cache, dw.tables,
                      torch.tensor([done + n], dtype=torch.int32, device="cuda"),
                      torch.tensor([0, n], dtype=torch.int32, device="cuda"), n, whole.scale)
        torch.cuda.synchronize()
        got[sub] = out
        done += n
    _, _, ref = _oracle(oracle_lib, whole)
    assert_close(got, ref, "chunks")
    assert_close(ref_whole, ref, "whole")


def test_prefill_full_size_sampled_rows(oracle_lib):
    """The benchmark's chunked_prefill workload in its launch configuration, checked on 768
    sampled rows (every sequence, tokens across the chunk including its first and last, all
    kv heads) against the oracle's row-by-row decode."""
    w = workloads.PREFILL_WORKLOADS["chunked_prefill"]()
    dw = DevicePrefill(w)
    out = dw.step().clone()
    assert bool(torch.isfinite(out.float()).all())
    kc, vc = oracle_lib.reshape_and_cache(w.key, w.value, w.key_cache, w.value_cache, w.slot_mapping)
    chunk = int(w.query_lens[0])
    assert np.all(w.query_lens == chunk)
    rng = np.random.default_rng(7)
    rows = []
    for b in range(w.num_seqs):
        toks = np.concatenate([[0, chunk - 1], rng.integers(0, chunk, size=30)])
        for i in toks:
            for h in rng.choice(w.num_q_heads, size=6, replace=False):
                rows.append((b, int(i), int(h)))
    q = w.query.view(w.num_seqs, chunk, w.num_q_heads, w.head_dim)
    ref = oracle_lib.decode_rows(rows, q, kc, vc, w.block_tables, w.context_lens, chunk, w.scale)
    got = torch.stack([out[int(w.query_start[b]) + i, h] for b, i, h in rows])
    assert_close(got, ref, "chunked_prefill sampled rows")
    assert torch.equal(dw.step(write=False), out)   # repeatable bits


def test_prefill_zero_scale_is_the_mean_of_visible_values(oracle_lib):
    """scale 0: every visible key has the same weight, so each row is the mean of the values
    it sees (the kernel takes the row maximum over raw scores; 0 must not turn masked keys
    into NaN)."""
    w = workloads.build_prefill("zero_scale", 5300, [300, 130, 77], [200, 5, 77], 32, 8, 128, scale=0.0)
    _, _, ref = _oracle(oracle_lib, w)
    out = DevicePrefill(w).step()
    assert_close(out, ref, "zero scale")
