"""Pins for the fp64 oracle: checks against things other than the oracle itself.

Every ``check_*`` function takes an ``oracle.Oracle`` and raises AssertionError
when the oracle disagrees with:
  * numbers printed on the vLLM pages (block counts, KV bytes, the paging figure),
  * brute-force attention over contiguous (un-paged) K/V on tiny inputs,
  * a library routine (torch scaled_dot_product_attention, fp64, CPU),
  * closed forms (one-token context, identical keys, zero scale),
  * invariants (block permutation, shared prefixes, GQA vs MHA, speculative
    rows vs shorter single-token calls, tiled online softmax and split/merge),
  * the copy-on-write rule of parallel sampling (a fork's writer copies the shared
    last block and writes there; the other candidates still read the original),
  * the sliding window (the most recent W tokens; entries before it may name the null
    block 0 and are never read),
  * the FP8 (E4M3) KV cache: the format's fixed values, torch's float8_e4m3fn conversion,
    the cache write's codes and attention over the dequantized pools.
The same checks run against deliberately broken builds of the oracle
(tests/test_oracle_mutants.py) to show that each planted mistake is caught.
"""

from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _bf16_round(x: np.ndarray) -> np.ndarray:
    """fp64 values rounded to bf16 (nearest even) and widened back, via torch."""
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).to(
        torch.float64).numpy()


def _bits(x: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


class Problem:
    """A tiny paged problem built from contiguous per-sequence K/V.

    The logical keys/values are drawn first; the pool is then filled by the
    page's address rule (block = table[t // bs], offset = t % bs) written here
    in numpy, so the brute-force references never read the pool.
    """

    def __init__(self, seed, ctxs, q=1, hq=4, hkv=2, d=16, bs=16, scale=None, extra_blocks=3,
                 same_keys=False):
        rng = np.random.default_rng(seed)
        self.B, self.q, self.hq, self.hkv, self.d, self.bs = len(ctxs), q, hq, hkv, d, bs
        self.ctxs = [int(c) for c in ctxs]
        self.scale = (1.0 / math.sqrt(d)) if scale is None else float(scale)
        nblk = [-(-c // bs) for c in self.ctxs]
        self.nb = sum(nblk) + extra_blocks
        perm = rng.permutation(self.nb)
        width = max(nblk) + 1
        self.tables = np.zeros((self.B, width), dtype=np.int32)
        cur = 0
        for b, n in enumerate(nblk):
            self.tables[b, :n] = perm[cur:cur + n]
            cur += n
        self.K = []
        self.V = []
        for c in self.ctxs:
            k = _bf16_round(rng.standard_normal((c, hkv, d)))
            if same_keys:
                k[:] = k[0]
            self.K.append(k)
            self.V.append(_bf16_round(rng.standard_normal((c, hkv, d))))
        self.Q = _bf16_round(rng.standard_normal((self.B, q, hq, d)))
        pool_k = _bf16_round(rng.standard_normal((self.nb, bs, hkv, d)))
        pool_v = _bf16_round(rng.standard_normal((self.nb, bs, hkv, d)))
        for b in range(self.B):
            for t in range(self.ctxs[b]):
                blk = self.tables[b, t // bs]
                pool_k[blk, t % bs] = self.K[b][t]
                pool_v[blk, t % bs] = self.V[b][t]
        self.pool_k, self.pool_v = pool_k, pool_v

    def run(self, oracle, pool_k=None, pool_v=None, tables=None, ctxs=None, Q=None, q=None,
            scale=None, window=0):
        pk = self.pool_k if pool_k is None else pool_k
        pv = self.pool_v if pool_v is None else pool_v
        qq = self.Q if Q is None else Q
        return oracle.decode(_bits(qq), _bits(pk), _bits(pv),
                             self.tables if tables is None else tables,
                             np.asarray(self.ctxs if ctxs is None else ctxs, dtype=np.int32),
                             self.q if q is None else q,
                             self.scale if scale is None else scale, window=window)


def brute_force(p: Problem) -> np.ndarray:
    """Textbook attention on the contiguous K/V, one row at a time."""
    g = p.hq // p.hkv
    out = np.zeros((p.B, p.q, p.hq, p.d))
    for b in range(p.B):
        for i in range(p.q):
            last = p.ctxs[b] - p.q + i
            for h in range(p.hq):
                kv = h // g
                s = np.array([p.scale * float(np.dot(p.Q[b, i, h], p.K[b][t, kv]))
                              for t in range(last + 1)])
                w = np.exp(s - s.max())
                out[b, i, h] = (w[:, None] * p.V[b][:last + 1, kv]).sum(0) / w.sum()
    return out


def library_attention(p: Problem) -> np.ndarray:
    """torch scaled_dot_product_attention in fp64 on the contiguous K/V."""
    g = p.hq // p.hkv
    out = np.zeros((p.B, p.q, p.hq, p.d))
    for b in range(p.B):
        c = p.ctxs[b]
        qb = torch.from_numpy(p.Q[b]).permute(1, 0, 2)[None]               # [1,hq,q,d]
        kb = torch.from_numpy(p.K[b]).permute(1, 0, 2).repeat_interleave(g, 0)[None]
        vb = torch.from_numpy(p.V[b]).permute(1, 0, 2).repeat_interleave(g, 0)[None]
        pos = torch.arange(c)[None, :]
        qpos = (c - p.q + torch.arange(p.q))[:, None]
        mask = pos <= qpos                                                   # [q, ctx]
        o = torch.nn.functional.scaled_dot_product_attention(qb, kb, vb, attn_mask=mask,
                                                             scale=p.scale)
        out[b] = o[0].permute(1, 0, 2).numpy()
    return out


def _close(a, b, tol=1e-10, what=""):
    err = float(np.max(np.abs(np.asarray(a) - np.asarray(b)))) if np.size(a) else 0.0
    assert err <= tol, f"{what}: max |diff| {err:.3e} > {tol:.1e}"


# ---------------------------------------------------------------- page numbers

def check_bf16_widening(oracle):
    known = {0x3F80: 1.0, 0xC000: -2.0, 0x3F81: 1.0 + 2.0 ** -7, 0x0000: 0.0,
             0x4049: 3.140625, 0x0001: 2.0 ** -133}
    for bits, val in known.items():
        assert oracle.bf16_to_f64(bits) == val, hex(bits)
    rng = np.random.default_rng(5)
    pats = rng.integers(0, 0x7F7F, size=256).astype(np.uint16)
    ref = torch.from_numpy(pats.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle.bf16_to_f64(int(x)) for x in pats])
    assert np.array_equal(got, ref), "bf16 widening differs from torch"


def check_block_counts_golden(oracle):
    data = json.load(open(os.path.join(GOLDEN, "page_numbers.json")))
    for row in data["block_counts"]:
        n = oracle.blocks_for_tokens(row["tokens"], row["block_size"])
        assert n == row["blocks"], row["cite"]
        if "empty_slots" in row:
            assert n * row["block_size"] - row["tokens"] == row["empty_slots"], row["cite"]
            assert (n * row["block_size"] - row["tokens"]) / (n * row["block_size"]) == \
                row["waste_fraction"], row["cite"]


def check_kv_bytes_golden(oracle):
    data = json.load(open(os.path.join(GOLDEN, "page_numbers.json")))
    for row in data["kv_bytes"]:
        per_tok = oracle.kv_bytes_per_token(row["layers"], row["kv_heads"], row["head_dim"],
                                            row["bytes_per_value"])
        if "bytes_per_token" in row:
            assert per_tok == row["bytes_per_token"], row["cite"]
            assert per_tok * row["context"] == row["bytes_per_request"], row["cite"]
        if "gib_per_request" in row:
            assert per_tok * row["context"] / 2 ** 30 == row["gib_per_request"], row["cite"]


def check_mapping_example(oracle):
    """The paging figure: table [0, 3, 7] puts tokens 0..47 in slots 0-15/48-63/112-127.

    Pool value channel 0 holds each physical slot's number (exact in bf16). With
    scale 0 and one query row per position, row i averages the slots of tokens
    0..i, so consecutive rows reveal the slot each token was read from.
    """
    ex = json.load(open(os.path.join(GOLDEN, "block_mapping_example.json")))
    bs, table, ctx = ex["block_size"], ex["block_table"], ex["context_len"]
    nb, d = 8, 8
    pool_k = np.zeros((nb, bs, 1, d))
    pool_v = np.zeros((nb, bs, 1, d))
    for blk in range(nb):
        for off in range(bs):
            pool_v[blk, off, 0, 0] = blk * bs + off
    q = np.zeros((1, ctx, 1, d))
    out = oracle.decode(_bits(q), _bits(pool_k), _bits(pool_v),
                        np.array([table], dtype=np.int32), np.array([ctx], dtype=np.int32),
                        ctx, 0.0)
    means = out[0, :, 0, 0]
    slots = [round(means[0])] + [round(means[i] * (i + 1) - means[i - 1] * i)
                                 for i in range(1, ctx)]
    expected = [s for lo, hi in ex["expected_slot_ranges"] for s in range(lo, hi + 1)]
    assert slots == expected, f"{ex['cite']}: got {slots}"


# ------------------------------------------------------------ reference checks

BRUTE_CASES = [
    dict(seed=11, ctxs=[1, 17, 33, 5], q=1, hq=4, hkv=2, d=16),
    dict(seed=12, ctxs=[40, 16, 23], q=3, hq=6, hkv=3, d=8),
    dict(seed=13, ctxs=[6, 31, 48], q=6, hq=8, hkv=2, d=16, scale=0.7),
    dict(seed=14, ctxs=[20, 9], q=2, hq=2, hkv=2, d=32, bs=8),
]


def check_brute_force(oracle):
    for case in BRUTE_CASES:
        p = Problem(**case)
        _close(p.run(oracle), brute_force(p), what=f"brute force {case}")


def check_library_attention(oracle):
    for case in BRUTE_CASES:
        p = Problem(**case)
        _close(p.run(oracle), library_attention(p), what=f"torch sdpa {case}")


def check_closed_forms(oracle):
    # one visible key: out == v_0 exactly
    p = Problem(seed=21, ctxs=[1, 1, 1], q=1, hq=4, hkv=2, d=16)
    out = p.run(oracle)
    for b in range(p.B):
        for h in range(p.hq):
            assert np.array_equal(out[b, 0, h], p.V[b][0, h // 2]), "ctx=1 must return v0"
    # identical keys: uniform weights, out == mean of the visible values
    p = Problem(seed=22, ctxs=[7, 19, 33], q=3, hq=4, hkv=2, d=16, same_keys=True)
    out = p.run(oracle)
    for b in range(p.B):
        for i in range(p.q):
            last = p.ctxs[b] - p.q + i
            for h in range(p.hq):
                _close(out[b, i, h], p.V[b][:last + 1, h // 2].mean(0), 1e-12, "identical keys")
    # zero scale: also the mean of the visible values
    p = Problem(seed=23, ctxs=[5, 30], q=2, hq=2, hkv=1, d=8, scale=0.0)
    out = p.run(oracle)
    for b in range(p.B):
        for i in range(p.q):
            last = p.ctxs[b] - p.q + i
            for h in range(p.hq):
                _close(out[b, i, h], p.V[b][:last + 1, 0].mean(0), 1e-12, "zero scale")


# ----------------------------------------------------------------- invariants

def check_block_permutation(oracle):
    p = Problem(seed=31, ctxs=[33, 50, 2], q=2, hq=4, hkv=2, d=16, extra_blocks=6)
    base = p.run(oracle)
    sigma = np.random.default_rng(32).permutation(p.nb)
    pk = np.empty_like(p.pool_k)
    pv = np.empty_like(p.pool_v)
    pk[sigma] = p.pool_k
    pv[sigma] = p.pool_v
    tables = sigma[p.tables].astype(np.int32)
    assert np.array_equal(p.run(oracle, pool_k=pk, pool_v=pv, tables=tables), base), \
        "physical block placement changed the output"


def check_unwritten_slots_ignored(oracle):
    """Pool slots that no sequence sees (past a context, or in blocks no table names) may
    hold any bits: NaN or Inf there leaves every output bit unchanged."""
    p = Problem(seed=36, ctxs=[17, 40, 5, 33], q=2, hq=4, hkv=2, d=16, extra_blocks=4)
    base = p.run(oracle)
    live = np.zeros((p.nb, p.bs), dtype=bool)
    for b, c in enumerate(p.ctxs):
        for t in range(c):
            live[p.tables[b, t // p.bs], t % p.bs] = True
    assert (~live).sum() > 0
    pk, pv = p.pool_k.copy(), p.pool_v.copy()
    pk[~live] = np.nan
    pv[~live] = np.inf
    pv[~live & (np.arange(p.bs)[None, :] % 2 == 0)] = np.nan
    assert np.array_equal(p.run(oracle, pool_k=pk, pool_v=pv), base), \
        "a slot outside every context reached the output"


def check_shared_prefix(oracle):
    """Two sequences sharing prefix blocks equal their unshared copies."""
    rng = np.random.default_rng(41)
    bs, hkv, hq, d = 16, 2, 4, 16
    nb = 12
    pk = _bf16_round(rng.standard_normal((nb, bs, hkv, d)))
    pv = _bf16_round(rng.standard_normal((nb, bs, hkv, d)))
    # sequence 0 and 1 share blocks 3, 5 (32 tokens); tails live in 7 and 9
    shared = np.array([[3, 5, 7], [3, 5, 9]], dtype=np.int32)
    ctxs = np.array([40, 45], dtype=np.int32)
    # unshared copy: prefix blocks duplicated into 0, 1 (for seq 1)
    pk2, pv2 = pk.copy(), pv.copy()
    pk2[[0, 1]] = pk[[3, 5]]
    pv2[[0, 1]] = pv[[3, 5]]
    unshared = np.array([[3, 5, 7], [0, 1, 9]], dtype=np.int32)
    Q = _bf16_round(rng.standard_normal((2, 1, hq, d)))
    a = oracle.decode(_bits(Q), _bits(pk), _bits(pv), shared, ctxs, 1, 0.25)
    b = oracle.decode(_bits(Q), _bits(pk2), _bits(pv2), unshared, ctxs, 1, 0.25)
    assert np.array_equal(a, b), "shared prefix blocks changed the output"


def check_gqa_equals_repeated_mha(oracle):
    p = Problem(seed=51, ctxs=[21, 38], q=2, hq=6, hkv=2, d=16)
    g = p.hq // p.hkv
    pk = np.repeat(p.pool_k, g, axis=2)
    pv = np.repeat(p.pool_v, g, axis=2)
    gqa = p.run(oracle)
    mha = p.run(oracle, pool_k=pk, pool_v=pv)
    assert np.array_equal(gqa, mha), "GQA differs from MHA with repeated kv heads"


def check_spec_rows_equal_short_calls(oracle):
    p = Problem(seed=61, ctxs=[30, 17], q=4, hq=4, hkv=2, d=16)
    full = p.run(oracle)
    for i in range(p.q):
        ctxs = [c - (p.q - 1 - i) for c in p.ctxs]
        one = p.run(oracle, ctxs=ctxs, Q=p.Q[:, i:i + 1].copy(), q=1)
        assert np.array_equal(full[:, i], one[:, 0]), f"speculative row {i}"


def _online_softmax(scores, values, tile):
    """Tile-by-tile running max / running sum, rescaled (vLLM study notes §4.3.1)."""
    m, l = -np.inf, 0.0
    o = np.zeros(values.shape[1])
    for s0 in range(0, len(scores), tile):
        s = scores[s0:s0 + tile]
        m_new = max(m, s.max())
        pw = np.exp(s - m_new)
        alpha = np.exp(m - m_new) if m > -np.inf else 0.0
        o = o * alpha + pw @ values[s0:s0 + tile]
        l = l * alpha + pw.sum()
        m = m_new
    return o, m, l


def check_online_and_split_merge(oracle):
    """Tiled online softmax, and split partials merged by log-sum-exp, equal the oracle."""
    p = Problem(seed=71, ctxs=[70, 129, 16], q=3, hq=4, hkv=2, d=16)
    ref = p.run(oracle)
    g = p.hq // p.hkv
    for b in range(p.B):
        for i in range(p.q):
            last = p.ctxs[b] - p.q + i
            for h in range(p.hq):
                kv = h // g
                s = p.scale * (p.K[b][:last + 1, kv] @ p.Q[b, i, h])
                v = p.V[b][:last + 1, kv]
                o, m, l = _online_softmax(s, v, 16)
                _close(o / l, ref[b, i, h], 1e-12, "online softmax")
                parts = [_online_softmax(s[c:c + 32], v[c:c + 32], 16)
                         for c in range(0, len(s), 32)]
                M = max(pm for _, pm, _ in parts)
                L = sum(pl * np.exp(pm - M) for _, pm, pl in parts)
                O = sum(po * np.exp(pm - M) for po, pm, _ in parts)
                _close(O / L, ref[b, i, h], 1e-12, "split + merge")


# ---------------------------------------------------------------- cache write

def check_cache_write(oracle):
    rng = np.random.default_rng(81)
    bs, hkv, d, nb = 16, 2, 8, 10
    tables = np.array([[4, 1, 8], [6, 2, 0]], dtype=np.int32)
    positions = [(0, 35), (1, 16), (1, 17), (0, 0)]
    slots = np.array([tables[b, t // bs] * bs + t % bs for b, t in positions] + [-1],
                     dtype=np.int64)
    T = len(slots)
    key = _bits(rng.standard_normal((T, hkv, d)))
    val = _bits(rng.standard_normal((T, hkv, d)))
    kc0 = _bits(rng.standard_normal((nb, bs, hkv, d)))
    vc0 = _bits(rng.standard_normal((nb, bs, hkv, d)))
    kc, vc = oracle.reshape_and_cache(key, val, kc0, vc0, slots)
    written = np.zeros((nb, bs), dtype=bool)
    for t, (b, pos) in enumerate(positions):
        blk, off = tables[b, pos // bs], pos % bs      # position -> table, not slot
        assert np.array_equal(kc[blk, off], key[t]), f"key of token {t}"
        assert np.array_equal(vc[blk, off], val[t]), f"value of token {t}"
        written[blk, off] = True
    assert np.array_equal(kc[~written], kc0[~written]), "stray key write"
    assert np.array_equal(vc[~written], vc0[~written]), "stray value write"
    bad = np.array([nb * bs + 3], dtype=np.int64)
    try:
        oracle.reshape_and_cache(key[:1], val[:1], kc0, vc0, bad)
    except ValueError:
        pass
    else:
        raise AssertionError("out-of-range slot not reported")


def _attend_rows(q, K, V, scale):
    """Textbook attention of one query token's heads over contiguous K/V [t][hkv][d]."""
    hq, hkv = q.shape[0], K.shape[1]
    out = np.zeros((hq, q.shape[1]))
    for h in range(hq):
        kv = h // (hq // hkv)
        s = scale * (K[:, kv] @ q[h])
        w = np.exp(s - s.max())
        out[h] = (w[:, None] * V[:, kv]).sum(0) / w.sum()
    return out


def check_copy_on_write(oracle):
    """The parallel-sampling fork of the copy-on-write rule (golden/copy_on_write.json):
    the candidates share every prompt block; a candidate about to write into the shared
    last block gets a copy first, writes there, and the others still read the original."""
    g = json.load(open(os.path.join(GOLDEN, "copy_on_write.json")))
    bs, n, L, writers = g["block_size"], g["parallel_samples"], g["prompt_tokens"], g["writers"]
    rng = np.random.default_rng(91)
    hq, hkv, d, nb = 4, 2, 8, 12
    pk = _bf16_round(rng.standard_normal((nb, bs, hkv, d)))
    pv = _bf16_round(rng.standard_normal((nb, bs, hkv, d)))
    prompt = [5, 2, 9]                                      # physical blocks of the prompt
    K = _bf16_round(rng.standard_normal((L, hkv, d)))
    V = _bf16_round(rng.standard_normal((L, hkv, d)))
    for t in range(L):
        pk[prompt[t // bs], t % bs] = K[t]
        pv[prompt[t // bs], t % bs] = V[t]
    tables = np.array([prompt] * n, dtype=np.int32)
    free = [b for b in range(nb) if b not in prompt]
    # the rule: a write into a block referenced by more than one table copies it first
    mapping = []
    for w in writers:
        blk = tables[w, L // bs]
        refs = int((tables[:, L // bs] == blk).sum())
        assert refs > g["copy_when_ref_count_above"]
        dst = free.pop(0)
        mapping.append([blk, dst])
        tables[w, L // bs] = dst
    for w in writers:   # after the copies every block a writer writes has one reference
        assert int((tables == tables[w, L // bs]).sum()) == 1
    kc, vc = oracle.copy_blocks(_bits(pk), _bits(pv), mapping + [[-1, 0]])
    newk = _bf16_round(rng.standard_normal((len(writers), hkv, d)))
    newv = _bf16_round(rng.standard_normal((len(writers), hkv, d)))
    slots = np.array([tables[w, L // bs] * bs + L % bs for w in writers], dtype=np.int64)
    kc, vc = oracle.reshape_and_cache(_bits(newk), _bits(newv), kc, vc, slots)
    # every candidate attends over its own logical sequence, built here without the pool
    Q = _bf16_round(rng.standard_normal((n, 1, hq, d)))
    ctxs = np.array([L + 1 if b in writers else L for b in range(n)], dtype=np.int32)
    out = oracle.decode(_bits(Q), kc, vc, tables, ctxs, 1, 1.0 / math.sqrt(d))
    for b in range(n):
        Kb, Vb = K, V
        if b in writers:
            Kb = np.concatenate([K, newk[writers.index(b)][None]])
            Vb = np.concatenate([V, newv[writers.index(b)][None]])
        _close(out[b, 0], _attend_rows(Q[b, 0], Kb, Vb, 1.0 / math.sqrt(d)), what=f"candidate {b}")
    # bit level: the source block is untouched, each copy equals it except the written
    # token, and no other block changed
    k0, v0 = _bits(pk), _bits(pv)
    for j, (src, dst) in enumerate(mapping):
        for pool, pool0, new in ((kc, k0, newk), (vc, v0, newv)):
            assert np.array_equal(pool[src], pool0[src]), "source block changed"
            exp = pool0[src].copy()
            exp[L % bs] = _bits(new[j])
            assert np.array_equal(pool[dst], exp), f"copy {j} differs from its source"
    others = [b for b in range(nb) if b not in [m[1] for m in mapping]]
    assert np.array_equal(kc[others], k0[others]) and np.array_equal(vc[others], v0[others]), "stray write"
    kc2, vc2 = oracle.copy_blocks(k0, v0, np.zeros((0, 2), dtype=np.int64))
    assert np.array_equal(kc2, k0) and np.array_equal(vc2, v0), "empty mapping changed the pools"
    for bad in ([[1, 3], [2, 3]], [[1, 3], [3, 4]], [[0, nb]]):
        try:
            oracle.copy_blocks(k0, v0, bad)
        except ValueError:
            continue
        raise AssertionError(f"mapping {bad} not rejected")


def _brute_force_window(p, window):
    """Textbook attention over the keys max(0, pos - W + 1) .. pos of the contiguous K/V."""
    g = p.hq // p.hkv
    out = np.zeros((p.B, p.q, p.hq, p.d))
    for b in range(p.B):
        for i in range(p.q):
            last = p.ctxs[b] - p.q + i
            first = max(0, last - window + 1)
            for h in range(p.hq):
                kv = h // g
                keys = range(first, last + 1)
                s = np.array([p.scale * float(np.dot(p.Q[b, i, h], p.K[b][t, kv])) for t in keys])
                w = np.exp(s - s.max())
                out[b, i, h] = (w[:, None] * p.V[b][first:last + 1, kv]).sum(0) / w.sum()
    return out


def check_sliding_window(oracle):
    """golden/sliding_window.json: the most recent W tokens only; positions before the window
    may point at the null block 0, whose contents are never read."""
    g = json.load(open(os.path.join(GOLDEN, "sliding_window.json")))
    p = Problem(seed=101, ctxs=[37, 50, 5, 16], q=3, hq=4, hkv=2, d=16, extra_blocks=4)
    for W in (1, 2, 7, 16, 17, 33, 64):
        _close(p.run(oracle, window=W), _brute_force_window(p, W), tol=1e-10, what=f"window {W}")
    # a one-token window is the query's own value row exactly
    out1 = p.run(oracle, window=1)
    for b in range(p.B):
        for i in range(p.q):
            last = p.ctxs[b] - p.q + i
            for h in range(p.hq):
                assert np.array_equal(out1[b, i, h], p.V[b][last, h // (p.hq // p.hkv)]), "W=1 closed form"
    # a window at least as long as every context is no window
    assert np.array_equal(p.run(oracle, window=max(p.ctxs)), p.run(oracle)), "W >= ctx"
    # the null block: relabel so that block 0 is unused, fill it with NaN, point every entry
    # wholly before a sequence's window at it
    null = g["null_block"]
    used = set(int(x) for b in range(p.B) for x in p.tables[b, :-(-p.ctxs[b] // p.bs)])
    spare = next(x for x in range(p.nb) if x not in used)
    tables = p.tables.copy()
    pk, pv = p.pool_k.copy(), p.pool_v.copy()
    if null in used:   # swap the contents and names of block `null` and the spare block
        pk[[null, spare]] = pk[[spare, null]]
        pv[[null, spare]] = pv[[spare, null]]
        tables = np.where(p.tables == null, spare, p.tables).astype(np.int32)
    W = 7
    ref = p.run(oracle, pool_k=pk, pool_v=pv, tables=tables, window=W)
    pk[null] = np.nan
    pv[null] = np.nan
    for b in range(p.B):
        first = max(0, p.ctxs[b] - p.q - W + 1)   # row 0's first visible key
        tables[b, :first // p.bs] = null
    got = p.run(oracle, pool_k=pk, pool_v=pv, tables=tables, window=W)
    assert np.array_equal(got, ref), "an entry before the window was read"
    # a library routine: torch scaled_dot_product_attention in fp64 with the window as a mask
    g_ = p.hq // p.hkv
    for W in (3, 16, 40):
        got = p.run(oracle, window=W)
        for b in range(p.B):
            c = p.ctxs[b]
            qb = torch.from_numpy(p.Q[b]).permute(1, 0, 2)[None]
            kb = torch.from_numpy(p.K[b]).permute(1, 0, 2).repeat_interleave(g_, 0)[None]
            vb = torch.from_numpy(p.V[b]).permute(1, 0, 2).repeat_interleave(g_, 0)[None]
            pos = torch.arange(c)[None, :]
            qpos = (c - p.q + torch.arange(p.q))[:, None]
            mask = (pos <= qpos) & (pos > qpos - W)
            o = torch.nn.functional.scaled_dot_product_attention(qb, kb, vb, attn_mask=mask, scale=p.scale)
            _close(got[b], o[0].permute(1, 0, 2).numpy(), tol=1e-10, what=f"window {W} vs SDPA, seq {b}")
    # visible key counts: min(W, pos + 1), through weights on a one-hot value pattern
    q1 = Problem(seed=103, ctxs=[30], q=1, hq=1, hkv=1, d=16, same_keys=True)
    for W in (1, 5, 30, 40):
        o = q1.run(oracle, window=W)[0, 0, 0]
        n = min(W, 30)
        assert np.allclose(o, q1.V[0][30 - n:30, 0].mean(0), atol=1e-12), f"visible keys for W={W}"


def _torch_fp8_codes(x32: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x32, dtype=np.float32)).to(torch.float8_e4m3fn).view(
        torch.uint8).numpy()


def _torch_fp8_values(codes: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn).to(
        torch.float64).numpy()


def check_fp8_format(oracle):
    """golden/fp8_e4m3.json (values fixed by the format's definition), torch.float8_e4m3fn (a
    library conversion) on every code and on a dense sweep of [-448, 448] with every tie, and
    the round trip of every code."""
    g = json.load(open(os.path.join(GOLDEN, "fp8_e4m3.json")))
    for table in ("codes", "saturate"):
        xs = np.array([float(k) for k in g[table]], dtype=np.float32)
        want = np.array(list(g[table].values()), dtype=np.uint8)
        got = oracle.fp8_encode(xs)
        assert np.array_equal(got, want), (table, xs[got != want], got[got != want])
    for k, c in g["codes"].items():
        assert oracle.fp8_decode([c])[0] == float(k) and math.copysign(1, oracle.fp8_decode([c])[0]) == \
            math.copysign(1, float(k)), k
    codes = np.arange(256, dtype=np.uint8)
    mine, ref = oracle.fp8_decode(codes), _torch_fp8_values(codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan) and np.array_equal(mine[~nan], ref[~nan]), "decode vs torch"
    vals = np.unique(ref[~nan])
    mids = ((vals[1:] + vals[:-1]) / 2).astype(np.float32)
    x = np.concatenate([np.arange(-448 * 1024, 448 * 1024 + 1) / 1024.0, mids, -mids,
                        np.random.default_rng(7).uniform(-448, 448, 100000)]).astype(np.float32)
    bad = oracle.fp8_encode(x) != _torch_fp8_codes(x)
    assert not bad.any(), ("encode vs torch", x[bad][:5])
    finite = codes[~nan]
    assert np.array_equal(oracle.fp8_encode(oracle.fp8_decode(finite).astype(np.float32)), finite), "round trip"


def check_fp8_cache_and_attention(oracle):
    """The FP8 cache write stores the codes torch gives for the fp32 quotients x / scale, and
    FP8 attention equals brute force over the contiguous K/V dequantized with torch."""
    rng = np.random.default_rng(111)
    bs, hkv, hq, d, q = 16, 2, 4, 16, 2
    ctxs = [20, 37, 5]
    ks, vs = 0.05, 0.02
    nb = sum(-(-c // bs) for c in ctxs) + 3
    perm = rng.permutation(nb)
    tables = np.zeros((len(ctxs), max(-(-c // bs) for c in ctxs)), dtype=np.int32)
    cur = 0
    for b, c in enumerate(ctxs):
        n = -(-c // bs)
        tables[b, :n] = perm[cur:cur + n]
        cur += n
    finite = np.array([c for c in range(256) if c & 0x7F != 0x7F], dtype=np.uint8)
    kc0 = rng.choice(finite, size=(nb, bs, hkv, d)).astype(np.uint8)
    vc0 = rng.choice(finite, size=(nb, bs, hkv, d)).astype(np.uint8)
    # the step's new tokens: the last q positions of each sequence
    slots = np.array([int(tables[b, p // bs]) * bs + p % bs for b, c in enumerate(ctxs)
                      for p in range(c - q, c)], dtype=np.int64)
    key = _bf16_round(rng.standard_normal((len(slots), hkv, d)) * 3)
    val = _bf16_round(rng.standard_normal((len(slots), hkv, d)) * 3)
    kc, vc = oracle.reshape_and_cache_fp8(_bits(key), _bits(val), kc0, vc0, slots, ks, vs)
    written = np.zeros((nb, bs), dtype=bool)
    for t, sl in enumerate(slots):
        blk, off = divmod(int(sl), bs)
        assert np.array_equal(kc[blk, off], _torch_fp8_codes(key[t].astype(np.float32) / np.float32(ks))), t
        assert np.array_equal(vc[blk, off], _torch_fp8_codes(val[t].astype(np.float32) / np.float32(vs))), t
        written[blk, off] = True
    assert np.array_equal(kc[~written], kc0[~written]) and np.array_equal(vc[~written], vc0[~written])
    Q = _bf16_round(rng.standard_normal((len(ctxs), q, hq, d)))
    scale = 1.0 / math.sqrt(d)
    out = oracle.decode_fp8(_bits(Q), kc, vc, tables, np.array(ctxs, dtype=np.int32), q, scale, ks, vs)
    kd, vd = _torch_fp8_values(kc) * ks, _torch_fp8_values(vc) * vs
    for b, c in enumerate(ctxs):
        K = np.stack([kd[tables[b, t // bs], t % bs] for t in range(c)])
        V = np.stack([vd[tables[b, t // bs], t % bs] for t in range(c)])
        for i in range(q):
            last = c - q + i
            _close(out[b, i], _attend_rows(Q[b, i], K[:last + 1], V[:last + 1], scale), what=f"fp8 seq {b} row {i}")
        # the same against torch scaled_dot_product_attention (fp64) on the dequantized K/V
        g_ = hq // hkv
        qb = torch.from_numpy(Q[b]).permute(1, 0, 2)[None]
        kb = torch.from_numpy(K).permute(1, 0, 2).repeat_interleave(g_, 0)[None]
        vb = torch.from_numpy(V).permute(1, 0, 2).repeat_interleave(g_, 0)[None]
        mask = torch.arange(c)[None, :] <= (c - q + torch.arange(q))[:, None]
        o = torch.nn.functional.scaled_dot_product_attention(qb, kb, vb, attn_mask=mask, scale=scale)
        _close(out[b], o[0].permute(1, 0, 2).numpy(), tol=1e-10, what=f"fp8 seq {b} vs SDPA")


def check_chunked_prefill(oracle):
    """Chunked prefill (vLLM study notes §3.5; "vLLM 深度解析" §5.4): a prompt is attended
    in chunks of many query tokens, each chunk causal within itself over the keys already
    in the pool. Pinned at q = 64 and 200 against brute force and torch SDPA, and by the
    property chunking relies on: the rows of a prompt attended as two chunks (the first
    with context = its length, the second over the whole prompt) equal the rows of one
    chunk over the whole prompt."""
    for case in (dict(seed=91, ctxs=[64, 100], q=64, hq=4, hkv=2, d=16),
                 dict(seed=92, ctxs=[200, 233], q=200, hq=4, hkv=1, d=16, bs=16)):
        p = Problem(**case)
        got = p.run(oracle)
        _close(got, library_attention(p), what=f"chunked prefill sdpa q={p.q}")
        bf = brute_force(p)
        _close(got, bf, what=f"chunked prefill brute force q={p.q}")
    # one chunk of 96 over a 96-token prompt == chunks of 40 and 56
    p = Problem(seed=93, ctxs=[96, 96], q=96, hq=4, hkv=2, d=16)
    whole = p.run(oracle)
    first = p.run(oracle, ctxs=[40, 40], Q=p.Q[:, :40].copy(), q=40)
    second = p.run(oracle, Q=p.Q[:, 40:].copy(), q=56)
    assert np.array_equal(whole[:, :40], first), "first chunk differs from the whole prompt's rows"
    assert np.array_equal(whole[:, 40:], second), "second chunk differs from the whole prompt's rows"


ALL_CHECKS = [
    check_bf16_widening,
    check_block_counts_golden,
    check_kv_bytes_golden,
    check_mapping_example,
    check_brute_force,
    check_library_attention,
    check_closed_forms,
    check_block_permutation,
    check_unwritten_slots_ignored,
    check_shared_prefix,
    check_gqa_equals_repeated_mha,
    check_spec_rows_equal_short_calls,
    check_online_and_split_merge,
    check_cache_write,
    check_copy_on_write,
    check_sliding_window,
    check_fp8_format,
    check_fp8_cache_and_attention,
    check_chunked_prefill,
]
