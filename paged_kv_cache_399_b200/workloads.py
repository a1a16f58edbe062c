"""Seeded synthetic inputs for the paged KV-cache hot path.

This module holds no attention arithmetic: it only draws context lengths,
block tables, slot mappings and bf16 ~N(0, 1) tensors, the way a serving
engine's block manager would hand them to the kernels. Both the CUDA tests and
the fp64 oracle read the same objects built here.

Workloads (sizes follow the decode shapes that the vLLM pages discuss: the
16-token block of "vLLM 深度实战" §3.2 and the Llama shapes of the vLLM study
notes §1.2.2):

* ``tiny``            4 seqs x 1 query token, 4 q heads / 2 kv heads, head_dim 64,
                      context U[1, 80], a 64-block pool drawn without replacement,
                      scale 1/8; the slot mapping writes each sequence's newest token.
* ``llama8b``         64 x 1, 32/8 heads, head_dim 128, context U[512, 4096], pool
                      1.25x the blocks needed, shuffled.
* ``llama70b_long``   4 x 1, 64/8 heads, head_dim 128, contexts 32k/64k/96k/128k,
                      pool 1.25x the blocks needed, shuffled.
* ``prefix_sharing``  16 prompts x 8 samples, 32/8 heads: the 8 samples of a prompt
                      map their first 2048 tokens to the same 128 physical blocks,
                      then private tails of U[1, 256] tokens.
* ``spec_verify``     32 seqs x 6 query tokens (causal inside the window), 32/8 heads,
                      context lognormal(ln 2048, 0.8) clipped to [16, 16384]; the slot
                      mapping writes all 6 new tokens.
* ``sliding_window``  16 x 1, 32/8 heads, head_dim 128, a 4096-token sliding window over
                      contexts U[8192, 32768]; entries before the window name the null
                      block 0.
* ``llama8b_fp8``     the llama8b shapes over FP8 (E4M3) pools, one scale 0.01 per pool
                      (the FP8 KV cache of the vLLM study notes §4.2).

Chunked prefill (``PREFILL_WORKLOADS``; the vLLM study notes §3.5):

* ``chunked_prefill`` 4 prompts of 4096 tokens, each attending its last 512-token chunk over
                      the pool (3584 earlier tokens + the chunk, causal), 32/8 heads, D 128.

Copy-on-write block copies (``make_copy``; the copy rule of the vLLM study notes
§3.2.2):

* ``cow_fork``        the fork of 16 prompts (U[1, 2048] tokens) into 8 samples each:
                      7 copies of every partly filled last prompt block, 8 kv heads,
                      head_dim 128 (32 KB per block and pool).
* ``cow_bulk``        8192 copies in a 20480-block pool (same block shape), sources
                      with repeats, distinct destinations.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

BLOCK_SIZE = 16


@dataclass
class Workload:
    name: str
    seed: int
    num_seqs: int
    q_per_seq: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    scale: float
    context_lens: np.ndarray          # int32 [B]
    block_tables: np.ndarray          # int32 [B, max_blocks_per_seq]
    num_blocks: int
    query: torch.Tensor               # bf16 [B, q, H_q, D]
    key: torch.Tensor                 # bf16 [T, H_kv, D], T = B * q
    value: torch.Tensor               # bf16 [T, H_kv, D]
    slot_mapping: np.ndarray          # int64 [T]
    key_cache: torch.Tensor           # bf16 [NB, bs, H_kv, D], pool before the write
    value_cache: torch.Tensor         # bf16 [NB, bs, H_kv, D]
    blocks_used: np.ndarray = field(default=None)   # int32 [B] blocks owned per sequence
    shared_groups: list = field(default_factory=list)  # [(members, prefix_tokens)]
    window: int = 0                   # sliding window in tokens, 0 = none
    kv_dtype: str = "bf16"            # "bf16", or "fp8_e4m3": uint8 pools of E4M3 codes
    k_scale: float = 1.0              # fp8_e4m3: value of a key code = code * k_scale
    v_scale: float = 1.0

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def num_tokens(self) -> int:
        return int(self.slot_mapping.shape[0])

    def describe(self) -> str:
        return (f"{self.name}: B={self.num_seqs} q={self.q_per_seq} H_q={self.num_q_heads} "
                f"H_kv={self.num_kv_heads} D={self.head_dim} bs={self.block_size} "
                f"ctx[min/mean/max]={int(self.context_lens.min())}/"
                f"{float(self.context_lens.mean()):.0f}/{int(self.context_lens.max())} "
                f"NB={self.num_blocks} seed={self.seed}" + (f" window={self.window}" if self.window else "")
                + (f" kv=fp8_e4m3 k_scale={self.k_scale:g} v_scale={self.v_scale:g}"
                   if self.kv_dtype == "fp8_e4m3" else ""))


def _blocks(n_tokens: int, block_size: int) -> int:
    return -(-int(n_tokens) // block_size)


def _randn_bf16(shape, gen: torch.Generator, chunk: int = 1 << 24) -> torch.Tensor:
    """bf16 ~N(0,1): fp32 normal draws rounded to nearest even, in chunks."""
    out = torch.empty(shape, dtype=torch.bfloat16)
    flat = out.view(-1)
    n = flat.numel()
    for start in range(0, n, chunk):
        stop = min(n, start + chunk)
        flat[start:stop] = torch.randn(stop - start, generator=gen, dtype=torch.float32).to(
            torch.bfloat16)
    return out


def build_workload(name: str, seed: int, context_lens, q_per_seq: int, num_q_heads: int,
                   num_kv_heads: int, head_dim: int, scale: float | None = None,
                   block_size: int = BLOCK_SIZE, pool_factor: float = 1.25,
                   num_blocks: int | None = None, share_groups=None,
                   max_blocks_per_seq: int | None = None, window: int = 0) -> Workload:
    """General builder.

    share_groups: optional list of (member_sequence_ids, prefix_tokens); the
    members map their first prefix_tokens (a multiple of block_size) to the same
    physical blocks. All other blocks are private. Physical ids come from one
    seeded permutation of the pool, so no two sequences alias a private block.

    window > 0: a sliding window of that many tokens. Only the blocks a sequence's rows
    can see are allocated; the table entries wholly before the first row's window point
    at the null block 0, which is reserved (the vLLM study notes, §5.5).
    """
    rng = np.random.default_rng(seed)
    gen = torch.Generator().manual_seed(seed)
    ctx = np.asarray(context_lens, dtype=np.int64)
    B = int(ctx.shape[0])
    if np.any(ctx < q_per_seq):
        raise ValueError("every context must hold its q_per_seq new tokens")
    need = np.array([_blocks(c, block_size) for c in ctx], dtype=np.int64)
    # first block a row of the sequence sees (0 without a window)
    lo_blk = np.array([max(0, int(c) - q_per_seq - window + 1) // block_size if window > 0 else 0
                       for c in ctx], dtype=np.int64)
    share_groups = list(share_groups or [])
    if window > 0 and share_groups:
        raise ValueError("a sliding window with shared prefixes is not generated")
    shared_prefix_blocks = np.zeros(B, dtype=np.int64)
    leader = np.arange(B)
    for members, prefix_tokens in share_groups:
        if prefix_tokens % block_size:
            raise ValueError("shared prefixes cover whole blocks")
        for m in members:
            shared_prefix_blocks[m] = prefix_tokens // block_size
            leader[m] = members[0]
    distinct = int((need - lo_blk).sum() - sum(shared_prefix_blocks[m] for members, _ in share_groups
                                                for m in members[1:]))
    reserved = 1 if window > 0 else 0   # the null block
    if num_blocks is None:
        num_blocks = int(math.ceil(pool_factor * distinct)) + reserved
    if num_blocks < distinct + reserved:
        raise ValueError("pool too small")
    perm = (reserved + rng.permutation(num_blocks - reserved)).astype(np.int64)
    width = int(max_blocks_per_seq or need.max())
    tables = np.zeros((B, width), dtype=np.int32)  # padding entries point at block 0
    cursor = 0
    for b in range(B):
        start = int(lo_blk[b])   # entries before it stay 0: the null block
        if shared_prefix_blocks[b] and leader[b] != b:
            start = int(shared_prefix_blocks[b])
            tables[b, :start] = tables[leader[b], :start]
        n = int(need[b]) - start
        tables[b, start:start + n] = perm[cursor:cursor + n]
        cursor += n
    # new tokens of this step: the last q_per_seq positions of every sequence
    slots = np.empty(B * q_per_seq, dtype=np.int64)
    for b in range(B):
        for i in range(q_per_seq):
            p = int(ctx[b]) - q_per_seq + i
            slots[b * q_per_seq + i] = int(tables[b, p // block_size]) * block_size + p % block_size
    if scale is None:
        scale = 1.0 / math.sqrt(head_dim)
    query = _randn_bf16((B, q_per_seq, num_q_heads, head_dim), gen)
    key = _randn_bf16((B * q_per_seq, num_kv_heads, head_dim), gen)
    value = _randn_bf16((B * q_per_seq, num_kv_heads, head_dim), gen)
    key_cache = _randn_bf16((num_blocks, block_size, num_kv_heads, head_dim), gen)
    value_cache = _randn_bf16((num_blocks, block_size, num_kv_heads, head_dim), gen)
    return Workload(name=name, seed=seed, num_seqs=B, q_per_seq=q_per_seq,
                    num_q_heads=num_q_heads, num_kv_heads=num_kv_heads, head_dim=head_dim,
                    block_size=block_size, scale=float(scale),
                    context_lens=ctx.astype(np.int32), block_tables=tables,
                    num_blocks=int(num_blocks), query=query, key=key, value=value,
                    slot_mapping=slots, key_cache=key_cache, value_cache=value_cache,
                    blocks_used=need.astype(np.int32), shared_groups=share_groups, window=int(window))


def with_fp8_pools(w: Workload, k_scale: float = 0.01, v_scale: float = 0.01,
                   name: str | None = None) -> Workload:
    """The same workload over FP8 KV pools: the pools' prior contents become E4M3 codes of
    the bf16 values over the pool scale (torch's float8_e4m3fn conversion, magnitudes clipped
    to the format's 448 first). The step's new K/V rows stay bf16: the FP8 cache write turns
    them into codes. The default scale 0.01 maps the ~N(0, 1) values onto the code range
    (|x| up to 4.48 before the codes saturate)."""
    import copy
    f = copy.copy(w)

    def codes(pool: torch.Tensor, scale: float) -> torch.Tensor:
        x = (pool.float() / scale).clamp_(-448.0, 448.0)
        return x.to(torch.float8_e4m3fn).view(torch.uint8)

    f.key_cache = codes(w.key_cache, k_scale)
    f.value_cache = codes(w.value_cache, v_scale)
    f.kv_dtype, f.k_scale, f.v_scale = "fp8_e4m3", float(k_scale), float(v_scale)
    f.name = name or (w.name + "_fp8")
    return f


def tiny(seed: int = 1000) -> Workload:
    rng = np.random.default_rng(seed + 7919)
    ctx = rng.integers(1, 80, size=4, endpoint=True)
    return build_workload("tiny", seed, ctx, 1, 4, 2, 64, scale=1.0 / 8.0, num_blocks=64)


def llama8b(seed: int = 1001, num_seqs: int = 64) -> Workload:
    rng = np.random.default_rng(seed + 7919)
    ctx = rng.integers(512, 4096, size=num_seqs, endpoint=True)
    return build_workload("llama8b", seed, ctx, 1, 32, 8, 128)


def llama70b_long(seed: int = 1002, context_lens=(32768, 65536, 98304, 131072)) -> Workload:
    return build_workload("llama70b_long", seed, list(context_lens), 1, 64, 8, 128)


def prefix_sharing(seed: int = 1003, prompts: int = 16, samples: int = 8,
                   prefix_tokens: int = 2048, max_tail: int = 256) -> Workload:
    rng = np.random.default_rng(seed + 7919)
    tails = rng.integers(1, max_tail, size=prompts * samples, endpoint=True)
    ctx = prefix_tokens + tails
    groups = [(list(range(p * samples, (p + 1) * samples)), prefix_tokens)
              for p in range(prompts)]
    return build_workload("prefix_sharing", seed, ctx, 1, 32, 8, 128, share_groups=groups)


def spec_verify(seed: int = 1004, num_seqs: int = 32, q_per_seq: int = 6) -> Workload:
    rng = np.random.default_rng(seed + 7919)
    ctx = np.rint(rng.lognormal(mean=math.log(2048.0), sigma=0.8, size=num_seqs))
    ctx = np.clip(ctx, 16, 16384).astype(np.int64)
    return build_workload("spec_verify", seed, ctx, q_per_seq, 32, 8, 128)


@dataclass
class CopyWorkload:
    """The copy-on-write block copies of one step: the pools and the {source,
    destination} pairs the block manager hands to pa_copy_blocks."""
    name: str
    seed: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    mapping: np.ndarray               # int64 [n, 2] {source, destination}
    key_cache: torch.Tensor           # bf16 [NB, bs, H_kv, D]
    value_cache: torch.Tensor

    @property
    def block_bytes(self) -> int:
        return self.block_size * self.num_kv_heads * self.head_dim * 2

    @property
    def num_pairs(self) -> int:
        return int((self.mapping >= 0).all(axis=1).sum())

    def describe(self) -> str:
        return (f"{self.name}: {self.num_pairs} block copies of {self.block_bytes} B per pool "
                f"(H_kv={self.num_kv_heads} D={self.head_dim} bs={self.block_size}), "
                f"NB={self.num_blocks} seed={self.seed}")


def _bits_bf16(shape, gen: torch.Generator) -> torch.Tensor:
    """Uniformly random 16-bit patterns as bf16 (NaN and infinity patterns included):
    a copy must move every pattern unchanged."""
    return torch.randint(-32768, 32768, shape, generator=gen, dtype=torch.int32).to(
        torch.int16).view(torch.bfloat16)


def cow_fork(seed: int = 1005, prompts: int = 16, samples: int = 8, max_prompt: int = 2048,
             num_kv_heads: int = 8, head_dim: int = 128) -> CopyWorkload:
    """The copy-on-write step of a parallel-sampling fork (the prefix-sharing shape: 16
    prompts x 8 samples, 8 kv heads, head_dim 128): the samples of a prompt share all of
    its blocks; every sample but the first writes its next token into the prompt's last
    block, so when that block is partly filled it is copied once per such sample. Prompt
    lengths U[1, max_prompt]; pool 1.25x the blocks needed, shuffled."""
    rng = np.random.default_rng(seed + 7919)
    gen = torch.Generator().manual_seed(seed)
    lens = rng.integers(1, max_prompt, size=prompts, endpoint=True)
    prompt_blocks = [_blocks(n, BLOCK_SIZE) for n in lens]
    copies = sum(samples - 1 for n in lens if n % BLOCK_SIZE)
    num_blocks = int(math.ceil(1.25 * (sum(prompt_blocks) + copies)))
    perm = rng.permutation(num_blocks).astype(np.int64)
    cursor = sum(prompt_blocks)
    pairs = []
    start = 0
    for n, nb in zip(lens, prompt_blocks):
        last = int(perm[start + nb - 1])
        start += nb
        if n % BLOCK_SIZE == 0:
            continue  # the next token opens a new block: nothing shared is written
        for _ in range(samples - 1):
            pairs.append([last, int(perm[cursor])])
            cursor += 1
    shape = (num_blocks, BLOCK_SIZE, num_kv_heads, head_dim)
    return CopyWorkload("cow_fork", seed, num_kv_heads, head_dim, BLOCK_SIZE, num_blocks,
                        np.asarray(pairs, dtype=np.int64).reshape(-1, 2),
                        _bits_bf16(shape, gen), _bits_bf16(shape, gen))


def cow_bulk(seed: int = 1006, pairs: int = 8192, num_blocks: int = 20480, num_kv_heads: int = 8,
             head_dim: int = 128) -> CopyWorkload:
    """A burst of copies large enough to time the copy against HBM bandwidth (many forks
    at once, e.g. beam search over a large batch): sources drawn with repeats from one half
    of a shuffled pool, destinations distinct blocks of the other half."""
    rng = np.random.default_rng(seed + 7919)
    gen = torch.Generator().manual_seed(seed)
    perm = rng.permutation(num_blocks).astype(np.int64)
    half = num_blocks // 2
    if pairs > num_blocks - half:
        raise ValueError("pool too small for the destinations")
    src = rng.choice(perm[:half], size=pairs, replace=True)
    dst = perm[half:half + pairs]
    shape = (num_blocks, BLOCK_SIZE, num_kv_heads, head_dim)
    return CopyWorkload("cow_bulk", seed, num_kv_heads, head_dim, BLOCK_SIZE, num_blocks,
                        np.stack([src, dst], axis=1).astype(np.int64),
                        _bits_bf16(shape, gen), _bits_bf16(shape, gen))


COPY_WORKLOADS = {
    "cow_fork": cow_fork,
    "cow_bulk": cow_bulk,
}


def make_copy(name: str, seed: int | None = None) -> CopyWorkload:
    fn = COPY_WORKLOADS[name]
    return fn() if seed is None else fn(seed)


def sliding_window(seed: int = 1007, num_seqs: int = 16, window: int = 4096) -> Workload:
    """A Mistral-7B-shaped decode layer with a sliding window (32 q heads, 8 kv heads,
    head_dim 128, window 4096): contexts U[8192, 32768], so every sequence reads the last
    4096 tokens of a longer context; the blocks before the window are the null block."""
    rng = np.random.default_rng(seed + 7919)
    ctx = rng.integers(8192, 32768, size=num_seqs, endpoint=True)
    return build_workload("sliding_window", seed, ctx, 1, 32, 8, 128, window=window)


def llama8b_fp8(seed: int = 1008) -> Workload:
    """The Llama-3.1-8B-shaped decode layer over FP8 (E4M3) KV pools, scale 0.01 per pool."""
    return with_fp8_pools(llama8b(seed), name="llama8b_fp8")


@dataclass
class PrefillWorkload:
    """One chunked-prefill step: every sequence attends a chunk of qlen_b new tokens (the
    last qlen_b positions of its context) over the paged pool, causal within the chunk.
    The chunk tokens' K/V are written first through the slot mapping."""
    name: str
    seed: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    scale: float
    context_lens: np.ndarray          # int32 [B], including the chunk
    query_start: np.ndarray           # int32 [B + 1]
    block_tables: np.ndarray          # int32 [B, max_blocks_per_seq]
    num_blocks: int
    query: torch.Tensor               # bf16 [T, H_q, D]
    key: torch.Tensor                 # bf16 [T, H_kv, D]: the chunk tokens' K
    value: torch.Tensor               # bf16 [T, H_kv, D]
    slot_mapping: np.ndarray          # int64 [T]
    key_cache: torch.Tensor           # bf16 [NB, bs, H_kv, D], pool before the write
    value_cache: torch.Tensor

    @property
    def num_seqs(self) -> int:
        return int(self.context_lens.shape[0])

    @property
    def query_lens(self) -> np.ndarray:
        return np.diff(self.query_start)

    @property
    def max_query_len(self) -> int:
        return int(self.query_lens.max()) if self.num_seqs else 0

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def num_tokens(self) -> int:
        return int(self.query_start[-1])

    def describe(self) -> str:
        ql = self.query_lens
        return (f"{self.name}: B={self.num_seqs} chunk[min/mean/max]={int(ql.min())}/{float(ql.mean()):.0f}/"
                f"{int(ql.max())} T={self.num_tokens} H_q={self.num_q_heads} H_kv={self.num_kv_heads} "
                f"D={self.head_dim} bs={self.block_size} ctx[min/mean/max]={int(self.context_lens.min())}/"
                f"{float(self.context_lens.mean()):.0f}/{int(self.context_lens.max())} NB={self.num_blocks} "
                f"seed={self.seed}")


def build_prefill(name: str, seed: int, context_lens, query_lens, num_q_heads: int, num_kv_heads: int,
                  head_dim: int, scale: float | None = None, block_size: int = BLOCK_SIZE,
                  pool_factor: float = 1.25) -> PrefillWorkload:
    """Sequences with the given contexts, each ending in a chunk of query_lens[b] new tokens;
    blocks from one seeded permutation of a pool pool_factor x the blocks needed; bf16
    ~N(0, 1) values."""
    rng = np.random.default_rng(seed)
    gen = torch.Generator().manual_seed(seed)
    ctx = np.asarray(context_lens, dtype=np.int64)
    ql = np.asarray(query_lens, dtype=np.int64)
    if ctx.shape != ql.shape or np.any(ql < 0) or np.any(ql > ctx):
        raise ValueError("every chunk lies inside its context")
    B = int(ctx.shape[0])
    need = np.array([_blocks(c, block_size) for c in ctx], dtype=np.int64)
    num_blocks = int(math.ceil(pool_factor * int(need.sum()))) + 1
    perm = rng.permutation(num_blocks).astype(np.int64)
    width = int(max(1, need.max()))
    tables = np.zeros((B, width), dtype=np.int32)
    cursor = 0
    for b in range(B):
        tables[b, :need[b]] = perm[cursor:cursor + need[b]]
        cursor += int(need[b])
    qstart = np.zeros(B + 1, dtype=np.int32)
    qstart[1:] = np.cumsum(ql)
    T = int(qstart[-1])
    slots = np.empty(T, dtype=np.int64)
    for b in range(B):
        for i in range(int(ql[b])):
            pos = int(ctx[b]) - int(ql[b]) + i
            slots[qstart[b] + i] = int(tables[b, pos // block_size]) * block_size + pos % block_size
    return PrefillWorkload(
        name=name, seed=seed, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads, head_dim=head_dim,
        block_size=block_size, scale=float(1.0 / math.sqrt(head_dim) if scale is None else scale),
        context_lens=ctx.astype(np.int32), query_start=qstart, block_tables=tables, num_blocks=num_blocks,
        query=_randn_bf16((T, num_q_heads, head_dim), gen), key=_randn_bf16((T, num_kv_heads, head_dim), gen),
        value=_randn_bf16((T, num_kv_heads, head_dim), gen), slot_mapping=slots,
        key_cache=_randn_bf16((num_blocks, block_size, num_kv_heads, head_dim), gen),
        value_cache=_randn_bf16((num_blocks, block_size, num_kv_heads, head_dim), gen))


def chunked_prefill(seed: int = 1009, num_seqs: int = 4, chunk: int = 512, context: int = 4096) -> PrefillWorkload:
    """A chunked-prefill step of a Llama-3.1-8B-shaped layer (32 q heads, 8 kv heads,
    head_dim 128): 4 prompts of 4096 tokens whose last 512-token chunk is attended now over
    the 3584 tokens already in the pool plus itself (the chunk size of the vLLM study
    notes §3.5 is 2048; 512 keeps four prompts in one step)."""
    return build_prefill("chunked_prefill", seed, [context] * num_seqs, [chunk] * num_seqs, 32, 8, 128)


PREFILL_WORKLOADS = {"chunked_prefill": chunked_prefill}


WORKLOADS = {
    "tiny": tiny,
    "llama8b": llama8b,
    "llama70b_long": llama70b_long,
    "prefix_sharing": prefix_sharing,
    "spec_verify": spec_verify,
    "sliding_window": sliding_window,
    "llama8b_fp8": llama8b_fp8,
}


def make(name: str, seed: int | None = None) -> Workload:
    fn = WORKLOADS[name]
    return fn() if seed is None else fn(seed)
