/*
 * pa.h -- C ABI of the B200 (sm_100a) paged KV-cache hot path.
 *
 * The operations, as the vLLM pages describe them:
 *   pa_reshape_and_cache  writes this step's new K/V rows into the paged pool at
 *                         the slots named by slot_mapping
 *                         ("vLLM 深度实战：从 PagedAttention 到 Speculative Decoding",
 *                          §3.3: block_table and slot_mapping address the blocks);
 *   pa_decode             attention softmax(q K^T * scale) V computed straight over
 *                         the scattered blocks through each sequence's block table
 *                         (same page §3.3; vLLM study notes, zihan-zhang.net, §3.2
 *                          page-table walk and §4.3.1 online softmax), with GQA
 *                         head groups and causal masking of multi-token
 *                         (speculative-verify) queries (vLLM study notes §1.1.1);
 *   pa_copy_blocks        the copy-on-write block copy behind shared blocks
 *                         (vLLM study notes §3.2.2);
 *   pa_reshape_and_cache_fp8  the cache write into FP8 (E4M3) pools with one scale per
 *                         pool (vLLM study notes §4.2);
 *   pa_decode_fp8         pa_decode over such FP8 pools (same notes §4.2: an FP8 KV cache
 *                         halves attention's memory traffic);
 *   pa_prefill            chunked-prefill attention: many query tokens per sequence over
 *                         the paged pool, causal within the chunk (same notes §3.5);
 *   pa_decode_partial,    one sequence's blocks split over several GPUs: each computes the
 *   pa_merge_partials     attention over its range of table entries as unnormalised pieces,
 *                         and the pieces gathered from all of them merge by the log-sum-exp
 *                         rule of split softmax (same notes §4.3.1).
 *
 * Conventions shared by every call
 *   - All data pointers are DEVICE pointers on the current CUDA device (the one
 *     exception: pa_copy_blocks' block_mapping is a host array); the library
 *     never allocates, frees or synchronises (except pa_validate and
 *     pa_get_device_error, which are synchronous debug calls). All work is enqueued
 *     on `stream` (a cudaStream_t; NULL = legacy default stream). The caller owns
 *     every buffer and must keep it alive until the stream has executed the work.
 *   - bf16 tensors are passed as raw 16-bit storage.
 *   - Shapes (row-major, innermost last):
 *       key, value     [num_tokens][num_kv_heads][head_dim]; token rows may be
 *                      `*_token_stride` elements apart (>= num_kv_heads*head_dim)
 *       key_cache,
 *       value_cache    [num_blocks][block_size][num_kv_heads][head_dim]
 *                      (token-major block, head_dim innermost)
 *       slot_mapping   int64 [num_tokens]; slot = physical_block * block_size +
 *                      offset; a negative slot skips the token
 *       query, out     [num_seqs][q_per_seq][num_q_heads][head_dim]
 *       block_tables   int32 [num_seqs][max_blocks_per_seq]; entry j is the
 *                      physical block holding tokens j*block_size ..
 *                      j*block_size + block_size - 1 of the sequence
 *       context_lens   int32 [num_seqs]; tokens of the sequence INCLUDING its
 *                      q_per_seq new ones (already written by pa_reshape_and_cache)
 *   - Query token i of a sequence sits at position pos = context_len - q_per_seq + i and
 *     attends to positions 0 .. pos (pos - W + 1 .. pos under a plan's sliding window W).
 *     Query head h reads kv head h / (num_q_heads / num_kv_heads).
 *   - Supported: block_size 16, head_dim 64 or 128, num_q_heads % num_kv_heads == 0,
 *     1 <= q_per_seq <= 16. Anything else returns PA_ERR_UNSUPPORTED before any
 *     launch. A tcgen05 plan also needs num_seqs * num_kv_heads * row chunks below 2^28,
 *     and that times (max_blocks_per_seq / 8 + 1) below 2^35 (its in-kernel range scan).
 *     There is no CPU fallback.
 *   - Errors: host-side argument checks run before any launch and return a status
 *     with nothing enqueued. Device-resident values (slots, block ids, context
 *     lengths) are preconditions: 0 <= slot < num_blocks*block_size or slot < 0,
 *     0 <= block id < num_blocks for the first ceil(context_len/block_size)
 *     entries of each table row (with a sliding window, for the entries from the
 *     window's first block on: the ones before it are never read), q_per_seq <= context_len <=
 *     max_blocks_per_seq*block_size. pa_validate checks them on request. A launch
 *     failure returns PA_ERR_CUDA. Kernels never trap: a bounded wait that times
 *     out records a code that pa_get_device_error returns.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define PA_API __attribute__((visibility("default")))
#else
#define PA_API
#endif

typedef struct CUstream_st* pa_stream_t; /* identical to cudaStream_t */

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1,   /* null / misaligned pointer, bad size or stride */
  PA_ERR_UNSUPPORTED = 2,   /* valid but outside the supported set above */
  PA_ERR_WORKSPACE = 3,     /* split plan without a large enough workspace */
  PA_ERR_OUT_OF_RANGE = 4,  /* pa_validate found a bad slot / block id / length;
                               pa_copy_blocks was given a block id past the pool */
  PA_ERR_CUDA = 5,          /* a CUDA runtime call or launch failed */
  PA_ERR_DEVICE = 6         /* pa_get_device_error: a kernel reported a timeout */
} pa_status_t;

/* Decode kernels. */
typedef enum {
  PA_PATH_AUTO = 0,   /* heuristic (pa_decode_plan): tcgen05 for head_dim 128 with more
                         than 16 rows (GQA group x q_per_seq) per kv head or with prefix
                         sharing, else the mma.sync tiles (the CUDA-core kernel for <= 2
                         rows) */
  PA_PATH_SINGLE = 1, /* CUDA-core kernel: warp-shuffle reductions, fp32 FMA */
  PA_PATH_TILE = 2,   /* tensor-core kernel: mma.sync m16n8k16 bf16 -> fp32 */
  PA_PATH_TCGEN05 = 3 /* 5th-generation tensor cores, head_dim 128 only: tcgen05.mma with
                         the 128 tokens of a tile on M and 16 or 32 query rows on N,
                         accumulators in tensor memory, TMA producer warps, one issuing
                         thread, two softmax warpgroups; always its own persistent
                         schedule (PA_SCHEDULE_PERSISTENT, no pre-pass, no split length) */
} pa_path_t;

/* How the work is spread over CTAs. */
typedef enum {
  PA_SCHEDULE_AUTO = 0,
  PA_SCHEDULE_GRID = 1,       /* one CTA per (kv head, sequence, context split of
                                 split_blocks blocks) + a log-sum-exp merge kernel */
  PA_SCHEDULE_PERSISTENT = 2  /* mma.sync / CUDA-core paths: a one-CTA pre-pass reads
                                 context_lens and cuts all (sequence, kv head, block)
                                 work into num_ctas equal shares; one resident CTA per
                                 share; pieces of an output are merged by the CTA that
                                 finishes it. tcgen05 path: num_ctas CTAs cut the
                                 8-block tiles into equal ranges themselves; range-cut
                                 units are merged by a second kernel */
} pa_schedule_t;

/* Element type of the KV pools a plan is for. */
typedef enum {
  PA_KV_BF16 = 0,     /* bf16 values: pa_decode */
  PA_KV_FP8_E4M3 = 1  /* E4M3 codes with one fp32 scale per pool: pa_decode_fp8 (mma.sync
                         tensor-core tiles only: PA_PATH_TILE, either schedule) */
} pa_kv_dtype_t;

/* Optional hints for pa_decode_plan; zero-initialised = all automatic. */
typedef struct {
  int32_t path;          /* pa_path_t */
  int32_t schedule;      /* pa_schedule_t */
  int32_t split_blocks;  /* grid schedule: blocks per split (0 = heuristic); a nonzero
                            value makes the automatic path a grid one */
  int32_t share_prefix;  /* 1 = adjacent sequences whose block tables start with the
                            same physical blocks (parallel sampling, beam search, a
                            common system prompt) are detected on the device and their
                            common prefix blocks are read once for all of them (up to
                            32 / (GQA group x q_per_seq) sequences per read; tensor-core
                            kernels only); 0 = off */
  int32_t sliding_window; /* > 0: each query token attends to the most recent
                            sliding_window tokens only, keys pos - W + 1 .. pos (vLLM
                            study notes §3.6.3); table entries wholly before every row's
                            window are never read (the pages point them at the null
                            block 0, §5.5). Grid schedule on the mma.sync or CUDA-core
                            path, or the tcgen05 path; with share_prefix or the mma.sync
                            persistent schedule: PA_ERR_UNSUPPORTED. 0 = no window */
  int32_t kv_cache_dtype; /* pa_kv_dtype_t of the pools the plan will decode (0 = bf16) */
} pa_plan_hints_t;

/* A decode plan; fill it with pa_decode_plan and treat it as opaque. */
typedef struct {
  int32_t path;          /* PA_PATH_SINGLE, PA_PATH_TILE or PA_PATH_TCGEN05 */
  int32_t schedule;      /* PA_SCHEDULE_GRID or PA_SCHEDULE_PERSISTENT */
  int32_t split_blocks;  /* grid: blocks per split */
  int32_t num_splits;    /* grid: ceil(max_blocks_per_seq / split_blocks) (see
                            sliding_window) */
  int32_t rows_per_cta;  /* query rows (GQA group x q_per_seq) one CTA holds; tcgen05:
                            the MMA's N (16 or 32) */
  int32_t num_ctas;      /* persistent: CTAs launched (resident slots of the device); a
                            caller may lower or raise it (the workspace size follows) */
  int32_t share_cap;     /* sequences per shared-prefix unit, 0 = off */
  int32_t share_split_blocks; /* grid with sharing: blocks per split of a shared prefix */
  int32_t sliding_window; /* tokens of the sliding window, 0 = none; with a window,
                            num_splits covers the window's blocks,
                            ceil(min(max_blocks_per_seq, ceil((W + q_per_seq - 1) / 16) + 1)
                            / split_blocks) */
  int32_t kv_cache_dtype; /* pa_kv_dtype_t: pa_decode takes PA_KV_BF16 plans only,
                            pa_decode_fp8 PA_KV_FP8_E4M3 plans only */
} pa_plan_t;

/* Write the step's new K/V into the pool: for each token t with slot s =
 * slot_mapping[t] >= 0, key_cache[s / block_size][s % block_size][:][:] = key[t]
 * and likewise value -> value_cache. Bit-exact copy; every other pool byte is left
 * untouched. Requirements: 16-byte aligned key, value, key_cache, value_cache;
 * token strides in elements with stride*2 a multiple of 16; num_kv_heads*head_dim*2
 * a multiple of 16. Duplicate slots in one call are a precondition violation (the
 * surviving row is unspecified). num_tokens == 0 is a no-op. */
PA_API pa_status_t pa_reshape_and_cache(const void* key, const void* value,
                                 int64_t key_token_stride, int64_t value_token_stride,
                                 void* key_cache, void* value_cache,
                                 const int64_t* slot_mapping, int64_t num_tokens,
                                 int32_t num_kv_heads, int32_t head_dim,
                                 int64_t num_blocks, int32_t block_size,
                                 pa_stream_t stream);

/* FP8 KV cache write (vLLM study notes §4.2, --kv-cache-dtype fp8). The pools hold E4M3
 * codes (uint8 [num_blocks][block_size][num_kv_heads][head_dim]); each bf16 element x of
 * key[t] (value[t]) is stored at the slot pa_reshape_and_cache would use as the E4M3 code of
 * the fp32 quotient x / k_scale (x / v_scale): round to nearest, ties to even, saturating at
 * +-448 (no infinities in E4M3). k_scale, v_scale: finite, > 0, one per pool, chosen by the
 * caller. Same layouts, strides, alignment, slot and error rules as pa_reshape_and_cache;
 * num_kv_heads*head_dim must be a multiple of 16. pa_decode_fp8 reads the codes back as
 * code * scale. */
PA_API pa_status_t pa_reshape_and_cache_fp8(const void* key, const void* value,
                                     int64_t key_token_stride, int64_t value_token_stride,
                                     void* key_cache, void* value_cache,
                                     const int64_t* slot_mapping, int64_t num_tokens,
                                     int32_t num_kv_heads, int32_t head_dim,
                                     int64_t num_blocks, int32_t block_size, float k_scale,
                                     float v_scale, pa_stream_t stream);

/* Choose a plan from host-known shape values only (no device read). hints may be
 * NULL. The heuristic reads the SM count of the current device and the occupancy of
 * the chosen kernel. */
PA_API pa_status_t pa_decode_plan(int32_t num_seqs, int32_t q_per_seq, int32_t num_q_heads,
                           int32_t num_kv_heads, int32_t head_dim,
                           int32_t max_blocks_per_seq, const pa_plan_hints_t* hints,
                           pa_plan_t* plan);

/* Workspace bytes pa_decode (or pa_decode_fp8) needs for `plan` (NULL = enough for the
 * heuristic plan of these shapes over bf16 pools and over FP8 pools, so that NULL works for
 * both calls when they too are given plan NULL; 0 for invalid shapes or plans). Grid schedule: split partials, 0 when there is one split. Persistent
 * schedule: the pre-pass tables, per-output counters and record lists, and a pool of
 * fp32 partial records (a few MB for the shapes above). tcgen05: two fp32 records of
 * rows_per_cta rows per CTA, a descriptor per CTA and, with sharing, one prefix
 * length per window (about 5 MB for 148 CTAs). */
PA_API size_t pa_decode_workspace_size(const pa_plan_t* plan, int32_t num_seqs,
                                int32_t q_per_seq, int32_t num_q_heads,
                                int32_t num_kv_heads, int32_t head_dim,
                                int32_t max_blocks_per_seq);

/* Paged decode attention. out[b][i][h][:] = sum_t softmax_t(scale * q.k_t) v_t over
 * the visible positions t of sequence b, rounded to bf16 (nearest even) from fp32
 * accumulation. A row with no visible key (context_len < q_per_seq, a precondition
 * violation) yields 0. plan NULL = heuristic. workspace: 16-byte aligned device
 * buffer of at least pa_decode_workspace_size(plan, ...) bytes, may be NULL when
 * that size is 0; its contents need no initialisation and are scratch afterwards
 * (the persistent schedule's pre-pass resets its counters on every call; every
 * tcgen05 CTA rewrites its descriptor on every call). Pool slots outside every
 * sequence's context may hold any bits, NaN included: they never reach the output.
 * Reads query/block_tables/context_lens/caches only after the preceding work on
 * the stream has completed (programmatic dependent launch is used to hide the
 * launch latency). num_seqs == 0 is a no-op. */
PA_API pa_status_t pa_decode(void* out, const void* query, const void* key_cache,
                      const void* value_cache, const int32_t* block_tables,
                      const int32_t* context_lens, int32_t num_seqs, int32_t q_per_seq,
                      int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                      int32_t block_size, int32_t max_blocks_per_seq, int64_t num_blocks,
                      float scale, const pa_plan_t* plan, void* workspace,
                      size_t workspace_bytes, pa_stream_t stream);

/* Paged decode over FP8 KV pools (vLLM study notes §4.2, --kv-cache-dtype fp8: half the
 * cache bytes, so half the memory traffic of attention). key_cache and value_cache hold E4M3
 * codes (uint8 [num_blocks][block_size][num_kv_heads][head_dim], as pa_reshape_and_cache_fp8
 * writes them); element (t, h, d) of a pool has the value code's value * k_scale (v_scale).
 * Result: pa_decode's definition over those values, i.e.
 *   out[b][i][h][:] = sum_t softmax_t(scale * k_scale * q . code_k_t) * v_scale * code_v_t,
 * rounded to bf16 from fp32 accumulation. The codes are widened to f16 exactly and the products
 * run on f16 tensor cores with fp32 accumulators; each query row is scaled by a power of two
 * before its f16 conversion (and the scores back), so any finite bf16 query is accepted.
 * k_scale, v_scale: finite, > 0 (else PA_ERR_INVALID_ARG). plan: NULL = pa_decode_plan's
 * heuristic for FP8 pools, else a plan made with hints.kv_cache_dtype = PA_KV_FP8_E4M3 (a bf16
 * plan is PA_ERR_INVALID_ARG). Everything else -- shapes, layouts, alignment, workspace, the
 * sliding window and prefix sharing of the plan, ownership, streams, errors -- is pa_decode's.
 * Code 0x7F / 0xFF (NaN) in a slot outside every context is harmless, as in pa_decode. */
PA_API pa_status_t pa_decode_fp8(void* out, const void* query, const void* key_cache,
                                 const void* value_cache, const int32_t* block_tables,
                                 const int32_t* context_lens, int32_t num_seqs, int32_t q_per_seq,
                                 int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                 int32_t block_size, int32_t max_blocks_per_seq, int64_t num_blocks,
                                 float scale, float k_scale, float v_scale, const pa_plan_t* plan,
                                 void* workspace, size_t workspace_bytes, pa_stream_t stream);

/* Chunked-prefill paged attention (vLLM study notes, zihan-zhang.net, §3.5 Chunked prefill;
 * "vLLM 深度解析：连续批处理与内存高效推理" §5.4): each sequence attends a chunk of its prompt --
 * many query tokens at once -- over the paged pool, causal within the chunk. The chunk's K/V
 * must already be in the pool (pa_reshape_and_cache with the chunk's slots).
 *   query, out     bf16 [num_query_tokens][num_q_heads][head_dim]: the chunks of all
 *                  sequences, concatenated; sequence b's chunk is rows
 *                  query_start[b] .. query_start[b+1]-1 (qlen_b = their count, may be 0)
 *   query_start    int32 [num_seqs + 1], DEVICE array, non-decreasing, query_start[0] = 0,
 *                  query_start[num_seqs] = num_query_tokens
 *   context_lens   int32 [num_seqs]: tokens of the sequence including its chunk
 *   block_tables, key_cache, value_cache: as pa_decode (bf16 pools)
 * Chunk token i of sequence b sits at position pos = context_lens[b] - qlen_b + i and
 * attends to keys 0 .. pos: out row = sum_t softmax_t(scale * q . k_t) v_t over them, rounded
 * to bf16 from fp32 accumulation (tensor cores: tcgen05.mma, bf16 operands, fp32
 * accumulators in tensor memory). max_query_len: host-known bound on every qlen_b (sizes
 * the grid). scale: finite and >= 0 (else PA_ERR_INVALID_ARG). Supported: head_dim 128,
 * block_size 16, 128 % (num_q_heads / num_kv_heads) == 0 (else PA_ERR_UNSUPPORTED). Preconditions (device data): qlen_b <= max_query_len and
 * qlen_b <= context_lens[b] <= max_blocks_per_seq * block_size, block ids as for pa_decode;
 * a sequence with context_lens[b] < qlen_b gets no rows written. No workspace; nothing is
 * allocated; asynchronous on `stream`; host argument errors as pa_decode's. Zero sequences,
 * tokens or max_query_len is a no-op. */
PA_API pa_status_t pa_prefill(void* out, const void* query, const void* key_cache, const void* value_cache,
                              const int32_t* block_tables, const int32_t* context_lens,
                              const int32_t* query_start, int32_t num_seqs, int32_t num_query_tokens,
                              int32_t max_query_len, int32_t num_q_heads, int32_t num_kv_heads,
                              int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq,
                              int64_t num_blocks, float scale, pa_stream_t stream);

/* Size of the fixed scratch array pa_decode_static_scratch uses (16 MiB, held on
 * every GPU that loads the library until the process exits). */
#define PA_STATIC_SCRATCH_BYTES (16u * 1024u * 1024u)

/* pa_decode for callers that cannot allocate device memory where they decode: code
 * inside another framework's memory pool that has already claimed the GPU's memory,
 * loops that must avoid the implicit synchronisation of cudaMalloc/cudaFree, or
 * plug-in hosts that forbid allocation in their execute step. The source pages have
 * no counterpart to this call; it exists for such callers only.
 * Same arguments and result as pa_decode without the workspace: the split path's
 * partial records go to a PA_STATIC_SCRATCH_BYTES array compiled into the library.
 * The caller still provides every input and output buffer. It calls no allocator.
 * - A plan whose pa_decode_workspace_size exceeds PA_STATIC_SCRATCH_BYTES is
 *   rejected with PA_ERR_WORKSPACE before anything is launched (pass an explicit
 *   plan with longer splits, or use pa_decode).
 * - The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current) and caches it for the life of the
 *   process; make that first call before any stream capture. Do not use this call
 *   after cudaDeviceReset (or any teardown of the device's primary context) in the
 *   same process: the array then lives at a new address that the cache does not see.
 * - All calls share the one array per device and it keeps the last call's contents;
 *   nothing in it needs to start at zero. Calls whose GPU work overlaps (unordered
 *   streams) race on it: keep them ordered on one stream. */
PA_API pa_status_t pa_decode_static_scratch(void* out, const void* query, const void* key_cache,
                                     const void* value_cache, const int32_t* block_tables,
                                     const int32_t* context_lens, int32_t num_seqs,
                                     int32_t q_per_seq, int32_t num_q_heads,
                                     int32_t num_kv_heads, int32_t head_dim,
                                     int32_t block_size, int32_t max_blocks_per_seq,
                                     int64_t num_blocks, float scale, const pa_plan_t* plan,
                                     pa_stream_t stream);

/* Debug check of the device-resident preconditions (synchronous: waits for
 * `stream`). Counts context lengths outside [q_per_seq, max_blocks_per_seq *
 * block_size], used block-table entries outside [0, num_blocks) and slots >=
 * num_blocks*block_size. slot_mapping may be NULL (num_tokens ignored). On return
 * *num_bad (may be NULL) holds the count; the status is PA_ERR_OUT_OF_RANGE when
 * it is non-zero. */
PA_API pa_status_t pa_validate(const int32_t* block_tables, const int32_t* context_lens,
                        const int64_t* slot_mapping, int32_t num_seqs,
                        int32_t max_blocks_per_seq, int32_t q_per_seq,
                        int64_t num_tokens, int64_t num_blocks, int32_t block_size,
                        int64_t* num_bad, pa_stream_t stream);

/* Reads (and with reset != 0 clears) the device error word that kernels set when a
 * bounded wait times out (synchronous: waits for `stream`). *code = 0 means no
 * error; the status is PA_ERR_DEVICE when *code != 0. The first code set since the
 * last reset is kept:
 *   0x100 a decode wait timed out, 0x200 draining in-flight copies timed out,
 *   0x300 / 0x400 the persistent schedule's record pool / list is full,
 *   0x500 an inconsistent schedule or shared-memory layout, 0x600 the self-test. */
PA_API pa_status_t pa_get_device_error(uint32_t* code, int32_t reset, pa_stream_t stream);

/* Self-test of the failure path (no counterpart on the pages): enqueues one CTA that
 * waits on an mbarrier nothing completes; after the bounded-wait limit (about 1 s)
 * it records 0x600 in the device error word and returns, leaving the context usable.
 * Asynchronous; read the result with pa_get_device_error. */
PA_API pa_status_t pa_selftest_bounded_wait(pa_stream_t stream);

/* Copy-on-write block copy (vLLM study notes, zihan-zhang.net, §3.2.2 写时复制: a
 * sequence about to write into a block other sequences still reference first gets a copy
 * of it; "vLLM 深度解析：连续批处理与内存高效推理" §2.1 Copy on Write and §4.2, the forks of
 * parallel sampling and beam search). For each pair p of block_mapping ([num_pairs][2] =
 * {source, destination} physical block ids), every element of the source block -- its
 * block_size tokens x num_kv_heads x head_dim values -- is copied onto the destination
 * block, in key_cache and in value_cache. Bit-exact; every other block is left untouched.
 * A pair with a negative entry is padding and is skipped.
 *   block_mapping is a HOST array (the block manager decides the copies on the host). It
 *   is read during the call, its entries travel inside the launches (up to 2048 pairs a
 *   launch), and it may be reused as soon as the call returns.
 *   Host checks, before anything is enqueued: block_size 16, head_dim 64 or 128
 *   (else PA_ERR_UNSUPPORTED); num_kv_heads >= 1, num_pairs >= 0 (0 is a no-op), non-null
 *   16-byte aligned pools (else PA_ERR_INVALID_ARG); every id < num_blocks (else
 *   PA_ERR_OUT_OF_RANGE); destinations distinct and none of them also a source (else
 *   PA_ERR_INVALID_ARG: the result would depend on the order of the copies). */
PA_API pa_status_t pa_copy_blocks(void* key_cache, void* value_cache, int64_t num_blocks,
                                  int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                  const int64_t* block_mapping, int64_t num_pairs,
                                  pa_stream_t stream);

/* Context parallelism, step 1 (vLLM study notes §4.3.1: the softmax of a split context is
 * recovered from per-split maxima and sums). The table entries block_begin <= j < block_end
 * (positions 16j .. 16j+15) of every sequence are cut into num_pieces equal pieces
 * (ceil((block_end - block_begin) / num_pieces) entries each, the last ones shorter or empty);
 * for piece k, sequence b and query row (i, h), the attention of pa_decode restricted to the
 * visible keys of the piece, written unnormalised and part-major:
 *   part_o [num_pieces][num_seqs][q_per_seq][num_q_heads][head_dim] fp32: sum_t 2^(s_t - m) v_t
 *   part_ml [num_pieces][num_seqs][q_per_seq][num_q_heads][2] fp32: {m, l = sum_t 2^(s_t - m)}
 * with s_t the score in log2 units (q.k * scale * log2 e) and m the largest s_t of the piece
 * (o / l and m + log2 l are what a merge needs); m = -inf, l = 0 and o = 0 when no key of the
 * piece is visible. Positions are the sequence's own (key 16j + r, query row i at
 * context_len - q_per_seq + i), so every GPU of a split passes the full context_lens and a block
 * table whose entries [block_begin, block_end) name blocks of its own pool (the other entries
 * are not read). bf16 pools only; same checks and preconditions as pa_decode, plus 0 <=
 * block_begin <= block_end <= max_blocks_per_seq and 1 <= num_pieces <= 65535 (else
 * PA_ERR_INVALID_ARG) and 16-byte aligned part_o / part_ml. Grid schedule, one CTA per (kv
 * head, sequence, piece); no workspace. */
PA_API pa_status_t pa_decode_partial(float* part_o, float* part_ml, const void* query, const void* key_cache,
                                     const void* value_cache, const int32_t* block_tables,
                                     const int32_t* context_lens, int32_t num_seqs, int32_t q_per_seq,
                                     int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                     int32_t block_size, int32_t max_blocks_per_seq, int64_t num_blocks,
                                     float scale, int32_t block_begin, int32_t block_end, int32_t num_pieces,
                                     pa_stream_t stream);

/* Pieces for pa_decode_partial over ranges of range_blocks table entries: the split count the
 * decode heuristic takes for tables of that length on this device (host-known values only; the
 * same on every GPU of a group, so the gathered pieces have one shape); 0 for bad shapes. */
PA_API int32_t pa_decode_partial_pieces(int32_t num_seqs, int32_t q_per_seq, int32_t num_q_heads,
                                        int32_t num_kv_heads, int32_t head_dim, int32_t range_blocks);

/* Context parallelism, between steps 1 and 2 (on each GPU, so that the exchange carries one
 * record per row): the num_parts pieces of each row (part_o / part_ml laid out as
 * pa_decode_partial writes them) combined into one record of the same form, rec_o
 * [num_seqs][q][H_q][D] = sum_k 2^(m_k - M) o_k and rec_ml [num_seqs][q][H_q][2] = {M, sum_k
 * 2^(m_k - M) l_k}, M the largest m_k (-inf, 0 and o = 0 when every piece is empty). Checks as
 * pa_merge_partials. */
PA_API pa_status_t pa_combine_partials(float* rec_o, float* rec_ml, const float* part_o, const float* part_ml,
                                       int32_t num_parts, int32_t num_seqs, int32_t q_per_seq,
                                       int32_t num_q_heads, int32_t head_dim, pa_stream_t stream);

/* Context parallelism, step 2: out[b][i][h] = sum_k 2^(m_k - M) o_k / sum_k 2^(m_k - M) l_k over
 * num_parts pieces laid out part-major (part_o [num_parts][num_seqs][q][H_q][D], part_ml
 * [num_parts][num_seqs][q][H_q][2], as an all-gather of every GPU's pa_decode_partial pieces
 * leaves them: num_parts = GPUs x num_pieces),
 * M the largest m_k; a row whose pieces are all empty gets zeros. Pieces over disjoint ranges that
 * together cover every context give pa_decode's result. bf16 out [num_seqs][q][H_q][D]; head_dim
 * 64 or 128; 16-byte aligned buffers (else PA_ERR_INVALID_ARG / PA_ERR_UNSUPPORTED). */
PA_API pa_status_t pa_merge_partials(void* out, const float* part_o, const float* part_ml, int32_t num_parts,
                                     int32_t num_seqs, int32_t q_per_seq, int32_t num_q_heads,
                                     int32_t head_dim, pa_stream_t stream);

/* Static description of a status code. */
PA_API const char* pa_status_string(pa_status_t status);

/* ABI version (major * 10000 + minor * 100 + patch). 1.1 added pa_decode_fp8, pa_prefill
 * and the kv_cache_dtype fields at the end of pa_plan_hints_t and pa_plan_t; 1.2 added
 * pa_decode_partial, pa_decode_partial_pieces, pa_combine_partials and pa_merge_partials. */
PA_API int32_t pa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
