// Internal interface between the host API (pa_api.cpp) and the kernels
// (pa_kernels.cu). Not part of the public ABI.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "pa.h"

namespace pa {

constexpr int kBlockSize = 16;   // tokens per KV block
constexpr int kWarpsPerCta = 4;  // decode CTA = 4 warps, each with its own TMA pipeline

// Kernel families (pa_path_t values) and schedules (pa_schedule_t values).
constexpr int kPathSingle = 1;
constexpr int kPathTile = 2;
constexpr int kPathTcgen05 = 3;
constexpr int kScheduleGrid = 1;
constexpr int kSchedulePersistent = 2;

// Largest rows one CTA holds for each family.
constexpr int kTileMaxRows = 32;   // 4 n-tiles of 8 rows
constexpr int kSingleMaxRows = 8;
constexpr int kTcmMaxRows = 32;   // tcgen05 kernel: query rows of a unit (the MMA's N)

// Persistent schedule: header written by the pre-pass, read by the decode CTAs.
struct SchedHeader {
  long long work;   // total work units (blocks x kv-head sub-units), W
  int pool;         // partial records handed out so far
  int pad[13];
};

struct DecodeParams {
  uint16_t* out;                 // bf16 [B][q][H_q][D]
  const uint16_t* query;         // bf16 [B][q][H_q][D]
  const int32_t* block_tables;   // [B][max_blocks]
  const int32_t* context_lens;   // [B]
  int32_t num_seqs, q_per_seq, num_q_heads, num_kv_heads, group;  // group = H_q / H_kv
  int32_t rows;                  // group * q_per_seq query rows per (sequence, kv head)
  int32_t max_blocks;
  int64_t num_blocks;             // pool size (blocks)
  int32_t rows_per_cta;          // rows the kernel instance holds (ROWS)
  int32_t row_chunks;            // ceil(rows / rows_per_cta)
  float scale_log2;              // scale * log2(e) (E4M3 pools: times the key pool's scale)
  float v_scale;                 // E4M3 pools: the value pool's scale (1 for bf16 pools)
  int32_t window;                // sliding window in tokens (grid schedule only); 0 = none

  // grid schedule: split partials for the merge kernel; with prefix sharing also the
  // shared-prefix splits (a 1-D grid: shared CTAs, then the sequences' own CTAs)
  int32_t split_blocks, num_splits;
  int32_t share_split_blocks, share_splits, share_windows;
  float* ws_o;                   // fp32 [B][num_splits][q*H_q][D]
  float2* ws_ml;                 // fp32 [B][num_splits][q*H_q] (m in log2 units, l)

  // persistent schedule
  int32_t num_ctas;              // persistent grid size
  int32_t share_cap;             // >= 2: members per shared-prefix unit; 0: no prefix sharing
  int32_t target_rows;           // rows of one output target (<= rows_per_cta)
  int32_t list_cap;              // record list capacity per target
  int32_t pool_cap;              // record pool capacity
  int32_t rec_stride;            // floats per record: target_rows * D + 2 * target_rows
  SchedHeader* hdr;
  long long* seq_start;          // [B] first work unit of the sequence's bands
  int4* seq_info;                // [B] {P_b shared prefix blocks, members if leader else 0, nblk, ctx}
  int32_t* cta_seq;              // [num_ctas] sequence holding the CTA's first unit
  int32_t* arrive;               // [targets] blocks merged so far
  int32_t* list_len;             // [targets]
  int2* list;                    // [targets][list_cap] {piece start block, record slot}
  float* records;                // [pool_cap][rec_stride]; tcgen05 path: [2 * num_ctas][rec_stride]

  // tcgen05 path: per CTA, the unit whose first piece it holds when that unit continues
  // in later CTAs: {record slot, last CTA with a piece, sequence, unit}, or {-1, ...}
  int4* tc_desc;
  int32_t tc_group;              // tcgen05 path: CTAs per group (a divisor of num_kv_heads)
  int32_t* win_prefix;           // tcgen05 path with prefix sharing: shared blocks per window
  // tcgen05 path: query tokens of one TMA box of Q rows ({64 of D, group heads, q_box
  // tokens}: the rows of one row chunk, or of a shared-prefix window); 0 = Q rows are
  // loaded with plain loads (a group that does not divide the MMA's N)
  int32_t q_box;
  // context parallelism (grid schedule): only table entries [range_lo, range_hi) of every
  // sequence are read, cut into num_splits pieces, and every CTA writes its (o, m, l) record
  // part-major ([piece][sequence][row]), never the output; num_parts > 0: the merge combines
  // num_parts such records per row, laid out [part][sequence][row] (gathered pieces)
  int32_t range_lo, range_hi, partial_only, num_parts;
  // num_parts > 0 with partial_only: the merge writes one fp32 record per row instead of the
  // output (o against the row's M [sequence][row][D], {M, L} [sequence][row])
  float* rec_o;
  float2* rec_ml;
};

// Host-side checks of a decode call's shapes and (when non-null) its plan, the ones
// pa_decode runs before anything else; returns a pa_status_t value. The workspace size
// query and the static-scratch entry point run them first, because the sizes divide by
// plan and shape fields.
int check_decode_args(const pa_plan_t* plan, int32_t num_seqs, int32_t q_per_seq, int32_t num_q_heads,
                      int32_t num_kv_heads, int32_t head_dim, int32_t max_blocks_per_seq);

// KV pool element types.
constexpr int kKvBf16 = 0;
constexpr int kKvE4M3 = 1;

// Launch the decode (pre-pass + persistent kernel, or grid kernel + merge) over pools of
// element type kv_dtype. tmap_q: the query map of a tcgen05 plan with p.q_box > 0 (else
// unused).
cudaError_t launch_decode(const DecodeParams& p, int path, int schedule, int head_dim, int kv_dtype,
                          const CUtensorMap& tmap_k, const CUtensorMap& tmap_v, const CUtensorMap& tmap_q,
                          cudaStream_t stream);

// Chunked-prefill attention (pa_prefill.cuh): one CTA per (kv head, sequence, tile of
// 128 / G chunk tokens counted from the chunk's end), max_tiles tiles per sequence.
struct PrefillParams {
  uint16_t* out;                 // bf16 [T][H_q][D]
  const uint16_t* query;         // bf16 [T][H_q][D]
  const int32_t* block_tables;   // [B][max_blocks]
  const int32_t* context_lens;   // [B], including the chunk's tokens
  const int32_t* query_start;    // [B + 1], first token of each sequence's chunk in query/out
  int32_t num_seqs, num_q_heads, num_kv_heads, group, max_blocks;
  int32_t tile_tokens;           // chunk tokens per CTA: 128 / group
  int64_t num_blocks;            // pool size (blocks)
  float scale_log2;              // scale * log2(e)
};
cudaError_t launch_prefill(const PrefillParams& p, int max_tiles, const CUtensorMap& tmap_k,
                           const CUtensorMap& tmap_v, cudaStream_t stream);

// The merge of a gathered set of p.num_parts partial decodes (p.ws_o, p.ws_ml laid out
// [part][sequence][row]) into p.out.
cudaError_t launch_merge_partials(const DecodeParams& p, int head_dim, cudaStream_t stream);

// Resident CTAs per SM of the decode kernel launch_decode would use.
int decode_ctas_per_sm(int path, int schedule, int head_dim, int rows_per_cta, int kv_dtype);

cudaError_t launch_cache_write(const uint16_t* key, const uint16_t* value, int64_t key_stride,
                               int64_t value_stride, uint16_t* key_cache, uint16_t* value_cache,
                               const int64_t* slots, int64_t num_tokens, int32_t row_elems,
                               int64_t num_slots, cudaStream_t stream);

// Synchronous debug check; *bad receives the number of violations.
cudaError_t run_validate(const int32_t* block_tables, const int32_t* context_lens,
                         const int64_t* slots, int32_t num_seqs, int32_t max_blocks,
                         int32_t q_per_seq, int64_t num_tokens, int64_t num_blocks,
                         int64_t* bad, cudaStream_t stream);

cudaError_t read_device_error(uint32_t* code, bool reset, cudaStream_t stream);

// Launch the bounded-wait self-test kernel (about one wait limit long).
cudaError_t run_selftest_wait(cudaStream_t stream);

}  // namespace pa
