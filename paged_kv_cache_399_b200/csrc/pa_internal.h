// Internal interface between the host API (pa_api.cpp) and the kernels
// (pa_kernels.cu). Not part of the public ABI.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace pa {

constexpr int kBlockSize = 16;   // tokens per KV block
constexpr int kWarpsPerCta = 4;  // decode CTA = 4 warps, each with its own TMA pipeline

struct DecodeParams {
  uint16_t* out;                 // bf16 [B][q][H_q][D]
  const uint16_t* query;         // bf16 [B][q][H_q][D]
  const int32_t* block_tables;   // [B][max_blocks]
  const int32_t* context_lens;   // [B]
  float* ws_o;                   // fp32 [B][num_splits][q*H_q][D]   (split plans only)
  float2* ws_ml;                 // fp32 [B][num_splits][q*H_q] (m in log2 units, l)
  int32_t num_seqs, q_per_seq, num_q_heads, num_kv_heads, group;  // group = H_q / H_kv
  int32_t rows;                  // group * q_per_seq query rows per kv head
  int32_t max_blocks, split_blocks, num_splits, row_chunks, rows_per_cta;
  float scale_log2;              // scale * log2(e)
};

// Kernel families (pa_path_t values).
constexpr int kPathSingle = 1;
constexpr int kPathTile = 2;

// Largest rows_per_cta each family is instantiated for.
constexpr int kTileMaxRows = 32;   // 4 n-tiles of 8 rows
constexpr int kSingleMaxRows = 8;

// Launch the decode kernel of `path` (and the merge kernel when num_splits > 1).
cudaError_t launch_decode(const DecodeParams& p, int path, int head_dim,
                          const CUtensorMap& tmap_k, const CUtensorMap& tmap_v,
                          cudaStream_t stream);

// Resident CTAs per SM of the decode kernel that launch_decode would use.
int decode_ctas_per_sm(int path, int head_dim, int rows_per_cta);

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

}  // namespace pa
