// Copy-on-write block copy (vLLM study notes, zihan-zhang.net, §3.2.2 写时复制; "vLLM
// 深度解析：连续批处理与内存高效推理" §2.1 Copy on Write and §4.2 reference counts): when a
// sequence is about to write into a block that other sequences still reference (the
// samples of a parallel-sampling fork, the beams of a beam search), the block manager
// gives it a fresh block holding a copy of the shared one. This file is the copy: for
// each {source, destination} pair every byte of the source block is copied onto the
// destination block, in the key pool and in the value pool.
//
// A pure HBM-bandwidth kernel: each byte is read once and written once. The mapping
// comes from the host (the block manager decides the copies there) and travels inside
// the launch parameters, so nothing is staged in device memory. Work items are
// (pair, pool, 32 KB chunk); each thread keeps kUnroll 16-byte loads in flight before
// it stores them, and the grid is kCtasPerSm CTAs per SM (one wave) or the item count.
//
// Self-contained: shares no code with the decode kernels.

#include <algorithm>
#include <cstdint>
#include <cuda_runtime.h>
#include <mutex>
#include <vector>

#include "pa.h"

namespace pa_copy {

constexpr int kThreads = 256;
constexpr int kUnroll = 8;                            // 16-byte words in flight per thread
constexpr int64_t kChunkWords = kThreads * kUnroll;   // 32 KB per work item
constexpr int kBlockSize = 16;
constexpr int kCtasPerSm = 4;                         // 128 KB of loads in flight per SM

template <int kCap>
struct CopyArgs {
  uint4* pool[2];      // key pool, value pool, as 16-byte words
  int64_t words;       // 16-byte words per block
  int32_t chunks;      // work items per (pair, pool)
  int32_t num_pairs;
  int32_t src[kCap];
  int32_t dst[kCap];
};

__device__ __forceinline__ uint4 load_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.cs.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void store_stream(uint4* p, const uint4& v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

template <int kCap>
__global__ void __launch_bounds__(kThreads, kCtasPerSm) copy_blocks_kernel(const __grid_constant__ CopyArgs<kCap> a) {
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the pools may come from the previous kernel
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int64_t items = static_cast<int64_t>(a.num_pairs) * 2 * a.chunks;
  for (int64_t it = blockIdx.x; it < items; it += gridDim.x) {
    const int64_t pp = it / a.chunks;  // (pair, pool)
    const int part = static_cast<int>(it - pp * a.chunks);
    const int pair = static_cast<int>(pp >> 1);
    uint4* base = a.pool[pp & 1];
    const uint4* s = base + static_cast<int64_t>(a.src[pair]) * a.words;
    uint4* d = base + static_cast<int64_t>(a.dst[pair]) * a.words;
    const int64_t w0 = part * kChunkWords + threadIdx.x;
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t w = w0 + u * kThreads;
      if (w < a.words) v[u] = load_stream(s + w);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t w = w0 + u * kThreads;
      if (w < a.words) store_stream(d + w, v[u]);
    }
  }
}

int sm_count() {
  static std::mutex mu;
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (dev < 64 && cached[dev] > 0) return cached[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (dev < 64) cached[dev] = n;
  return n;
}

template <int kCap>
cudaError_t launch(void* key_cache, void* value_cache, int64_t words, const int64_t* mapping, int64_t first,
                   int n, int sms, cudaStream_t stream) {
  CopyArgs<kCap> a;
  a.pool[0] = static_cast<uint4*>(key_cache);
  a.pool[1] = static_cast<uint4*>(value_cache);
  a.words = words;
  a.chunks = static_cast<int32_t>((words + kChunkWords - 1) / kChunkWords);
  a.num_pairs = 0;
  for (int i = 0; i < n; ++i) {
    const int64_t s = mapping[2 * (first + i)], d = mapping[2 * (first + i) + 1];
    if (s < 0 || d < 0) continue;  // padding
    a.src[a.num_pairs] = static_cast<int32_t>(s);
    a.dst[a.num_pairs] = static_cast<int32_t>(d);
    ++a.num_pairs;
  }
  if (a.num_pairs == 0) return cudaSuccess;
  const int64_t items = static_cast<int64_t>(a.num_pairs) * 2 * a.chunks;
  const int64_t resident = static_cast<int64_t>(sms) * kCtasPerSm;
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>(items, resident));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, copy_blocks_kernel<kCap>, a);
}

constexpr int kSmallCap = 128;
constexpr int kLargeCap = 2048;

}  // namespace pa_copy

extern "C" PA_API pa_status_t pa_copy_blocks(void* key_cache, void* value_cache, int64_t num_blocks,
                                             int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                             const int64_t* block_mapping, int64_t num_pairs,
                                             pa_stream_t stream) {
  using namespace pa_copy;
  if (num_pairs < 0 || num_blocks <= 0 || num_kv_heads <= 0) return PA_ERR_INVALID_ARG;
  if (block_size != kBlockSize || (head_dim != 64 && head_dim != 128)) return PA_ERR_UNSUPPORTED;
  if (num_blocks > INT32_MAX) return PA_ERR_UNSUPPORTED;
  if (num_pairs == 0) return PA_OK;
  if (!key_cache || !value_cache || !block_mapping) return PA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(key_cache) | reinterpret_cast<uintptr_t>(value_cache)) & 15u)
    return PA_ERR_INVALID_ARG;
  // ids inside the pool; destinations distinct and never a source (else the result would
  // depend on the order of the copies). A bitmap of the pool's blocks, kept per thread
  // and cleared after use, makes this O(pairs).
  for (int64_t i = 0; i < 2 * num_pairs; ++i)
    if (block_mapping[i] >= num_blocks) return PA_ERR_OUT_OF_RANGE;
  thread_local std::vector<uint64_t> marks;
  const size_t words_needed = static_cast<size_t>((num_blocks + 63) / 64);
  if (marks.size() < words_needed) marks.assign(words_needed, 0);
  auto mark = [&](int64_t b) { return (marks[b >> 6] >> (b & 63)) & 1u; };
  pa_status_t verdict = PA_OK;
  int64_t marked = 0;  // pairs whose destination was marked
  for (; marked < num_pairs; ++marked) {
    const int64_t s = block_mapping[2 * marked], d = block_mapping[2 * marked + 1];
    if (s < 0 || d < 0) continue;
    if (mark(d)) {
      verdict = PA_ERR_INVALID_ARG;
      break;
    }
    marks[d >> 6] |= 1ull << (d & 63);
  }
  for (int64_t i = 0; verdict == PA_OK && i < num_pairs; ++i) {
    const int64_t s = block_mapping[2 * i], d = block_mapping[2 * i + 1];
    if (s >= 0 && d >= 0 && mark(s)) verdict = PA_ERR_INVALID_ARG;
  }
  for (int64_t i = 0; i < marked; ++i) {
    const int64_t s = block_mapping[2 * i], d = block_mapping[2 * i + 1];
    if (s >= 0 && d >= 0) marks[d >> 6] &= ~(1ull << (d & 63));
  }
  if (verdict != PA_OK) return verdict;
  const int sms = sm_count();
  if (sms <= 0) return PA_ERR_CUDA;
  const int64_t words = static_cast<int64_t>(block_size) * num_kv_heads * head_dim * 2 / 16;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  for (int64_t first = 0; first < num_pairs; first += kLargeCap) {
    const int n = static_cast<int>(std::min<int64_t>(kLargeCap, num_pairs - first));
    const cudaError_t e = n <= kSmallCap ? launch<kSmallCap>(key_cache, value_cache, words, block_mapping, first, n, sms, st)
                                         : launch<kLargeCap>(key_cache, value_cache, words, block_mapping, first, n, sms, st);
    if (e != cudaSuccess) return PA_ERR_CUDA;
  }
  return PA_OK;
}
