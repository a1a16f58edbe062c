// FP8 KV cache write (vLLM study notes, zihan-zhang.net, §4.2: an FP8 KV cache,
// --kv-cache-dtype fp8, doubles the cache's capacity and halves attention's memory traffic).
// The format is E4M3 (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits, no
// infinities, largest finite 448) with one fp32 scale per pool passed by the caller: each
// bf16 element x of the step's new K (V) rows is stored as the E4M3 code of the fp32
// quotient x / k_scale (x / v_scale), rounded to nearest with ties to even and saturated at
// +-448, at the pool position the slot mapping names.
//
// A pure bandwidth kernel: each thread reads 16 bf16 elements (two 16-byte loads), divides
// them by the pool scale (IEEE division, so that the stored code is the one the fp32 quotient
// determines) and converts pairs with cvt.rn.satfinite.e4m3x2.f32, then writes 16 codes with
// one 16-byte store. Self-contained: shares no code with the decode kernels.

#include <cmath>
#include <cstdint>
#include <cuda_runtime.h>

#include "pa.h"

namespace pa_fp8 {

constexpr int kBlockSize = 16;
constexpr int kThreads = 256;

// Two fp32 values -> two E4M3 codes (round to nearest even, saturating): lo in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__global__ void __launch_bounds__(kThreads)
cache_write_fp8_kernel(const uint16_t* __restrict__ key, const uint16_t* __restrict__ value,
                       int64_t key_stride, int64_t value_stride, uint8_t* __restrict__ key_cache,
                       uint8_t* __restrict__ value_cache, const int64_t* __restrict__ slots,
                       int64_t num_tokens, int32_t row_elems, int64_t num_slots, float k_scale,
                       float v_scale) {
  asm volatile("griddepcontrol.wait;" ::: "memory");  // inputs may come from the previous kernel
  const int chunks = row_elems / 16;                    // 16-element pieces of one row
  const int64_t per_token = 2 * static_cast<int64_t>(chunks);
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= num_tokens * per_token) return;
  const int64_t t = idx / per_token;
  const int rem = static_cast<int>(idx - t * per_token);
  const bool is_v = rem >= chunks;
  const int ch = is_v ? rem - chunks : rem;
  const int64_t slot = __ldg(slots + t);
  if (slot < 0 || slot >= num_slots) return;  // padding, or outside the pool: nothing written
  const uint4* src =
      reinterpret_cast<const uint4*>((is_v ? value : key) + t * (is_v ? value_stride : key_stride) + ch * 16);
  const float s = is_v ? v_scale : k_scale;
  const uint4 a = __ldg(src), b = __ldg(src + 1);
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};  // bf16 pairs, element 2i in the low half
  uint32_t out[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float f0 = __uint_as_float(w[2 * i] << 16), f1 = __uint_as_float(w[2 * i] & 0xFFFF0000u);
    const float f2 = __uint_as_float(w[2 * i + 1] << 16), f3 = __uint_as_float(w[2 * i + 1] & 0xFFFF0000u);
    out[i] = e4m3x2(__fdiv_rn(f0, s), __fdiv_rn(f1, s)) | (e4m3x2(__fdiv_rn(f2, s), __fdiv_rn(f3, s)) << 16);
  }
  uint8_t* dst = (is_v ? value_cache : key_cache) + slot * row_elems + ch * 16;
  *reinterpret_cast<uint4*>(dst) = make_uint4(out[0], out[1], out[2], out[3]);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace pa_fp8

extern "C" PA_API pa_status_t pa_reshape_and_cache_fp8(const void* key, const void* value,
                                                       int64_t key_token_stride, int64_t value_token_stride,
                                                       void* key_cache, void* value_cache,
                                                       const int64_t* slot_mapping, int64_t num_tokens,
                                                       int32_t num_kv_heads, int32_t head_dim,
                                                       int64_t num_blocks, int32_t block_size, float k_scale,
                                                       float v_scale, pa_stream_t stream) {
  using namespace pa_fp8;
  if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || num_blocks <= 0) return PA_ERR_INVALID_ARG;
  if (!(std::isfinite(k_scale) && k_scale > 0.f && std::isfinite(v_scale) && v_scale > 0.f))
    return PA_ERR_INVALID_ARG;
  if (block_size != kBlockSize) return PA_ERR_UNSUPPORTED;
  const int64_t row_elems = static_cast<int64_t>(num_kv_heads) * head_dim;
  if (row_elems % 16 != 0 || row_elems > INT32_MAX) return PA_ERR_UNSUPPORTED;
  if (key_token_stride < row_elems || value_token_stride < row_elems) return PA_ERR_INVALID_ARG;
  if ((key_token_stride * 2) % 16 != 0 || (value_token_stride * 2) % 16 != 0) return PA_ERR_INVALID_ARG;
  if (num_tokens == 0) return PA_OK;
  if (!key || !value || !key_cache || !value_cache || !slot_mapping) return PA_ERR_INVALID_ARG;
  if (!aligned16(key) || !aligned16(value) || !aligned16(key_cache) || !aligned16(value_cache) ||
      (reinterpret_cast<uintptr_t>(slot_mapping) & 7u))
    return PA_ERR_INVALID_ARG;
  if (num_tokens > (int64_t{1} << 30)) return PA_ERR_UNSUPPORTED;
  const int64_t threads = num_tokens * 2 * (row_elems / 16);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((threads + kThreads - 1) / kThreads));
  cfg.blockDim = dim3(kThreads);
  cfg.stream = reinterpret_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(
      &cfg, cache_write_fp8_kernel, static_cast<const uint16_t*>(key), static_cast<const uint16_t*>(value),
      key_token_stride, value_token_stride, static_cast<uint8_t*>(key_cache), static_cast<uint8_t*>(value_cache),
      slot_mapping, num_tokens, static_cast<int32_t>(row_elems), num_blocks * kBlockSize, k_scale, v_scale);
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
