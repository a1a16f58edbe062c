// pa_decode_static_scratch: paged decode with its split-context scratch taken from
// a fixed array compiled into this library, so the caller allocates nothing.
//
// Who needs it: callers that cannot call cudaMalloc where they decode -- code that
// runs inside another framework's device-memory pool which has already reserved the
// GPU's memory (a fresh cudaMalloc there fails or fragments the pool), serving loops
// that must not pay the implicit device synchronisation of cudaMalloc/cudaFree, and
// plug-in hosts whose execute callbacks forbid allocation. They still pass every
// input and output buffer; only the fp32 partial records of the split path (o, m, l
// per split and query row) live in the array below.
//
// Sharing: every call on a device uses the same array and it keeps what the last
// call wrote. Nothing in it has to start at zero: each record the merge kernel
// reads was written earlier in the same call. Two calls whose work overlaps on the
// GPU (different streams, no ordering between them) race on the array and give
// wrong results; order such calls on one stream or use pa_decode with separate
// workspaces.

#include "pa.h"

#include <cuda_runtime.h>

#include <mutex>

#include "pa_internal.h"

namespace {

// File-scope scratch, PA_STATIC_SCRATCH_BYTES on every GPU that loads this library,
// held until the process exits. Host code must not use this name as an address:
// it is a host-side stand-in, so the device address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_static_scratch[PA_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

// Device address of g_static_scratch on the current device, looked up once per
// device (with that device current) and cached. Returns nullptr on failure.
void* scratch_address() {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess) return nullptr;
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace

extern "C" PA_API pa_status_t pa_decode_static_scratch(
    void* out, const void* query, const void* key_cache, const void* value_cache,
    const int32_t* block_tables, const int32_t* context_lens, int32_t num_seqs, int32_t q_per_seq,
    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
    int32_t max_blocks_per_seq, int64_t num_blocks, float scale, const pa_plan_t* plan,
    pa_stream_t stream) {
  pa_plan_t local;
  if (plan == nullptr) {
    const pa_status_t st = pa_decode_plan(num_seqs, q_per_seq, num_q_heads, num_kv_heads, head_dim,
                                          max_blocks_per_seq, nullptr, &local);
    if (st != PA_OK) return st;
    plan = &local;
  } else {
    // the same shape and plan checks pa_decode runs, before the size below is computed
    const int st = pa::check_decode_args(plan, num_seqs, q_per_seq, num_q_heads, num_kv_heads, head_dim,
                                         max_blocks_per_seq);
    if (st != PA_OK) return static_cast<pa_status_t>(st);
  }
  const size_t need = pa_decode_workspace_size(plan, num_seqs, q_per_seq, num_q_heads, num_kv_heads,
                                               head_dim, max_blocks_per_seq);
  if (need > PA_STATIC_SCRATCH_BYTES) return PA_ERR_WORKSPACE;  // plan too large for the array
  void* scratch = nullptr;
  if (need > 0) {
    scratch = scratch_address();
    if (scratch == nullptr) return PA_ERR_CUDA;
  }
  return pa_decode(out, query, key_cache, value_cache, block_tables, context_lens, num_seqs,
                   q_per_seq, num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                   num_blocks, scale, plan, scratch, need > 0 ? PA_STATIC_SCRATCH_BYTES : 0, stream);
}
