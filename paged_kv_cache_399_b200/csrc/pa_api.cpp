// Host side of the C ABI declared in include/pa.h: argument checks, the plan
// heuristic, TMA descriptors for the paged pool, and the kernel launches.
// Nothing here touches device data; all work is enqueued on the caller's stream.

#include "pa.h"

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "pa_internal.h"

namespace {

using pa::DecodeParams;

constexpr int32_t kVersion = 10200;  // 1.2.0

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// ----------------------------------------------------------------- device facts

struct DeviceInfo {
  int sms = 0;
};

DeviceInfo device_info() {
  static std::mutex mu;
  static DeviceInfo cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DeviceInfo{148};
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev].sms == 0) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
      sms = 148;
    cache[dev].sms = sms;
  }
  return cache[dev];
}

// ----------------------------------------------------------------- TMA descriptors

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// The pool [num_blocks][16][H_kv][D] as a 3-D tensor {D, H_kv, num_blocks*16}; one
// box is {64, 1, 16}: half of head_dim for one kv head over the 16 tokens of a block,
// 128-byte swizzled in shared memory.
// E4M3 pools ([num_blocks][16][H_kv][D] bytes): one box is {D, 1, 16}, a whole block of one
// kv head (16 rows of D bytes), with the 128-byte swizzle at D = 128 and the 64-byte one at
// D = 64.
bool encode_pool_map_uncached(CUtensorMap* map, const void* base, int64_t num_blocks, int32_t num_kv_heads,
                              int32_t head_dim, int kv_dtype);

// The maps of the last few pools this thread used: encoding costs microseconds of host
// time on every call otherwise, and a decode loop passes the same two pools each step.
bool encode_pool_map(CUtensorMap* map, const void* base, int64_t num_blocks, int32_t num_kv_heads,
                     int32_t head_dim, int kv_dtype) {
  struct Entry {
    const void* base;
    int64_t num_blocks;
    int32_t num_kv_heads, head_dim, kv_dtype;
    CUtensorMap map;
  };
  thread_local Entry cache[4] = {};
  thread_local int next = 0;
  for (const Entry& e : cache)
    if (e.base == base && e.base != nullptr && e.num_blocks == num_blocks && e.num_kv_heads == num_kv_heads &&
        e.head_dim == head_dim && e.kv_dtype == kv_dtype) {
      *map = e.map;
      return true;
    }
  if (!encode_pool_map_uncached(map, base, num_blocks, num_kv_heads, head_dim, kv_dtype)) return false;
  cache[next] = Entry{base, num_blocks, num_kv_heads, head_dim, kv_dtype, *map};
  next = (next + 1) & 3;
  return true;
}

bool encode_pool_map_uncached(CUtensorMap* map, const void* base, int64_t num_blocks, int32_t num_kv_heads,
                              int32_t head_dim, int kv_dtype) {
  auto fn = encode_fn();
  if (!fn) return false;
  const bool e4m3 = kv_dtype == pa::kKvE4M3;
  const cuuint64_t elem = e4m3 ? 1 : 2;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(num_kv_heads),
                        static_cast<cuuint64_t>(num_blocks) * pa::kBlockSize};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_dim) * elem,
                           static_cast<cuuint64_t>(head_dim) * num_kv_heads * elem};
  cuuint32_t box[3] = {e4m3 ? static_cast<cuuint32_t>(head_dim) : 64u, 1, static_cast<cuuint32_t>(pa::kBlockSize)};
  cuuint32_t elem_strides[3] = {1, 1, 1};
  const CUtensorMapSwizzle swz =
      (e4m3 && head_dim == 64) ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  CUresult r = fn(map, e4m3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                  const_cast<void*>(base), dims, strides, box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Query rows of the tcgen05 decode as TMA boxes: the query [tokens][H_q][D] as a 3-D map
// {D, H_q, tokens}, box {64 of D, group heads, box_tokens tokens} with the 128-byte swizzle
// (the layout of the kernel's K-major Q operand). Cached like the pool maps.
bool encode_query_map(CUtensorMap* map, const void* base, int64_t tokens, int32_t num_q_heads, int32_t head_dim,
                      int32_t group, int32_t box_tokens) {
  struct Entry {
    const void* base;
    int64_t tokens;
    int32_t num_q_heads, head_dim, group, box_tokens;
    CUtensorMap map;
  };
  thread_local Entry cache[4] = {};
  thread_local int next = 0;
  for (const Entry& e : cache)
    if (e.base == base && e.base != nullptr && e.tokens == tokens && e.num_q_heads == num_q_heads &&
        e.head_dim == head_dim && e.group == group && e.box_tokens == box_tokens) {
      *map = e.map;
      return true;
    }
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(num_q_heads),
                        static_cast<cuuint64_t>(tokens)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_dim) * 2,
                           static_cast<cuuint64_t>(head_dim) * num_q_heads * 2};
  cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(group), static_cast<cuuint32_t>(box_tokens)};
  cuuint32_t elem_strides[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
                  elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  cache[next] = Entry{base, tokens, num_q_heads, head_dim, group, box_tokens, *map};
  next = (next + 1) & 3;
  return true;
}

// ----------------------------------------------------------------- plan

// Blocks of one sequence's table that a decode reads: every block without a window; with
// a window of W tokens at most the blocks spanning the last W + q - 1 positions.
int32_t window_span_blocks(int32_t window, int32_t q_per_seq, int32_t max_blocks_per_seq) {
  if (window <= 0) return max_blocks_per_seq;
  const int64_t span = ceil_div(static_cast<int64_t>(window) + q_per_seq - 1, pa::kBlockSize) + 1;
  return static_cast<int32_t>(span < max_blocks_per_seq ? span : max_blocks_per_seq);
}

int rows_per_cta_for(int path, int rows) {
  if (path == pa::kPathTcgen05) return rows <= 16 ? 16 : pa::kTcmMaxRows;
  if (path == pa::kPathTile) {
    const int r8 = static_cast<int>(ceil_div(rows, 8)) * 8;
    return r8 < pa::kTileMaxRows ? r8 : pa::kTileMaxRows;
  }
  int r = 1;
  while (r < rows && r < pa::kSingleMaxRows) r <<= 1;
  return r;
}

pa_status_t check_shapes(int32_t num_seqs, int32_t q_per_seq, int32_t num_q_heads,
                         int32_t num_kv_heads, int32_t head_dim, int32_t max_blocks_per_seq) {
  if (num_seqs < 0 || q_per_seq <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 ||
      max_blocks_per_seq <= 0 || head_dim <= 0)
    return PA_ERR_INVALID_ARG;
  if (num_q_heads % num_kv_heads != 0) return PA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (q_per_seq > 16) return PA_ERR_UNSUPPORTED;
  if (num_seqs > 65535) return PA_ERR_UNSUPPORTED;  // grid y
  if (static_cast<int64_t>(max_blocks_per_seq) * pa::kBlockSize > INT32_MAX) return PA_ERR_UNSUPPORTED;
  return PA_OK;
}

// Members of one shared-prefix unit: as many sequences as fit the tile kernel's rows.
int share_cap_for(int rows) { return rows <= pa::kTileMaxRows / 2 ? pa::kTileMaxRows / rows : 0; }

pa_status_t make_plan(int32_t num_seqs, int32_t q_per_seq, int32_t num_q_heads, int32_t num_kv_heads,
                      int32_t head_dim, int32_t max_blocks_per_seq, const pa_plan_hints_t* hints,
                      pa_plan_t* plan) {
  pa_status_t st = check_shapes(num_seqs, q_per_seq, num_q_heads, num_kv_heads, head_dim,
                                max_blocks_per_seq);
  if (st != PA_OK) return st;
  pa_plan_hints_t h = {};
  if (hints) h = *hints;
  if (h.path != PA_PATH_AUTO && h.path != PA_PATH_SINGLE && h.path != PA_PATH_TILE &&
      h.path != PA_PATH_TCGEN05)
    return PA_ERR_INVALID_ARG;
  if (h.schedule != PA_SCHEDULE_AUTO && h.schedule != PA_SCHEDULE_GRID &&
      h.schedule != PA_SCHEDULE_PERSISTENT)
    return PA_ERR_INVALID_ARG;
  if (h.split_blocks < 0 || h.share_prefix < 0 || h.share_prefix > 1 || h.sliding_window < 0)
    return PA_ERR_INVALID_ARG;
  if (h.kv_cache_dtype != PA_KV_BF16 && h.kv_cache_dtype != PA_KV_FP8_E4M3) return PA_ERR_INVALID_ARG;
  // E4M3 pools are read by the mma.sync tensor-core tiles (grid or persistent schedule)
  const bool e4m3 = h.kv_cache_dtype == PA_KV_FP8_E4M3;
  if (e4m3 && (h.path == PA_PATH_SINGLE || h.path == PA_PATH_TCGEN05)) return PA_ERR_UNSUPPORTED;
  // a sliding window runs on the grid schedule of the mma.sync and CUDA-core kernels and on
  // the tcgen05 kernel (its own schedule); not with prefix sharing or the mma.sync
  // persistent schedule
  if (h.sliding_window > 0 &&
      (h.share_prefix || (h.schedule == PA_SCHEDULE_PERSISTENT && h.path != PA_PATH_TCGEN05)))
    return PA_ERR_UNSUPPORTED;
  const int group = num_q_heads / num_kv_heads;
  const int rows = group * q_per_seq;
  int schedule = h.schedule == PA_SCHEDULE_AUTO ? PA_SCHEDULE_GRID : h.schedule;
  int share_cap = 0;
  if (h.share_prefix) {
    share_cap = share_cap_for(rows);
    if (share_cap < 2 || h.path == PA_PATH_SINGLE) return PA_ERR_UNSUPPORTED;
  }
  if (h.path == PA_PATH_TCGEN05) {
    // tokens-on-M tensor-core kernel: head_dim 128, its own persistent equal-tile schedule
    if (head_dim != 128 || h.schedule == PA_SCHEDULE_GRID) return PA_ERR_UNSUPPORTED;
    schedule = PA_SCHEDULE_PERSISTENT;
  }
  int path = h.path;
  if (path == PA_PATH_AUTO && e4m3) path = PA_PATH_TILE;
  if (path == PA_PATH_AUTO) {
    // measured on B200: the tcgen05 kernel wins for head_dim 128 with more than 16 rows per
    // kv head or with prefix sharing; mma.sync tiles win below that; CUDA cores for <= 2 rows
    if (head_dim == 128 && (rows > 16 || share_cap > 0) && h.schedule != PA_SCHEDULE_GRID &&
        h.split_blocks == 0) {
      path = PA_PATH_TCGEN05;
      schedule = PA_SCHEDULE_PERSISTENT;
    } else {
      path = (rows <= 2 && share_cap == 0) ? PA_PATH_SINGLE : PA_PATH_TILE;
    }
  }
  // a shared-prefix unit holds share_cap sequences' rows in one CTA (32 rows)
  const int rpc = share_cap ? pa::kTileMaxRows : rows_per_cta_for(path, rows);
  const int64_t row_chunks = ceil_div(rows, rpc);
  if (num_kv_heads * row_chunks > 65535) return PA_ERR_UNSUPPORTED;  // grid x
  const int slots = device_info().sms * pa::decode_ctas_per_sm(path, schedule, head_dim, rpc, h.kv_cache_dtype);
  plan->kv_cache_dtype = h.kv_cache_dtype;
  plan->path = path;
  plan->schedule = schedule;
  plan->rows_per_cta = rpc;
  plan->share_cap = share_cap;
  plan->share_split_blocks = 0;
  plan->sliding_window = h.sliding_window;
  // blocks one sequence reads: all of its table, or the span of the window
  const int32_t span = window_span_blocks(h.sliding_window, q_per_seq, max_blocks_per_seq);
  if (schedule == PA_SCHEDULE_PERSISTENT) {
    plan->num_ctas = slots;
    plan->split_blocks = max_blocks_per_seq;
    plan->num_splits = 1;
    return PA_OK;
  }
  if (share_cap) {
    // the bulk of the work is the shared prefixes: at most ceil(B / cap) chunk windows
    // per kv head; cut the longest possible prefix into as many splits as fill one wave
    // of resident CTAs (long CTAs amortise their prologue and the records they write)
    const int64_t units = ceil_div(num_seqs, share_cap) * num_kv_heads;
    int64_t splits = static_cast<int64_t>(slots) / units;
    if (splits < 1) splits = 1;
    int64_t sb = ceil_div(ceil_div(max_blocks_per_seq, splits), pa::kWarpsPerCta) * pa::kWarpsPerCta;
    if (sb < 4 * pa::kWarpsPerCta) sb = 4 * pa::kWarpsPerCta;
    plan->share_split_blocks = static_cast<int32_t>(sb < max_blocks_per_seq ? sb : max_blocks_per_seq);
  }
  int split_blocks = h.split_blocks;
  if (split_blocks == 0) {
    // Host-known values only: units of (sequence, kv head, row chunk) against the
    // number of resident CTAs. Enough units: one split. Otherwise cut the longest
    // possible context into pieces so that about four waves of CTAs exist (contexts of
    // different lengths leave many splits empty). With a sliding window every sequence
    // reads about the same span, so about 1.5 waves of longer splits suffice (measured
    // on B200: fewer, longer splits beat the four-wave rule there). Over E4M3 pools the
    // tile core is bound by its per-block instructions, not by the loads, and three waves
    // measured faster than four. Splits are made equal, so that no short last split is
    // left over.
    const int64_t units = static_cast<int64_t>(num_seqs) * num_kv_heads * row_chunks;
    if (units >= 2 * static_cast<int64_t>(slots) || units == 0) {
      split_blocks = span;
    } else {
      const int64_t target = h.sliding_window > 0 ? 3 * static_cast<int64_t>(slots) / 2
                             : (e4m3 ? 3 : 4) * static_cast<int64_t>(slots);
      const int64_t splits = ceil_div(target, units);
      const int64_t floor_sb = (h.sliding_window > 0 ? 4 : 8) * pa::kWarpsPerCta;
      int64_t sb = ceil_div(span, splits);
      sb = ceil_div(sb, pa::kWarpsPerCta) * pa::kWarpsPerCta;
      if (sb < floor_sb) sb = floor_sb;
      if (sb < span) {  // equal splits
        const int64_t n = ceil_div(span, sb);
        sb = ceil_div(ceil_div(span, n), pa::kWarpsPerCta) * pa::kWarpsPerCta;
      }
      split_blocks = static_cast<int32_t>(sb < span ? sb : span);
    }
  }
  const int64_t num_splits = ceil_div(span, split_blocks);
  if (num_splits > 65535) return PA_ERR_UNSUPPORTED;  // grid z
  plan->split_blocks = split_blocks;
  plan->num_splits = static_cast<int32_t>(num_splits);
  plan->num_ctas = 0;
  return PA_OK;
}

// Byte layout of the persistent schedule's workspace.
struct PersistentLayout {
  size_t hdr, seq_start, seq_info, cta_seq, arrive, list_len, list, records, total;
  int32_t target_rows, list_cap, pool_cap, rec_stride;
};

size_t align256(size_t x) { return (x + 255) & ~size_t{255}; }

PersistentLayout persistent_layout(const pa_plan_t& plan, int32_t num_seqs, int32_t q_per_seq,
                                   int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim) {
  PersistentLayout L = {};
  const int64_t rows = static_cast<int64_t>(num_q_heads / num_kv_heads) * q_per_seq;
  const int64_t rc = ceil_div(rows, plan.rows_per_cta);
  const int64_t targets = static_cast<int64_t>(num_seqs) * num_kv_heads * rc;
  const int64_t P = plan.num_ctas;
  L.target_rows = static_cast<int32_t>(rows < plan.rows_per_cta ? rows : plan.rows_per_cta);
  L.list_cap = static_cast<int32_t>(2 * P + 4);
  // records: one per non-direct private piece (<= targets + P) plus, with prefix
  // sharing, up to share_cap per shared piece (<= H_kv * B/2 shared sub-units + P)
  int64_t pool = targets + P;
  if (plan.share_cap >= 2) pool += plan.share_cap * (num_kv_heads * ceil_div(num_seqs, 2) + P);
  L.pool_cap = static_cast<int32_t>(pool);
  // o rows then (m, l) pairs, rounded to 4 floats so every record is 16-byte aligned
  L.rec_stride = (L.target_rows * head_dim + 2 * L.target_rows + 3) & ~3;
  size_t off = 0;
  L.hdr = off; off = align256(off + sizeof(pa::SchedHeader));
  L.seq_start = off; off = align256(off + sizeof(long long) * num_seqs);
  L.seq_info = off; off = align256(off + 16 * static_cast<size_t>(num_seqs));
  L.cta_seq = off; off = align256(off + 4 * static_cast<size_t>(P));
  L.arrive = off; off = align256(off + 4 * static_cast<size_t>(targets));
  L.list_len = off; off = align256(off + 4 * static_cast<size_t>(targets));
  L.list = off; off = align256(off + 8 * static_cast<size_t>(targets) * L.list_cap);
  L.records = off; off = align256(off + 4 * static_cast<size_t>(pool) * L.rec_stride);
  L.total = off;
  return L;
}

// Records of the grid schedule with prefix sharing: [B][share splits][q*H_q] for the
// shared prefixes, then [B][num_splits][q*H_q] for the sequences' own blocks. The
// share-split count is derived from share_split_blocks and the plan's split_blocks x
// num_splits (= the table width rounded up).
size_t share_records(const pa_plan_t& plan, int32_t num_seqs, int32_t q_per_seq, int32_t num_q_heads) {
  const int64_t width = static_cast<int64_t>(plan.split_blocks) * plan.num_splits;
  const int64_t ssplits = plan.share_split_blocks > 0 ? ceil_div(width, plan.share_split_blocks) : 0;
  return static_cast<size_t>(num_seqs) * (ssplits + plan.num_splits) * q_per_seq * num_q_heads;
}

// Workspace of the tcgen05 path: two partial records per CTA, then one piece descriptor
// per CTA. A record holds rows_per_cta rows of O (fp32) and their (m, l) pairs.
int32_t tcm_rec_stride(const pa_plan_t& plan, int32_t head_dim) {
  return plan.rows_per_cta * head_dim + 2 * plan.rows_per_cta;
}
size_t tcm_desc_offset(const pa_plan_t& plan, int32_t head_dim) {
  return align256(static_cast<size_t>(2) * plan.num_ctas * tcm_rec_stride(plan, head_dim) * 4);
}

// With prefix sharing the shared-prefix length of every window of share_cap sequences
// follows the descriptors.
size_t tcm_prefix_offset(const pa_plan_t& plan, int32_t head_dim) {
  return align256(tcm_desc_offset(plan, head_dim) + 16 * static_cast<size_t>(plan.num_ctas));
}

size_t workspace_bytes_for(const pa_plan_t& plan, int32_t num_seqs, int32_t q_per_seq,
                           int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim) {
  if (plan.path == PA_PATH_TCGEN05) {
    if (num_seqs == 0) return 0;
    if (plan.share_cap > 1)
      return tcm_prefix_offset(plan, head_dim) + 4 * static_cast<size_t>(ceil_div(num_seqs, plan.share_cap));
    return tcm_desc_offset(plan, head_dim) + 16 * static_cast<size_t>(plan.num_ctas);
  }
  if (plan.schedule == PA_SCHEDULE_PERSISTENT) {
    if (num_seqs == 0) return 0;
    return persistent_layout(plan, num_seqs, q_per_seq, num_q_heads, num_kv_heads, head_dim).total;
  }
  if (plan.share_cap) {  // records of the shared-prefix splits and of the own splits + seq_info
    const size_t recs = share_records(plan, num_seqs, q_per_seq, num_q_heads);
    return align256(recs * (static_cast<size_t>(head_dim) + 2) * 4) + 16 * static_cast<size_t>(num_seqs);
  }
  if (plan.num_splits <= 1) return 0;
  return static_cast<size_t>(num_seqs) * plan.num_splits * q_per_seq * num_q_heads *
         (static_cast<size_t>(head_dim) + 2) * 4;
}

pa_status_t check_plan(const pa_plan_t& plan, int32_t q_per_seq, int32_t num_q_heads,
                       int32_t num_kv_heads, int32_t max_blocks_per_seq) {
  if (plan.path != PA_PATH_SINGLE && plan.path != PA_PATH_TILE && plan.path != PA_PATH_TCGEN05)
    return PA_ERR_INVALID_ARG;
  if (plan.kv_cache_dtype != PA_KV_BF16 && plan.kv_cache_dtype != PA_KV_FP8_E4M3) return PA_ERR_INVALID_ARG;
  if (plan.kv_cache_dtype == PA_KV_FP8_E4M3 && plan.path != PA_PATH_TILE) return PA_ERR_INVALID_ARG;
  if (plan.sliding_window < 0) return PA_ERR_INVALID_ARG;
  if (plan.sliding_window > 0 &&
      (plan.share_cap != 0 || (plan.path != PA_PATH_TCGEN05 && plan.schedule != PA_SCHEDULE_GRID)))
    return PA_ERR_UNSUPPORTED;
  const int rows = num_q_heads / num_kv_heads * q_per_seq;
  if (plan.path == PA_PATH_TCGEN05) {
    if (plan.schedule != PA_SCHEDULE_PERSISTENT || plan.share_split_blocks != 0 || plan.num_ctas <= 0 ||
        plan.num_ctas > (1 << 20))
      return PA_ERR_INVALID_ARG;
    if (plan.share_cap != 0)
      return plan.share_cap == share_cap_for(rows) && plan.rows_per_cta == pa::kTcmMaxRows ? PA_OK
                                                                                            : PA_ERR_INVALID_ARG;
    return plan.rows_per_cta == rows_per_cta_for(plan.path, rows) ? PA_OK : PA_ERR_INVALID_ARG;
  }
  if (plan.schedule == PA_SCHEDULE_PERSISTENT) {
    if (plan.num_ctas <= 0 || plan.num_ctas > (1 << 20)) return PA_ERR_INVALID_ARG;
    if (plan.share_split_blocks != 0) return PA_ERR_INVALID_ARG;  // grid-only field
    if (plan.share_cap != 0) {
      if (plan.path != PA_PATH_TILE || plan.share_cap != share_cap_for(rows) ||
          plan.rows_per_cta != pa::kTileMaxRows)
        return PA_ERR_INVALID_ARG;
      return PA_OK;
    }
  } else if (plan.schedule == PA_SCHEDULE_GRID) {
    if (plan.split_blocks <= 0) return PA_ERR_INVALID_ARG;
    if (plan.num_splits !=
        ceil_div(window_span_blocks(plan.sliding_window, q_per_seq, max_blocks_per_seq), plan.split_blocks))
      return PA_ERR_INVALID_ARG;
    if (plan.share_cap != 0) {
      if (plan.path != PA_PATH_TILE || plan.share_cap != share_cap_for(rows) ||
          plan.rows_per_cta != pa::kTileMaxRows || plan.share_split_blocks <= 0)
        return PA_ERR_INVALID_ARG;
      return PA_OK;
    }
    if (plan.share_split_blocks != 0) return PA_ERR_INVALID_ARG;
  } else {
    return PA_ERR_INVALID_ARG;
  }
  if (plan.rows_per_cta != rows_per_cta_for(plan.path, rows)) return PA_ERR_INVALID_ARG;
  return PA_OK;
}

// pa_decode and pa_decode_fp8: the pools hold bf16 values, or E4M3 codes with one scale
// per pool (k_scale, v_scale; 1 for bf16 pools).
// A partial decode (context parallelism): table entries [lo, hi) of every sequence only, its
// records written to part_o / part_ml.
struct PartialArgs {
  int32_t lo, hi, pieces;
  float* part_o;
  float* part_ml;
};

// Grid plan of a partial decode: the mma.sync tiles, or the CUDA-core kernel for up to 2 rows;
// `pieces` splits of the range (0: as many as the split heuristic takes for a table of the
// range's length). Returns the plan's status.
pa_status_t partial_plan(int32_t num_seqs, int32_t q_per_seq, int32_t num_q_heads, int32_t num_kv_heads,
                         int32_t head_dim, int32_t lo, int32_t hi, int32_t pieces, pa_plan_t* plan) {
  const int32_t span = hi > lo ? hi - lo : 1;
  pa_plan_hints_t h = {};
  h.schedule = PA_SCHEDULE_GRID;
  h.path = q_per_seq * (num_q_heads / num_kv_heads) <= 2 ? PA_PATH_SINGLE : PA_PATH_TILE;
  if (pieces > 0) h.split_blocks = static_cast<int32_t>(ceil_div(span, pieces));
  const pa_status_t st = make_plan(num_seqs, q_per_seq, num_q_heads, num_kv_heads, head_dim, span, &h, plan);
  if (st == PA_OK && pieces > 0) plan->num_splits = pieces;
  return st;
}

pa_status_t decode_impl(void* out, const void* query, const void* key_cache, const void* value_cache,
                        const int32_t* block_tables, const int32_t* context_lens, int32_t num_seqs,
                        int32_t q_per_seq, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                        int32_t block_size, int32_t max_blocks_per_seq, int64_t num_blocks, float scale,
                        int kv_dtype, float k_scale, float v_scale, const pa_plan_t* plan, void* workspace,
                        size_t workspace_bytes, pa_stream_t stream, const PartialArgs* part = nullptr) {
  pa_status_t st = check_shapes(num_seqs, q_per_seq, num_q_heads, num_kv_heads, head_dim,
                                max_blocks_per_seq);
  if (st != PA_OK) return st;
  if (block_size != pa::kBlockSize) return PA_ERR_UNSUPPORTED;
  if (num_blocks <= 0 || !std::isfinite(scale)) return PA_ERR_INVALID_ARG;
  if (!(std::isfinite(k_scale) && k_scale > 0.f && std::isfinite(v_scale) && v_scale > 0.f))
    return PA_ERR_INVALID_ARG;
  if (num_blocks * pa::kBlockSize > INT32_MAX) return PA_ERR_UNSUPPORTED;  // TMA coordinate range
  if (num_seqs == 0) return PA_OK;
  if ((!out && !part) || !query || !key_cache || !value_cache || !block_tables || !context_lens)
    return PA_ERR_INVALID_ARG;
  if ((out && !aligned16(out)) || !aligned16(query) || !aligned16(key_cache) || !aligned16(value_cache) ||
      (reinterpret_cast<uintptr_t>(block_tables) & 3u) || (reinterpret_cast<uintptr_t>(context_lens) & 3u))
    return PA_ERR_INVALID_ARG;
  pa_plan_t local;
  if (part) {
    // the range's pieces on the grid schedule; no workspace (the records go to the caller's
    // buffers)
    st = partial_plan(num_seqs, q_per_seq, num_q_heads, num_kv_heads, head_dim, part->lo, part->hi, part->pieces,
                      &local);
    if (st != PA_OK) return st;
    plan = &local;
  } else if (plan) {
    st = check_plan(*plan, q_per_seq, num_q_heads, num_kv_heads, max_blocks_per_seq);
    if (st == PA_OK && plan->kv_cache_dtype != kv_dtype) st = PA_ERR_INVALID_ARG;  // a plan for other pools
  } else {
    pa_plan_hints_t h = {};
    h.kv_cache_dtype = kv_dtype;
    st = make_plan(num_seqs, q_per_seq, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq, &h, &local);
    plan = &local;
  }
  if (st != PA_OK) return st;
  if (plan->path == PA_PATH_TCGEN05) {
    // the tcgen05 kernel's range scan adds (tiles, units with tiles) packed in one 64-bit word:
    // the units must stay below 2^28 and the tiles below 2^35 (bounds over every kv head)
    const int64_t rows = static_cast<int64_t>(num_q_heads / num_kv_heads) * q_per_seq;
    const int64_t units = static_cast<int64_t>(num_seqs) * num_kv_heads * ceil_div(rows, plan->rows_per_cta);
    const int64_t tiles = units * (max_blocks_per_seq / 8 + 1);
    if (units >= (int64_t{1} << 28) || tiles >= (int64_t{1} << 35)) return PA_ERR_UNSUPPORTED;
  }
  const size_t need =
      part ? 0 : workspace_bytes_for(*plan, num_seqs, q_per_seq, num_q_heads, num_kv_heads, head_dim);
  if (need > 0 && (!workspace || workspace_bytes < need || !aligned16(workspace))) return PA_ERR_WORKSPACE;

  CUtensorMap tk, tv, tq = {};
  if (!encode_pool_map(&tk, key_cache, num_blocks, num_kv_heads, head_dim, kv_dtype) ||
      !encode_pool_map(&tv, value_cache, num_blocks, num_kv_heads, head_dim, kv_dtype))
    return PA_ERR_CUDA;

  DecodeParams p = {};
  p.out = static_cast<uint16_t*>(out);
  p.query = static_cast<const uint16_t*>(query);
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.num_seqs = num_seqs;
  p.q_per_seq = q_per_seq;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = num_kv_heads;
  p.group = num_q_heads / num_kv_heads;
  p.rows = p.group * q_per_seq;
  p.max_blocks = max_blocks_per_seq;
  p.num_blocks = num_blocks;
  p.rows_per_cta = plan->rows_per_cta;
  p.row_chunks = static_cast<int32_t>(ceil_div(p.rows, p.rows_per_cta));
  p.scale_log2 = scale * k_scale * 1.4426950408889634f;
  p.v_scale = v_scale;
  p.split_blocks = plan->split_blocks;
  p.window = plan->sliding_window;
  p.num_splits = plan->num_splits;
  const int64_t rq = static_cast<int64_t>(q_per_seq) * num_q_heads;
  char* ws = static_cast<char*>(workspace);
  if (plan->path == PA_PATH_TCGEN05) {
    if (head_dim != 128) return PA_ERR_UNSUPPORTED;
    p.num_ctas = plan->num_ctas;
    p.share_cap = plan->share_cap;
    p.rec_stride = tcm_rec_stride(*plan, head_dim);
    p.records = reinterpret_cast<float*>(ws);
    if (plan->share_cap > 1) p.win_prefix = reinterpret_cast<int32_t*>(ws + tcm_prefix_offset(*plan, head_dim));
    p.tc_desc = reinterpret_cast<int4*>(ws + tcm_desc_offset(*plan, head_dim));
    // Q rows by TMA: a row chunk of N rows is N / G query tokens of G heads when G divides N;
    // a shared-prefix window is share_cap * q_per_seq tokens (share_cap * rows <= N)
    const int group = num_q_heads / num_kv_heads;
    if (plan->share_cap > 1)
      p.q_box = plan->share_cap * q_per_seq;
    else if (plan->rows_per_cta % group == 0)
      p.q_box = plan->rows_per_cta / group;
    if (p.q_box > 0 && !encode_query_map(&tq, query, static_cast<int64_t>(num_seqs) * q_per_seq, num_q_heads,
                                         head_dim, group, p.q_box))
      return PA_ERR_CUDA;
    // CTAs per group: the largest divisor of H_kv that the grid holds
    p.tc_group = 1;
    for (int sz = num_kv_heads; sz >= 1; --sz)
      if (num_kv_heads % sz == 0 && sz <= plan->num_ctas) {
        p.tc_group = sz;
        break;
      }
  } else if (plan->schedule == PA_SCHEDULE_PERSISTENT) {
    const PersistentLayout L = persistent_layout(*plan, num_seqs, q_per_seq, num_q_heads, num_kv_heads, head_dim);
    p.num_ctas = plan->num_ctas;
    p.share_cap = plan->share_cap;
    p.target_rows = L.target_rows;
    p.list_cap = L.list_cap;
    p.pool_cap = L.pool_cap;
    p.rec_stride = L.rec_stride;
    p.hdr = reinterpret_cast<pa::SchedHeader*>(ws + L.hdr);
    p.seq_start = reinterpret_cast<long long*>(ws + L.seq_start);
    p.seq_info = reinterpret_cast<int4*>(ws + L.seq_info);
    p.cta_seq = reinterpret_cast<int32_t*>(ws + L.cta_seq);
    p.arrive = reinterpret_cast<int32_t*>(ws + L.arrive);
    p.list_len = reinterpret_cast<int32_t*>(ws + L.list_len);
    p.list = reinterpret_cast<int2*>(ws + L.list);
    p.records = reinterpret_cast<float*>(ws + L.records);
  } else if (part) {
    p.partial_only = 1;
    p.range_lo = part->lo;
    p.range_hi = part->hi;
    p.ws_o = part->part_o;
    p.ws_ml = reinterpret_cast<float2*>(part->part_ml);
  } else if (need > 0) {
    const size_t recs = plan->share_cap ? share_records(*plan, num_seqs, q_per_seq, num_q_heads)
                                        : static_cast<size_t>(num_seqs) * plan->num_splits * rq;
    p.ws_o = reinterpret_cast<float*>(ws);
    p.ws_ml = reinterpret_cast<float2*>(reinterpret_cast<float*>(ws) + recs * head_dim);
    if (plan->share_cap) {
      p.share_cap = plan->share_cap;
      p.share_split_blocks = plan->share_split_blocks;
      p.share_splits = static_cast<int32_t>(
          ceil_div(static_cast<int64_t>(plan->split_blocks) * plan->num_splits, plan->share_split_blocks));
      p.share_windows = static_cast<int32_t>(ceil_div(num_seqs, plan->share_cap));
      p.seq_info = reinterpret_cast<int4*>(ws + align256(recs * (static_cast<size_t>(head_dim) + 2) * 4));
    }
  }
  cudaError_t e = pa::launch_decode(p, plan->path, plan->schedule, head_dim, kv_dtype, tk, tv, tq,
                                    reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace

namespace pa {

int check_decode_args(const pa_plan_t* plan, int32_t num_seqs, int32_t q_per_seq, int32_t num_q_heads,
                      int32_t num_kv_heads, int32_t head_dim, int32_t max_blocks_per_seq) {
  const int st =
      check_shapes(num_seqs, q_per_seq, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq);
  if (st != PA_OK || plan == nullptr) return st;
  return check_plan(*plan, q_per_seq, num_q_heads, num_kv_heads, max_blocks_per_seq);
}

}  // namespace pa

extern "C" {

int32_t pa_version(void) { return kVersion; }

const char* pa_status_string(pa_status_t status) {
  switch (status) {
    case PA_OK: return "PA_OK";
    case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG: null/misaligned pointer or bad size";
    case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED: outside the supported shapes";
    case PA_ERR_WORKSPACE: return "PA_ERR_WORKSPACE: workspace missing or too small";
    case PA_ERR_OUT_OF_RANGE: return "PA_ERR_OUT_OF_RANGE: bad slot, block id or context length";
    case PA_ERR_CUDA: return "PA_ERR_CUDA: CUDA runtime error";
    case PA_ERR_DEVICE: return "PA_ERR_DEVICE: a kernel reported a bounded-wait timeout";
  }
  return "unknown pa_status_t";
}

pa_status_t pa_reshape_and_cache(const void* key, const void* value, int64_t key_token_stride,
                                 int64_t value_token_stride, void* key_cache, void* value_cache,
                                 const int64_t* slot_mapping, int64_t num_tokens,
                                 int32_t num_kv_heads, int32_t head_dim, int64_t num_blocks,
                                 int32_t block_size, pa_stream_t stream) {
  if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || num_blocks <= 0)
    return PA_ERR_INVALID_ARG;
  if (block_size != pa::kBlockSize) return PA_ERR_UNSUPPORTED;
  const int64_t row_elems = static_cast<int64_t>(num_kv_heads) * head_dim;
  if ((row_elems * 2) % 16 != 0 || row_elems > INT32_MAX) return PA_ERR_UNSUPPORTED;
  if (key_token_stride < row_elems || value_token_stride < row_elems) return PA_ERR_INVALID_ARG;
  if ((key_token_stride * 2) % 16 != 0 || (value_token_stride * 2) % 16 != 0) return PA_ERR_INVALID_ARG;
  if (num_tokens == 0) return PA_OK;
  if (!key || !value || !key_cache || !value_cache || !slot_mapping) return PA_ERR_INVALID_ARG;
  if (!aligned16(key) || !aligned16(value) || !aligned16(key_cache) || !aligned16(value_cache) ||
      (reinterpret_cast<uintptr_t>(slot_mapping) & 7u))
    return PA_ERR_INVALID_ARG;
  if (num_tokens > (int64_t{1} << 30)) return PA_ERR_UNSUPPORTED;
  cudaError_t e = pa::launch_cache_write(
      static_cast<const uint16_t*>(key), static_cast<const uint16_t*>(value), key_token_stride,
      value_token_stride, static_cast<uint16_t*>(key_cache), static_cast<uint16_t*>(value_cache),
      slot_mapping, num_tokens, static_cast<int32_t>(row_elems), num_blocks * pa::kBlockSize,
      reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status_t pa_decode_plan(int32_t num_seqs, int32_t q_per_seq, int32_t num_q_heads,
                           int32_t num_kv_heads, int32_t head_dim, int32_t max_blocks_per_seq,
                           const pa_plan_hints_t* hints, pa_plan_t* plan) {
  if (!plan) return PA_ERR_INVALID_ARG;
  return make_plan(num_seqs, q_per_seq, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                   hints, plan);
}

size_t pa_decode_workspace_size(const pa_plan_t* plan, int32_t num_seqs, int32_t q_per_seq,
                                int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                int32_t max_blocks_per_seq) {
  if (!plan) {
    // the heuristic plans for bf16 pools (pa_decode) and for E4M3 pools (pa_decode_fp8) may
    // differ (their kernels' occupancies do): the larger of the two serves both calls
    size_t need = 0;
    for (int dtype : {PA_KV_BF16, PA_KV_FP8_E4M3}) {
      pa_plan_hints_t h = {};
      h.kv_cache_dtype = dtype;
      pa_plan_t local;
      if (make_plan(num_seqs, q_per_seq, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq, &h, &local) !=
          PA_OK)
        continue;
      const size_t n = workspace_bytes_for(local, num_seqs, q_per_seq, num_q_heads, num_kv_heads, head_dim);
      if (n > need) need = n;
    }
    return need;
  }
  if (pa::check_decode_args(plan, num_seqs, q_per_seq, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq) !=
      PA_OK)
    return 0;  // the sizes below divide by plan and shape fields: never with bad ones
  return workspace_bytes_for(*plan, num_seqs, q_per_seq, num_q_heads, num_kv_heads, head_dim);
}

pa_status_t pa_decode(void* out, const void* query, const void* key_cache, const void* value_cache,
                      const int32_t* block_tables, const int32_t* context_lens, int32_t num_seqs,
                      int32_t q_per_seq, int32_t num_q_heads, int32_t num_kv_heads,
                      int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq,
                      int64_t num_blocks, float scale, const pa_plan_t* plan, void* workspace,
                      size_t workspace_bytes, pa_stream_t stream) {
  return decode_impl(out, query, key_cache, value_cache, block_tables, context_lens, num_seqs, q_per_seq,
                     num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks, scale,
                     PA_KV_BF16, 1.f, 1.f, plan, workspace, workspace_bytes, stream);
}

pa_status_t pa_decode_fp8(void* out, const void* query, const void* key_cache, const void* value_cache,
                          const int32_t* block_tables, const int32_t* context_lens, int32_t num_seqs,
                          int32_t q_per_seq, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                          int32_t block_size, int32_t max_blocks_per_seq, int64_t num_blocks, float scale,
                          float k_scale, float v_scale, const pa_plan_t* plan, void* workspace,
                          size_t workspace_bytes, pa_stream_t stream) {
  return decode_impl(out, query, key_cache, value_cache, block_tables, context_lens, num_seqs, q_per_seq,
                     num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks, scale,
                     PA_KV_FP8_E4M3, k_scale, v_scale, plan, workspace, workspace_bytes, stream);
}

pa_status_t pa_decode_partial(float* part_o, float* part_ml, const void* query, const void* key_cache,
                              const void* value_cache, const int32_t* block_tables, const int32_t* context_lens,
                              int32_t num_seqs, int32_t q_per_seq, int32_t num_q_heads, int32_t num_kv_heads,
                              int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq,
                              int64_t num_blocks, float scale, int32_t block_begin, int32_t block_end,
                              int32_t num_pieces, pa_stream_t stream) {
  if (block_begin < 0 || block_end < block_begin || block_end > max_blocks_per_seq || num_pieces <= 0 ||
      num_pieces > 65535)
    return PA_ERR_INVALID_ARG;
  if (num_seqs > 0 && (!part_o || !part_ml || !aligned16(part_o) || !aligned16(part_ml))) return PA_ERR_INVALID_ARG;
  const PartialArgs part{block_begin, block_end, num_pieces, part_o, part_ml};
  return decode_impl(nullptr, query, key_cache, value_cache, block_tables, context_lens, num_seqs, q_per_seq,
                     num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks, scale,
                     PA_KV_BF16, 1.f, 1.f, nullptr, nullptr, 0, stream, &part);
}

int32_t pa_decode_partial_pieces(int32_t num_seqs, int32_t q_per_seq, int32_t num_q_heads, int32_t num_kv_heads,
                                 int32_t head_dim, int32_t range_blocks) {
  if (range_blocks < 0 ||
      check_shapes(num_seqs, q_per_seq, num_q_heads, num_kv_heads, head_dim, range_blocks > 0 ? range_blocks : 1) !=
          PA_OK)
    return 0;
  pa_plan_t plan;
  if (partial_plan(num_seqs, q_per_seq, num_q_heads, num_kv_heads, head_dim, 0, range_blocks, 0, &plan) != PA_OK)
    return 0;
  return plan.num_splits;
}

pa_status_t pa_combine_partials(float* rec_o, float* rec_ml, const float* part_o, const float* part_ml,
                                int32_t num_parts, int32_t num_seqs, int32_t q_per_seq, int32_t num_q_heads,
                                int32_t head_dim, pa_stream_t stream) {
  if (num_parts <= 0 || num_seqs < 0 || q_per_seq <= 0 || num_q_heads <= 0) return PA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  const int64_t rows = static_cast<int64_t>(num_seqs) * q_per_seq * num_q_heads;
  if (rows > INT32_MAX || static_cast<int64_t>(num_parts) * rows > INT32_MAX) return PA_ERR_UNSUPPORTED;
  if (num_seqs == 0) return PA_OK;
  if (!rec_o || !rec_ml || !part_o || !part_ml || !aligned16(rec_o) || !aligned16(rec_ml) || !aligned16(part_o) ||
      !aligned16(part_ml))
    return PA_ERR_INVALID_ARG;
  DecodeParams p = {};
  p.num_seqs = num_seqs;
  p.q_per_seq = q_per_seq;
  p.num_q_heads = num_q_heads;
  p.num_parts = num_parts;
  p.partial_only = 1;
  p.ws_o = const_cast<float*>(part_o);
  p.ws_ml = reinterpret_cast<float2*>(const_cast<float*>(part_ml));
  p.rec_o = rec_o;
  p.rec_ml = reinterpret_cast<float2*>(rec_ml);
  return pa::launch_merge_partials(p, head_dim, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? PA_OK
             : PA_ERR_CUDA;
}

pa_status_t pa_merge_partials(void* out, const float* part_o, const float* part_ml, int32_t num_parts,
                              int32_t num_seqs, int32_t q_per_seq, int32_t num_q_heads, int32_t head_dim,
                              pa_stream_t stream) {
  if (num_parts <= 0 || num_seqs < 0 || q_per_seq <= 0 || num_q_heads <= 0) return PA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  const int64_t rows = static_cast<int64_t>(num_seqs) * q_per_seq * num_q_heads;
  if (rows > INT32_MAX || static_cast<int64_t>(num_parts) * rows > INT32_MAX) return PA_ERR_UNSUPPORTED;
  if (num_seqs == 0) return PA_OK;
  if (!out || !part_o || !part_ml || !aligned16(out) || !aligned16(part_o) || !aligned16(part_ml))
    return PA_ERR_INVALID_ARG;
  DecodeParams p = {};
  p.out = static_cast<uint16_t*>(out);
  p.num_seqs = num_seqs;
  p.q_per_seq = q_per_seq;
  p.num_q_heads = num_q_heads;
  p.num_parts = num_parts;
  p.ws_o = const_cast<float*>(part_o);
  p.ws_ml = reinterpret_cast<float2*>(const_cast<float*>(part_ml));
  return pa::launch_merge_partials(p, head_dim, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? PA_OK
             : PA_ERR_CUDA;
}

pa_status_t pa_prefill(void* out, const void* query, const void* key_cache, const void* value_cache,
                       const int32_t* block_tables, const int32_t* context_lens, const int32_t* query_start,
                       int32_t num_seqs, int32_t num_query_tokens, int32_t max_query_len, int32_t num_q_heads,
                       int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq,
                       int64_t num_blocks, float scale, pa_stream_t stream) {
  // the kernel takes each row's maximum over the raw scores, so the scale must not be negative
  if (num_seqs < 0 || num_query_tokens < 0 || max_query_len < 0 || num_q_heads <= 0 || num_kv_heads <= 0 ||
      head_dim <= 0 || max_blocks_per_seq <= 0 || num_blocks <= 0 || !std::isfinite(scale) || scale < 0.f)
    return PA_ERR_INVALID_ARG;
  if (num_q_heads % num_kv_heads != 0) return PA_ERR_INVALID_ARG;
  const int group = num_q_heads / num_kv_heads;
  // 128 query rows per CTA = 128 / G chunk tokens x the G heads of a kv head
  if (head_dim != 128 || block_size != pa::kBlockSize || 128 % group != 0) return PA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(max_blocks_per_seq) * pa::kBlockSize > INT32_MAX ||
      num_blocks * pa::kBlockSize > INT32_MAX)
    return PA_ERR_UNSUPPORTED;
  if (num_seqs == 0 || num_query_tokens == 0 || max_query_len == 0) return PA_OK;
  const int tile_tokens = 128 / group;
  const int64_t max_tiles = ceil_div(max_query_len, tile_tokens);
  if (num_seqs > 65535 || max_tiles > 65535) return PA_ERR_UNSUPPORTED;  // grid y, z
  if (!out || !query || !key_cache || !value_cache || !block_tables || !context_lens || !query_start)
    return PA_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(query) || !aligned16(key_cache) || !aligned16(value_cache) ||
      (reinterpret_cast<uintptr_t>(block_tables) & 3u) || (reinterpret_cast<uintptr_t>(context_lens) & 3u) ||
      (reinterpret_cast<uintptr_t>(query_start) & 3u))
    return PA_ERR_INVALID_ARG;
  CUtensorMap tk, tv;
  if (!encode_pool_map(&tk, key_cache, num_blocks, num_kv_heads, head_dim, pa::kKvBf16) ||
      !encode_pool_map(&tv, value_cache, num_blocks, num_kv_heads, head_dim, pa::kKvBf16))
    return PA_ERR_CUDA;
  pa::PrefillParams p = {};
  p.out = static_cast<uint16_t*>(out);
  p.query = static_cast<const uint16_t*>(query);
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.query_start = query_start;
  p.num_seqs = num_seqs;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = num_kv_heads;
  p.group = group;
  p.max_blocks = max_blocks_per_seq;
  p.tile_tokens = tile_tokens;
  p.num_blocks = num_blocks;
  p.scale_log2 = scale * 1.4426950408889634f;
  const cudaError_t e =
      pa::launch_prefill(p, static_cast<int>(max_tiles), tk, tv, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status_t pa_validate(const int32_t* block_tables, const int32_t* context_lens,
                        const int64_t* slot_mapping, int32_t num_seqs, int32_t max_blocks_per_seq,
                        int32_t q_per_seq, int64_t num_tokens, int64_t num_blocks,
                        int32_t block_size, int64_t* num_bad, pa_stream_t stream) {
  if (num_seqs < 0 || max_blocks_per_seq <= 0 || q_per_seq <= 0 || num_blocks <= 0 ||
      (slot_mapping && num_tokens < 0))
    return PA_ERR_INVALID_ARG;
  if (block_size != pa::kBlockSize) return PA_ERR_UNSUPPORTED;
  if (num_seqs > 0 && (!block_tables || !context_lens)) return PA_ERR_INVALID_ARG;
  int64_t bad = 0;
  cudaError_t e = pa::run_validate(block_tables, context_lens, slot_mapping, num_seqs,
                                   max_blocks_per_seq, q_per_seq, num_tokens, num_blocks, &bad,
                                   reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return PA_ERR_CUDA;
  if (num_bad) *num_bad = bad;
  return bad ? PA_ERR_OUT_OF_RANGE : PA_OK;
}

pa_status_t pa_selftest_bounded_wait(pa_stream_t stream) {
  return pa::run_selftest_wait(reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status_t pa_get_device_error(uint32_t* code, int32_t reset, pa_stream_t stream) {
  if (!code) return PA_ERR_INVALID_ARG;
  cudaError_t e = pa::read_device_error(code, reset != 0, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return PA_ERR_CUDA;
  return *code ? PA_ERR_DEVICE : PA_OK;
}

}  // extern "C"
