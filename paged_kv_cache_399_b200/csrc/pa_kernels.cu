// sm_100a kernels of the paged KV-cache hot path.
//
//   cache_write_kernel   slot_mapping scatter of the step's new K/V rows
//                        ("vLLM 深度实战：从 PagedAttention 到 Speculative Decoding" §3.3)
//   decode_tile_kernel   paged decode on tensor cores (mma.sync m16n8k16, bf16 -> fp32)
//   decode_single_kernel paged decode on CUDA cores (fp32 FMA, warp-shuffle reductions)
//   merge_kernel         log-sum-exp merge of split-context partials
//   validate_kernel      debug bounds check of slots / block ids / context lengths
//
// Both decode kernels walk each sequence's block table ("vLLM study notes"
// zihan-zhang.net §3.2: logical block -> physical block, then a contiguous read of
// the block) and keep a running max / running sum / rescaled output per query row
// (same notes §4.3.1, online softmax). Work unit = one CTA per (kv head, sequence,
// context split, row chunk); the CTA's 4 warps take the split's blocks round-robin,
// each warp with its own TMA pipeline, and are merged through shared memory.
//
// Pool layout [num_blocks][16][H_kv][D] bf16: the 16 rows of one (block, kv head)
// are D*2 bytes each, H_kv*D*2 bytes apart. One TMA box {64 elems, 1 head, 16
// tokens} moves one 2 KB half-tile with the 128-byte swizzle, so ldmatrix reads are
// bank-conflict free: 16-byte chunk c of tile row r sits at chunk c ^ (r & 7).

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cfloat>
#include <cstdint>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

__device__ unsigned int g_device_error = 0;

__device__ __forceinline__ void record_error(unsigned code) { atomicCAS(&g_device_error, 0u, code); }

constexpr unsigned kFull = 0xffffffffu;
constexpr int kHalfTileBytes = 16 * 64 * 2;  // 16 tokens x 64 bf16

template <int D>
struct TileGeom {
  static constexpr int kHalves = D / 64;
  static constexpr int kTileBytes = 16 * D * 2;      // one K or V block tile of a kv head
  static constexpr int kStageBytes = 2 * kTileBytes;  // K + V
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return p + ((1024u - (a & 1023u)) & 1023u);
}

// Byte offset of 16-byte chunk `c` (0..D/8-1) of token row `t` inside a K or V
// tile made of 128-byte-swizzled 2 KB halves.
__device__ __forceinline__ uint32_t tile_chunk_offset(int t, int c) {
  return static_cast<uint32_t>((c >> 3) * kHalfTileBytes + t * 128 + (((c & 7) ^ (t & 7)) << 4));
}

// ---------------------------------------------------------------------------
// Per-warp TMA pipeline over the blocks j = blk0 + warp + NW*k, k < n_my.
// ---------------------------------------------------------------------------
template <int D, int NW, int STAGES>
struct WarpPipe {
  uint8_t* stage_base;   // this warp's STAGES stage buffers
  uint64_t* bars;        // this warp's STAGES mbarriers
  const int32_t* trow;   // block table row of the sequence
  int blk0, warp, lane, n_my, kvh;
  int tchunk, tbase;     // 32 table entries cached in registers, lane k -> entry tbase+k
  int issued;

  __device__ __forceinline__ int table_entry(int k) const {
    return k < n_my ? __ldg(trow + blk0 + warp + NW * k) : 0;
  }
  __device__ __forceinline__ void init(uint8_t* smem, uint64_t* all_bars, const int32_t* row,
                                       int blk0_, int blk1, int warp_, int lane_, int kvh_) {
    warp = warp_;
    lane = lane_;
    blk0 = blk0_;
    kvh = kvh_;
    trow = row;
    stage_base = smem + warp * STAGES * TileGeom<D>::kStageBytes;
    bars = all_bars + warp * STAGES;
    const int span = blk1 - blk0;
    n_my = span > warp ? (span - warp + NW - 1) / NW : 0;
    tbase = 0;
    tchunk = table_entry(lane);
    issued = 0;
  }
  __device__ __forceinline__ uint8_t* kbuf(int s) const {
    return stage_base + s * TileGeom<D>::kStageBytes;
  }
  __device__ __forceinline__ uint8_t* vbuf(int s) const {
    return kbuf(s) + TileGeom<D>::kTileBytes;
  }
  // Called by all lanes, in increasing k.
  __device__ __forceinline__ void issue(int k, const CUtensorMap* tk, const CUtensorMap* tv) {
    if ((k & ~31) != tbase) {
      tbase = k & ~31;
      tchunk = table_entry(tbase + lane);
    }
    const int phys = __shfl_sync(kFull, tchunk, k & 31);
    const int s = k % STAGES;
    if (lane == 0) {
      fence_proxy_async_smem();
      uint64_t* bar = &bars[s];
      mbar_arrive_expect_tx(bar, TileGeom<D>::kStageBytes);
#pragma unroll
      for (int hf = 0; hf < TileGeom<D>::kHalves; ++hf)
        tma_load_3d(kbuf(s) + hf * kHalfTileBytes, tk, bar, hf * 64, kvh, phys * kBlockSize);
#pragma unroll
      for (int hf = 0; hf < TileGeom<D>::kHalves; ++hf)
        tma_load_3d(vbuf(s) + hf * kHalfTileBytes, tv, bar, hf * 64, kvh, phys * kBlockSize);
    }
    issued = k + 1;
  }
  // Uniform across the warp: true when stage of block k holds its data.
  __device__ __forceinline__ bool wait(int k) {
    const bool ok = mbar_wait_bounded(&bars[k % STAGES], (k / STAGES) & 1);
    return __all_sync(kFull, ok);
  }
  // After a timeout: wait (bounded) for every load still in flight.
  __device__ __forceinline__ void drain(int from) {
    for (int k = from; k < issued; ++k)
      if (!mbar_wait_bounded(&bars[k % STAGES], (k / STAGES) & 1)) record_error(kErrTimeoutDrain);
    __syncwarp();
  }
};

// ---------------------------------------------------------------------------
// Cross-warp combine of (m, l, O) and the final store.
//   ow:  NW regions of ROWS x OS fp32 (unnormalised O, row r, column d)
//   ml:  NW x ROWS (m in log2 units, l)
// One split: out = (sum_w O_w 2^(m_w - M)) / (sum_w l_w 2^(m_w - M)) as bf16.
// Several splits: the unnormalised sum and (M, L) go to the workspace.
// ---------------------------------------------------------------------------
template <int D, int ROWS, int NW>
__device__ __forceinline__ void cta_combine_store(const DecodeParams& p, const float* ow,
                                                  const float2* ml, int b, int kvh, int rc,
                                                  int split, bool single_split) {
  constexpr int OS = D + 4;
  constexpr int DC = D / 8;
  for (int task = threadIdx.x; task < ROWS * DC; task += NW * 32) {
    const int r = task / DC;
    const int dc = task % DC;
    const int rg = rc * p.rows_per_cta + r;
    if (rg >= p.rows) continue;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, ml[w * ROWS + r].x);
    float L = 0.f;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float2 mlw = ml[w * ROWS + r];
      const float wt = (mlw.x == -INFINITY) ? 0.f : fast_exp2(mlw.x - M);
      L += wt * mlw.y;
      const float4* src = reinterpret_cast<const float4*>(ow + (w * ROWS + r) * OS + dc * 8);
      const float4 x0 = src[0], x1 = src[1];
      acc[0] += wt * x0.x; acc[1] += wt * x0.y; acc[2] += wt * x0.z; acc[3] += wt * x0.w;
      acc[4] += wt * x1.x; acc[5] += wt * x1.y; acc[6] += wt * x1.z; acc[7] += wt * x1.w;
    }
    const int i = rg / p.group;
    const int h = kvh * p.group + rg % p.group;
    const int rq = i * p.num_q_heads + h;
    if (single_split) {
      const float inv = L > 0.f ? 1.f / L : 0.f;
      uint4 v;
      v.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
      v.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
      v.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
      v.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
      const size_t off = ((static_cast<size_t>(b) * p.q_per_seq + i) * p.num_q_heads + h) * D + dc * 8;
      *reinterpret_cast<uint4*>(p.out + off) = v;
    } else {
      const size_t rec = (static_cast<size_t>(b) * p.num_splits + split) * (p.q_per_seq * p.num_q_heads) + rq;
      float4* dst = reinterpret_cast<float4*>(p.ws_o + rec * D + dc * 8);
      dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
      if (dc == 0) p.ws_ml[rec] = make_float2(M, L);
    }
  }
}

// Rows of a sequence with no visible key at all (context_len 0) get zeros.
template <int D, int NW>
__device__ void store_zero_rows(const DecodeParams& p, int b, int kvh, int rc) {
  constexpr int DC = D / 8;
  for (int task = threadIdx.x; task < p.rows_per_cta * DC; task += NW * 32) {
    const int rg = rc * p.rows_per_cta + task / DC;
    if (rg >= p.rows) continue;
    const int i = rg / p.group;
    const int h = kvh * p.group + rg % p.group;
    const size_t off = ((static_cast<size_t>(b) * p.q_per_seq + i) * p.num_q_heads + h) * D + (task % DC) * 8;
    *reinterpret_cast<uint4*>(p.out + off) = make_uint4(0, 0, 0, 0);
  }
}

template <int D, int ROWS, int NW, int STAGES>
struct DecodeSmem {
  static constexpr int kStages = NW * STAGES * TileGeom<D>::kStageBytes;
  static constexpr int kMerge = NW * ROWS * (D + 4) * 4;
  static constexpr int kBytes = (kStages > kMerge ? kStages : kMerge) + 1024;  // + alignment slack
};

// ---------------------------------------------------------------------------
// Tensor-core decode. Per warp and per 16-token block:
//   S^T[16 tok][8 rows] = K[16 tok][D] . Q^T[D][8 rows]   (A = K via ldmatrix, B = Q regs)
//   online softmax on S^T in registers (a row's 16 scores sit in 8 lanes)
//   O^T[D][8 rows] += V^T[D][16 tok] . P^T[16 tok][8 rows] (A = V via ldmatrix.trans,
//                                                            B = P^T via movmatrix)
// NT n-tiles of 8 rows: rows = GQA group x query tokens, row r = i * group + g.
// ---------------------------------------------------------------------------
template <int D, int NT, int NW, int STAGES>
__global__ void __launch_bounds__(NW * 32)
decode_tile_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmap_k,
                   const __grid_constant__ CUtensorMap tmap_v) {
  constexpr int ROWS = NT * 8;
  constexpr int KSTEPS = D / 16;
  constexpr int OS = D + 4;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bars[NW * STAGES];
  __shared__ float2 ml_s[NW * ROWS];

  uint8_t* smem = align1024(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int kvh = blockIdx.x / p.row_chunks;
  const int rc = blockIdx.x % p.row_chunks;
  const int b = blockIdx.y;
  const int split = blockIdx.z;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NW * STAGES; ++i) mbar_init(&bars[i], 1);
    fence_barrier_init();
    tma_prefetch_desc(&tmap_k);
    tma_prefetch_desc(&tmap_v);
  }
  __syncthreads();
  grid_dependency_wait();  // inputs may be produced by the previous kernel on the stream

  const int ctx = __ldg(p.context_lens + b);
  const int nblk = min(max(ctx, 0) + kBlockSize - 1, p.max_blocks * kBlockSize) / kBlockSize;
  const int blk0 = split * p.split_blocks;
  if (blk0 >= nblk) {
    if (split == 0) store_zero_rows<D, NW>(p, b, kvh, rc);
    grid_launch_dependents();
    return;
  }
  const int blk1 = min(nblk, blk0 + p.split_blocks);
  const bool single_split = (nblk + p.split_blocks - 1) / p.split_blocks == 1;

  WarpPipe<D, NW, STAGES> pipe;
  pipe.init(smem, bars, p.block_tables + static_cast<size_t>(b) * p.max_blocks, blk0, blk1, warp,
            lane, kvh);
#pragma unroll
  for (int s = 0; s < STAGES; ++s)
    if (s < pipe.n_my) pipe.issue(s, &tmap_k, &tmap_v);

  // Q^T fragments (B operand): row n = lane/4, k pairs 2*(lane%4) and +8.
  uint32_t qf[NT][KSTEPS][2];
  int lim[NT][2];  // last visible key position of the thread's two rows per n-tile
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int rg = rc * ROWS + nt * 8 + (lane >> 2);
    const bool valid = rg < p.rows;
    const int i = valid ? rg / p.group : 0;
    const int h = kvh * p.group + (valid ? rg % p.group : 0);
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
        p.query + ((static_cast<size_t>(b) * p.q_per_seq + i) * p.num_q_heads + h) * D);
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      qf[nt][kk][0] = valid ? __ldg(qrow + kk * 8 + (lane & 3)) : 0u;
      qf[nt][kk][1] = valid ? __ldg(qrow + kk * 8 + 4 + (lane & 3)) : 0u;
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int r = rc * ROWS + nt * 8 + 2 * (lane & 3) + e;
      lim[nt][e] = r < p.rows ? ctx - p.q_per_seq + r / p.group : ctx - 1;
    }
  }

  const float c = p.scale_log2;
  float m_run[NT][2], l_run[NT][2];
  float o[KSTEPS][NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    m_run[nt][0] = m_run[nt][1] = -INFINITY;
    l_run[nt][0] = l_run[nt][1] = 0.f;
  }
#pragma unroll
  for (int mt = 0; mt < KSTEPS; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[mt][nt][e] = 0.f;

  // ldmatrix lane roles
  const int lm = lane >> 3;         // which 8x8 matrix this lane addresses
  const int lr = lane & 7;          // row inside it
  const int k_tok = lr + (lm & 1) * 8, k_chk = lm >> 1;   // K (non-transposed A)
  const int v_tok = lr + (lm >> 1) * 8, v_chk = lm & 1;   // V (transposed A)

  for (int k = 0; k < pipe.n_my; ++k) {
    if (!pipe.wait(k)) {
      if (lane == 0) record_error(kErrTimeoutDecode);
      pipe.drain(k);
      break;
    }
    const int s = k % STAGES;
    const uint32_t kb = smem_u32(pipe.kbuf(s));
    const uint32_t vb = smem_u32(pipe.vbuf(s));
    const int tb = (blk0 + warp + NW * k) * kBlockSize;

    float sc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      uint32_t a0, a1, a2, a3;
      ldmatrix_x4(kb + tile_chunk_offset(k_tok, 2 * kk + k_chk), a0, a1, a2, a3);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(sc[nt], a0, a1, a2, a3, qf[nt][kk][0], qf[nt][kk][1]);
    }

    // scores in log2 units, then the causal / end-of-context mask (only blocks
    // reaching past the first query position need it)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sc[nt][e] *= c;
    if (tb + kBlockSize - 1 > ctx - p.q_per_seq) {
      const int t0 = tb + (lane >> 2);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        if (t0 > lim[nt][0]) sc[nt][0] = -INFINITY;
        if (t0 > lim[nt][1]) sc[nt][1] = -INFINITY;
        if (t0 + 8 > lim[nt][0]) sc[nt][2] = -INFINITY;
        if (t0 + 8 > lim[nt][1]) sc[nt][3] = -INFINITY;
      }
    }

    uint32_t pb[NT][2];
    float alpha[NT][2];
    bool rescale = false;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float mx = fmaxf(sc[nt][e], sc[nt][e + 2]);
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
        const float m_new = fmaxf(m_run[nt][e], mx);
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
        alpha[nt][e] = fast_exp2(m_run[nt][e] - m_use);
        rescale |= alpha[nt][e] != 1.f;
        const float p0 = fast_exp2(sc[nt][e] - m_use);
        const float p1 = fast_exp2(sc[nt][e + 2] - m_use);
        sc[nt][e] = p0;
        sc[nt][e + 2] = p1;
        l_run[nt][e] = fmaf(l_run[nt][e], alpha[nt][e], p0 + p1);
        m_run[nt][e] = m_new;
      }
      pb[nt][0] = movmatrix_trans(pack_bf16x2(sc[nt][0], sc[nt][1]));
      pb[nt][1] = movmatrix_trans(pack_bf16x2(sc[nt][2], sc[nt][3]));
    }
    if (__any_sync(kFull, rescale)) {
#pragma unroll
      for (int mt = 0; mt < KSTEPS; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          o[mt][nt][0] *= alpha[nt][0];
          o[mt][nt][1] *= alpha[nt][1];
          o[mt][nt][2] *= alpha[nt][0];
          o[mt][nt][3] *= alpha[nt][1];
        }
    }
#pragma unroll
    for (int mt = 0; mt < KSTEPS; ++mt) {
      uint32_t a0, a1, a2, a3;
      ldmatrix_x4_trans(vb + tile_chunk_offset(v_tok, 2 * mt + v_chk), a0, a1, a2, a3);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(o[mt][nt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
    }
    __syncwarp();
    if (k + STAGES < pipe.n_my) pipe.issue(k + STAGES, &tmap_k, &tmap_v);
  }

  // row sums: a row's partial sums live in the 8 lanes sharing lane % 4
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float l = l_run[nt][e];
      l += __shfl_xor_sync(kFull, l, 4);
      l += __shfl_xor_sync(kFull, l, 8);
      l += __shfl_xor_sync(kFull, l, 16);
      l_run[nt][e] = l;
    }

  grid_launch_dependents();
  __syncthreads();  // every warp is done with its stage buffers
  float* ow = reinterpret_cast<float*>(smem) + warp * ROWS * OS;
#pragma unroll
  for (int mt = 0; mt < KSTEPS; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int r = nt * 8 + 2 * (lane & 3);
      const int d = mt * 16 + (lane >> 2);
      ow[r * OS + d] = o[mt][nt][0];
      ow[(r + 1) * OS + d] = o[mt][nt][1];
      ow[r * OS + d + 8] = o[mt][nt][2];
      ow[(r + 1) * OS + d + 8] = o[mt][nt][3];
    }
  if (lane < 4) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        ml_s[warp * ROWS + nt * 8 + 2 * lane + e] = make_float2(m_run[nt][e], l_run[nt][e]);
      }
  }
  __syncthreads();
  cta_combine_store<D, ROWS, NW>(p, reinterpret_cast<const float*>(smem), ml_s, b, kvh, rc, split,
                                 single_split);
}

// ---------------------------------------------------------------------------
// CUDA-core decode. Per warp and per 16-token block:
//   QK^T: lane (t = lane/2, half = lane%2) dots token t with every row over its
//         half of head_dim (fp32 FMA), the two halves are joined by one shuffle;
//   online softmax: row max over the 16 tokens by 4 xor-shuffles;
//   PV:   lane owns D/32 output columns; p broadcast through shared memory.
// ROWS query rows (GQA group x query tokens) per CTA, Q held in shared memory.
// ---------------------------------------------------------------------------
template <int D, int ROWS, int NW, int STAGES>
__global__ void __launch_bounds__(NW * 32)
decode_single_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmap_k,
                     const __grid_constant__ CUtensorMap tmap_v) {
  constexpr int OS = D + 4;
  constexpr int CPL = D / 16;  // 16-byte chunks of a row each lane of a pair covers
  constexpr int DPL = D / 32;  // output columns per lane
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bars[NW * STAGES];
  __shared__ float2 ml_s[NW * ROWS];
  __shared__ __align__(16) float q_s[ROWS][D];
  __shared__ __align__(16) float p_s[NW][16][ROWS];

  uint8_t* smem = align1024(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int kvh = blockIdx.x / p.row_chunks;
  const int rc = blockIdx.x % p.row_chunks;
  const int b = blockIdx.y;
  const int split = blockIdx.z;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NW * STAGES; ++i) mbar_init(&bars[i], 1);
    fence_barrier_init();
    tma_prefetch_desc(&tmap_k);
    tma_prefetch_desc(&tmap_v);
  }
  __syncthreads();
  grid_dependency_wait();

  const int ctx = __ldg(p.context_lens + b);
  const int nblk = min(max(ctx, 0) + kBlockSize - 1, p.max_blocks * kBlockSize) / kBlockSize;
  const int blk0 = split * p.split_blocks;
  if (blk0 >= nblk) {
    if (split == 0) store_zero_rows<D, NW>(p, b, kvh, rc);
    grid_launch_dependents();
    return;
  }
  const int blk1 = min(nblk, blk0 + p.split_blocks);
  const bool single_split = (nblk + p.split_blocks - 1) / p.split_blocks == 1;

  WarpPipe<D, NW, STAGES> pipe;
  pipe.init(smem, bars, p.block_tables + static_cast<size_t>(b) * p.max_blocks, blk0, blk1, warp,
            lane, kvh);
#pragma unroll
  for (int s = 0; s < STAGES; ++s)
    if (s < pipe.n_my) pipe.issue(s, &tmap_k, &tmap_v);

  for (int idx = threadIdx.x; idx < ROWS * D / 2; idx += NW * 32) {
    const int r = idx / (D / 2);
    const int d2 = idx % (D / 2);
    const int rg = rc * ROWS + r;
    float lo = 0.f, hi = 0.f;
    if (rg < p.rows) {
      const int h = kvh * p.group + rg % p.group;
      const uint32_t v = __ldg(reinterpret_cast<const uint32_t*>(
          p.query + ((static_cast<size_t>(b) * p.q_per_seq + rg / p.group) * p.num_q_heads + h) * D) + d2);
      lo = bf16_lo(v);
      hi = bf16_hi(v);
    }
    q_s[r][2 * d2] = lo;
    q_s[r][2 * d2 + 1] = hi;
  }
  int lim[ROWS];
#pragma unroll
  for (int r = 0; r < ROWS; ++r) {
    const int rg = rc * ROWS + r;
    lim[r] = rg < p.rows ? ctx - p.q_per_seq + rg / p.group : ctx - 1;
  }
  __syncthreads();

  const float c = p.scale_log2;
  float m_run[ROWS], l_run[ROWS], o[ROWS][DPL];
#pragma unroll
  for (int r = 0; r < ROWS; ++r) {
    m_run[r] = -INFINITY;
    l_run[r] = 0.f;
#pragma unroll
    for (int e = 0; e < DPL; ++e) o[r][e] = 0.f;
  }
  const int t_me = lane >> 1;   // token of this lane for QK^T
  const int half = lane & 1;
  // PV: columns [lane*DPL, lane*DPL + DPL) -> chunk and byte offset inside it
  const int pv_chunk = (lane * DPL) / 8;
  const int pv_byte = ((lane * DPL) % 8) * 2;

  for (int k = 0; k < pipe.n_my; ++k) {
    if (!pipe.wait(k)) {
      if (lane == 0) record_error(kErrTimeoutDecode);
      pipe.drain(k);
      break;
    }
    const int s = k % STAGES;
    const uint8_t* kt = pipe.kbuf(s);
    const uint8_t* vt = pipe.vbuf(s);
    const int tb = (blk0 + warp + NW * k) * kBlockSize;

    float sc[ROWS];
#pragma unroll
    for (int r = 0; r < ROWS; ++r) sc[r] = 0.f;
#pragma unroll
    for (int ci = 0; ci < CPL; ++ci) {
      // the two lanes of a pair start half a row apart and walk the 8 chunk
      // positions in a rotated order so that they never share a bank group
      const int cc = half * CPL + (ci ^ (half * (CPL / 2)));
      const uint4 kv = *reinterpret_cast<const uint4*>(kt + tile_chunk_offset(t_me, cc));
      float kf[8] = {bf16_lo(kv.x), bf16_hi(kv.x), bf16_lo(kv.y), bf16_hi(kv.y),
                     bf16_lo(kv.z), bf16_hi(kv.z), bf16_lo(kv.w), bf16_hi(kv.w)};
#pragma unroll
      for (int r = 0; r < ROWS; ++r) {
        const float4 q0 = *reinterpret_cast<const float4*>(&q_s[r][cc * 8]);
        const float4 q1 = *reinterpret_cast<const float4*>(&q_s[r][cc * 8 + 4]);
        float a = sc[r];
        a = fmaf(q0.x, kf[0], a); a = fmaf(q0.y, kf[1], a); a = fmaf(q0.z, kf[2], a);
        a = fmaf(q0.w, kf[3], a); a = fmaf(q1.x, kf[4], a); a = fmaf(q1.y, kf[5], a);
        a = fmaf(q1.z, kf[6], a); a = fmaf(q1.w, kf[7], a);
        sc[r] = a;
      }
    }
    const int t_glob = tb + t_me;
    const bool masked_blk = tb + kBlockSize - 1 > ctx - p.q_per_seq;
    bool rescale = false;
    float alpha[ROWS];
#pragma unroll
    for (int r = 0; r < ROWS; ++r) {
      float sv = (sc[r] + __shfl_xor_sync(kFull, sc[r], 1)) * c;  // log2 units
      if (masked_blk && t_glob > lim[r]) sv = -INFINITY;
      float mx = sv;
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
      const float m_new = fmaxf(m_run[r], mx);
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      alpha[r] = fast_exp2(m_run[r] - m_use);
      rescale |= alpha[r] != 1.f;
      const float pr = fast_exp2(sv - m_use);
      l_run[r] = fmaf(l_run[r], alpha[r], half == 0 ? pr : 0.f);
      m_run[r] = m_new;
      if (half == 0) p_s[warp][t_me][r] = pr;
    }
    if (rescale) {  // m_run is warp-uniform, so is alpha
#pragma unroll
      for (int r = 0; r < ROWS; ++r)
#pragma unroll
        for (int e = 0; e < DPL; ++e) o[r][e] *= alpha[r];
    }
    __syncwarp();
#pragma unroll 4
    for (int t = 0; t < kBlockSize; ++t) {
      const uint8_t* vrow = vt + tile_chunk_offset(t, pv_chunk) + pv_byte;
      float vf[DPL];
      if constexpr (DPL == 4) {
        const uint2 vv = *reinterpret_cast<const uint2*>(vrow);
        vf[0] = bf16_lo(vv.x); vf[1] = bf16_hi(vv.x); vf[2] = bf16_lo(vv.y); vf[3] = bf16_hi(vv.y);
      } else {
        const uint32_t vv = *reinterpret_cast<const uint32_t*>(vrow);
        vf[0] = bf16_lo(vv); vf[1] = bf16_hi(vv);
      }
#pragma unroll
      for (int r = 0; r < ROWS; ++r) {
        const float pr = p_s[warp][t][r];
#pragma unroll
        for (int e = 0; e < DPL; ++e) o[r][e] = fmaf(pr, vf[e], o[r][e]);
      }
    }
    __syncwarp();
    if (k + STAGES < pipe.n_my) pipe.issue(k + STAGES, &tmap_k, &tmap_v);
  }

#pragma unroll
  for (int r = 0; r < ROWS; ++r) {
    float l = l_run[r];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) l += __shfl_xor_sync(kFull, l, off);
    l_run[r] = l;
  }
  grid_launch_dependents();
  __syncthreads();
  float* ow = reinterpret_cast<float*>(smem) + warp * ROWS * OS;
#pragma unroll
  for (int r = 0; r < ROWS; ++r)
#pragma unroll
    for (int e = 0; e < DPL; ++e) ow[r * OS + lane * DPL + e] = o[r][e];
  if (lane == 0) {
#pragma unroll
    for (int r = 0; r < ROWS; ++r)
      ml_s[warp * ROWS + r] = make_float2(m_run[r], l_run[r]);
  }
  __syncthreads();
  cta_combine_store<D, ROWS, NW>(p, reinterpret_cast<const float*>(smem), ml_s, b, kvh, rc, split,
                                 single_split);
}

// ---------------------------------------------------------------------------
// Log-sum-exp merge of split partials: one warp per (sequence, query token, head).
// M = max_s m_s, L = sum_s l_s 2^(m_s - M), out = sum_s o_s 2^(m_s - M) / L.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(128) merge_kernel(const DecodeParams p) {
  constexpr int DPL = D / 32;
  grid_dependency_wait();
  const int RQ = p.q_per_seq * p.num_q_heads;
  const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= p.num_seqs * RQ) return;
  const int b = row / RQ;
  const int rq = row % RQ;
  const int ctx = __ldg(p.context_lens + b);
  const int nblk = min(max(ctx, 0) + kBlockSize - 1, p.max_blocks * kBlockSize) / kBlockSize;
  const int ns = (nblk + p.split_blocks - 1) / p.split_blocks;
  if (ns <= 1) return;  // written directly by the decode kernel
  const size_t base = static_cast<size_t>(b) * p.num_splits * RQ + rq;
  float M = -INFINITY;
  for (int s = 0; s < ns; ++s) M = fmaxf(M, p.ws_ml[base + static_cast<size_t>(s) * RQ].x);
  float L = 0.f, acc[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
  for (int s = 0; s < ns; ++s) {
    const size_t rec = base + static_cast<size_t>(s) * RQ;
    const float2 ml = p.ws_ml[rec];
    const float w = (ml.x == -INFINITY) ? 0.f : fast_exp2(ml.x - M);
    L += w * ml.y;
    const float* src = p.ws_o + rec * D + lane * DPL;
    if constexpr (DPL == 4) {
      const float4 x = *reinterpret_cast<const float4*>(src);
      acc[0] += w * x.x; acc[1] += w * x.y; acc[2] += w * x.z; acc[3] += w * x.w;
    } else {
      const float2 x = *reinterpret_cast<const float2*>(src);
      acc[0] += w * x.x; acc[1] += w * x.y;
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  const int i = rq / p.num_q_heads;
  const int h = rq % p.num_q_heads;
  uint16_t* dst = p.out + ((static_cast<size_t>(b) * p.q_per_seq + i) * p.num_q_heads + h) * D + lane * DPL;
  if constexpr (DPL == 4) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(acc[0] * inv, acc[1] * inv),
                                                pack_bf16x2(acc[2] * inv, acc[3] * inv));
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  }
}

// ---------------------------------------------------------------------------
// Cache write: one warp per (token, K|V) row of row_elems bf16 = row_elems*2 bytes,
// copied in 16-byte vectors. Slots outside [0, num_slots) are skipped.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
cache_write_kernel(const uint16_t* __restrict__ key, const uint16_t* __restrict__ value,
                   int64_t key_stride, int64_t value_stride, uint16_t* __restrict__ key_cache,
                   uint16_t* __restrict__ value_cache, const int64_t* __restrict__ slots,
                   int64_t num_tokens, int32_t row_elems, int64_t num_slots) {
  grid_dependency_wait();
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= 2 * num_tokens) return;
  const int64_t t = wid >> 1;
  const bool is_v = wid & 1;
  const int64_t slot = __ldg(slots + t);
  if (slot < 0 || slot >= num_slots) return;
  const uint4* src = reinterpret_cast<const uint4*>((is_v ? value : key) + t * (is_v ? value_stride : key_stride));
  uint4* dst = reinterpret_cast<uint4*>((is_v ? value_cache : key_cache) + slot * row_elems);
  const int n16 = row_elems / 8;
  for (int v = lane; v < n16; v += 32) dst[v] = __ldg(src + v);
}

// ---------------------------------------------------------------------------
// Debug bounds check (one thread per sequence or token).
// ---------------------------------------------------------------------------
__global__ void validate_kernel(const int32_t* block_tables, const int32_t* context_lens,
                                const int64_t* slots, int32_t num_seqs, int32_t max_blocks,
                                int32_t q_per_seq, int64_t num_tokens, int64_t num_blocks,
                                unsigned long long* bad) {
  const int64_t id = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  unsigned long long n = 0;
  if (id < num_seqs) {
    const int ctx = context_lens[id];
    if (ctx < q_per_seq || ctx > max_blocks * kBlockSize) {
      ++n;
    } else {
      const int nb = (ctx + kBlockSize - 1) / kBlockSize;
      for (int j = 0; j < nb; ++j) {
        const int blk = block_tables[id * static_cast<int64_t>(max_blocks) + j];
        if (blk < 0 || blk >= num_blocks) ++n;
      }
    }
  }
  if (slots != nullptr && id < num_tokens) {
    const int64_t s = slots[id];
    if (s >= num_blocks * kBlockSize) ++n;
  }
  if (n) atomicAdd(bad, n);
}

__device__ unsigned long long g_validate_count = 0;

// ---------------------------------------------------------------------------
// Host-side launchers
// ---------------------------------------------------------------------------
namespace {

template <typename Kernel>
cudaError_t launch_pdl(Kernel kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, p, tk, tv);
}

template <int D, int NT>
constexpr int tile_stages() { return 2; }

// Opt a kernel into its dynamic shared memory size once per device. `done_mask`
// (bit d: done on device d) must be owned by the kernel instance itself.
template <typename Kernel>
cudaError_t configure_smem(Kernel kernel, int smem, unsigned long long& done_mask) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (done_mask & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess) done_mask |= bit;
  return e;
}

template <int D, int NT>
cudaError_t launch_tile(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv,
                        cudaStream_t stream, int* occupancy) {
  constexpr int ST = tile_stages<D, NT>();
  constexpr int smem = DecodeSmem<D, NT * 8, kWarpsPerCta, ST>::kBytes;
  auto kernel = decode_tile_kernel<D, NT, kWarpsPerCta, ST>;
  static unsigned long long done_mask = 0;  // one per template instance
  cudaError_t e = configure_smem(kernel, smem, done_mask);
  if (e != cudaSuccess) return e;
  if (occupancy) return cudaOccupancyMaxActiveBlocksPerMultiprocessor(occupancy, kernel, kWarpsPerCta * 32, smem);
  dim3 grid(p.num_kv_heads * p.row_chunks, p.num_seqs, p.num_splits);
  return launch_pdl(kernel, grid, dim3(kWarpsPerCta * 32), smem, stream, p, tk, tv);
}

template <int D, int ROWS>
cudaError_t launch_single(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv,
                          cudaStream_t stream, int* occupancy) {
  constexpr int ST = 2;
  constexpr int smem = DecodeSmem<D, ROWS, kWarpsPerCta, ST>::kBytes;
  auto kernel = decode_single_kernel<D, ROWS, kWarpsPerCta, ST>;
  static unsigned long long done_mask = 0;  // one per template instance
  cudaError_t e = configure_smem(kernel, smem, done_mask);
  if (e != cudaSuccess) return e;
  if (occupancy) return cudaOccupancyMaxActiveBlocksPerMultiprocessor(occupancy, kernel, kWarpsPerCta * 32, smem);
  dim3 grid(p.num_kv_heads * p.row_chunks, p.num_seqs, p.num_splits);
  return launch_pdl(kernel, grid, dim3(kWarpsPerCta * 32), smem, stream, p, tk, tv);
}

template <int D>
cudaError_t dispatch_rows(int path, int rows_per_cta, const DecodeParams& p, const CUtensorMap& tk,
                          const CUtensorMap& tv, cudaStream_t stream, int* occ) {
  if (path == kPathTile) {
    switch (rows_per_cta) {
      case 8: return launch_tile<D, 1>(p, tk, tv, stream, occ);
      case 16: return launch_tile<D, 2>(p, tk, tv, stream, occ);
      case 24: return launch_tile<D, 3>(p, tk, tv, stream, occ);
      case 32: return launch_tile<D, 4>(p, tk, tv, stream, occ);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (rows_per_cta) {
    case 1: return launch_single<D, 1>(p, tk, tv, stream, occ);
    case 2: return launch_single<D, 2>(p, tk, tv, stream, occ);
    case 4: return launch_single<D, 4>(p, tk, tv, stream, occ);
    case 8: return launch_single<D, 8>(p, tk, tv, stream, occ);
    default: return cudaErrorInvalidValue;
  }
}

template <int D>
cudaError_t launch_merge(const DecodeParams& p, cudaStream_t stream) {
  const long rows = static_cast<long>(p.num_seqs) * p.q_per_seq * p.num_q_heads;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((rows + 3) / 4));
  cfg.blockDim = dim3(128);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, merge_kernel<D>, p);
}

}  // namespace

cudaError_t launch_decode(const DecodeParams& p, int path, int head_dim, const CUtensorMap& tk,
                          const CUtensorMap& tv, cudaStream_t stream) {
  cudaError_t e = head_dim == 128 ? dispatch_rows<128>(path, p.rows_per_cta, p, tk, tv, stream, nullptr)
                                  : dispatch_rows<64>(path, p.rows_per_cta, p, tk, tv, stream, nullptr);
  if (e != cudaSuccess || p.num_splits <= 1) return e;
  return head_dim == 128 ? launch_merge<128>(p, stream) : launch_merge<64>(p, stream);
}

int decode_ctas_per_sm(int path, int head_dim, int rows_per_cta) {
  DecodeParams dummy = {};
  CUtensorMap tm = {};
  int occ = 0;
  cudaError_t e = head_dim == 128 ? dispatch_rows<128>(path, rows_per_cta, dummy, tm, tm, nullptr, &occ)
                                  : dispatch_rows<64>(path, rows_per_cta, dummy, tm, tm, nullptr, &occ);
  return e == cudaSuccess && occ > 0 ? occ : 1;
}

cudaError_t launch_cache_write(const uint16_t* key, const uint16_t* value, int64_t key_stride,
                               int64_t value_stride, uint16_t* key_cache, uint16_t* value_cache,
                               const int64_t* slots, int64_t num_tokens, int32_t row_elems,
                               int64_t num_slots, cudaStream_t stream) {
  const int64_t threads = 2 * num_tokens * 32;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((threads + 255) / 256));
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, cache_write_kernel, key, value, key_stride, value_stride, key_cache,
                            value_cache, slots, num_tokens, row_elems, num_slots);
}

cudaError_t run_validate(const int32_t* block_tables, const int32_t* context_lens,
                         const int64_t* slots, int32_t num_seqs, int32_t max_blocks,
                         int32_t q_per_seq, int64_t num_tokens, int64_t num_blocks,
                         int64_t* bad, cudaStream_t stream) {
  unsigned long long zero = 0, count = 0;
  cudaError_t e = cudaMemcpyToSymbolAsync(g_validate_count, &zero, sizeof zero, 0,
                                          cudaMemcpyHostToDevice, stream);
  if (e != cudaSuccess) return e;
  const int64_t n = slots ? (num_tokens > num_seqs ? num_tokens : num_seqs) : num_seqs;
  if (n > 0) {
    unsigned long long* dcount = nullptr;
    e = cudaGetSymbolAddress(reinterpret_cast<void**>(&dcount), g_validate_count);
    if (e != cudaSuccess) return e;
    validate_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, stream>>>(
        block_tables, context_lens, slots, num_seqs, max_blocks, q_per_seq, num_tokens, num_blocks,
        dcount);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  e = cudaMemcpyFromSymbolAsync(&count, g_validate_count, sizeof count, 0, cudaMemcpyDeviceToHost,
                                stream);
  if (e != cudaSuccess) return e;
  e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return e;
  *bad = static_cast<int64_t>(count);
  return cudaSuccess;
}

cudaError_t read_device_error(uint32_t* code, bool reset, cudaStream_t stream) {
  unsigned int v = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_device_error, sizeof v, 0, cudaMemcpyDeviceToHost, stream);
  if (e != cudaSuccess) return e;
  if (reset) {
    static const unsigned int zero = 0;
    e = cudaMemcpyToSymbolAsync(g_device_error, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, stream);
    if (e != cudaSuccess) return e;
  }
  e = cudaStreamSynchronize(stream);
  *code = v;
  return e;
}

}  // namespace pa
