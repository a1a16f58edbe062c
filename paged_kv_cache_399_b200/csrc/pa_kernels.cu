// sm_100a kernels of the paged KV-cache hot path.
//
//   cache_write_kernel       slot_mapping scatter of the step's new K/V rows
//                            ("vLLM 深度实战：从 PagedAttention 到 Speculative Decoding" §3.3)
//   sched_prepass_kernel     persistent schedule: equal-work partition of all
//                            (sequence, kv head, block) units, optional detection of
//                            adjacent sequences sharing prefix blocks
//   decode_persistent_kernel paged decode, one CTA per resident slot, each over an
//                            equal share of the work; partial results are merged by
//                            the CTA that completes an output
//   decode_grid_kernel       paged decode, one CTA per (kv head, sequence, split)
//   merge_kernel             log-sum-exp merge of the grid schedule's split partials
//   validate_kernel          debug bounds check of slots / block ids / context lengths
//   selftest_wait_kernel     the bounded-wait failure path, taken without a fault
// and, from pa_tcgen05.cuh, the 5th-generation tensor-core path:
//   decode_tcm_kernel        tokens on M, tcgen05.mma with TMEM accumulators, persistent
//                            equal-tile schedule over windows of sequences
//   tcm_merge_kernel         merge of the units a tile range boundary cuts
//   tcm_share_prepass        common table prefix of each window (prefix sharing)
//
// Two compute cores run inside the mma.sync / CUDA-core decode kernels:
//   TileCore   tensor cores: mma.sync m16n8k16 bf16 -> fp32 on S^T = K Q^T and
//              O^T += V^T P^T, online softmax on the accumulator fragments;
//   SimtCore   CUDA cores: fp32 FMA dot products, warp-shuffle max / sum.
// Both walk a sequence's block table ("vLLM study notes", zihan-zhang.net §3.2: logical
// block -> physical block, contiguous read inside a block) and keep a running max,
// running sum and rescaled output per query row (same notes §4.3.1). Partial states
// (m, l, o) of disjoint key ranges combine by the same rescaling: out =
// sum_k o_k 2^(m_k - M) / sum_k l_k 2^(m_k - M), M = max_k m_k (log2 units).
//
// Pool layout [num_blocks][16][H_kv][D] bf16: the 16 rows of one (block, kv head) are
// D*2 bytes each, H_kv*D*2 bytes apart. One TMA box {64 elems, 1 head, 16 tokens}
// moves one 2 KB half-tile with the 128-byte swizzle, so ldmatrix reads are bank-
// conflict free: 16-byte chunk c of tile row r sits at chunk c ^ (r & 7). Every CTA
// warp owns a private STAGES-deep TMA pipeline (one mbarrier per stage).

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cfloat>
#include <climits>
#include <mutex>
#include <cstdint>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

__device__ unsigned int g_device_error = 0;

__device__ __forceinline__ void record_error(unsigned code) { atomicCAS(&g_device_error, 0u, code); }

constexpr unsigned kErrRecordPool = 0x300u;
constexpr unsigned kErrRecordList = 0x400u;
constexpr unsigned kErrSchedule = 0x500u;
constexpr unsigned kErrSelftest = 0x600u;

constexpr unsigned kFull = 0xffffffffu;
constexpr int kHalfTileBytes = 16 * 64 * 2;  // 16 tokens x 64 bf16

// One block of one kv head as it sits in a pipeline stage. bf16 pools: D/64 TMA boxes of
// 16 tokens x 64 elements (2 KB each, 128-byte swizzle). E4M3 pools: one box of 16 tokens x
// D bytes (128-byte swizzle at D = 128, 64-byte at D = 64).
template <int D, bool kFp8 = false>
struct TileGeom {
  static constexpr int kD = D;
  static constexpr bool kE4M3 = kFp8;
  static constexpr int kBoxes = kFp8 ? 1 : D / 64;                // TMA boxes per K (or V) tile
  static constexpr int kBoxBytes = kFp8 ? 16 * D : kHalfTileBytes;
  static constexpr int kTileBytes = kBoxes * kBoxBytes;          // one K or V block tile of a kv head
  static constexpr int kStageBytes = 2 * kTileBytes;             // K + V
  // element (x) coordinate of box hf: bf16 boxes cover 64 elements each
  static __device__ __forceinline__ int box_x(int hf) { return kFp8 ? 0 : hf * 64; }
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return p + ((1024u - (a & 1023u)) & 1023u);
}

// Byte offset of 16-byte chunk `c` (0..D/8-1) of token row `t` inside a K or V tile
// made of 128-byte-swizzled 2 KB halves.
__device__ __forceinline__ uint32_t tile_chunk_offset(int t, int c) {
  return static_cast<uint32_t>((c >> 3) * kHalfTileBytes + t * 128 + (((c & 7) ^ (t & 7)) << 4));
}

__device__ __forceinline__ int num_blocks_of(const DecodeParams& p, int ctx) {
  return min(max(ctx, 0) + kBlockSize - 1, p.max_blocks * kBlockSize) / kBlockSize;
}

// Sliding window: the first block holding a key that some query row of a sequence with
// ctx tokens sees (its first query token's window start); 0 without a window.
__device__ __forceinline__ int window_first_block(const DecodeParams& p, int ctx) {
  return p.window > 0 ? max(0, ctx - p.q_per_seq - p.window + 1) / kBlockSize : 0;
}

// ---------------------------------------------------------------------------
// A segment: consecutive blocks [blk0, blk1) of one kv head, for a set of query rows.
// Private: rows row0 .. row0+nrows-1 of sequence b0. Shared: `members` sequences
// b0 .. b0+members-1 that map these blocks to the same physical blocks; local row r
// is row r % rows of member r / rows.
// ---------------------------------------------------------------------------
struct Seg {
  int b0, members, kvh, row0, nrows, blk0, blk1;
  bool shared;
};

__device__ __forceinline__ bool seg_row(const DecodeParams& p, const Seg& s, int r, int& b, int& i,
                                        int& h) {
  if (r >= s.nrows) return false;
  int m = 0, rr = s.row0 + r;
  if (s.shared) {
    m = r / p.rows;
    rr = r - m * p.rows;
  }
  b = s.b0 + m;
  i = rr / p.group;
  h = s.kvh * p.group + (rr - i * p.group);
  return true;
}

__device__ __forceinline__ size_t out_offset(const DecodeParams& p, int b, int i, int h, int D) {
  return ((static_cast<size_t>(b) * p.q_per_seq + i) * p.num_q_heads + h) * D;
}

// ---------------------------------------------------------------------------
// Per-warp TMA pipeline over the blocks j = blk0 + warp + NW*k, k < n_my.
// ---------------------------------------------------------------------------
template <class Geom, int NW, int STAGES>
struct WarpPipe {
  uint8_t* stage_base;   // this warp's STAGES stage buffers
  uint64_t* bars;        // this warp's STAGES mbarriers
  const int32_t* trow;   // block table row of the sequence
  int blk0, warp, lane, n_my, kvh;
  int tchunk, tbase;     // 32 table entries cached in registers, lane k -> entry tbase+k
  int issued;
  uint32_t phase_base;   // loads issued on this warp's barriers before this run

  // Block index (within the sequence) of this warp's k-th block of the run.
  __device__ __forceinline__ int block_of(int k) const { return blk0 + warp + NW * k; }
  __device__ __forceinline__ int table_entry(int k) const {
    return k < n_my ? __ldg(trow + block_of(k)) : 0;
  }
  __device__ __forceinline__ void init(uint8_t* smem, uint64_t* all_bars, int warp_, int lane_) {
    warp = warp_;
    lane = lane_;
    stage_base = smem + warp * STAGES * Geom::kStageBytes;
    bars = all_bars + warp * STAGES;
    phase_base = 0;
    issued = 0;
    n_my = 0;
  }
  // Start a new run of blocks [blk0_, blk1_) of kv head kvh_. The barrier phases
  // continue from the previous run.
  __device__ __forceinline__ void start(const int32_t* row, int blk0_, int blk1_, int kvh_) {
    phase_base += issued;
    blk0 = blk0_;
    kvh = kvh_;
    trow = row;
    const int span = blk1_ - blk0_;
    n_my = span > warp ? (span - warp + NW - 1) / NW : 0;
    tbase = 0;
    tchunk = table_entry(lane);
    issued = 0;
  }
  __device__ __forceinline__ uint8_t* kbuf(int s) const {
    return stage_base + s * Geom::kStageBytes;
  }
  __device__ __forceinline__ uint8_t* vbuf(int s) const { return kbuf(s) + Geom::kTileBytes; }
  __device__ __forceinline__ int stage_of(int k) const { return (phase_base + k) % STAGES; }
  __device__ __forceinline__ uint32_t parity_of(int k) const { return ((phase_base + k) / STAGES) & 1; }
  // Called by all lanes, in increasing k.
  __device__ __forceinline__ void issue(int k, const CUtensorMap* tk, const CUtensorMap* tv) {
    if ((k & ~31) != tbase) {
      tbase = k & ~31;
      tchunk = table_entry(tbase + lane);
    }
    const int phys = __shfl_sync(kFull, tchunk, k & 31);
    const int s = stage_of(k);
    if (lane == 0) {
      fence_proxy_async_smem();
      uint64_t* bar = &bars[s];
      mbar_arrive_expect_tx(bar, Geom::kStageBytes);
#pragma unroll
      for (int hf = 0; hf < Geom::kBoxes; ++hf)
        tma_load_3d(kbuf(s) + hf * Geom::kBoxBytes, tk, bar, Geom::box_x(hf), kvh, phys * kBlockSize);
#pragma unroll
      for (int hf = 0; hf < Geom::kBoxes; ++hf)
        tma_load_3d(vbuf(s) + hf * Geom::kBoxBytes, tv, bar, Geom::box_x(hf), kvh, phys * kBlockSize);
    }
    issued = k + 1;
  }
  // Uniform across the warp: true when the stage of block k holds its data.
  __device__ __forceinline__ bool wait(int k) {
    const bool ok = mbar_wait_bounded(&bars[stage_of(k)], parity_of(k));
    return __all_sync(kFull, ok);
  }
  // After a timeout: wait (bounded) for every load still in flight, then stop.
  __device__ __forceinline__ void drain(int from) {
    for (int k = from; k < issued; ++k)
      if (!mbar_wait_bounded(&bars[stage_of(k)], parity_of(k))) record_error(kErrTimeoutDrain);
    __syncwarp();
  }
};

// ---------------------------------------------------------------------------
// Tensor-core core. Per warp and per 16-token block:
//   S^T[16 tok][8 rows] = K[16 tok][D] . Q^T[D][8 rows]   (A = K via ldmatrix, B = Q regs)
//   online softmax on S^T in registers (a row's 16 scores sit in 8 lanes)
//   O^T[D][8 rows] += V^T[D][16 tok] . P^T[16 tok][8 rows] (A = V via ldmatrix.trans,
//                                                            B = P^T via movmatrix)
// NT n-tiles of 8 rows; only the first nt_active carry real rows in a segment.
//
// kFp8: the pools hold E4M3 codes (vLLM study notes §4.2, --kv-cache-dtype fp8) with one
// scale per pool. The tile bytes are widened in registers, exactly, to f16
// (cvt.rn.f16x2.e4m3x2; every E4M3 value is an f16 value) and the products run as f16
// mma.sync with fp32 accumulators:
//   K: ldmatrix over byte pairs gives a lane four consecutive codes of one token, so the
//      k index of a 16-wide step is the head-dim order permuted as k 2c,2c+1 <-> d 4c,4c+1
//      and k 2c+8,2c+9 <-> d 4c+2,4c+3 (c = lane % 4); Q's fragments use the same order,
//      which leaves every dot product unchanged;
//   V: ldmatrix.trans over byte pairs gives a lane two tokens x two head-dim columns; one
//      byte permute pairs the tokens of each column, so the m index of a 16-row tile is
//      the head-dim order permuted as m g <-> d 2g and m g+8 <-> d 2g+1 (g = lane / 4),
//      undone when O is written out;
//   Q: each row is scaled by a power of two 2^s (exact) that puts its largest magnitude in
//      [2^14, 2^15) before the f16 conversion, so no bf16 query overflows f16; the scores
//      are multiplied back by 2^-s. k_scale is folded into the softmax scale by the host and
//      v_scale is applied to O once, before it leaves the core.
// ---------------------------------------------------------------------------

// Four E4M3 codes -> two f16 pairs: lo = codes 0, 1 (code 0 in the low half), hi = codes 2, 3.
__device__ __forceinline__ void e4m3x4_to_f16x2(uint32_t x, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 c01, c23;\n\t"
      "mov.b32 {c01, c23}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, c01;\n\t"
      "cvt.rn.f16x2.e4m3x2 %1, c23;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(x));
}

__device__ __forceinline__ uint32_t byte_perm(uint32_t x, uint32_t sel) {
  uint32_t y;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(y) : "r"(x), "r"(0u), "r"(sel));
  return y;
}

// Two fp32 -> packed f16x2 (round to nearest even); `lo` in the low half.
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t v;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(v) : "f"(hi), "f"(lo));
  return v;
}

// D = A(16x16, row) * B(16x8, col) + D, f16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Byte offset of 16-byte chunk `c` of token row `t` inside an E4M3 tile of D-byte rows, as TMA
// swizzles it: 128-byte swizzle for D = 128, 64-byte swizzle for D = 64.
template <int D>
__device__ __forceinline__ uint32_t e4m3_chunk_offset(int t, int c) {
  if constexpr (D == 128)
    return static_cast<uint32_t>(t * 128 + ((c ^ (t & 7)) << 4));
  else
    return static_cast<uint32_t>(t * 64 + ((c ^ ((t >> 1) & 3)) << 4));
}

template <int D, int NT, bool kFp8 = false>
struct TileCore {
  using Geom = TileGeom<D, kFp8>;
  // stages per warp: with E4M3 tiles (half the bytes) 3 stages and 4 CTAs per SM for 8 rows
  // keep the bf16 core's bytes in flight with a third more warps to hide the conversions
  static constexpr int kStages = kFp8 ? (NT == 1 ? 3 : 4) : 2;
  static constexpr int ROWS = NT * 8;
  static constexpr int KSTEPS = D / 16;
  static constexpr bool kNeedsQSmem = false;
  uint32_t qf[NT][KSTEPS][2];
  int lim[NT][2];
  float m_run[NT][2], l_run[NT][2];
  float o[KSTEPS][NT][4];
  float rs[NT][2];  // kFp8: 2^-s of the rows of this lane's score columns (1 otherwise)
  float v_scale;
  int nt_active;
  int vlim;  // largest row limit of the segment: no row sees a token past it

  __device__ __forceinline__ void begin(const DecodeParams& p, const Seg& s, int ctx, int lane) {
    nt_active = (s.nrows + 7) >> 3;
    v_scale = p.v_scale;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      int b = 0, i = 0, h = 0;
      const bool valid = seg_row(p, s, nt * 8 + (lane >> 2), b, i, h);
      const uint32_t* qrow = reinterpret_cast<const uint32_t*>(p.query + out_offset(p, b, i, h, D));
      if constexpr (!kFp8) {
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
          qf[nt][kk][0] = valid ? __ldg(qrow + kk * 8 + (lane & 3)) : 0u;
          qf[nt][kk][1] = valid ? __ldg(qrow + kk * 8 + 4 + (lane & 3)) : 0u;
        }
        rs[nt][0] = rs[nt][1] = 1.f;
      } else {
        // lane (g, c) holds d = 32*kc + 4c .. 4c+3 (step 2kc) and 32*kc + 16 + 4c .. (step 2kc+1)
        const uint2* q2 = reinterpret_cast<const uint2*>(qrow);
        uint2 raw[KSTEPS];
        float mx = 0.f;
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
          raw[kk] = valid ? __ldg(q2 + kk * 4 + (lane & 3)) : make_uint2(0u, 0u);
          mx = fmaxf(mx, fmaxf(fmaxf(fabsf(bf16_lo(raw[kk].x)), fabsf(bf16_hi(raw[kk].x))),
                               fmaxf(fabsf(bf16_lo(raw[kk].y)), fabsf(bf16_hi(raw[kk].y)))));
        }
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
        // 2^s with the row's largest magnitude in [2^14, 2^15) (s clamped: a row that small is 0)
        int sh = 0;
        if (mx > 0.f) sh = 14 - (static_cast<int>((__float_as_uint(mx) >> 23) & 0xFFu) - 127);
        sh = min(max(sh, -100), 100);
        const float up = __uint_as_float(static_cast<uint32_t>(127 + sh) << 23);
        const float down = __uint_as_float(static_cast<uint32_t>(127 - sh) << 23);
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
          qf[nt][kk][0] = pack_f16x2(bf16_lo(raw[kk].x) * up, bf16_hi(raw[kk].x) * up);
          qf[nt][kk][1] = pack_f16x2(bf16_lo(raw[kk].y) * up, bf16_hi(raw[kk].y) * up);
        }
        // this lane's score columns are rows 2c and 2c+1, whose factors sit in lanes 4 * row
        rs[nt][0] = __shfl_sync(kFull, down, 8 * (lane & 3));
        rs[nt][1] = __shfl_sync(kFull, down, 8 * (lane & 3) + 4);
      }
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const bool v = seg_row(p, s, nt * 8 + 2 * (lane & 3) + e, b, i, h);
        lim[nt][e] = v ? ctx - p.q_per_seq + i : ctx - 1;
      }
      m_run[nt][0] = m_run[nt][1] = -INFINITY;
      l_run[nt][0] = l_run[nt][1] = 0.f;
    }
    int vl = lim[0][0];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) vl = max(vl, max(lim[nt][0], lim[nt][1]));
    vl = max(vl, __shfl_xor_sync(kFull, vl, 1));
    vlim = max(vl, __shfl_xor_sync(kFull, vl, 2));
#pragma unroll
    for (int mt = 0; mt < KSTEPS; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[mt][nt][e] = 0.f;
  }

  // win > 0: sliding window (a row with last visible key lim sees keys lim - win + 1 ..
  // lim); vlo: no row of the segment sees a key before it (INT_MIN without a window)
  __device__ __forceinline__ void block(const uint8_t* kt, const uint8_t* vt, int tb, bool need_mask,
                                        float c, int lane, float*, int win, int vlo) {
    const uint32_t kb = smem_u32(kt);
    const uint32_t vb = smem_u32(vt);
    const int lm = lane >> 3, lr = lane & 7;
    float sc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
    if constexpr (!kFp8) {
      const int k_tok = lr + (lm & 1) * 8, k_chk = lm >> 1;  // K (non-transposed A)
#pragma unroll
      for (int kk = 0; kk < KSTEPS; ++kk) {
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4(kb + tile_chunk_offset(k_tok, 2 * kk + k_chk), a0, a1, a2, a3);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          if (nt < nt_active) mma_bf16_16816(sc[nt], a0, a1, a2, a3, qf[nt][kk][0], qf[nt][kk][1]);
      }
    } else {
      // matrices: tokens 0-7 / 8-15 x the two 16-byte chunks of a 32-byte column group
      const int k_tok = lr + (lm & 1) * 8, k_chk = lm >> 1;
#pragma unroll
      for (int kc = 0; kc < D / 32; ++kc) {
        uint32_t r0, r1, r2, r3;
        ldmatrix_x4(kb + e4m3_chunk_offset<D>(k_tok, 2 * kc + k_chk), r0, r1, r2, r3);
        uint32_t a0, a1, a2, a3;
        e4m3x4_to_f16x2(r0, a0, a2);  // token g: d 4c,4c+1 | 4c+2,4c+3 of the first chunk
        e4m3x4_to_f16x2(r1, a1, a3);  // token g + 8
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          if (nt < nt_active) mma_f16_16816(sc[nt], a0, a1, a2, a3, qf[nt][2 * kc][0], qf[nt][2 * kc][1]);
        e4m3x4_to_f16x2(r2, a0, a2);  // the second chunk
        e4m3x4_to_f16x2(r3, a1, a3);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          if (nt < nt_active)
            mma_f16_16816(sc[nt], a0, a1, a2, a3, qf[nt][2 * kc + 1][0], qf[nt][2 * kc + 1][1]);
      }
    }
    // scores in log2 units, then the causal / end-of-context mask
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const float c0 = kFp8 ? c * rs[nt][0] : c, c1 = kFp8 ? c * rs[nt][1] : c;
      sc[nt][0] *= c0;
      sc[nt][1] *= c1;
      sc[nt][2] *= c0;
      sc[nt][3] *= c1;
    }
    if (need_mask) {
      const int t0 = tb + (lane >> 2);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        if (t0 > lim[nt][0]) sc[nt][0] = -INFINITY;
        if (t0 > lim[nt][1]) sc[nt][1] = -INFINITY;
        if (t0 + 8 > lim[nt][0]) sc[nt][2] = -INFINITY;
        if (t0 + 8 > lim[nt][1]) sc[nt][3] = -INFINITY;
      }
      if (win > 0) {  // keys before a row's window: t <= lim - win
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          if (t0 + win <= lim[nt][0]) sc[nt][0] = -INFINITY;
          if (t0 + win <= lim[nt][1]) sc[nt][1] = -INFINITY;
          if (t0 + 8 + win <= lim[nt][0]) sc[nt][2] = -INFINITY;
          if (t0 + 8 + win <= lim[nt][1]) sc[nt][3] = -INFINITY;
        }
      }
    }
    uint32_t pb[NT][2];
    float alpha[NT][2];
    bool rescale = false;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      alpha[nt][0] = alpha[nt][1] = 1.f;
      pb[nt][0] = pb[nt][1] = 0u;
      if (nt >= nt_active) continue;
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
      if constexpr (!kFp8) {
        pb[nt][0] = movmatrix_trans(pack_bf16x2(sc[nt][0], sc[nt][1]));
        pb[nt][1] = movmatrix_trans(pack_bf16x2(sc[nt][2], sc[nt][3]));
      } else {
        pb[nt][0] = movmatrix_trans(pack_f16x2(sc[nt][0], sc[nt][1]));
        pb[nt][1] = movmatrix_trans(pack_f16x2(sc[nt][2], sc[nt][3]));
      }
    }
    // Slots of the last block past the context, and slots before every row's window, may
    // hold any bits (NaN too): their p is 0, but 0 * NaN is NaN, so their V elements are
    // cleared in the operand fragments (a0/a1 hold tokens 2c, 2c+1 and a2/a3 tokens
    // 2c+8, 2c+9 of the block, c = lane & 3).
    const bool vmask = need_mask && (tb + kBlockSize - 1 > vlim || tb < vlo);
    uint32_t vm_lo = ~0u, vm_hi = ~0u;
    if (vmask) {
      const int t = tb + 2 * (lane & 3);
      auto keep = [&](int tt) { return tt <= vlim && tt >= vlo; };
      vm_lo = (keep(t) ? 0x0000FFFFu : 0u) | (keep(t + 1) ? 0xFFFF0000u : 0u);
      vm_hi = (keep(t + 8) ? 0x0000FFFFu : 0u) | (keep(t + 9) ? 0xFFFF0000u : 0u);
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
    if constexpr (!kFp8) {
      const int v_tok = lr + (lm >> 1) * 8, v_chk = lm & 1;  // V (transposed A)
#pragma unroll
      for (int mt = 0; mt < KSTEPS; ++mt) {
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4_trans(vb + tile_chunk_offset(v_tok, 2 * mt + v_chk), a0, a1, a2, a3);
        if (vmask) {
          a0 &= vm_lo;
          a1 &= vm_lo;
          a2 &= vm_hi;
          a3 &= vm_hi;
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          if (nt < nt_active) mma_bf16_16816(o[mt][nt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
      }
    } else {
      // matrices: tokens 0-7 / 8-15 x the two 16-byte chunks of a 32-byte column group; a
      // lane receives tokens 2c, 2c+1 x codes 2g, 2g+1 of each (tokens 2c+8, 2c+9 from the
      // second), and the byte permute 3120 pairs the two tokens of each code column
      const int v_tok = lr + (lm & 1) * 8, v_chk = lm >> 1;
#pragma unroll
      for (int kc = 0; kc < D / 32; ++kc) {
        uint32_t r0, r1, r2, r3;
        ldmatrix_x4_trans(vb + e4m3_chunk_offset<D>(v_tok, 2 * kc + v_chk), r0, r1, r2, r3);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t a0, a1, a2, a3;
          e4m3x4_to_f16x2(byte_perm(half ? r2 : r0, 0x3120u), a0, a1);  // tokens 2c, 2c+1: d 2g | 2g+1
          e4m3x4_to_f16x2(byte_perm(half ? r3 : r1, 0x3120u), a2, a3);  // tokens 2c+8, 2c+9
          if (vmask) {
            a0 &= vm_lo;
            a1 &= vm_lo;
            a2 &= vm_hi;
            a3 &= vm_hi;
          }
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            if (nt < nt_active) mma_f16_16816(o[2 * kc + half][nt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
        }
      }
    }
  }

  // Row sums across the 8 lanes of a row, then O and (m, l) of this warp to smem.
  __device__ __forceinline__ void finish(float* ow, float2* ml, int lane) {
    constexpr int OS = D + 4;
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
#pragma unroll
    for (int mt = 0; mt < KSTEPS; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        if (nt >= nt_active) continue;
        const int r = nt * 8 + 2 * (lane & 3);
        if constexpr (!kFp8) {
          const int d = mt * 16 + (lane >> 2);
          ow[r * OS + d] = o[mt][nt][0];
          ow[(r + 1) * OS + d] = o[mt][nt][1];
          ow[r * OS + d + 8] = o[mt][nt][2];
          ow[(r + 1) * OS + d + 8] = o[mt][nt][3];
        } else {
          // m g <-> d 2g, m g+8 <-> d 2g+1 (see block); the pool's V scale applies here once
          const int d = mt * 16 + 2 * (lane >> 2);
          *reinterpret_cast<float2*>(ow + r * OS + d) = make_float2(o[mt][nt][0] * v_scale, o[mt][nt][2] * v_scale);
          *reinterpret_cast<float2*>(ow + (r + 1) * OS + d) =
              make_float2(o[mt][nt][1] * v_scale, o[mt][nt][3] * v_scale);
        }
      }
    if (lane < 4) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e)
          ml[nt * 8 + 2 * lane + e] = make_float2(m_run[nt][e], l_run[nt][e]);
    }
  }
};

// ---------------------------------------------------------------------------
// CUDA-core core. Per warp and per 16-token block:
//   QK^T: lane (t = lane/2, half = lane%2) dots token t with every row over its half
//         of head_dim (fp32 FMA); the two halves are joined by one shuffle;
//   online softmax: row max over the 16 tokens by 4 xor-shuffles;
//   PV:   lane owns D/32 output columns; p is broadcast through shared memory.
// Q of the segment's rows is staged in shared memory as fp32 by the whole CTA.
// ---------------------------------------------------------------------------
template <int D, int ROWS_>
struct SimtCore {
  using Geom = TileGeom<D>;
  static constexpr int kStages = 2;
  static constexpr int ROWS = ROWS_;
  static constexpr int CPL = D / 16;  // 16-byte chunks of a row each lane of a pair covers
  static constexpr int DPL = D / 32;  // output columns per lane
  static constexpr bool kNeedsQSmem = true;
  float m_run[ROWS], l_run[ROWS], o[ROWS][DPL];
  int lim[ROWS];
  int vlim;  // largest row limit of the segment: no row sees a token past it
  const float (*q_s)[D];
  float* p_w;  // this warp's [16][ROWS] probabilities

  // All threads of the CTA; a __syncthreads() must follow.
  static __device__ __forceinline__ void stage_q(const DecodeParams& p, const Seg& s, float (*qs)[D],
                                                 int nthreads) {
    for (int idx = threadIdx.x; idx < ROWS * D / 2; idx += nthreads) {
      const int r = idx / (D / 2);
      const int d2 = idx % (D / 2);
      int b, i, h;
      float lo = 0.f, hi = 0.f;
      if (seg_row(p, s, r, b, i, h)) {
        const uint32_t v = __ldg(reinterpret_cast<const uint32_t*>(p.query + out_offset(p, b, i, h, D)) + d2);
        lo = bf16_lo(v);
        hi = bf16_hi(v);
      }
      qs[r][2 * d2] = lo;
      qs[r][2 * d2 + 1] = hi;
    }
  }

  __device__ __forceinline__ void bind(const float (*qs)[D], float* pw) {
    q_s = qs;
    p_w = pw;
  }

  __device__ __forceinline__ void begin(const DecodeParams& p, const Seg& s, int ctx, int) {
#pragma unroll
    for (int r = 0; r < ROWS; ++r) {
      int b, i, h;
      lim[r] = seg_row(p, s, r, b, i, h) ? ctx - p.q_per_seq + i : ctx - 1;
      m_run[r] = -INFINITY;
      l_run[r] = 0.f;
#pragma unroll
      for (int e = 0; e < DPL; ++e) o[r][e] = 0.f;
    }
    vlim = lim[0];
#pragma unroll
    for (int r = 1; r < ROWS; ++r) vlim = max(vlim, lim[r]);
  }

  __device__ __forceinline__ void block(const uint8_t* kt, const uint8_t* vt, int tb, bool need_mask,
                                        float c, int lane, float*, int win, int vlo) {
    const int t_me = lane >> 1;
    const int half = lane & 1;
    float sc[ROWS];
#pragma unroll
    for (int r = 0; r < ROWS; ++r) sc[r] = 0.f;
#pragma unroll
    for (int ci = 0; ci < CPL; ++ci) {
      // the two lanes of a pair start half a row apart and walk the chunk positions in
      // a rotated order so that they never share a bank group
      const int cc = half * CPL + (ci ^ (half * (CPL / 2)));
      const uint4 kv = *reinterpret_cast<const uint4*>(kt + tile_chunk_offset(t_me, cc));
      const float kf[8] = {bf16_lo(kv.x), bf16_hi(kv.x), bf16_lo(kv.y), bf16_hi(kv.y),
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
    bool rescale = false;
    float alpha[ROWS];
#pragma unroll
    for (int r = 0; r < ROWS; ++r) {
      float sv = (sc[r] + __shfl_xor_sync(kFull, sc[r], 1)) * c;  // log2 units
      if (need_mask && (t_glob > lim[r] || (win > 0 && t_glob + win <= lim[r]))) sv = -INFINITY;
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
      if (half == 0) p_w[t_me * ROWS + r] = pr;
    }
    if (rescale) {  // m_run is warp-uniform, so is alpha
#pragma unroll
      for (int r = 0; r < ROWS; ++r)
#pragma unroll
        for (int e = 0; e < DPL; ++e) o[r][e] *= alpha[r];
    }
    __syncwarp();
    const int pv_chunk = (lane * DPL) / 8;
    const int pv_byte = ((lane * DPL) % 8) * 2;
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
      if (need_mask && (tb + t > vlim || tb + t < vlo)) {  // outside every row's keys: p = 0, V may be NaN
#pragma unroll
        for (int e = 0; e < DPL; ++e) vf[e] = 0.f;
      }
#pragma unroll
      for (int r = 0; r < ROWS; ++r) {
        const float pr = p_w[t * ROWS + r];
#pragma unroll
        for (int e = 0; e < DPL; ++e) o[r][e] = fmaf(pr, vf[e], o[r][e]);
      }
    }
    __syncwarp();
  }

  __device__ __forceinline__ void finish(float* ow, float2* ml, int lane) {
    constexpr int OS = D + 4;
#pragma unroll
    for (int r = 0; r < ROWS; ++r) {
      float l = l_run[r];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) l += __shfl_xor_sync(kFull, l, off);
      l_run[r] = l;
    }
#pragma unroll
    for (int r = 0; r < ROWS; ++r)
#pragma unroll
      for (int e = 0; e < DPL; ++e) ow[r * OS + lane * DPL + e] = o[r][e];
    if (lane == 0) {
#pragma unroll
      for (int r = 0; r < ROWS; ++r) ml[r] = make_float2(m_run[r], l_run[r]);
    }
  }
};

// ---------------------------------------------------------------------------
// Shared memory of a decode CTA and the per-segment driver.
// ---------------------------------------------------------------------------
template <class Geom, int ROWS, int NW, int STAGES>
struct DecodeSmem {
  static constexpr int D = Geom::kD;
  static constexpr int kStages = NW * STAGES * Geom::kStageBytes;
  static constexpr int kMerge = NW * ROWS * (D + 4) * 4;
  static constexpr int kBytes = (kStages > kMerge ? kStages : kMerge) + 1024;  // + alignment slack
};

// Static shared state; the q / p staging areas exist for the CUDA-core core only.
template <int D, int ROWS, int NW, int STAGES, bool kQ>
struct CtaState {
  uint64_t bars[NW * STAGES];
  float2 ml[NW * ROWS];
  int slot[kTileMaxRows];
  int last[kTileMaxRows];
  __align__(16) float q_s[kQ ? ROWS : 1][D];
  __align__(16) float p_s[NW][kQ ? 16 * ROWS : 1];
};

// Run one segment through the warps' pipelines; on return every warp's (m, l, O)
// sits in shared memory (ow: NW x ROWS x (D+4) fp32 over the stage buffers; st.ml).
template <class Core, int D, int NW, int STAGES, class State>
__device__ __forceinline__ void run_segment(const DecodeParams& p, const Seg& sg, int ctx,
                                            WarpPipe<typename Core::Geom, NW, STAGES>& pipe, Core& core, State& st,
                                            uint8_t* smem, const CUtensorMap* tk,
                                            const CUtensorMap* tv, int warp, int lane) {
  constexpr int OS = D + 4;
  const int32_t* trow = p.block_tables + static_cast<size_t>(sg.b0) * p.max_blocks;
  pipe.start(trow, sg.blk0, sg.blk1, sg.kvh);
#pragma unroll
  for (int s = 0; s < STAGES; ++s)
    if (s < pipe.n_my) pipe.issue(s, tk, tv);
  if constexpr (Core::kNeedsQSmem) {
    Core::stage_q(p, sg, st.q_s, NW * 32);
    core.bind(st.q_s, st.p_s[warp]);
    __syncthreads();
  }
  core.begin(p, sg, ctx, lane);
  const float c = p.scale_log2;
  const int first_masked = ctx - p.q_per_seq;  // blocks ending past this position need the mask
  // sliding window: the segment's first row (query token row0 / G) has the lowest window
  // start; blocks starting before ctx - win (the last query's window start) need the mask
  const int win = p.window;
  const int vlo = win > 0 ? ctx - p.q_per_seq + sg.row0 / p.group - win + 1 : INT_MIN;
  for (int k = 0; k < pipe.n_my; ++k) {
    if (!pipe.wait(k)) {
      if (lane == 0) record_error(kErrTimeoutDecode);
      pipe.drain(k);
      break;
    }
    const int s = pipe.stage_of(k);
    const int tb = pipe.block_of(k) * kBlockSize;
    const bool need_mask = !sg.shared && (tb + kBlockSize - 1 > first_masked || (win > 0 && tb < ctx - win));
    core.block(pipe.kbuf(s), pipe.vbuf(s), tb, need_mask, c, lane, nullptr, win, vlo);
    __syncwarp();
    if (k + STAGES < pipe.n_my) pipe.issue(k + STAGES, tk, tv);
  }
  __syncthreads();  // every warp is done with its stage buffers
  core.finish(reinterpret_cast<float*>(smem) + warp * Core::ROWS * OS, st.ml + warp * Core::ROWS, lane);
  __syncthreads();
}

// Cross-warp combine of local row r, 8 output columns starting at dc*8:
// M = max_w m_w, L = sum_w l_w 2^(m_w - M), acc = sum_w O_w 2^(m_w - M).
template <int D, int ROWS, int NW>
__device__ __forceinline__ void combine_row(const float* ow, const float2* ml, int r, int dc, float& M,
                                            float& L, float (&acc)[8]) {
  constexpr int OS = D + 4;
  M = -INFINITY;
#pragma unroll
  for (int w = 0; w < NW; ++w) M = fmaxf(M, ml[w * ROWS + r].x);
  L = 0.f;
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
}

__device__ __forceinline__ void store_bf16x8(uint16_t* dst, const float (&acc)[8], float inv) {
  uint4 v;
  v.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  v.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
  v.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
  v.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
  *reinterpret_cast<uint4*>(dst) = v;
}

template <int NW, int STAGES>
__device__ __forceinline__ void init_cta(uint64_t* bars, const CUtensorMap* tk, const CUtensorMap* tv) {
  if (threadIdx.x == 0) {
    for (int i = 0; i < NW * STAGES; ++i) mbar_init(&bars[i], 1);
    fence_barrier_init();
    tma_prefetch_desc(tk);
    tma_prefetch_desc(tv);
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------
// Persistent decode. CTA c covers work units [c*W/P, (c+1)*W/P) of the flattened
// list the pre-pass built: per sequence b, its shared-prefix band (leaders only:
// H_kv sub-units of P_b blocks, rows = members x rows) then its private band
// (H_kv x row_chunks sub-units of nblk_b - P_b blocks). A sub-unit cut by the CTA
// range, or a target that also has a shared part, is completed through partial
// records: each piece adds its block count to the target's arrival counter and the
// piece that brings it to nblk merges all of the target's records.
// ---------------------------------------------------------------------------
template <class Core, int D, int NW, int STAGES>
__global__ void __launch_bounds__(NW * 32)
decode_persistent_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmap_k,
                         const __grid_constant__ CUtensorMap tmap_v) {
  constexpr int ROWS = Core::ROWS;
  constexpr int DC = D / 8;
  extern __shared__ uint8_t smem_raw[];
  __shared__ CtaState<D, ROWS, NW, STAGES, Core::kNeedsQSmem> st;
  uint8_t* smem = align1024(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  init_cta<NW, STAGES>(st.bars, &tmap_k, &tmap_v);
  grid_dependency_wait();  // the pre-pass (and anything before it) has completed

  const long long W = __ldcg(&p.hdr->work);
  const long long pos_end = W * (blockIdx.x + 1) / gridDim.x;
  long long pos = W * blockIdx.x / gridDim.x;
  if (pos >= pos_end) {
    grid_launch_dependents();
    return;
  }
  WarpPipe<typename Core::Geom, NW, STAGES> pipe;
  pipe.init(smem, st.bars, warp, lane);
  Core core;
  const int H = p.num_kv_heads;
  const int RC = p.row_chunks;
  int b = __ldcg(p.cta_seq + blockIdx.x);
  if (b < 0 || b >= p.num_seqs) {  // inconsistent schedule tables
    record_error(kErrSchedule);
    grid_launch_dependents();
    return;
  }
  while (pos < pos_end && b < p.num_seqs) {
    const long long base = __ldcg(p.seq_start + b);
    const int4 info = __ldcg(p.seq_info + b);
    const int P_b = info.x, members = info.y, nblk = info.z;
    const long long sh_work = members > 0 ? static_cast<long long>(H) * P_b : 0;
    const int pv_len = nblk - P_b;
    const long long pv_work = static_cast<long long>(H) * RC * pv_len;
    if (pos >= base + sh_work + pv_work) {
      ++b;
      continue;
    }
    Seg sg;
    int rc = 0;
    long long len;
    if (pos < base + sh_work) {
      const long long off = pos - base;
      const int kvh = static_cast<int>(off / P_b);
      const int j = static_cast<int>(off - static_cast<long long>(kvh) * P_b);
      len = min(pos_end - pos, static_cast<long long>(P_b - j));
      sg = Seg{b, members, kvh, 0, members * p.rows, j, j + static_cast<int>(len), true};
    } else {
      const long long off = pos - base - sh_work;
      const int sub = static_cast<int>(off / pv_len);
      const int jo = static_cast<int>(off - static_cast<long long>(sub) * pv_len);
      rc = sub % RC;
      const int kvh = sub / RC;
      len = min(pos_end - pos, static_cast<long long>(pv_len - jo));
      sg = Seg{b, 1, kvh, rc * ROWS, min(ROWS, p.rows - rc * ROWS), P_b + jo,
               P_b + jo + static_cast<int>(len), false};
    }
    if (len <= 0) {  // cannot happen with consistent tables; never loop forever
      if (threadIdx.x == 0) record_error(kErrSchedule);
      break;
    }
    const int ctx = info.w;
    run_segment<Core, D, NW, STAGES>(p, sg, ctx, pipe, core, st, smem, &tmap_k, &tmap_v, warp, lane);
    const float* ow = reinterpret_cast<const float*>(smem);

    const bool direct = !sg.shared && P_b == 0 && sg.blk0 == 0 && sg.blk1 == nblk;
    if (direct) {
      for (int task = threadIdx.x; task < sg.nrows * DC; task += NW * 32) {
        const int r = task / DC, dc = task % DC;
        float M, L, acc[8];
        combine_row<D, ROWS, NW>(ow, st.ml, r, dc, M, L, acc);
        int bb, i, h;
        seg_row(p, sg, r, bb, i, h);
        store_bf16x8(p.out + out_offset(p, bb, i, h, D) + dc * 8, acc, L > 0.f ? 1.f / L : 0.f);
      }
    } else {
      // one partial record per output target (sequence, kv head, row chunk) touched
      const int tr = p.target_rows;
      if (threadIdx.x < sg.members) {
        int slot = atomicAdd(&p.hdr->pool, 1);
        if (slot >= p.pool_cap) {
          record_error(kErrRecordPool);
          slot = -1;
        }
        st.slot[threadIdx.x] = slot;
      }
      __syncthreads();
      for (int task = threadIdx.x; task < sg.nrows * DC; task += NW * 32) {
        const int r = task / DC, dc = task % DC;
        const int m = sg.shared ? r / p.rows : 0;
        const int rr = sg.shared ? r - m * p.rows : r;  // row inside the target
        const int slot = st.slot[m];
        if (slot < 0) continue;
        float M, L, acc[8];
        combine_row<D, ROWS, NW>(ow, st.ml, r, dc, M, L, acc);
        float* rec = p.records + static_cast<size_t>(slot) * p.rec_stride;
        float4* dst = reinterpret_cast<float4*>(rec + rr * D + dc * 8);
        __stcg(dst, make_float4(acc[0], acc[1], acc[2], acc[3]));
        __stcg(dst + 1, make_float4(acc[4], acc[5], acc[6], acc[7]));
        if (dc == 0) __stcg(reinterpret_cast<float2*>(rec + tr * D) + rr, make_float2(M, L));
      }
      __threadfence();
      __syncthreads();
      if (threadIdx.x < sg.members) {
        const int bm = sg.b0 + threadIdx.x;
        const int t = (bm * H + sg.kvh) * RC + rc;
        const int slot = st.slot[threadIdx.x];
        if (slot >= 0) {
          const int idx = atomicAdd(p.list_len + t, 1);
          if (idx < p.list_cap) {
            p.list[static_cast<size_t>(t) * p.list_cap + idx] = make_int2(sg.blk0, slot);
          } else {
            record_error(kErrRecordList);
          }
        }
        __threadfence();
        const int nb_m = num_blocks_of(p, __ldg(p.context_lens + bm));
        const int prev = atomicAdd(p.arrive + t, static_cast<int>(len));
        st.last[threadIdx.x] = (prev + static_cast<int>(len) == nb_m) ? 1 : 0;
      }
      __syncthreads();
      for (int m = 0; m < sg.members; ++m) {
        if (!st.last[m]) continue;  // uniform: shared memory flag
        // This piece completed target t: merge its records in order of their first
        // block (unique per target), so the result does not depend on arrival order.
        __threadfence();
        const int bm = sg.b0 + m;
        const int t = (bm * H + sg.kvh) * RC + rc;
        const int n = min(__ldcg(p.list_len + t), p.list_cap);
        const int2* lst = p.list + static_cast<size_t>(t) * p.list_cap;
        int2* raw = reinterpret_cast<int2*>(smem);  // stage buffers are free here
        int* sorted = reinterpret_cast<int*>(raw + n);
        for (int k = threadIdx.x; k < n; k += NW * 32) raw[k] = __ldcg(lst + k);
        __syncthreads();
        for (int k = threadIdx.x; k < n; k += NW * 32) {
          int rank = 0;
          for (int k2 = 0; k2 < n; ++k2) rank += raw[k2].x < raw[k].x;
          sorted[rank] = raw[k].y;
        }
        __syncthreads();
        const int rows_t = min(tr, p.rows - rc * ROWS);
        for (int task = threadIdx.x; task < rows_t * DC; task += NW * 32) {
          const int rr = task / DC, dc = task % DC;
          float M = -INFINITY;
          for (int k = 0; k < n; ++k) {
            const float* rec = p.records + static_cast<size_t>(sorted[k]) * p.rec_stride;
            M = fmaxf(M, __ldcg(reinterpret_cast<const float2*>(rec + tr * D) + rr).x);
          }
          float L = 0.f, acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
          for (int k = 0; k < n; ++k) {
            const float* rec = p.records + static_cast<size_t>(sorted[k]) * p.rec_stride;
            const float2 mlk = __ldcg(reinterpret_cast<const float2*>(rec + tr * D) + rr);
            const float wt = (mlk.x == -INFINITY) ? 0.f : fast_exp2(mlk.x - M);
            L += wt * mlk.y;
            const float4* src = reinterpret_cast<const float4*>(rec + rr * D + dc * 8);
            const float4 x0 = __ldcg(src), x1 = __ldcg(src + 1);
            acc[0] += wt * x0.x; acc[1] += wt * x0.y; acc[2] += wt * x0.z; acc[3] += wt * x0.w;
            acc[4] += wt * x1.x; acc[5] += wt * x1.y; acc[6] += wt * x1.z; acc[7] += wt * x1.w;
          }
          const int rg = rc * ROWS + rr;
          const int i = rg / p.group;
          const int h = sg.kvh * p.group + (rg - i * p.group);
          store_bf16x8(p.out + out_offset(p, bm, i, h, D) + dc * 8, acc, L > 0.f ? 1.f / L : 0.f);
        }
        __syncthreads();  // the sort buffer is reused by the next member
      }
    }
    __syncthreads();  // shared memory is reused by the next segment
    pos += len;
  }
  grid_launch_dependents();
}

// ---------------------------------------------------------------------------
// Pre-pass of the persistent schedule (one CTA of kPrepassThreads threads).
//   1. per sequence: nblk; with prefix sharing on, groups = maximal runs of adjacent
//      sequences whose first block is the same physical block, cut into chunks of
//      share_cap members; a chunk's shared prefix P = the leading blocks identical in
//      all members' tables, limited to blocks every member's query rows fully see.
//   2. work(b) = [leader: H_kv * P] + H_kv * row_chunks * (nblk - P_b); exclusive scan
//      -> seq_start; W = total; CTA c starts in the sequence holding unit c*W/P.
//   3. zero the arrival counters and record lists; zero outputs of empty sequences.
// ---------------------------------------------------------------------------
constexpr int kPrepassThreads = 1024;

__device__ __forceinline__ long long block_exclusive_scan(long long v, long long* warp_tot,
                                                          long long& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  long long x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const long long y = __shfl_up_sync(kFull, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    long long w = lane < kPrepassThreads / 32 ? warp_tot[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const long long y = __shfl_up_sync(kFull, w, off);
      if (lane >= off) w += y;
    }
    warp_tot[lane] = w;  // inclusive prefix over warps
  }
  __syncthreads();
  const long long before = (warp > 0 ? warp_tot[warp - 1] : 0) + x - v;
  total = warp_tot[kPrepassThreads / 32 - 1];
  __syncthreads();
  return before;
}

template <int D>
__global__ void __launch_bounds__(kPrepassThreads) sched_prepass_kernel(const DecodeParams p) {
  constexpr int T = kPrepassThreads;
  constexpr int kLook = 16;                 // >= share_cap - 1: lookahead past the chunk
  __shared__ long long warp_tot[T / 32];
  __shared__ int wmax[T / 32];
  __shared__ int s_g0carry;
  __shared__ int s_ctx[T + kLook];          // context lengths of the chunk (+ lookahead)
  __shared__ int s_gstart[T + kLook];       // 1: the sequence starts a new shared group
  __shared__ int s_lead[T];                 // leaders of this chunk with a possible shared prefix
  __shared__ int s_pmax[T];
  __shared__ int s_mem[T];
  __shared__ int s_bad[T];
  __shared__ int s_nlead;
  grid_dependency_wait();
  grid_launch_dependents();
  const int B = p.num_seqs;
  const int H = p.num_kv_heads;
  const int RC = p.row_chunks;
  const int cap = p.share_cap;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  // ---- pass 1: sharing, P_b, work(b) (kept in seq_start for now), W
  if (threadIdx.x == 0) s_g0carry = 0;
  __syncthreads();
  long long W = 0;
  for (int c0 = 0; c0 < B; c0 += T) {
    const int b = c0 + threadIdx.x;
    const bool in = b < B;
    // one round of independent loads: context lengths and group-start flags
    for (int idx = threadIdx.x; idx < T + kLook; idx += T) {
      const int bb = c0 + idx;
      int c = 0, g = 1;
      if (bb < B) {
        c = __ldg(p.context_lens + bb);
        if (cap >= 2 && bb > 0) {
          const int cprev = __ldg(p.context_lens + bb - 1);
          const int t0 = __ldg(p.block_tables + static_cast<size_t>(bb) * p.max_blocks);
          const int t1 = __ldg(p.block_tables + static_cast<size_t>(bb - 1) * p.max_blocks);
          g = (num_blocks_of(p, c) == 0 || num_blocks_of(p, cprev) == 0 || t0 != t1) ? 1 : 0;
        }
      }
      s_ctx[idx] = c;
      s_gstart[idx] = g;
    }
    if (threadIdx.x == 0) s_nlead = 0;
    __syncthreads();
    const int ctx = s_ctx[threadIdx.x];
    const int nblk = in ? num_blocks_of(p, ctx) : 0;
    int g0 = 0;
    if (cap >= 2) {
      // first sequence of b's group: inclusive max-scan of group start positions
      int v = (in && s_gstart[threadIdx.x]) ? b : -1;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(kFull, v, off);
        if (lane >= off) v = max(v, y);
      }
      if (lane == 31) wmax[warp] = v;
      __syncthreads();
      int before = s_g0carry;
      for (int w = 0; w < warp; ++w) before = max(before, wmax[w]);
      g0 = max(v, before);
      __syncthreads();
      if (threadIdx.x == T - 1) s_g0carry = g0;
      // chunk leaders: members, and the blocks every member's rows fully see
      if (in && (b - g0) % cap == 0) {
        int mem = 1;
        int pmax = (ctx - p.q_per_seq + 1) / kBlockSize;
        while (mem < cap && b + mem < B && !s_gstart[threadIdx.x + mem]) {
          pmax = min(pmax, (s_ctx[threadIdx.x + mem] - p.q_per_seq + 1) / kBlockSize);
          ++mem;
        }
        pmax = max(0, min(pmax, nblk));
        if (mem > 1 && pmax > 0) {
          const int k = atomicAdd(&s_nlead, 1);
          s_lead[k] = b;
          s_pmax[k] = pmax;
          s_mem[k] = mem;
          s_bad[k] = pmax;
        } else {
          p.seq_info[b] = make_int4(0, 0, nblk, ctx);
        }
      }
      __syncthreads();
      // longest common table prefix: warps take (leader, 32-block window) pairs; the
      // members' entries of a window are loaded together
      const int nlead = s_nlead;
      int npairs = 0;
      for (int k = 0; k < nlead; ++k) npairs += (s_pmax[k] + 31) / 32;
      for (int pr = warp; pr < npairs; pr += T / 32) {
        int k = 0, rem = pr;
        while (rem >= (s_pmax[k] + 31) / 32) {
          rem -= (s_pmax[k] + 31) / 32;
          ++k;
        }
        const int j = rem * 32 + lane;
        const int mem = s_mem[k];
        bool ok = true;
        if (j < s_pmax[k]) {
          const int32_t* t0 = p.block_tables + static_cast<size_t>(s_lead[k]) * p.max_blocks + j;
          const int ref = __ldg(t0);
          int vals[kLook];
#pragma unroll
          for (int m = 1; m < kLook; ++m)
            vals[m] = m < mem ? __ldg(t0 + static_cast<size_t>(m) * p.max_blocks) : ref;
#pragma unroll
          for (int m = 1; m < kLook; ++m) ok &= vals[m] == ref;
        }
        const unsigned badmask = __ballot_sync(kFull, !ok);
        if (badmask && lane == 0) atomicMin(&s_bad[k], rem * 32 + __ffs(badmask) - 1);
      }
      __syncthreads();
      for (int k = threadIdx.x; k < nlead; k += T) {
        const int P = s_bad[k];
        const int lb = s_lead[k] - c0;
        p.seq_info[s_lead[k]] = make_int4(P, P > 0 ? s_mem[k] : 0, num_blocks_of(p, s_ctx[lb]), s_ctx[lb]);
      }
    }
    __syncthreads();
    int P_b = 0, lead_members = 0;
    if (in && cap >= 2) {
      const int leader = g0 + ((b - g0) / cap) * cap;
      const int4 li = p.seq_info[leader];
      if (li.y > 0) P_b = li.x;  // the chunk has a shared unit
      if (leader == b) lead_members = li.y;
    }
    __syncthreads();  // every leader entry is read before any is rewritten
    long long work = 0;
    if (in) {
      p.seq_info[b] = make_int4(P_b, lead_members, nblk, ctx);
      work = (lead_members > 0 ? static_cast<long long>(H) * P_b : 0) +
             static_cast<long long>(H) * RC * (nblk - P_b);
      p.seq_start[b] = work;
    }
    long long tot;
    block_exclusive_scan(work, warp_tot, tot);
    W += tot;
  }
  __syncthreads();

  // ---- pass 2: starts, CTA assignment, counters
  const long long P = p.num_ctas;
  long long carry = 0;
  for (int c0 = 0; c0 < B; c0 += T) {
    const int b = c0 + threadIdx.x;
    const long long work = b < B ? p.seq_start[b] : 0;
    long long tot;
    const long long start = carry + block_exclusive_scan(work, warp_tot, tot);
    if (b < B) {
      p.seq_start[b] = start;
      if (W > 0 && work > 0) {
        const long long c_lo = (start * P + W - 1) / W;
        const long long c_hi = min(P, ((start + work) * P + W - 1) / W);
        for (long long c = c_lo; c < c_hi; ++c) p.cta_seq[c] = b;
      }
    }
    carry += tot;
  }
  const int targets = B * H * RC;
  for (int t = threadIdx.x; t < targets; t += T) {
    p.arrive[t] = 0;
    p.list_len[t] = 0;
  }
  // sequences without any block: outputs are zero
  for (int b = warp; b < B; b += T / 32) {
    if (num_blocks_of(p, __ldg(p.context_lens + b)) != 0) continue;
    uint16_t* dst = p.out + static_cast<size_t>(b) * p.q_per_seq * p.num_q_heads * D;
    for (int e = lane; e < p.q_per_seq * p.num_q_heads * D / 8; e += 32)
      reinterpret_cast<uint4*>(dst)[e] = make_uint4(0, 0, 0, 0);
  }
  if (threadIdx.x == 0) {
    p.hdr->work = W;
    p.hdr->pool = 0;
  }
}

// ---------------------------------------------------------------------------
// Grid decode: one CTA per (kv head x row chunk, sequence, split of split_blocks
// blocks). A sequence with one split writes bf16 directly; otherwise each split
// writes fp32 partials (o, m, l) for merge_kernel.
// ---------------------------------------------------------------------------
// Resident CTAs per SM the compiler must allow for (a register cap of 168): 3 for the
// cores that fit without spilling; the 24- and 32-row tensor-core cores keep their
// registers (they spill under the cap, which measured slower) and run 2 per SM; the 8-row
// E4M3 core runs 4 (a cap of 128).
template <class Core>
constexpr int min_ctas_per_sm() {
  if (Core::Geom::kE4M3 && Core::ROWS <= 8) return 4;  // the 8-row E4M3 core fits 4 per SM
  return Core::ROWS > 16 && !Core::kNeedsQSmem ? 2 : 3;
}

template <class Core, int D, int NW, int STAGES>
__global__ void __launch_bounds__(NW * 32, min_ctas_per_sm<Core>())
decode_grid_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmap_k,
                   const __grid_constant__ CUtensorMap tmap_v) {
  constexpr int ROWS = Core::ROWS;
  constexpr int DC = D / 8;
  extern __shared__ uint8_t smem_raw[];
  __shared__ CtaState<D, ROWS, NW, STAGES, Core::kNeedsQSmem> st;
  uint8_t* smem = align1024(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  init_cta<NW, STAGES>(st.bars, &tmap_k, &tmap_v);
  grid_dependency_wait();  // inputs may be produced by the previous kernel on the stream
  const int H = p.num_kv_heads;
  const int RQ = p.q_per_seq * p.num_q_heads;
  const float* ow = reinterpret_cast<const float*>(smem);
  WarpPipe<typename Core::Geom, NW, STAGES> pipe;
  pipe.init(smem, st.bars, warp, lane);
  Core core;

  // Grid layout. Without prefix sharing: x = kv head x row chunk, y = sequence,
  // z = split of split_blocks blocks. With prefix sharing, a 1-D grid: first the
  // shared CTAs (kv head, window of share_cap sequences, split of a shared prefix),
  // then the sequences' own CTAs (kv head, sequence, split of the blocks after the
  // shared prefix).
  int kvh, rc = 0, b = 0, z;
  bool shared_role = false;
  if (p.share_cap) {
    const long long idx = blockIdx.x;
    const long long n_sh = static_cast<long long>(H) * p.share_windows * p.share_splits;
    if (idx < n_sh) {
      shared_role = true;
      kvh = static_cast<int>(idx % H);
      b = static_cast<int>((idx / H) % p.share_windows) * p.share_cap;  // first sequence of the window
      z = static_cast<int>(idx / (static_cast<long long>(H) * p.share_windows));
    } else {
      const long long j = idx - n_sh;
      kvh = static_cast<int>(j % H);
      b = static_cast<int>((j / H) % p.num_seqs);
      z = static_cast<int>(j / (static_cast<long long>(H) * p.num_seqs));
    }
  } else {
    kvh = blockIdx.x / p.row_chunks;
    rc = blockIdx.x % p.row_chunks;
    b = blockIdx.y;
    z = blockIdx.z;
  }

  if (shared_role) {
    // every chunk leader of the window whose shared prefix reaches split z
    const int ssb = p.share_split_blocks;
    const int wend = min(p.num_seqs, b + p.share_cap);
    if (threadIdx.x < wend - b) {
      const int4 info = __ldcg(p.seq_info + b + threadIdx.x);
      st.slot[threadIdx.x] = info.x;  // shared prefix blocks
      st.last[threadIdx.x] = info.y;  // members if this sequence leads a chunk
    }
    __syncthreads();
    for (int L = b; L < wend; ++L) {
      const int P_L = st.slot[L - b], members = st.last[L - b];
      if (members == 0 || z * ssb >= P_L) continue;  // uniform
      const Seg sg{L, members, kvh, 0, members * p.rows, z * ssb, min(P_L, z * ssb + ssb), true};
      run_segment<Core, D, NW, STAGES>(p, sg, 0, pipe, core, st, smem, &tmap_k, &tmap_v, warp, lane);
      for (int task = threadIdx.x; task < sg.nrows * DC; task += NW * 32) {
        const int r = task / DC, dc = task % DC;
        float M, L2, acc[8];
        combine_row<D, ROWS, NW>(ow, st.ml, r, dc, M, L2, acc);
        int bb, i, h;
        seg_row(p, sg, r, bb, i, h);
        const size_t rec = (static_cast<size_t>(bb) * p.share_splits + z) * RQ + i * p.num_q_heads + h;
        float4* dst = reinterpret_cast<float4*>(p.ws_o + rec * D + dc * 8);
        dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
        if (dc == 0) p.ws_ml[rec] = make_float2(M, L2);
      }
      __syncthreads();  // shared memory is reused by the next segment
    }
    grid_launch_dependents();
    return;
  }

  const int ctx = __ldg(p.context_lens + b);
  const int nblk = num_blocks_of(p, ctx);
  const int S = p.num_splits;
  const int sb = p.split_blocks;
  // own blocks start after the shared prefix, or at the first block of the window; a partial
  // decode (context parallelism) reads table entries [range_lo, range_hi) only
  const int P_b = p.share_cap ? __ldcg(p.seq_info + b).x : window_first_block(p, ctx);
  const int lo_b = p.partial_only ? max(P_b, p.range_lo) : P_b;
  const int hi_b = p.partial_only ? min(nblk, p.range_hi) : nblk;
  Seg sg{b, 1, kvh, rc * ROWS, min(ROWS, p.rows - rc * ROWS), 0, 0, false};
  const int blk0 = lo_b + z * sb;
  if (blk0 >= hi_b) {
    if (p.partial_only) {  // no key of this piece: an empty record (weight 0 in the merge)
      for (int task = threadIdx.x; task < sg.nrows * DC; task += NW * 32) {
        int bb, i, h;
        seg_row(p, sg, task / DC, bb, i, h);
        const size_t rec = (static_cast<size_t>(z) * p.num_seqs + b) * RQ + i * p.num_q_heads + h;
        float4* dst = reinterpret_cast<float4*>(p.ws_o + rec * D + (task % DC) * 8);
        dst[0] = make_float4(0.f, 0.f, 0.f, 0.f);
        dst[1] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (task % DC == 0) p.ws_ml[rec] = make_float2(-INFINITY, 0.f);
      }
    } else if (z == 0 && nblk == 0) {  // no block at all: zero output
      for (int task = threadIdx.x; task < sg.nrows * DC; task += NW * 32) {
        int bb, i, h;
        seg_row(p, sg, task / DC, bb, i, h);
        *reinterpret_cast<uint4*>(p.out + out_offset(p, bb, i, h, D) + (task % DC) * 8) = make_uint4(0, 0, 0, 0);
      }
    }
    grid_launch_dependents();
    return;
  }
  sg.blk0 = blk0;
  sg.blk1 = min(hi_b, blk0 + sb);
  // the only piece of its outputs: write bf16 directly (a partial decode always writes records)
  const bool direct = !p.partial_only && (p.share_cap == 0 || P_b == 0) && nblk - P_b <= sb;
  run_segment<Core, D, NW, STAGES>(p, sg, ctx, pipe, core, st, smem, &tmap_k, &tmap_v, warp, lane);
  grid_launch_dependents();
  // own-block records follow the shared-prefix records when sharing is on
  const size_t region = p.share_cap ? static_cast<size_t>(p.num_seqs) * p.share_splits : 0;
  for (int task = threadIdx.x; task < sg.nrows * DC; task += NW * 32) {
    const int r = task / DC, dc = task % DC;
    float M, L, acc[8];
    combine_row<D, ROWS, NW>(ow, st.ml, r, dc, M, L, acc);
    int bb, i, h;
    seg_row(p, sg, r, bb, i, h);
    if (direct) {
      store_bf16x8(p.out + out_offset(p, bb, i, h, D) + dc * 8, acc, L > 0.f ? 1.f / L : 0.f);
    } else {
      // a partial decode's pieces are part-major ([piece][sequence][row]), as the merge of
      // gathered pieces reads them
      const size_t rec = p.partial_only ? (static_cast<size_t>(z) * p.num_seqs + b) * RQ + i * p.num_q_heads + h
                                        : (region + static_cast<size_t>(b) * S + z) * RQ + i * p.num_q_heads + h;
      float4* dst = reinterpret_cast<float4*>(p.ws_o + rec * D + dc * 8);
      dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
      if (dc == 0) p.ws_ml[rec] = make_float2(M, L);
    }
  }
}

// Prefix sharing for the grid schedule, one warp per sequence b. Sequences are cut
// into windows of share_cap aligned at multiples of share_cap; inside a window, a
// chunk is a maximal run of sequences whose block tables start with the same
// physical block. The chunk's shared prefix P = the leading table entries identical
// for all its members, limited to blocks every member's query rows fully see and to
// kShareScanBlocks. Every member computes the same chunk and P from the same data.
// seq_info[b] = {P (0: no shared part), members if b leads a chunk with P > 0, nblk, ctx}.
constexpr int kShareScanBlocks = 8192;

__global__ void __launch_bounds__(128) share_prepass_kernel(const DecodeParams p) {
  grid_dependency_wait();
  grid_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int b = blockIdx.x * 4 + (threadIdx.x >> 5);
  if (b >= p.num_seqs) return;
  const int cap = p.share_cap;  // 2..16
  const int W0 = (b / cap) * cap;
  const int span = min(cap, p.num_seqs - W0);
  int ctx_l = 0, nb_l = 0;
  bool gs = true;
  if (lane < span) {
    const int bb = W0 + lane;
    ctx_l = __ldg(p.context_lens + bb);
    nb_l = num_blocks_of(p, ctx_l);
    if (lane > 0) {
      const int nprev = num_blocks_of(p, __ldg(p.context_lens + bb - 1));
      gs = nb_l == 0 || nprev == 0 ||
           __ldg(p.block_tables + static_cast<size_t>(bb) * p.max_blocks) !=
               __ldg(p.block_tables + static_cast<size_t>(bb - 1) * p.max_blocks);
    }
  }
  const unsigned starts = __ballot_sync(kFull, lane < span && gs);  // bit 0 is always set
  const int m = b - W0;
  const unsigned upto = (m >= 31) ? kFull : ((2u << m) - 1u);
  const int Li = 31 - __clz(starts & upto);
  const unsigned above = starts & ~upto;
  const int Ni = above ? __ffs(above) - 1 : span;
  const int members = Ni - Li;
  const int leader = W0 + Li;
  int pm = (lane >= Li && lane < Ni) ? min((ctx_l - p.q_per_seq + 1) / kBlockSize, nb_l) : INT_MAX;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) pm = min(pm, __shfl_xor_sync(kFull, pm, off));
  const int pmax = max(0, min(pm, kShareScanBlocks));
  int P = 0;
  if (members > 1 && pmax > 0) {
    const int32_t* t0 = p.block_tables + static_cast<size_t>(leader) * p.max_blocks;
    P = pmax;
    // 128 table positions per round: the loads of a round are all issued before any
    // comparison, so a 2048-token prefix costs one round trip
    for (int j0 = 0; j0 < pmax && P == pmax; j0 += 128) {
      unsigned bad[4];
#pragma unroll
      for (int part = 0; part < 4; ++part) {
        const int j = j0 + part * 32 + lane;
        bool ok = true;
        if (j < pmax) {
          const int ref = __ldg(t0 + j);
          int vals[16];
#pragma unroll
          for (int mm = 1; mm < 16; ++mm)
            vals[mm] = mm < members ? __ldg(t0 + static_cast<size_t>(mm) * p.max_blocks + j) : ref;
#pragma unroll
          for (int mm = 1; mm < 16; ++mm) ok &= vals[mm] == ref;
        }
        bad[part] = __ballot_sync(kFull, !ok);
      }
#pragma unroll
      for (int part = 3; part >= 0; --part)
        if (bad[part]) P = j0 + part * 32 + __ffs(bad[part]) - 1;
    }
  }
  const int my_ctx = __shfl_sync(kFull, ctx_l, m);
  if (lane == 0)
    p.seq_info[b] = make_int4(P, (b == leader && P > 0) ? members : 0, num_blocks_of(p, my_ctx), my_ctx);
}

// Log-sum-exp merge of the grid schedule's split partials. One CTA per output row
// (sequence, query token, head) with MW warps: warp w folds splits w, w+MW, ... into
// (M_w, L_w, acc_w) with lanes over head_dim, and the CTA combines the MW states.
constexpr int kMergeMaxWarps = 8;

template <int D>
__global__ void __launch_bounds__(32 * kMergeMaxWarps) merge_kernel(const DecodeParams p) {
  constexpr int DPL = D / 32;
  __shared__ float2 s_ml[kMergeMaxWarps];
  __shared__ __align__(16) float s_acc[kMergeMaxWarps][D];
  grid_dependency_wait();
  const int RQ = p.q_per_seq * p.num_q_heads;
  const int row = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int MW = blockDim.x >> 5;
  const int b = row / RQ;
  const int rq = row % RQ;
  int nsh = 0, ns = p.num_parts;
  if (p.num_parts == 0) {
    const int ctx = __ldg(p.context_lens + b);
    const int nblk = num_blocks_of(p, ctx);
    const int sb = p.split_blocks;
    // records: the shared-prefix splits (region 0, with prefix sharing) then the
    // sequence's own splits (region 1 with prefix sharing, else region 0); with a sliding
    // window the own blocks start at the window's first block
    const int P_b = p.share_cap ? __ldcg(p.seq_info + b).x : window_first_block(p, ctx);
    nsh = (p.share_cap && P_b > 0) ? (P_b + p.share_split_blocks - 1) / p.share_split_blocks : 0;
    ns = nsh + (nblk - P_b + sb - 1) / sb;
    if (nsh == 0 && ns <= 1) return;  // written directly by the decode kernel (uniform per CTA)
  }
  const size_t own_region = p.share_cap ? static_cast<size_t>(p.num_seqs) * p.share_splits : 0;
  auto rec_of = [&](int k) -> size_t {
    if (p.num_parts > 0)  // gathered partial decodes: [part][sequence][row]
      return (static_cast<size_t>(k) * p.num_seqs + b) * RQ + rq;
    return (k < nsh ? static_cast<size_t>(b) * p.share_splits + k
                    : own_region + static_cast<size_t>(b) * p.num_splits + (k - nsh)) * RQ + rq;
  };
  // this warp's splits s = warp, warp + MW, ...: four at a time, their (m, l) and this lane's
  // slices of their o loaded together, folded in against the warp's running maximum
  float Mw = -INFINITY, Lw = 0.f, acc[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
  for (int s0 = warp; s0 < ns; s0 += 4 * MW) {
    float2 ml[4];
    float x[4][DPL];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int s = s0 + u * MW;
      ml[u] = make_float2(-INFINITY, 0.f);
#pragma unroll
      for (int e = 0; e < DPL; ++e) x[u][e] = 0.f;
      if (s < ns) {
        const size_t rec = rec_of(s);
        ml[u] = p.ws_ml[rec];
        const float* src = p.ws_o + rec * D + lane * DPL;
        if constexpr (DPL == 4) {
          const float4 v = *reinterpret_cast<const float4*>(src);
          x[u][0] = v.x; x[u][1] = v.y; x[u][2] = v.z; x[u][3] = v.w;
        } else {
          const float2 v = *reinterpret_cast<const float2*>(src);
          x[u][0] = v.x; x[u][1] = v.y;
        }
      }
    }
    float Mn = Mw;
#pragma unroll
    for (int u = 0; u < 4; ++u) Mn = fmaxf(Mn, ml[u].x);
    if (Mn == -INFINITY) continue;  // uniform over the warp: no key in these splits yet
    const float rs = Mw == -INFINITY ? 0.f : fast_exp2(Mw - Mn);  // what is folded in so far
    Lw *= rs;
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[e] *= rs;
    Mw = Mn;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float w = (ml[u].x == -INFINITY) ? 0.f : fast_exp2(ml[u].x - Mw);
      Lw += w * ml[u].y;
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[e] += w * x[u][e];
    }
  }
  if (lane == 0) s_ml[warp] = make_float2(Mw, Lw);
#pragma unroll
  for (int e = 0; e < DPL; ++e) s_acc[warp][lane * DPL + e] = acc[e];
  __syncthreads();
  float M = -INFINITY;
  for (int w = 0; w < MW; ++w) M = fmaxf(M, s_ml[w].x);
  float L = 0.f;
  for (int w = 0; w < MW; ++w) L += s_ml[w].x == -INFINITY ? 0.f : s_ml[w].y * fast_exp2(s_ml[w].x - M);
  if (p.num_parts > 0 && p.partial_only) {
    // combine into one record of the row (o against M, then {M, L}): [sequence][row] in ws_rec_*
    float* dst = p.rec_o + static_cast<size_t>(row) * D;
    for (int d = threadIdx.x; d < D; d += blockDim.x) {
      float v = 0.f;
      for (int w = 0; w < MW; ++w)
        v += s_ml[w].x == -INFINITY ? 0.f : fast_exp2(s_ml[w].x - M) * s_acc[w][d];
      dst[d] = v;
    }
    if (threadIdx.x == 0) p.rec_ml[row] = make_float2(M, L);
    return;
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  const int i = rq / p.num_q_heads;
  const int h = rq % p.num_q_heads;
  uint16_t* dst = p.out + out_offset(p, b, i, h, D);
  for (int d = threadIdx.x; d < D / 2; d += blockDim.x) {
    float v0 = 0.f, v1 = 0.f;
    for (int w = 0; w < MW; ++w) {
      const float wt = s_ml[w].x == -INFINITY ? 0.f : fast_exp2(s_ml[w].x - M);
      v0 += wt * s_acc[w][2 * d];
      v1 += wt * s_acc[w][2 * d + 1];
    }
    reinterpret_cast<uint32_t*>(dst)[d] = pack_bf16x2(v0 * inv, v1 * inv);
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

}  // namespace pa

#include "pa_tcgen05.cuh"
#include "pa_prefill.cuh"

namespace pa {

// ---------------------------------------------------------------------------
// Host-side launchers
// ---------------------------------------------------------------------------
namespace {

template <typename Kernel, typename... Args>
cudaError_t launch_pdl(Kernel kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args... args) {
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
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

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
  // ask for the largest shared-memory carveout, so that as many CTAs as the shared
  // memory allows are resident (the driver may otherwise pick a smaller one)
  if (e == cudaSuccess) e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e == cudaSuccess) done_mask |= bit;
  return e;
}

template <class Core, int D>
cudaError_t launch_core(const DecodeParams& p, int schedule, const CUtensorMap& tk,
                        const CUtensorMap& tv, cudaStream_t stream, int* occupancy) {
  constexpr int kStages = Core::kStages;
  constexpr int smem = DecodeSmem<typename Core::Geom, Core::ROWS, kWarpsPerCta, kStages>::kBytes;
  const dim3 block(kWarpsPerCta * 32);
  if (schedule == kSchedulePersistent) {
    auto kernel = decode_persistent_kernel<Core, D, kWarpsPerCta, kStages>;
    static unsigned long long done_mask = 0;  // one per template instance
    cudaError_t e = configure_smem(kernel, smem, done_mask);
    if (e != cudaSuccess) return e;
    if (occupancy) return cudaOccupancyMaxActiveBlocksPerMultiprocessor(occupancy, kernel, block.x, smem);
    e = launch_pdl(sched_prepass_kernel<D>, dim3(1), dim3(kPrepassThreads), 0, stream, p);
    if (e != cudaSuccess) return e;
    return launch_pdl(kernel, dim3(p.num_ctas), block, smem, stream, p, tk, tv);
  }
  auto kernel = decode_grid_kernel<Core, D, kWarpsPerCta, kStages>;
  static unsigned long long done_mask = 0;
  cudaError_t e = configure_smem(kernel, smem, done_mask);
  if (e != cudaSuccess) return e;
  if (occupancy) return cudaOccupancyMaxActiveBlocksPerMultiprocessor(occupancy, kernel, block.x, smem);
  if (p.share_cap) {
    e = launch_pdl(share_prepass_kernel, dim3(static_cast<unsigned>((p.num_seqs + 3) / 4)), dim3(128), 0,
                   stream, p);
    if (e != cudaSuccess) return e;
  }
  dim3 grid(p.num_kv_heads * p.row_chunks, p.num_seqs, p.num_splits);
  if (p.share_cap) {
    const long long ctas = static_cast<long long>(p.num_kv_heads) *
                           (static_cast<long long>(p.share_windows) * p.share_splits +
                            static_cast<long long>(p.num_seqs) * p.num_splits);
    grid = dim3(static_cast<unsigned>(ctas));
  }
  e = launch_pdl(kernel, grid, block, smem, stream, p, tk, tv);
  // a partial decode leaves its pieces to the merge of gathered pieces
  if (e != cudaSuccess || (p.num_splits <= 1 && !p.share_cap) || p.partial_only) return e;
  const long rows = static_cast<long>(p.num_seqs) * p.q_per_seq * p.num_q_heads;
  // about four records per warp, at most kMergeMaxWarps warps per row
  const int mw = max(1, min(kMergeMaxWarps, (p.num_splits + p.share_splits + 3) / 4));
  return launch_pdl(merge_kernel<D>, dim3(static_cast<unsigned>(rows)), dim3(32 * mw), 0, stream, p);
}

template <int D>
cudaError_t launch_merge_parts(const DecodeParams& p, cudaStream_t stream) {
  const long rows = static_cast<long>(p.num_seqs) * p.q_per_seq * p.num_q_heads;
  const int mw = max(1, min(kMergeMaxWarps, (p.num_parts + 3) / 4));
  return launch_pdl(merge_kernel<D>, dim3(static_cast<unsigned>(rows)), dim3(32 * mw), 0, stream, p);
}

template <int N>
cudaError_t launch_tcm(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& tq, cudaStream_t stream, int* occupancy) {
  constexpr int smem = tcm::Smem<N>::kBytes;
  // the sliding-window instance only for plans with a window
  auto kernel = p.window > 0 ? decode_tcm_kernel<N, true> : decode_tcm_kernel<N, false>;
  static unsigned long long done_mask[2] = {0, 0};  // one per instance
  cudaError_t e = configure_smem(kernel, smem, done_mask[p.window > 0 ? 1 : 0]);
  if (e != cudaSuccess) return e;
  if (occupancy) return cudaOccupancyMaxActiveBlocksPerMultiprocessor(occupancy, kernel, tcm::kThreads, smem);
  if (p.share_cap > 1) {
    const int windows = (p.num_seqs + p.share_cap - 1) / p.share_cap;
    e = launch_pdl(tcm_share_prepass, dim3(static_cast<unsigned>(windows)), dim3(256), 0, stream, p);
    if (e != cudaSuccess) return e;
  }
  e = launch_pdl(kernel, dim3(p.num_ctas), dim3(tcm::kThreads), smem, stream, p, tk, tv, tq);
  if (e != cudaSuccess) return e;
  return launch_pdl(tcm_merge_kernel<N>, dim3(p.num_ctas), dim3(tcm::kMergeThreads), 0, stream, p);
}

template <int D>
cudaError_t dispatch(int path, int schedule, int rows_per_cta, int kv_dtype, const DecodeParams& p,
                     const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq, cudaStream_t stream,
                     int* occ) {
  if (kv_dtype == kKvE4M3) {  // E4M3 pools: the tensor-core tiles widen the codes to f16
    if (path != kPathTile) return cudaErrorInvalidValue;
    switch (rows_per_cta) {
      case 8: return launch_core<TileCore<D, 1, true>, D>(p, schedule, tk, tv, stream, occ);
      case 16: return launch_core<TileCore<D, 2, true>, D>(p, schedule, tk, tv, stream, occ);
      case 24: return launch_core<TileCore<D, 3, true>, D>(p, schedule, tk, tv, stream, occ);
      case 32: return launch_core<TileCore<D, 4, true>, D>(p, schedule, tk, tv, stream, occ);
      default: return cudaErrorInvalidValue;
    }
  }
  if (kv_dtype != kKvBf16) return cudaErrorInvalidValue;
  if (path == kPathTcgen05) {
    if constexpr (D != tcm::kD) {
      return cudaErrorInvalidValue;
    } else {
      if (schedule != kSchedulePersistent) return cudaErrorInvalidValue;
      if (rows_per_cta == 16) return launch_tcm<16>(p, tk, tv, tq, stream, occ);
      if (rows_per_cta == 32) return launch_tcm<32>(p, tk, tv, tq, stream, occ);
      return cudaErrorInvalidValue;
    }
  }
  if (path == kPathTile) {
    switch (rows_per_cta) {
      case 8: return launch_core<TileCore<D, 1>, D>(p, schedule, tk, tv, stream, occ);
      case 16: return launch_core<TileCore<D, 2>, D>(p, schedule, tk, tv, stream, occ);
      case 24: return launch_core<TileCore<D, 3>, D>(p, schedule, tk, tv, stream, occ);
      case 32: return launch_core<TileCore<D, 4>, D>(p, schedule, tk, tv, stream, occ);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (rows_per_cta) {
    case 1: return launch_core<SimtCore<D, 1>, D>(p, schedule, tk, tv, stream, occ);
    case 2: return launch_core<SimtCore<D, 2>, D>(p, schedule, tk, tv, stream, occ);
    case 4: return launch_core<SimtCore<D, 4>, D>(p, schedule, tk, tv, stream, occ);
    case 8: return launch_core<SimtCore<D, 8>, D>(p, schedule, tk, tv, stream, occ);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_prefill(const PrefillParams& p, int max_tiles, const CUtensorMap& tk, const CUtensorMap& tv,
                           cudaStream_t stream) {
  static unsigned long long done_mask = 0;
  cudaError_t e = configure_smem(prefill_tcm_kernel, pfl::Smem::kBytes, done_mask);
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>(p.num_kv_heads), static_cast<unsigned>(p.num_seqs),
                  static_cast<unsigned>(max_tiles));
  return launch_pdl(prefill_tcm_kernel, grid, dim3(pfl::kThreads), pfl::Smem::kBytes, stream, p, tk, tv);
}

cudaError_t launch_decode(const DecodeParams& p, int path, int schedule, int head_dim, int kv_dtype,
                          const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq,
                          cudaStream_t stream) {
  return head_dim == 128 ? dispatch<128>(path, schedule, p.rows_per_cta, kv_dtype, p, tk, tv, tq, stream, nullptr)
                         : dispatch<64>(path, schedule, p.rows_per_cta, kv_dtype, p, tk, tv, tq, stream, nullptr);
}

cudaError_t launch_merge_partials(const DecodeParams& p, int head_dim, cudaStream_t stream) {
  return head_dim == 128 ? launch_merge_parts<128>(p, stream) : launch_merge_parts<64>(p, stream);
}

int decode_ctas_per_sm(int path, int schedule, int head_dim, int rows_per_cta, int kv_dtype) {
  // the occupancy query costs microseconds of host time: remember it per device and kernel
  struct Entry {
    int dev, path, schedule, head_dim, rows, kv_dtype, occ;
  };
  static std::mutex mu;
  static Entry cache[64];
  static int used = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
  {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i)
      if (cache[i].dev == dev && cache[i].path == path && cache[i].schedule == schedule &&
          cache[i].head_dim == head_dim && cache[i].rows == rows_per_cta && cache[i].kv_dtype == kv_dtype)
        return cache[i].occ;
  }
  DecodeParams dummy = {};
  CUtensorMap tm = {};
  int occ = 0;
  cudaError_t e =
      head_dim == 128 ? dispatch<128>(path, schedule, rows_per_cta, kv_dtype, dummy, tm, tm, tm, nullptr, &occ)
                      : dispatch<64>(path, schedule, rows_per_cta, kv_dtype, dummy, tm, tm, tm, nullptr, &occ);
  const int result = e == cudaSuccess && occ > 0 ? occ : 1;
  if (e == cudaSuccess && occ > 0 && dev >= 0) {
    std::lock_guard<std::mutex> lock(mu);
    if (used < 64) cache[used++] = Entry{dev, path, schedule, head_dim, rows_per_cta, kv_dtype, occ};
  }
  return result;
}

cudaError_t launch_cache_write(const uint16_t* key, const uint16_t* value, int64_t key_stride,
                               int64_t value_stride, uint16_t* key_cache, uint16_t* value_cache,
                               const int64_t* slots, int64_t num_tokens, int32_t row_elems,
                               int64_t num_slots, cudaStream_t stream) {
  const int64_t threads = 2 * num_tokens * 32;
  return launch_pdl(cache_write_kernel, dim3(static_cast<unsigned>((threads + 255) / 256)), dim3(256), 0,
                    stream, key, value, key_stride, value_stride, key_cache, value_cache, slots,
                    num_tokens, row_elems, num_slots);
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

// Self-test of the failure path: one thread waits on an mbarrier that nothing
// completes; the bounded wait gives up after its limit and the kernel records
// kErrSelftest and returns.
__global__ void selftest_wait_kernel() {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_barrier_init();
  if (!mbar_wait_bounded(&bar, 0)) record_error(kErrSelftest);
}

cudaError_t run_selftest_wait(cudaStream_t stream) {
  selftest_wait_kernel<<<1, 32, 0, stream>>>();
  return cudaGetLastError();
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
