// Paged decode on the 5th-generation tensor cores (tcgen05, accumulators in TMEM).
// Included by pa_kernels.cu (shares its helpers and device error word).
//
// One CTA per (kv head x row chunk, sequence, context split) of up to 32 query rows,
// three warps with fixed roles:
//   warp 1  TMA producer: tiles of 4 blocks (64 tokens) of K and of V, 3 stages;
//   warp 2  MMA issuer (one thread) and TMEM owner:
//             S_t = Q . K_t^T     M=128 (query rows, 32 used), N=64 tokens, K=head_dim
//             O  += P_t . V_t     M=128, N=head_dim, K=64 tokens (V is an MN-major operand
//                                 read straight from the TMA tile)
//           completions are signalled with tcgen05.commit on mbarriers;
//   warp 0  softmax, one thread per query row = TMEM lane: reads its row of S_t,
//           masks, keeps a reference maximum, writes P_t (bf16) to shared memory in the
//           128-byte-swizzled K-major layout, and rescales its row of O in TMEM only
//           when the row maximum grows by more than 2^8 over the reference (the result
//           is exact either way: numerator and denominator share the reference).
// TMEM: S double buffer in columns [0,64) and [64,128), O in [128, 128+head_dim).
// Shared memory: Q (32 rows), one P buffer, 3 stages of K and of V: 108 KB at head_dim
// 128, so two CTAs share an SM.
// Rows 32..127 of the A operands (Q, P) alias neighbouring shared memory: their
// products land in TMEM lanes 32..127, which nobody reads.

namespace pa {
namespace tc5 {

constexpr int kTileBlocks = 4;
constexpr int kTileTokens = kTileBlocks * kBlockSize;  // 64
constexpr int kStages = 3;
constexpr int kRows = 32;          // query rows per CTA: the softmax warp's 32 TMEM lanes
constexpr int kThreads = 96;
constexpr uint32_t kTmemCols = 256;
constexpr float kRescaleLog2 = 8.f;

template <int D>
struct Smem {
  static constexpr int kHalves = D / 64;
  static constexpr int kQ = kHalves * 4096;              // rows 0..31 of each 64-column half
  static constexpr int kP = 4096;                        // rows 0..31 x 64 tokens
  static constexpr int kKV = kTileBlocks * kHalves * kHalfTileBytes;  // one K or V stage
  static constexpr int offQ = 0;
  static constexpr int offP = kQ;
  static constexpr int offK = offP + kP;
  static constexpr int offV = offK + kStages * kKV;
  static constexpr int kUsed = offV + kStages * kKV;
  static constexpr int offBars = kUsed;                  // barriers, TMEM address, flags
  // no static shared memory: the dynamic buffer starts at the (1024-aligned) base of the
  // CTA's window, so two 113 KB CTAs fit an SM; at least 77 KB so that no more than two
  // CTAs (2 x 256 TMEM columns) share an SM and a TMEM allocation never waits
  static constexpr int kBytes = (kUsed + 256) > 77 * 1024 ? (kUsed + 256) : 77 * 1024;
  // descriptors of Q and P span 128 rows = 16 KB from their start: stay inside
  static_assert(offQ + (kHalves - 1) * 4096 + 16384 <= kUsed, "Q rows 32..127 must alias allocated smem");
  static_assert(offP + kP + 16384 <= kUsed, "P rows 32..127 must alias allocated smem");
};

struct Bars {
  uint64_t k_full[kStages], v_full[kStages], kv_empty[kStages];
  uint64_t s_full[2], s_free[2], p_full, p_free;
  uint64_t q_full, o_final, drain;
};

}  // namespace tc5

template <int D>
__global__ void __launch_bounds__(tc5::kThreads)
decode_tc5_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmap_k,
                  const __grid_constant__ CUtensorMap tmap_v) {
  using L = tc5::Smem<D>;
  constexpr int HALVES = D / 64;
  constexpr int KSTEPS = D / 16;
  constexpr int DC = D / 32;
  extern __shared__ __align__(1024) uint8_t smem[];
  static_assert(sizeof(tc5::Bars) + 8 <= 256, "barrier area");
  tc5::Bars& bars = *reinterpret_cast<tc5::Bars*>(smem + L::offBars);
  uint32_t& tmem_base_s = *reinterpret_cast<uint32_t*>(smem + L::offBars + sizeof(tc5::Bars));
  int& abort_s = *reinterpret_cast<int*>(smem + L::offBars + sizeof(tc5::Bars) + 4);
  if (smem_u32(smem) & 1023u) {  // the swizzled operand layouts need a 1024-aligned base
    if (threadIdx.x == 0) record_error(kErrSchedule);
    return;
  }
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int kvh = blockIdx.x / p.row_chunks;
  const int rc = blockIdx.x % p.row_chunks;
  const int b = blockIdx.y;
  const int split = blockIdx.z;

  if (threadIdx.x == 0) {
    uint64_t* all = reinterpret_cast<uint64_t*>(&bars);
    for (int i = 0; i < static_cast<int>(sizeof(tc5::Bars) / 8); ++i) mbar_init(all + i, 1);
    fence_barrier_init();
    tma_prefetch_desc(&tmap_k);
    tma_prefetch_desc(&tmap_v);
    abort_s = 0;
  }
  __syncthreads();
  grid_dependency_wait();

  const int ctx = __ldg(p.context_lens + b);
  const int nblk = num_blocks_of(p, ctx);
  const int blk0 = split * p.split_blocks;
  const Seg sg{b, 1, kvh, rc * tc5::kRows, min(tc5::kRows, p.rows - rc * tc5::kRows), blk0,
               min(nblk, blk0 + p.split_blocks), false};
  if (blk0 >= nblk) {  // uniform: nothing to read
    if (split == 0 && warp == 0) {
      int bb, i, h;
      if (seg_row(p, sg, lane, bb, i, h)) {
        uint4* dst = reinterpret_cast<uint4*>(p.out + out_offset(p, bb, i, h, D));
        for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
      }
    }
    grid_launch_dependents();
    return;
  }
  const int blk1 = sg.blk1;
  const int ntiles = (blk1 - blk0 + tc5::kTileBlocks - 1) / tc5::kTileBlocks;
  const bool single_split = (nblk + p.split_blocks - 1) / p.split_blocks == 1;

  if (warp == 2) {
    tmem_alloc(&tmem_base_s, tc5::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = tmem_base_s;
  const uint32_t sm = smem_u32(smem);
  const uint32_t q_s = sm + L::offQ;
  const uint32_t p_s = sm + L::offP;
  const uint32_t k_s = sm + L::offK;
  const uint32_t v_s = sm + L::offV;

  if (warp == 1) {
    // ------------------------------------------------------------ TMA producer
    const int32_t* trow = p.block_tables + static_cast<size_t>(b) * p.max_blocks;
    const int oob = static_cast<int>(p.num_blocks);  // block id past the pool: TMA fills zeros
    int t = 0;
    for (; t < ntiles; ++t) {
      const int s = t % tc5::kStages;
      if (t >= tc5::kStages) {
        const bool ok = mbar_wait_bounded(&bars.kv_empty[s], ((t / tc5::kStages) - 1) & 1);
        if (!__all_sync(kFull, ok)) {
          if (lane == 0) record_error(kErrTimeoutDecode);
          abort_s = 1;
          break;
        }
      }
      // lanes 0..3 read the tile's 4 block ids; blocks past the split use an id past the
      // pool, which the TMA fills with zeros
      const int blk = blk0 + t * tc5::kTileBlocks + lane;
      const int phys_l = (lane < tc5::kTileBlocks && blk < blk1) ? __ldg(trow + blk) : oob;
      int ph[tc5::kTileBlocks];
#pragma unroll
      for (int jj = 0; jj < tc5::kTileBlocks; ++jj) ph[jj] = __shfl_sync(kFull, phys_l, jj);
      if (lane == 0) {
        uint8_t* kdst = smem + L::offK + s * L::kKV;
        uint8_t* vdst = smem + L::offV + s * L::kKV;
        mbar_arrive_expect_tx(&bars.k_full[s], L::kKV);
        mbar_arrive_expect_tx(&bars.v_full[s], L::kKV);
#pragma unroll
        for (int jj = 0; jj < tc5::kTileBlocks; ++jj)
#pragma unroll
          for (int hf = 0; hf < HALVES; ++hf) {
            const int off = hf * (tc5::kTileBlocks * kHalfTileBytes) + jj * kHalfTileBytes;
            tma_load_3d(kdst + off, &tmap_k, &bars.k_full[s], hf * 64, kvh, ph[jj] * kBlockSize);
            tma_load_3d(vdst + off, &tmap_v, &bars.v_full[s], hf * 64, kvh, ph[jj] * kBlockSize);
          }
      }
      __syncwarp();
    }
    if (abort_s) {  // wait (bounded) for the loads still in flight before leaving
      for (int u = max(0, t - tc5::kStages); u < t; ++u) {
        const int s = u % tc5::kStages;
        if (!mbar_wait_bounded(&bars.k_full[s], (u / tc5::kStages) & 1) ||
            !mbar_wait_bounded(&bars.v_full[s], (u / tc5::kStages) & 1))
          record_error(kErrTimeoutDrain);
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, tc5::kTileTokens, 0, 0);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, 0, 1);
      bool ok = mbar_wait_bounded(&bars.q_full, 0);
      for (int t = 0; ok && t <= ntiles; ++t) {
        if (t < ntiles) {
          const int s = t % tc5::kStages;
          ok = mbar_wait_bounded(&bars.k_full[s], (t / tc5::kStages) & 1);
          if (ok && t >= 2) ok = mbar_wait_bounded(&bars.s_free[t & 1], ((t >> 1) - 1) & 1);
          if (!ok) break;
          tc_fence_after_sync();
          const uint32_t kst = k_s + s * L::kKV;
#pragma unroll
          for (int k = 0; k < KSTEPS; ++k) {
            const uint64_t ad = smem_desc_sw128(q_s + (k >> 2) * 4096 + (k & 3) * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(kst + (k >> 2) * (tc5::kTileBlocks * kHalfTileBytes) +
                                                    (k & 3) * 32, 16, 1024);
            tc_mma_bf16(tmem + (t & 1) * tc5::kTileTokens, ad, bd, idesc_s, k > 0 ? 1u : 0u);
          }
          tc_commit(&bars.s_full[t & 1]);
        }
        if (t >= 1) {
          const int u = t - 1;
          const int su = u % tc5::kStages;
          ok = mbar_wait_bounded(&bars.p_full, u & 1);
          if (ok) ok = mbar_wait_bounded(&bars.v_full[su], (u / tc5::kStages) & 1);
          if (!ok) break;
          tc_fence_after_sync();
          const uint32_t vst = v_s + su * L::kKV;
#pragma unroll
          for (int kk = 0; kk < tc5::kTileTokens / 16; ++kk) {
            const uint64_t ad = smem_desc_sw128(p_s + kk * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(vst + kk * 2048, tc5::kTileBlocks * kHalfTileBytes, 1024);
            tc_mma_bf16(tmem + 128, ad, bd, idesc_o, (u > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(&bars.p_free);
          tc_commit(&bars.kv_empty[su]);
        }
      }
      if (!ok) {
        record_error(kErrTimeoutDecode);
        abort_s = 1;
      }
      tc_commit(&bars.o_final);
      // every MMA issued so far has completed once o_final flips
      if (!mbar_wait_bounded(&bars.o_final, 0)) record_error(kErrTimeoutDrain);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax (warp 0)
    const int r = lane;
    int bb = 0, qi = 0, qh = 0;
    const bool valid = seg_row(p, sg, r, bb, qi, qh);
    {  // Q row r -> shared memory (128-byte swizzle, K-major), zeros for padded rows
      const uint4* qsrc = reinterpret_cast<const uint4*>(p.query + out_offset(p, bb, qi, qh, D));
#pragma unroll
      for (int hf = 0; hf < HALVES; ++hf)
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 v = valid ? __ldg(qsrc + hf * 8 + c) : make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4*>(smem + L::offQ + hf * 4096 + r * 128 + ((c ^ (r & 7)) << 4)) = v;
        }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.q_full);
    }
    const int lim = valid ? ctx - p.q_per_seq + qi : ctx - 1;
    const int end_tok = min(ctx, blk1 * kBlockSize);
    // The sequence's last block, when partly filled, is in this split's tile zero_tile:
    // its slots past the context may hold any bits (NaN too), and although their p is 0,
    // 0 * NaN is NaN, so those V rows are cleared in shared memory before the PV reads them.
    const int zero_tile = (blk1 == nblk && (ctx & (kBlockSize - 1))) ? (nblk - 1 - blk0) / tc5::kTileBlocks : -1;
    const float c = p.scale_log2;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int t = 0; t < ntiles && ok; ++t) {
      ok = __all_sync(kFull, mbar_wait_bounded(&bars.s_full[t & 1], (t >> 1) & 1));
      if (!ok) break;
      tc_fence_after_sync();
      uint32_t sv[tc5::kTileTokens];
      tmem_ld32(tmem + (t & 1) * tc5::kTileTokens, *reinterpret_cast<uint32_t(*)[32]>(sv));
      tmem_ld32(tmem + (t & 1) * tc5::kTileTokens + 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32));
      tc_wait_ld();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.s_free[t & 1]);

      const int tok0 = (blk0 + t * tc5::kTileBlocks) * kBlockSize;
      const bool edge = tok0 + tc5::kTileTokens > min(end_tok, ctx - p.q_per_seq + 1);
      float x[tc5::kTileTokens];
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};  // 4 independent chains
#pragma unroll
      for (int j = 0; j < tc5::kTileTokens; ++j) {
        float v = __uint_as_float(sv[j]) * c;
        if (edge && (tok0 + j >= end_tok || tok0 + j > lim)) v = -INFINITY;
        x[j] = v;
        mx4[j & 3] = fmaxf(mx4[j & 3], v);
      }
      const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
      const bool need = mx > m_ref + tc5::kRescaleLog2 || (m_ref == -INFINITY && mx != -INFINITY);
      if (__any_sync(kFull, need)) {
        const float new_ref = need ? mx : m_ref;
        const float alpha = (m_ref == -INFINITY) ? 0.f : fast_exp2(m_ref - new_ref);
        l *= alpha;
        if (t > 0) {  // O holds tiles 0..t-1 once the PV of tile t-1 has completed
          ok = __all_sync(kFull, mbar_wait_bounded(&bars.p_free, (t - 1) & 1));
          if (!ok) break;
          tc_fence_after_sync();
#pragma unroll
          for (int ch = 0; ch < DC; ++ch) {
            uint32_t o[32];
            tmem_ld32(tmem + 128 + ch * 32, o);
            tc_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(tmem + 128 + ch * 32, o);
          }
          tc_wait_st();
        }
        m_ref = new_ref;
      }
      if (t >= 1) {  // the PV of tile t-1 reads the P buffer: wait until it has completed
        ok = __all_sync(kFull, mbar_wait_bounded(&bars.p_free, (t - 1) & 1));
        if (!ok) break;
      }
      if (t == zero_tile) {
        const int su = t % tc5::kStages;
        ok = __all_sync(kFull, mbar_wait_bounded(&bars.v_full[su], (t / tc5::kStages) & 1));
        if (!ok) break;
        const int jj = (nblk - 1 - blk0) % tc5::kTileBlocks;
        const int r0 = ctx & (kBlockSize - 1);  // first unwritten row of the block
        const int nrow = kBlockSize - r0;
        uint8_t* vblk = smem + L::offV + su * L::kKV + jj * kHalfTileBytes;
        for (int idx = lane; idx < HALVES * nrow * 8; idx += 32) {
          const int hf = idx / (nrow * 8);
          const int rem = idx - hf * (nrow * 8);
          *reinterpret_cast<uint4*>(vblk + hf * (tc5::kTileBlocks * kHalfTileBytes) +
                                    (r0 + (rem >> 3)) * 128 + (rem & 7) * 16) = make_uint4(0, 0, 0, 0);
        }
      }
      const float mref_use = (m_ref == -INFINITY) ? 0.f : m_ref;
      float ps4[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t pk[tc5::kTileTokens / 2];
#pragma unroll
      for (int j = 0; j < tc5::kTileTokens; j += 2) {
        const float p0 = fast_exp2(x[j] - mref_use);
        const float p1 = fast_exp2(x[j + 1] - mref_use);
        ps4[(j >> 1) & 3] += p0 + p1;
        pk[j / 2] = pack_bf16x2(p0, p1);
      }
      l += (ps4[0] + ps4[1]) + (ps4[2] + ps4[3]);
      uint8_t* prow = smem + L::offP + r * 128;
#pragma unroll
      for (int ch = 0; ch < 8; ++ch)
        *reinterpret_cast<uint4*>(prow + ((ch ^ (r & 7)) << 4)) =
            make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
      fence_proxy_async_smem();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.p_full);
    }
    if (!ok) {
      if (lane == 0) record_error(kErrTimeoutDecode);
      abort_s = 1;
    }
    // epilogue: wait for the last PV, then O row r -> output or partial record
    const bool done = __all_sync(kFull, mbar_wait_bounded(&bars.o_final, 0));
    tc_fence_after_sync();
    if (!done) record_error(kErrTimeoutDecode);
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const int rq = qi * p.num_q_heads + qh;
    const size_t rec = (static_cast<size_t>(b) * p.num_splits + split) * (p.q_per_seq * p.num_q_heads) + rq;
#pragma unroll
    for (int ch = 0; ch < DC; ++ch) {
      uint32_t o[32];
      tmem_ld32(tmem + 128 + ch * 32, o);
      tc_wait_ld();
      if (!valid || !done) continue;
      if (single_split) {
        uint4* dst = reinterpret_cast<uint4*>(p.out + out_offset(p, bb, qi, qh, D) + ch * 32);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          float a[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) a[e] = __uint_as_float(o[q4 * 8 + e]);
          store_bf16x8(reinterpret_cast<uint16_t*>(dst + q4), a, inv);
        }
      } else {
        float4* dst = reinterpret_cast<float4*>(p.ws_o + rec * D + ch * 32);
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4)
          dst[q4] = make_float4(__uint_as_float(o[4 * q4]), __uint_as_float(o[4 * q4 + 1]),
                                __uint_as_float(o[4 * q4 + 2]), __uint_as_float(o[4 * q4 + 3]));
      }
    }
    if (valid && done && !single_split) p.ws_ml[rec] = make_float2(m_ref, l);
  }
  grid_launch_dependents();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 2) tmem_dealloc(tmem, tc5::kTmemCols);
}

}  // namespace pa
