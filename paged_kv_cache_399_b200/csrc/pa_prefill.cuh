// Chunked-prefill paged attention on the 5th-generation tensor cores (vLLM study notes,
// zihan-zhang.net, §3.5 "Chunked prefill": a long prompt is attended in chunks of many
// query tokens, batched with decode steps; "vLLM 深度解析" §5.4 Chunked Prefill). A chunk's
// K/V are already in the paged pool (written by pa_reshape_and_cache); its query token i
// sits at position ctx - qlen + i and sees keys 0 .. that position, i.e. the sequence's
// earlier context plus the chunk up to itself (causal). Included by pa_kernels.cu (shares
// its device helpers and error word).
//
// This is a contraction with hundreds of query rows per kv head, so the query rows go on the
// MMA's M dimension (the decode kernels put the keys there):
//   S[128 rows][64 keys] = Q[128 rows][D] . K^T[D][64 keys]      K-major A (Q) and B (K)
//   softmax per row over the tile's 64 keys: thread r owns row r (TMEM lane r) and the
//   whole tile row, so no thread waits for another's maximum; the running reference
//   maximum moves only when a tile's maximum exceeds it by more than 2^8 (numerator and
//   denominator share the reference, so the result is exact either way);
//   O[128 rows][D] += P[128 rows][64 keys] . V[64 keys][D]       A = P from TMEM (written
//                                                                over the tile's scores),
//                                                                MN-major B (V)
// Two CTAs share an SM (96 KB of shared memory and 256 TMEM columns each), so the softmax
// of one runs while the other's MMAs do, and each SM sub-partition holds a softmax warp of
// both.
// A CTA owns 128 rows = 128 / G consecutive chunk tokens x the G query heads of one kv head
// (GQA: every row of a CTA reads the same K/V), and walks the key tiles of 4 blocks from
// the sequence's first block to the block of its last row's position.
//
// Roles: warps 0-3 load Q, run the softmax and the epilogue; warp 4 issues the K boxes and
// warp 5 the V boxes (8 TMA boxes of 2 KB per tile each); warp 6 holds the TMEM allocation
// and one of its threads issues the MMAs (S of a tile as soon as its K has landed and an S
// buffer is free, i.e. the PV of the tile two before has read its P; PV of a tile as soon as
// its P is in TMEM and its V in shared memory). A K stage is released when its S completes,
// a V stage when its PV completes.
// TMEM: S double buffer in columns [0, 128) (a tile's P, bf16 pairs, over the first 32
// columns of its S), O in [128, 256).
// Shared memory: Q (32 KB), 2 K stages and 2 V stages of 16 KB, barriers.

namespace pa {

namespace pfl {

// Three-input maximum and paired f32 arithmetic (sm_100): half the instructions of the
// softmax's maximum, scaling and row sums.
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
// (a.x * b + c, a.y * b + c) and (a.x + b.x, a.y + b.y) as single paired instructions
__device__ __forceinline__ float2 fma2(float2 a, float b, float c) {
  unsigned long long r;
  const float2 bb = make_float2(b, b), cc = make_float2(c, c);
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r)
      : "l"(*reinterpret_cast<const unsigned long long*>(&a)), "l"(*reinterpret_cast<const unsigned long long*>(&bb)),
        "l"(*reinterpret_cast<const unsigned long long*>(&cc)));
  return *reinterpret_cast<float2*>(&r);
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  unsigned long long r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r)
      : "l"(*reinterpret_cast<const unsigned long long*>(&a)), "l"(*reinterpret_cast<const unsigned long long*>(&b)));
  return *reinterpret_cast<float2*>(&r);
}

constexpr int kD = 128;
constexpr int kRows = 128;                        // query rows of a CTA: the MMA's M
constexpr int kTileBlocks = 4;
constexpr int kKeys = kTileBlocks * kBlockSize;   // 64 keys per tile
constexpr int kStages = 2;
constexpr int kThreads = 224;                     // 7 warps
constexpr int kCtasPerSm = 2;
constexpr int kSoftmaxWarps = 4;                  // one warpgroup: thread r owns row r
constexpr int kKWarp = 4, kVWarp = 5, kMmaWarp = 6;
constexpr int kHalfBytes = kKeys * 128;           // one 64-column half of a K or V tile: 8 KB
constexpr int kTileBytes = 2 * kHalfBytes;        // 16 KB
constexpr int kRowsHalfBytes = kRows * 128;       // one 64-column half of Q, or P: 16 KB
constexpr float kRescaleLog2 = 8.f;
constexpr uint32_t kTmemCols = 256;               // S double buffer + O (a power of 2)
constexpr uint32_t kTmemO = 2 * kKeys;            // column of O

struct Smem {
  static constexpr int offQ = 0;
  static constexpr int offK = offQ + 2 * kRowsHalfBytes;
  static constexpr int offV = offK + kStages * kTileBytes;
  static constexpr int offBars = offV + kStages * kTileBytes;
  static constexpr int kBytes = offBars + 256;
  static_assert(offK % 1024 == 0 && offV % 1024 == 0, "swizzled operands");
  // two CTAs per SM: 228 KB of shared memory less 1 KB reserved per CTA
  static_assert(kCtasPerSm * (kBytes + 1024) <= 228 * 1024, "shared memory of two CTAs");
};

struct Bars {
  uint64_t k_full[kStages], k_empty[kStages], v_full[kStages], v_empty[kStages];
  uint64_t s_full[2], p_full[2], pv_done[2], q_full, drain;
};

// Byte offset of 16-byte chunk c (0..15) of row r in a 128-row operand of two 64-column
// halves, 128-byte swizzled (the layout TMA writes for K/V and the one Q and P use).
__device__ __forceinline__ uint32_t row_chunk_offset(int r, int c) {
  return static_cast<uint32_t>((c >> 3) * kRowsHalfBytes + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}


}  // namespace pfl

__global__ void __launch_bounds__(pfl::kThreads, pfl::kCtasPerSm)
prefill_tcm_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap tmap_k,
                   const __grid_constant__ CUtensorMap tmap_v) {
  using L = pfl::Smem;
  using pfl::kKeys;
  using pfl::kStages;
  using pfl::kTileBlocks;
  constexpr int D = pfl::kD;
  extern __shared__ __align__(1024) uint8_t smem[];
  pfl::Bars& bars = *reinterpret_cast<pfl::Bars*>(smem + L::offBars);
  uint32_t& tmem_base_s = *reinterpret_cast<uint32_t*>(smem + L::offBars + sizeof(pfl::Bars));
  static_assert(sizeof(pfl::Bars) + 16 <= 256, "barrier area");
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (smem_u32(smem) & 1023u) {  // the swizzled operand layouts need a 1024-aligned base
    if (threadIdx.x == 0) record_error(kErrSchedule);
    return;
  }
  // grid: x = kv head, y = sequence, z = tile counted from the chunk's end (the tiles that
  // see the most keys start first)
  const int kvh = blockIdx.x;
  const int b = blockIdx.y;
  if (threadIdx.x == 0) {
    uint64_t* all = reinterpret_cast<uint64_t*>(&bars);
    for (int i = 0; i < static_cast<int>(sizeof(pfl::Bars) / 8); ++i) mbar_init(all + i, 1);
    for (int i = 0; i < 2; ++i) mbar_init(&bars.p_full[i], pfl::kSoftmaxWarps);  // one arrival per softmax warp
    mbar_init(&bars.q_full, pfl::kSoftmaxWarps);
    fence_barrier_init();
    tma_prefetch_desc(&tmap_k);
    tma_prefetch_desc(&tmap_v);
  }
  grid_dependency_wait();
  const int qs = __ldg(p.query_start + b);
  const int qlen = __ldg(p.query_start + b + 1) - qs;
  const int ctx = __ldg(p.context_lens + b);
  const int TT = p.tile_tokens;
  const int ntiles = qlen > 0 ? (qlen + TT - 1) / TT : 0;
  const int rt = static_cast<int>(blockIdx.z);
  // nothing to do: past the chunk's tiles, or a context shorter than the chunk (a
  // precondition violation; no position would be valid)
  if (rt >= ntiles || ctx < qlen) {
    grid_launch_dependents();
    return;
  }
  const int tile = ntiles - 1 - rt;
  const int tok0 = tile * TT;
  const int ntok = min(TT, qlen - tok0);
  const int pos0 = ctx - qlen + tok0;          // position of the CTA's first token
  const int kmax = pos0 + ntok - 1;            // position of its last token: the last key seen
  const int nk = kmax / kKeys + 1;             // key tiles 0 .. nk-1
  const int nblk = min((ctx + kBlockSize - 1) / kBlockSize, p.max_blocks);

  if (warp == pfl::kMmaWarp) {
    tmem_alloc(&tmem_base_s, pfl::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = tmem_base_s;
  const uint32_t sm = smem_u32(smem);

  if (warp == pfl::kKWarp || warp == pfl::kVWarp) {
    // ------------------------------------------------------------ TMA producers
    // lanes 0..7 issue the tile's 8 boxes (half = lane / 4, block = lane % 4); lanes 0..3
    // read the next tile's block ids while this one is issued
    const bool is_k = warp == pfl::kKWarp;
    const CUtensorMap* tmap = is_k ? &tmap_k : &tmap_v;
    uint64_t* full = is_k ? bars.k_full : bars.v_full;
    uint64_t* empty = is_k ? bars.k_empty : bars.v_empty;
    const int stage_off = is_k ? L::offK : L::offV;
    const int32_t* trow = p.block_tables + static_cast<size_t>(b) * p.max_blocks;
    const int oob = static_cast<int>(p.num_blocks);  // block id past the pool: TMA fills zeros
    auto block_id = [&](int j) {
      const int blk = j * kTileBlocks + lane;
      return (lane < kTileBlocks && blk < nblk) ? __ldg(trow + blk) : oob;
    };
    int phys_next = block_id(0);
    bool ok = true;
    int j = 0;
    for (; j < nk; ++j) {
      const int s = j % kStages;
      const int ph = __shfl_sync(kFull, phys_next, lane & (kTileBlocks - 1));
      if (j + 1 < nk) phys_next = block_id(j + 1);
      if (j >= kStages) ok = __all_sync(kFull, mbar_wait_bounded(&empty[s], ((j / kStages) - 1) & 1));
      if (!ok) break;
      if (lane == 0) mbar_arrive_expect_tx(&full[s], pfl::kTileBytes);
      __syncwarp();
      const int hf = lane / kTileBlocks, jj = lane & (kTileBlocks - 1);
      if (lane < 2 * kTileBlocks)
        tma_load_3d(smem + stage_off + s * pfl::kTileBytes + hf * pfl::kHalfBytes + jj * kHalfTileBytes, tmap,
                    &full[s], hf * 64, kvh, ph * kBlockSize);
      __syncwarp();
    }
    if (!ok) {
      if (lane == 0) record_error(kErrTimeoutDecode);
      for (int u = max(0, j - kStages); u < j; ++u)
        if (!mbar_wait_bounded(&full[u % kStages], (u / kStages) & 1) && lane == 0) record_error(kErrTimeoutDrain);
    }
  } else if (warp == pfl::kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc_s = idesc_bf16_f32(128, kKeys, 0, 0);  // Q K-major, K K-major
    constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, 0, 1);      // P K-major, V MN-major
    int gs = 0, gp = 0;  // next tile to issue S for / PV for
    bool ok = true;
    unsigned long long idle_since = 0;
    unsigned idle_polls = 0;
    // slots of the sequence's partly filled last block past the context: V rows to clear
    // before the PV of the tile holding that block (their p is 0, but 0 * NaN is NaN)
    const int last_blk = nblk - 1;
    const int last_fill = ctx - last_blk * kBlockSize;  // 1..16 tokens used in the last block
    while (gp < nk) {
      bool progressed = false;
      bool pv_ready = false;
      if (lane == 0)
        pv_ready = gp < gs && mbar_test_wait(&bars.p_full[gp & 1], (gp >> 1) & 1) &&
                   mbar_test_wait(&bars.v_full[gp % kStages], (gp / kStages) & 1);
      if (__shfl_sync(kFull, pv_ready, 0)) {
        const int jj = last_blk - gp * kTileBlocks;
        if (last_fill < kBlockSize && jj >= 0 && jj < kTileBlocks) {
          mbar_test_wait(&bars.v_full[gp % kStages], (gp / kStages) & 1);  // every lane sees the data
          uint8_t* vblk = smem + L::offV + (gp % kStages) * pfl::kTileBytes + jj * kHalfTileBytes;
          const int nrow = kBlockSize - last_fill;
          for (int idx = lane; idx < 2 * nrow * 8; idx += 32) {
            const int hf = idx / (nrow * 8);
            const int rem = idx - hf * (nrow * 8);
            *reinterpret_cast<uint4*>(vblk + hf * pfl::kHalfBytes + (last_fill + (rem >> 3)) * 128 + (rem & 7) * 16) =
                make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
          __syncwarp();
        }
        if (lane == 0) {
          tc_fence_after_sync();
          const uint32_t vst = sm + L::offV + (gp % kStages) * pfl::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < kKeys / 16; ++kk) {
            // A = P in TMEM: keys 16kk .. 16kk+15 of each row = columns 8kk .. 8kk+7 of the S
            // buffer the tile's scores came from
            const uint32_t ta = tmem + (gp & 1) * kKeys + kk * 8;
            // B = V: keys 16kk .. 16kk+15 (rows of the tile) x all D columns (MN-major)
            const uint64_t bd = smem_desc_sw128(vst + kk * 2048, pfl::kHalfBytes, 1024);
            tc_mma_bf16_ta(tmem + pfl::kTmemO, ta, bd, idesc_o, (gp == 0 && kk == 0) ? 0u : 1u);
          }
          tc_commit(&bars.pv_done[gp & 1]);
          tc_commit(&bars.v_empty[gp % kStages]);
        }
        __syncwarp();
        ++gp;
        progressed = true;
      }
      if (gs < nk && gs < gp + 3) {  // S of tile j+2 may run while the softmax of tile j does
        const int s = gs % kStages;
        bool s_ready = false;
        if (lane == 0)
          s_ready = (gs > 0 || mbar_test_wait(&bars.q_full, 0)) &&
                    mbar_test_wait(&bars.k_full[s], (gs / kStages) & 1) &&
                    (gs < 2 || mbar_test_wait(&bars.pv_done[gs & 1], ((gs >> 1) - 1) & 1));
        if (__shfl_sync(kFull, s_ready, 0)) {
          if (lane == 0) {
            tc_fence_after_sync();
            const uint32_t kst = sm + L::offK + s * pfl::kTileBytes;
            const uint32_t qst = sm + L::offQ;
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
              const uint64_t ad = smem_desc_sw128(qst + (k >> 2) * pfl::kRowsHalfBytes + (k & 3) * 32, 16, 1024);
              const uint64_t bd = smem_desc_sw128(kst + (k >> 2) * pfl::kHalfBytes + (k & 3) * 32, 16, 1024);
              tc_mma_bf16(tmem + (gs & 1) * kKeys, ad, bd, idesc_s, k > 0 ? 1u : 0u);
            }
            tc_commit(&bars.s_full[gs & 1]);
            tc_commit(&bars.k_empty[s]);
          }
          __syncwarp();
          ++gs;
          progressed = true;
        }
      }
      if (progressed) {
        idle_since = 0;
        idle_polls = 0;
      } else if ((++idle_polls & 63) == 0) {  // the clock is read once every 64 idle polls
        const unsigned long long now = __shfl_sync(kFull, global_timer_ns(), 0);
        if (idle_since == 0) {
          idle_since = now;
        } else if (now - idle_since > kWaitLimitNs) {
          ok = false;
          break;
        }
      }
    }
    if (lane == 0) {
      if (!ok) record_error(kErrTimeoutDecode);
      tc_commit(&bars.drain);  // every MMA issued so far has completed once drain flips
      if (!mbar_wait_bounded(&bars.drain, 0)) record_error(kErrTimeoutDrain);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ Q, softmax, epilogue
    const int r = threadIdx.x;                 // row = TMEM lane
    const int tt = r / p.group;                // chunk token of the row (within the CTA)
    const int h = kvh * p.group + (r - tt * p.group);
    const bool valid = tt < ntok;
    const int pos = valid ? pos0 + tt : -1;    // the row's position: keys 0 .. pos visible
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t o_col = tmem + lane_off + pfl::kTmemO;
    const size_t row_off = (static_cast<size_t>(qs + tok0 + tt) * p.num_q_heads + h) * D;
    {  // the Q row -> shared memory, 128-byte swizzled K-major; zeros for rows past the chunk
      const uint4* src = reinterpret_cast<const uint4*>(p.query + row_off);
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const uint4 v = valid ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(smem + L::offQ + pfl::row_chunk_offset(r, c)) = v;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.q_full);
    }
    const float cs = p.scale_log2;             // > 0 or 0: the maximum commutes with it
    float mref = -INFINITY, l = 0.f;
    bool ok = true;
    auto wait = [&](uint64_t* bar, uint32_t parity) {
      if (ok) ok = __all_sync(kFull, mbar_wait_bounded(bar, parity));
    };
    for (int j = 0; j < nk; ++j) {
      wait(&bars.s_full[j & 1], (j >> 1) & 1);
      tc_fence_after_sync();
      uint32_t sv[kKeys];
      tmem_ld32(tmem + lane_off + (j & 1) * kKeys, *reinterpret_cast<uint32_t(*)[32]>(sv));
      tmem_ld32(tmem + lane_off + (j & 1) * kKeys + 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32));
      tc_wait_ld();
      // keys past the row's position are masked (the chunk is causal; keys past every row's
      // position are past the context or belong to later chunk tokens): only tiles that reach
      // past the row's position take the mask. The maximum is taken over the raw scores
      // (the scale is >= 0) and the scale is applied once, in the exponent's FMA.
      const int k0 = j * kKeys;
      const bool edge = k0 + kKeys - 1 > pos;
      const int nvis = edge ? min(kKeys, max(0, pos - k0 + 1)) : kKeys;  // keys k < nvis are visible
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      if (edge) {
#pragma unroll
        for (int k = 0; k < kKeys; ++k)
          if (k < nvis) m4[k & 3] = fmaxf(m4[k & 3], __uint_as_float(sv[k]));
      } else {
#pragma unroll
        for (int k = 0; k < kKeys; k += 2)
          m4[(k >> 1) & 3] = pfl::max3(m4[(k >> 1) & 3], __uint_as_float(sv[k]), __uint_as_float(sv[k + 1]));
      }
      const float rmx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      const float mx = rmx == -INFINITY ? -INFINITY : rmx * cs;   // the tile's row maximum, log2 units
      // move the reference when the tile's maximum exceeds it by more than 2^8; O (TMEM) is
      // rescaled by the whole warp whenever one of its rows moved (tcgen05.ld/st are
      // warp-collective), the other rows by 1
      const bool need = mx > mref + pfl::kRescaleLog2 || (mref == -INFINITY && mx != -INFINITY);
      float alpha = 1.f;
      if (need) {
        alpha = mref == -INFINITY ? 0.f : fast_exp2(mref - mx);
        l *= alpha;
      }
      const bool rescale = __any_sync(kFull, need && j > 0 && mref != -INFINITY);
      if (need) mref = mx;
      const float mu = mref == -INFINITY ? 0.f : mref;
      // p = 2^(s * scale - reference): one FMA and one exponential per key
      uint32_t pk[kKeys / 2];
      float2 la = make_float2(0.f, 0.f), lb = make_float2(0.f, 0.f);
#pragma unroll
      for (int k = 0; k < kKeys; k += 2) {
        const float2 x = pfl::fma2(make_float2(__uint_as_float(sv[k]), __uint_as_float(sv[k + 1])), cs, -mu);
        float p0 = fast_exp2(x.x);
        float p1 = fast_exp2(x.y);
        if (edge) {
          p0 = k < nvis ? p0 : 0.f;
          p1 = k + 1 < nvis ? p1 : 0.f;
        }
        if (k & 2) lb = pfl::add2(lb, make_float2(p0, p1)); else la = pfl::add2(la, make_float2(p0, p1));
        pk[k / 2] = pack_bf16x2(p0, p1);
      }
      l += (la.x + la.y) + (lb.x + lb.y);
      // O holds the earlier tiles once the PV of tile j-1 has completed: the rescale of O
      // comes before this tile's PV is released
      if (rescale) {
        wait(&bars.pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1);
        tc_fence_after_sync();
#pragma unroll
        for (int q4 = 0; q4 < D / 32; ++q4) {
          uint32_t ov[32];
          tmem_ld32(o_col + q4 * 32, ov);
          tc_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
          tmem_st32(o_col + q4 * 32, ov);
        }
        tc_wait_st();
      }
      // P over the tile's scores in TMEM (the S buffer is taken again only by S of tile j+2,
      // which waits for this tile's PV)
      tmem_st32(tmem + lane_off + (j & 1) * kKeys, pk);
      tc_wait_st();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.p_full[j & 1]);
    }
    // ---- epilogue: O / l once the last PV has completed
    wait(&bars.pv_done[(nk - 1) & 1], ((nk - 1) >> 1) & 1);
    tc_fence_after_sync();
    const float inv = l > 0.f ? 1.f / l : 0.f;
    uint4* dst = reinterpret_cast<uint4*>(p.out + row_off);
#pragma unroll
    for (int q4 = 0; q4 < D / 32; ++q4) {
      uint32_t ov[32];
      tmem_ld32(o_col + q4 * 32, ov);
      tc_wait_ld();
      if (ok && valid) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
          dst[q4 * 4 + c] = make_uint4(
              pack_bf16x2(__uint_as_float(ov[8 * c]) * inv, __uint_as_float(ov[8 * c + 1]) * inv),
              pack_bf16x2(__uint_as_float(ov[8 * c + 2]) * inv, __uint_as_float(ov[8 * c + 3]) * inv),
              pack_bf16x2(__uint_as_float(ov[8 * c + 4]) * inv, __uint_as_float(ov[8 * c + 5]) * inv),
              pack_bf16x2(__uint_as_float(ov[8 * c + 6]) * inv, __uint_as_float(ov[8 * c + 7]) * inv));
      }
    }
    tc_fence_before_sync();
    if (!ok && lane == 0) record_error(kErrTimeoutDecode);
  }
  grid_launch_dependents();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == pfl::kMmaWarp) tmem_dealloc(tmem, pfl::kTmemCols);
}

}  // namespace pa
