// Paged decode on the 5th-generation tensor cores (tcgen05, accumulators in TMEM), with
// the tokens of a tile on the MMA's M dimension. Included by pa_kernels.cu (shares its
// helpers and device error word).
//
// Work. A unit is (sequence, kv head, row chunk of N query rows); its blocks are cut into
// tiles of 8 blocks = 128 tokens. The CTAs of the persistent grid form groups of S
// (a divisor of H_kv); CTA li of a group takes the kv heads li, li + S, ... . All groups
// walk the same enumeration of (sequence, kv-head index, row chunk, tile) and split it
// into equal contiguous ranges, one per group, computed in the kernel from context_lens
// (no pre-pass); the S CTAs of a group therefore read the kv-head slices of the same
// blocks at about the same time. A unit cut by a range boundary leaves partial records,
// combined afterwards by tcm_merge_kernel.
//
// Per tile, with Q of the unit's N (16 or 32) rows:
//   S^T[128 tok][N]  = K[128 tok][D] . Q^T[D][N]           tcgen05.mma M=128, K-major A and B
//   softmax over the tile's 128 tokens: thread t of the softmax warpgroup owns token t
//   (TMEM lane t) and all N columns; the column maxima are reduced across the 128
//   threads, and the running reference maximum of a column moves only when the tile
//   maximum exceeds it by more than 2^8 (the output is exact either way, since
//   numerator and denominator share the reference);
//   O^T[D][N] += V^T[D][128 tok] . P^T[128 tok][N]         tcgen05.mma M=D=128, MN-major A
//                                                          (the TMA tile) and B (P^T)
// Roles: warps 0-7 softmax and epilogue in two warpgroups, each over TMEM lanes 0..127 and
// owning half of the N columns (its own maxima, references, P^T half and O^T half);
// warp 8 TMA producer of K and Q loads, warp 10 TMA producer of V (one warp issues about
// 16 2-KB boxes per us, so K and V get a warp each), warp 9 MMA issuer (one thread) and
// TMEM owner. The issuer polls both of its
// inputs and issues whichever MMA is ready: the S of the next tile once its K has
// landed, the PV of the oldest tile once its P^T is written; a K stage is released
// when its S completes, a V stage when its PV completes.
// TMEM columns: S double buffer [0, 2N), O double buffer (by unit parity) [2N, 4N).
// Shared memory: 2 Q buffers, 2 P^T buffers, 3 stages of K and 3 of V (32 KB each).

namespace pa {
namespace tcm {

constexpr int kD = 128;
constexpr int kTileBlocks = 8;
constexpr int kTileTokens = kTileBlocks * kBlockSize;   // 128
constexpr int kKStages = 3;  // a K stage is released as soon as its S has completed
constexpr int kVStages = 3;  // a V stage is held until the PV, after the tile's softmax
constexpr int kSoftmaxWarps = 8;   // two warpgroups, each owning half of the N columns
constexpr int kThreads = 352;
constexpr int kProducerWarp = 8;   // K boxes and Q rows
constexpr int kMmaWarp = 9;
constexpr int kVProducerWarp = 10; // V boxes
constexpr float kRescaleLog2 = 8.f;
constexpr int kHalfBytes = kTileBlocks * kHalfTileBytes;  // one 64-column half of a tile
constexpr int kStageBytes = 2 * kHalfBytes;               // K or V of one tile
constexpr int kPGroupBytes = kTileTokens * 16;            // P^T: 8 columns x 128 tokens

template <int N>
struct Smem {
  static constexpr int kQ = 2 * N * 128;             // 2 halves x N rows x 128 B, 128-B swizzle
  static constexpr int kP = (N / 8) * kPGroupBytes;  // 128 tokens x N bf16, core matrices
  static constexpr int offQ = 0;
  static constexpr int offP = offQ + 2 * kQ;
  static constexpr int offK = offP + 2 * kP;
  static constexpr int offV = offK + kKStages * kStageBytes;
  static constexpr int offRed = offV + kVStages * kStageBytes;  // [2 wg][3][4 warps][N/2] floats
  static constexpr int offScan = offRed + 2 * 3 * 4 * (N / 2) * 4;  // [11] int64, then the start
  static constexpr int offBars = offScan + 128;
  static constexpr int kBytes = offBars + 256;
  static_assert(offK % 1024 == 0 && kQ % 1024 == 0, "swizzled operands need 1024-B alignment");
};

struct Bars {
  uint64_t k_full[kKStages], k_empty[kKStages], v_full[kVStages], v_empty[kVStages];
  uint64_t q_full[2], q_empty[2], s_full[2], s_free[2], p_full[2], pv_done[2];
  uint64_t drain;
};

// Position in the CTA's tile range: sequence b, unit k (kv head x row chunk) of it,
// tile x of the unit.
struct Walk {
  int b, k, x, ctx, nblk, tiles;
  __device__ __forceinline__ void seq(const DecodeParams& p) {
    ctx = b < p.num_seqs ? __ldg(p.context_lens + b) : 0;
    nblk = num_blocks_of(p, ctx);
    ctx = min(ctx, nblk * kBlockSize);
    tiles = (nblk + kTileBlocks - 1) / kTileBlocks;
  }
  __device__ __forceinline__ void next(const DecodeParams& p, int upb) {
    if (++x < tiles) return;
    x = 0;
    if (++k < upb) return;
    k = 0;
    do {
      ++b;
      seq(p);
    } while (tiles == 0 && b < p.num_seqs);
  }
};

// Named barrier of one softmax warpgroup (ids 1 and 2).
__device__ __forceinline__ void named_sync_softmax(int wg) {
  asm volatile("bar.sync %0, 128;" ::"r"(1 + wg) : "memory");
}

// Column reduction of a warp: lane l holds V values (columns 0..V-1); on return every
// lane holds the reduction over all 32 lanes of column (l % V). Halving exchange: at
// each step a lane keeps the half of its columns selected by one lane bit and sends
// the other half to the partner lane (31 shuffles for V = 32).
template <int V, bool kMax>
__device__ __forceinline__ float column_reduce(float (&v)[V], int lane) {
#pragma unroll
  for (int h = V / 2; h >= 1; h >>= 1) {
    const bool upper = (lane & h) != 0;
#pragma unroll
    for (int k = 0; k < h; ++k) {
      const float send = upper ? v[k] : v[k + h];
      const float keep = upper ? v[k + h] : v[k];
      const float got = __shfl_xor_sync(kFull, send, h);
      v[k] = kMax ? fmaxf(keep, got) : keep + got;
    }
  }
  float r = v[0];
#pragma unroll
  for (int o = V; o < 32; o <<= 1) {
    const float got = __shfl_xor_sync(kFull, r, o);
    r = kMax ? fmaxf(r, got) : r + got;
  }
  return r;
}

}  // namespace tcm

template <int N>
__global__ void __launch_bounds__(tcm::kThreads, 1)
decode_tcm_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmap_k,
                  const __grid_constant__ CUtensorMap tmap_v) {
  using L = tcm::Smem<N>;
  using tcm::kKStages;
  using tcm::kVStages;
  using tcm::kTileBlocks;
  using tcm::kTileTokens;
  constexpr int D = tcm::kD;
  extern __shared__ __align__(1024) uint8_t smem[];
  static_assert(sizeof(tcm::Bars) + 16 <= 256, "barrier area");
  static_assert(tcm::kThreads / 32 * 8 <= 96, "scan area");
  tcm::Bars& bars = *reinterpret_cast<tcm::Bars*>(smem + L::offBars);
  uint32_t& tmem_base_s = *reinterpret_cast<uint32_t*>(smem + L::offBars + sizeof(tcm::Bars));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  if (smem_u32(smem) & 1023u) {  // the swizzled operand layouts need a 1024-aligned base
    if (threadIdx.x == 0) {
      record_error(kErrSchedule);
      p.tc_desc[c] = make_int4(-1, 0, 0, 0);
    }
    return;
  }
  if (threadIdx.x == 0) {
    uint64_t* all = reinterpret_cast<uint64_t*>(&bars);
    for (int i = 0; i < static_cast<int>(sizeof(tcm::Bars) / 8); ++i) mbar_init(all + i, 1);
    for (int i = 0; i < 2; ++i) {  // one arrival per softmax warp
      mbar_init(&bars.s_free[i], tcm::kSoftmaxWarps);
      mbar_init(&bars.p_full[i], tcm::kSoftmaxWarps);
    }
    fence_barrier_init();
    tma_prefetch_desc(&tmap_k);
    tma_prefetch_desc(&tmap_v);
  }
  grid_dependency_wait();

  // ---- this CTA's group, kv-head set and tile range [t0, t1) of the W tiles every group
  // walks: prefix sums over the sequences
  const int S = p.tc_group;
  const int li = c % S;
  const int NG = static_cast<int>(gridDim.x) / S;
  const int upb = (p.num_kv_heads / S) * p.row_chunks;  // units per sequence of one CTA
  long long* wsum = reinterpret_cast<long long*>(smem + L::offScan);
  int* start = reinterpret_cast<int*>(smem + L::offScan + 96);
  long long W, t0, t1;
  int NGe;  // groups that take part: at most one per tile, so that every range is non-empty
  {
    const int B = p.num_seqs;
    const int chunk = (B + tcm::kThreads - 1) / tcm::kThreads;
    const int s0 = min(B, static_cast<int>(threadIdx.x) * chunk), s1 = min(B, s0 + chunk);
    long long local = 0;
    for (int b = s0; b < s1; ++b) {
      const int nb = num_blocks_of(p, __ldg(p.context_lens + b));
      local += static_cast<long long>((nb + kTileBlocks - 1) / kTileBlocks) * upb;
    }
    long long v = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long nv = __shfl_up_sync(kFull, v, o);
      if (lane >= o) v += nv;
    }
    if (lane == 31) wsum[warp] = v;
    __syncthreads();
    long long base = 0;
    W = 0;
    for (int w2 = 0; w2 < tcm::kThreads / 32; ++w2) {
      if (w2 < warp) base += wsum[w2];
      W += wsum[w2];
    }
    NGe = static_cast<int>(min(static_cast<long long>(NG), W));
    const int gi = c / S;
    t0 = gi < NGe ? static_cast<long long>(gi) * W / NGe : 0;
    t1 = gi < NGe ? static_cast<long long>(gi + 1) * W / NGe : 0;
    const long long excl = base + v - local;
    if (local > 0 && t0 < t1 && t0 >= excl && t0 < excl + local) {
      long long acc = excl;
      for (int b = s0; b < s1; ++b) {
        const int nb = num_blocks_of(p, __ldg(p.context_lens + b));
        const long long tb = static_cast<long long>((nb + kTileBlocks - 1) / kTileBlocks) * upb;
        if (t0 < acc + tb) {
          start[0] = b;
          start[1] = static_cast<int>(t0 - acc);
          break;
        }
        acc += tb;
      }
    }
    __syncthreads();
  }
  const int n = static_cast<int>(t1 - t0);
  if (n <= 0) {  // uniform: no tiles for this CTA
    if (threadIdx.x == 0) p.tc_desc[c] = make_int4(-1, 0, 0, 0);
    grid_launch_dependents();
    return;
  }
  // unit k of a sequence -> kv head and row chunk of this CTA
  auto unit_kvh = [&](int k) { return li + S * (k / p.row_chunks); };
  auto unit_rc = [&](int k) { return k % p.row_chunks; };
  tcm::Walk w0;
  w0.b = start[0];
  w0.seq(p);
  w0.k = start[1] / w0.tiles;
  w0.x = start[1] - w0.k * w0.tiles;

  if (warp == tcm::kMmaWarp) {
    tmem_alloc(&tmem_base_s, 4 * N < 32 ? 32 : 4 * N);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = tmem_base_s;
  const uint32_t sm = smem_u32(smem);

  if (warp == tcm::kProducerWarp || warp == tcm::kVProducerWarp) {
    // ------------------------------------------------------------ TMA producers
    // Lanes 0..15 issue a tile's 16 boxes (half = lane / 8, block = lane % 8) of K (warp 4)
    // or V (warp 6); lanes 0..7 load the next tile's block ids while this one is issued.
    const bool is_k = warp == tcm::kProducerWarp;
    const CUtensorMap* tmap = is_k ? &tmap_k : &tmap_v;
    uint64_t* full = is_k ? bars.k_full : bars.v_full;
    uint64_t* empty = is_k ? bars.k_empty : bars.v_empty;
    const int stage_off = is_k ? L::offK : L::offV;
    tcm::Walk w = w0;
    const int oob = static_cast<int>(p.num_blocks);  // block id past the pool: TMA fills zeros
    auto block_id = [&](const tcm::Walk& at) {
      const int blk = at.x * kTileBlocks + lane;
      return (lane < kTileBlocks && blk < at.nblk)
                 ? __ldg(p.block_tables + static_cast<size_t>(at.b) * p.max_blocks + blk)
                 : oob;
    };
    int phys_next = block_id(w);
    int j = -1, g = 0;
    bool ok = true;
    for (; g < n; ++g) {
      if (is_k && (g == 0 || w.x == 0)) {
        ++j;
        if (j >= 2) ok = __all_sync(kFull, mbar_wait_bounded(&bars.q_empty[j & 1], ((j >> 1) - 1) & 1));
        if (!ok) break;
        // Q rows of the unit -> Q[j & 1], 128-byte swizzled K-major; zeros for padded rows
        const int kvh = unit_kvh(w.k);
        const int rc = unit_rc(w.k);
        const int nrows = min(N, p.rows - rc * N);
        uint8_t* qb = smem + L::offQ + (j & 1) * L::kQ;
        if (lane < N) {
          const int r = lane;
          const bool valid = r < nrows;
          const int rr = rc * N + r;
          const int i = valid ? rr / p.group : 0;
          const int gg = valid ? rr - i * p.group : 0;
          const uint4* src = reinterpret_cast<const uint4*>(
              p.query + (static_cast<size_t>(w.b * p.q_per_seq + i) * p.num_q_heads + kvh * p.group + gg) * D);
#pragma unroll
          for (int ch = 0; ch < D / 8; ++ch) {
            const uint4 v = valid ? __ldg(src + ch) : make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4*>(qb + (ch >> 3) * (N * 128) + r * 128 + (((ch & 7) ^ (r & 7)) << 4)) = v;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.q_full[j & 1]);
      }
      const int stages = is_k ? kKStages : kVStages;
      const int s = g % stages;
      const int kvh = unit_kvh(w.k);
      const int ph = __shfl_sync(kFull, phys_next, lane & (kTileBlocks - 1));
      tcm::Walk wn = w;
      wn.next(p, upb);
      if (g + 1 < n) phys_next = block_id(wn);
      if (g >= stages) ok = __all_sync(kFull, mbar_wait_bounded(&empty[s], ((g / stages) - 1) & 1));
      if (!ok) break;
      if (lane == 0) mbar_arrive_expect_tx(&full[s], tcm::kStageBytes);
      __syncwarp();
      const int hf = lane >> 3, jj = lane & (kTileBlocks - 1);
      if (lane < 2 * kTileBlocks)
        tma_load_3d(smem + stage_off + s * tcm::kStageBytes + hf * tcm::kHalfBytes + jj * kHalfTileBytes, tmap,
                    &full[s], hf * 64, kvh, ph * kBlockSize);
      __syncwarp();
      w = wn;
    }
    if (!ok) {
      if (lane == 0) record_error(kErrTimeoutDecode);
      // wait (bounded) for the loads still in flight before leaving
      const int stages = is_k ? kKStages : kVStages;
      for (int u = max(0, g - stages); u < g; ++u)
        if (!mbar_wait_bounded(&full[u % stages], (u / stages) & 1) && lane == 0) record_error(kErrTimeoutDrain);
    }
  } else if (warp == tcm::kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, N, 0, 0);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, N, 1, 1);
      tcm::Walk w = w0;      // position of the next S
      int js = -1;           // unit counter of the S issued last
      int gs = 0, gp = 0;    // next tile to issue S for / PV for (gp <= gs <= gp + 3)
      int ring = 0;          // per tile in flight: bit 2(g&3) O buffer, bit 2(g&3)+1 first of unit
      bool ok = true;
      unsigned long long idle_since = 0;
      unsigned idle_polls = 0;
      while (gp < n) {
        bool progressed = false;
        if (gp < gs && mbar_test_wait(&bars.p_full[gp & 1], (gp >> 1) & 1) &&
            mbar_test_wait(&bars.v_full[gp % kVStages], (gp / kVStages) & 1)) {
          const int sh = 2 * (gp & 3);
          const int obuf = (ring >> sh) & 1;
          const bool first = (ring >> (sh + 1)) & 1;
          tc_fence_after_sync();
          const uint32_t vst = sm + L::offV + (gp % kVStages) * tcm::kStageBytes;
          const uint32_t pst = sm + L::offP + (gp & 1) * L::kP;
#pragma unroll
          for (int kk = 0; kk < kTileTokens / 16; ++kk) {
            const uint64_t ad = smem_desc_sw128(vst + kk * 2048, tcm::kHalfBytes, 1024);
            const uint64_t bd = smem_desc_noswizzle(pst + kk * 256, 128, tcm::kPGroupBytes);
            tc_mma_bf16(tmem + 2 * N + obuf * N, ad, bd, idesc_o, (first && kk == 0) ? 0u : 1u);
          }
          tc_commit(&bars.pv_done[gp & 1]);
          tc_commit(&bars.v_empty[gp % kVStages]);
          ++gp;
          progressed = true;
        }
        if (gs < n && gs - gp < 3) {
          const bool first = gs == 0 || w.x == 0;
          const int jn = first ? js + 1 : js;
          const int s = gs % kKStages;
          if ((!first || mbar_test_wait(&bars.q_full[jn & 1], (jn >> 1) & 1)) &&
              mbar_test_wait(&bars.k_full[s], (gs / kKStages) & 1) &&
              (gs < 2 || mbar_test_wait(&bars.s_free[gs & 1], ((gs >> 1) - 1) & 1))) {
            js = jn;
            const int obuf = js & 1;
            const bool last = gs == n - 1 || w.x == w.tiles - 1;
            tc_fence_after_sync();
            const uint32_t kst = sm + L::offK + s * tcm::kStageBytes;
            const uint32_t qst = sm + L::offQ + obuf * L::kQ;
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
              const uint64_t ad = smem_desc_sw128(kst + (k >> 2) * tcm::kHalfBytes + (k & 3) * 32, 16, 1024);
              const uint64_t bd = smem_desc_sw128(qst + (k >> 2) * (N * 128) + (k & 3) * 32, 16, 1024);
              tc_mma_bf16(tmem + (gs & 1) * N, ad, bd, idesc_s, k > 0 ? 1u : 0u);
            }
            tc_commit(&bars.s_full[gs & 1]);
            tc_commit(&bars.k_empty[s]);
            if (last) tc_commit(&bars.q_empty[obuf]);
            const int sh = 2 * (gs & 3);
            ring = (ring & ~(3 << sh)) | (obuf << sh) | ((first ? 1 : 0) << (sh + 1));
            w.next(p, upb);
            ++gs;
            progressed = true;
          }
        }
        if (progressed) {
          idle_since = 0;
          idle_polls = 0;
        } else if ((++idle_polls & 63) == 0) {  // the clock is read once every 64 idle polls
          const unsigned long long now = global_timer_ns();
          if (idle_since == 0) {
            idle_since = now;
          } else if (now - idle_since > kWaitLimitNs) {
            ok = false;
            break;
          }
        }
      }
      if (!ok) record_error(kErrTimeoutDecode);
      tc_commit(&bars.drain);  // every MMA issued so far has completed once drain flips
      if (!mbar_wait_bounded(&bars.drain, 0)) record_error(kErrTimeoutDrain);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    constexpr int NC = N / 2;  // columns of this warpgroup
    const int wg = warp >> 2;
    const int cb = wg * NC;    // first column of this warpgroup
    const int t = (warp & 3) * 32 + lane;  // token of the tile = TMEM lane = head-dim index in O^T
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    float* red = reinterpret_cast<float*>(smem + L::offRed) + wg * 3 * 4 * NC;
    const float cs = p.scale_log2;
    tcm::Walk w = w0;
    int j = -1, first_x = 0, kvh = 0, rc = 0, nrows = 0, minlim = 0;
    float mref_c = -INFINITY;  // reference maximum of column cb + (lane % NC)
    float mref[NC], lpart[NC];
    int lim[NC];
    // A bounded wait that gives up makes `ok` false for good: the later waits are skipped
    // and nothing more is written to global memory, but every warp still passes every
    // named barrier, so none of a warpgroup's four warps is left waiting for the others.
    bool ok = true;
    auto wait = [&](uint64_t* bar, uint32_t parity) {
      if (ok) ok = __all_sync(kFull, mbar_wait_bounded(bar, parity));
    };
    // A unit piece whose output is written one tile later: by then its last PV is done.
    struct Pending {
      bool on, complete;
      int g, obuf, b, kvh, rc, nrows, slot;
      float L_c, m_c;  // l and the reference maximum of column cb + (lane % NC)
    } pend;
    pend.on = false;
    auto flush = [&](Pending& e) {
      e.on = false;
      wait(&bars.pv_done[e.g & 1], (e.g >> 1) & 1);
      tc_fence_after_sync();
      uint32_t ov[NC];
      tmem_ld<NC>(tmem + lane_off + 2 * N + e.obuf * N + cb, ov);
      tc_wait_ld();
      tc_fence_before_sync();
      if (!ok) return;  // nothing is written after a timeout
      if (e.complete) {
        int i = (e.rc * N + cb) / p.group, gg = e.rc * N + cb - i * p.group;
#pragma unroll
        for (int r = 0; r < NC; ++r) {
          const float lr = __shfl_sync(kFull, e.L_c, r);
          if (cb + r < e.nrows) {
            const float inv = lr > 0.f ? 1.f / lr : 0.f;
            p.out[(static_cast<size_t>(e.b * p.q_per_seq + i) * p.num_q_heads + e.kvh * p.group + gg) * D + t] =
                static_cast<uint16_t>(pack_bf16x2(__uint_as_float(ov[r]) * inv, 0.f) & 0xFFFFu);
          }
          if (++gg == p.group) {
            gg = 0;
            ++i;
          }
        }
      } else {
        float* rec = p.records + static_cast<size_t>(e.slot) * p.rec_stride;
#pragma unroll
        for (int r = 0; r < NC; ++r)
          if (cb + r < e.nrows) rec[(cb + r) * D + t] = __uint_as_float(ov[r]);
        if (t < NC && cb + t < e.nrows) reinterpret_cast<float2*>(rec + N * D)[cb + t] = make_float2(e.m_c, e.L_c);
      }
    };
    for (int g = 0; g < n; ++g) {
      const bool first = g == 0 || w.x == 0;
      const bool last = g == n - 1 || w.x == w.tiles - 1;
      if (first) {
        ++j;
        first_x = w.x;
        kvh = unit_kvh(w.k);
        rc = unit_rc(w.k);
        nrows = min(N, p.rows - rc * N);
        int i = (rc * N + cb) / p.group, gg = rc * N + cb - i * p.group;
        minlim = w.ctx - p.q_per_seq + (rc * N) / p.group;
#pragma unroll
        for (int r = 0; r < NC; ++r) {
          lim[r] = cb + r < nrows ? w.ctx - p.q_per_seq + i : w.ctx - 1;
          if (++gg == p.group) {
            gg = 0;
            ++i;
          }
          mref[r] = -INFINITY;
          lpart[r] = 0.f;
        }
        mref_c = -INFINITY;
      }
      // ---- S^T of this tile: this warpgroup's NC scores of token t
      wait(&bars.s_full[g & 1], (g >> 1) & 1);
      tc_fence_after_sync();
      uint32_t sv[NC];
      tmem_ld<NC>(tmem + lane_off + (g & 1) * N + cb, sv);
      tc_wait_ld();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.s_free[g & 1]);
      const int tok = w.x * kTileTokens + t;
      const bool edge = w.x * kTileTokens + kTileTokens - 1 > minlim;
      float x[NC], tmp[NC];
#pragma unroll
      for (int r = 0; r < NC; ++r) {
        float v = __uint_as_float(sv[r]) * cs;
        if (edge && tok > lim[r]) v = -INFINITY;
        x[r] = v;
        tmp[r] = v;
      }
      // ---- column maxima over the 128 tokens
      const float wmax = tcm::column_reduce<NC, true>(tmp, lane);
      float* rb = red + (g & 1) * 4 * NC;
      if (lane < NC) rb[(warp & 3) * NC + lane] = wmax;
      tcm::named_sync_softmax(wg);
      const int jc = lane % NC;
      const float M = fmaxf(fmaxf(rb[jc], rb[NC + jc]), fmaxf(rb[2 * NC + jc], rb[3 * NC + jc]));
      const bool need = M > mref_c + tcm::kRescaleLog2 || (mref_c == -INFINITY && M != -INFINITY);
      if (__any_sync(kFull, need)) {  // the same decision in the warpgroup's four warps
        const float nm = need ? M : mref_c;
        const float alpha_c = need ? (mref_c == -INFINITY ? 0.f : fast_exp2(mref_c - nm)) : 1.f;
        mref_c = nm;
        float alpha[NC];
#pragma unroll
        for (int r = 0; r < NC; ++r) {
          mref[r] = __shfl_sync(kFull, mref_c, r);
          alpha[r] = __shfl_sync(kFull, alpha_c, r);
          lpart[r] *= alpha[r];
        }
        if (!first) {  // O holds this unit's earlier tiles once the PV of tile g-1 is done
          wait(&bars.pv_done[(g - 1) & 1], ((g - 1) >> 1) & 1);
          tc_fence_after_sync();
          uint32_t ov[NC];
          const uint32_t oaddr = tmem + lane_off + 2 * N + (j & 1) * N + cb;
          tmem_ld<NC>(oaddr, ov);
          tc_wait_ld();
#pragma unroll
          for (int r = 0; r < NC; ++r) ov[r] = __float_as_uint(__uint_as_float(ov[r]) * alpha[r]);
          tmem_st<NC>(oaddr, ov);
          tc_wait_st();
        }
      }
      // ---- probabilities, bf16 pairs (column 2q in the low half)
      uint32_t pk[NC / 2];
#pragma unroll
      for (int r = 0; r < NC; r += 2) {
        const float p0 = fast_exp2(x[r] - (mref[r] == -INFINITY ? 0.f : mref[r]));
        const float p1 = fast_exp2(x[r + 1] - (mref[r + 1] == -INFINITY ? 0.f : mref[r + 1]));
        lpart[r] += p0;
        lpart[r + 1] += p1;
        pk[r / 2] = pack_bf16x2(p0, p1);
      }
      // the P^T buffer of this tile was read by the PV of tile g-2
      if (g >= 2) wait(&bars.pv_done[g & 1], ((g >> 1) - 1) & 1);
      if (wg == 0 && w.x == w.tiles - 1 && (w.ctx & (kBlockSize - 1))) {
        // The sequence's last block is partly filled: its slots past the context may hold
        // any bits (NaN too), and although their p is 0, 0 * NaN is NaN, so those V rows
        // are cleared before the PV reads them.
        const int s = g % kVStages;
        wait(&bars.v_full[s], (g / kVStages) & 1);
        const int jj = (w.nblk - 1) - w.x * kTileBlocks;
        const int r0 = w.ctx & (kBlockSize - 1);
        const int nrow = kBlockSize - r0;
        uint8_t* vblk = smem + L::offV + s * tcm::kStageBytes + jj * kHalfTileBytes;
        for (int idx = t; idx < 2 * nrow * 8; idx += 128) {
          const int hf = idx / (nrow * 8);
          const int rem = idx - hf * (nrow * 8);
          *reinterpret_cast<uint4*>(vblk + hf * tcm::kHalfBytes + (r0 + (rem >> 3)) * 128 + (rem & 7) * 16) =
              make_uint4(0, 0, 0, 0);
        }
      }
      uint8_t* pb = smem + L::offP + (g & 1) * L::kP + (cb / 8) * tcm::kPGroupBytes;
#pragma unroll
      for (int q8 = 0; q8 < NC / 8; ++q8)
        *reinterpret_cast<uint4*>(pb + q8 * tcm::kPGroupBytes + t * 16) =
            make_uint4(pk[4 * q8], pk[4 * q8 + 1], pk[4 * q8 + 2], pk[4 * q8 + 3]);
      fence_proxy_async_smem();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.p_full[g & 1]);

      // ---- the previous unit's output, now that its last PV has had a tile's time
      if (pend.on) flush(pend);
      if (last) {
        // ---- end of the unit's piece: l now; O^T / l after the next tile (deferred)
        float ls[NC];
#pragma unroll
        for (int r = 0; r < NC; ++r) ls[r] = lpart[r];
        const float wl = tcm::column_reduce<NC, false>(ls, lane);
        float* rl = red + 2 * 4 * NC;
        if (lane < NC) rl[(warp & 3) * NC + lane] = wl;
        tcm::named_sync_softmax(wg);
        pend.on = true;
        pend.g = g;
        pend.obuf = j & 1;
        pend.b = w.b;
        pend.kvh = kvh;
        pend.rc = rc;
        pend.nrows = nrows;
        pend.complete = first_x == 0 && w.x == w.tiles - 1;
        pend.slot = j == 0 ? 2 * c : 2 * c + 1;
        pend.L_c = (rl[jc] + rl[NC + jc]) + (rl[2 * NC + jc] + rl[3 * NC + jc]);
        pend.m_c = mref_c;
        if (g == n - 1 && wg == 0 && t == 0) {
          // the merge descriptor: this CTA's last unit continues in the next CTAs and
          // started here, so this CTA holds its first piece
          int4 dsc = make_int4(-1, 0, 0, 0);
          if (w.x != w.tiles - 1 && (j > 0 || first_x == 0)) {
            const long long E = t1 + (w.tiles - 1 - w.x);  // end tile (exclusive) of the unit
            dsc = make_int4(j == 0 ? 2 * c : 2 * c + 1, static_cast<int>((E * NGe - 1) / W) * S + li, w.b, w.k);
          }
          p.tc_desc[c] = dsc;
        }
      }
      w.next(p, upb);
    }
    if (pend.on) flush(pend);
    if (!ok) {
      if (lane == 0) record_error(kErrTimeoutDecode);
      if (wg == 0 && t == 0) p.tc_desc[c] = make_int4(-1, 0, 0, 0);
    }
  }
  grid_launch_dependents();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == tcm::kMmaWarp) tmem_dealloc(tmem, 4 * N < 32 ? 32 : 4 * N);
}

// Combines the partial records of every unit cut by a range boundary (one CTA per
// decode CTA; the descriptor of CTA c names the unit whose first piece c holds and the
// last CTA c1 with a piece of it: the pieces are in record slots desc.x, then 2c' for
// c' = c+S, c+2S, ..., c1 (the same CTA of the following groups), in that order), then
// writes zeros for sequences with no keys.
template <int N>
__global__ void __launch_bounds__(128) tcm_merge_kernel(const DecodeParams p) {
  constexpr int D = tcm::kD;
  grid_dependency_wait();
  const int c = blockIdx.x;
  const int d = threadIdx.x;
  const int4 dsc = p.tc_desc[c];
  if (dsc.x >= 0) {
    const int b = dsc.z;
    const int S = p.tc_group;
    const int kvh = c % S + S * (dsc.w / p.row_chunks);
    const int rc = dsc.w % p.row_chunks;
    const int nrows = min(N, p.rows - rc * N);
    const int pieces = 1 + (dsc.y - c) / S;
    int i = (rc * N) / p.group, gg = rc * N - i * p.group;
    for (int r = 0; r < nrows; ++r) {
      float M = -INFINITY;
      for (int k = 0; k < pieces; ++k) {
        const int slot = k == 0 ? dsc.x : 2 * (c + k * S);
        M = fmaxf(M, reinterpret_cast<const float2*>(p.records + static_cast<size_t>(slot) * p.rec_stride + N * D)[r].x);
      }
      float acc = 0.f, l = 0.f;
      if (M != -INFINITY) {
        for (int k = 0; k < pieces; ++k) {
          const int slot = k == 0 ? dsc.x : 2 * (c + k * S);
          const float* rec = p.records + static_cast<size_t>(slot) * p.rec_stride;
          const float2 ml = reinterpret_cast<const float2*>(rec + N * D)[r];
          const float wk = ml.x == -INFINITY ? 0.f : fast_exp2(ml.x - M);
          l = fmaf(ml.y, wk, l);
          acc = fmaf(rec[r * D + d], wk, acc);
        }
      }
      const float inv = l > 0.f ? 1.f / l : 0.f;
      p.out[(static_cast<size_t>(b * p.q_per_seq + i) * p.num_q_heads + kvh * p.group + gg) * D + d] =
          static_cast<uint16_t>(pack_bf16x2(acc * inv, 0.f) & 0xFFFFu);
      if (++gg == p.group) {
        gg = 0;
        ++i;
      }
    }
  }
  // sequences without a visible key (context length 0) get zero rows
  const int rq = p.q_per_seq * p.num_q_heads;
  for (int b = c; b < p.num_seqs; b += gridDim.x) {
    if (num_blocks_of(p, __ldg(p.context_lens + b)) != 0) continue;
    uint16_t* o = p.out + static_cast<size_t>(b) * rq * D;
    for (int e = d; e < rq * D; e += blockDim.x) o[e] = 0;
  }
}

}  // namespace pa
