// Paged decode on the 5th-generation tensor cores (tcgen05, accumulators in TMEM), with
// the tokens of a tile on the MMA's M dimension. Included by pa_kernels.cu (shares its
// helpers and device error word).
//
// Work. A unit is (sequence, kv head, row chunk of N query rows); its blocks are cut into
// tiles of 8 blocks = 128 tokens. The CTAs of the persistent grid form groups of S
// (a divisor of H_kv); CTA li of a group takes the kv heads li, li + S, ... . All groups
// walk the same enumeration of (sequence, kv-head index, row chunk, tile) and split it
// into contiguous ranges of equal cost, one per group, computed in the kernel from
// context_lens (no pre-pass): a tile costs kCostTile, and the start of a unit costs
// kCostUnit more (its first tile, the previous unit's epilogue; measured at about one
// tile period). The S CTAs of a group therefore read the kv-head slices of the same
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
// Range cost: tile kCostTile, start of a unit kCostUnit extra. Windows are summed as
// (tiles << kPackShift) + units with tiles, one 64-bit add per window.
constexpr int kCostTile = 4;
constexpr int kCostUnit = 4;
constexpr int kPackShift = 28;
constexpr int kHalfBytes = kTileBlocks * kHalfTileBytes;  // one 64-column half of a tile
constexpr int kStageBytes = 2 * kHalfBytes;               // K or V of one tile
constexpr int kPGroupBytes = kTileTokens * 16;            // P^T: 8 columns x 128 tokens
constexpr int kMergeThreads = 1024;  // one warp per row of a unit (N <= 32)

template <int N>
struct Smem {
  static constexpr int kQ = 2 * N * 128;             // 2 halves x N rows x 128 B, 128-B swizzle
  static constexpr int kP = (N / 8) * kPGroupBytes;  // 128 tokens x N bf16, core matrices
  static constexpr int offQ = 0;
  static constexpr int offP = offQ + 2 * kQ;
  static constexpr int offK = offP + 2 * kP;
  static constexpr int offV = offK + kKStages * kStageBytes;
  // per softmax warpgroup: [3][4 warps][N/2] floats (2 maxima buffers, 1 sum), [2][4] votes
  static constexpr int kRedWg = 3 * 4 * (N / 2) + 8;
  static constexpr int offRed = offV + kVStages * kStageBytes;
  static constexpr int offScan = offRed + 2 * kRedWg * 4;     // [11] int64, then the start
  static constexpr int offBars = offScan + 128;
  static constexpr int kBytes = offBars + 256;
  static_assert(offK % 1024 == 0 && kQ % 1024 == 0, "swizzled operands need 1024-B alignment");
};

struct Bars {
  uint64_t k_full[kKStages], k_empty[kKStages], v_full[kVStages], v_empty[kVStages];
  uint64_t q_full[2], q_empty[2], s_full[2], s_free[2], p_full[2], pv_done[2];
  uint64_t drain;
};

// Tiles of every unit of window w (one thread, for the partition scan). kWin: the plan has a
// sliding window (a member's own blocks start at its window's first block).
template <bool kWin>
__device__ __forceinline__ int window_tiles(const DecodeParams& p, int w) {
  const int cap = p.share_cap > 1 ? p.share_cap : 1;
  const int b0 = w * cap;
  const int m = min(cap, p.num_seqs - b0);
  if (m <= 0) return 0;
  const int P = cap > 1 ? __ldg(p.win_prefix + w) : 0;
  int tiles = (P + kTileBlocks - 1) / kTileBlocks;
  for (int jj = 0; jj < m; ++jj) {
    const int cx = __ldg(p.context_lens + b0 + jj);
    const int nb = num_blocks_of(p, cx);
    // own blocks: after the shared prefix, from the sliding window's first block on
    const int lo = kWin ? min(nb, max(P, window_first_block(p, cx))) : P;
    tiles += (nb - lo + kTileBlocks - 1) / kTileBlocks;
  }
  return tiles;
}

// Position in the CTA's tile range, kept by a whole warp. A window is `cap` consecutive
// sequences (cap = 1 without prefix sharing) whose tables may start with the same P
// physical blocks; its units are (kv-head index, row chunk) of this CTA, and every unit
// walks the window's tiles: the shared prefix (P blocks, read once for all members) then
// each member's own blocks (with a sliding window, from its window's first block). Lane jj
// holds member jj's context length and blocks, so moving between members takes shuffles,
// not loads. kWin: the plan has a sliding window.
template <bool kWin>
struct Walk {
  int w, k, x;          // window, unit of the window, tile of the unit
  int b0, m, P, tiles;  // window: first sequence, members, shared blocks, tiles of a unit
  int j, y, seg;        // segment: member j (-1: the shared prefix), its tile y, its tiles
  int ctx, nblk, lo;    // member j: context length (clamped to its blocks), blocks, first own block
  int lctx, lnblk, llo; // this lane's member

  __device__ __forceinline__ int own_tiles_lane() const {
    return (lnblk - llo + kTileBlocks - 1) / kTileBlocks;
  }
  __device__ __forceinline__ void member(int jj) {
    ctx = __shfl_sync(kFull, lctx, jj);
    nblk = __shfl_sync(kFull, lnblk, jj);
    lo = kWin ? __shfl_sync(kFull, llo, jj) : P;
  }
  __device__ __forceinline__ void window(const DecodeParams& p) {
    const int lane = threadIdx.x & 31;
    const int cap = p.share_cap > 1 ? p.share_cap : 1;
    b0 = w * cap;
    m = min(cap, p.num_seqs - b0);
    tiles = 0;
    lctx = 0;
    lnblk = 0;
    llo = 0;
    if (m <= 0) return;
    P = cap > 1 ? __ldg(p.win_prefix + w) : 0;
    if (lane < m) {
      lctx = __ldg(p.context_lens + b0 + lane);
      lnblk = num_blocks_of(p, lctx);
      llo = kWin ? min(lnblk, max(P, window_first_block(p, lctx))) : P;
      lctx = min(lctx, lnblk * kBlockSize);
    }
    int t = lane < m ? own_tiles_lane() : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(kFull, t, o);
    tiles = t + (P + kTileBlocks - 1) / kTileBlocks;
  }
  __device__ __forceinline__ void seek(int xx) {
    const int lane = threadIdx.x & 31;
    x = xx;
    int r = xx;
    const int sh = (P + kTileBlocks - 1) / kTileBlocks;
    if (r < sh) {
      j = -1;
      y = r;
      seg = sh;
      ctx = 0;
      nblk = P;
      return;
    }
    r -= sh;
    // member holding own tile r: inclusive prefix sum of the members' own tiles
    int ot = lane < m ? own_tiles_lane() : 0;
    int incl = ot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(kFull, incl, o);
      if (lane >= o) incl += v;
    }
    const unsigned past = __ballot_sync(kFull, lane < m && incl <= r);  // members wholly before r
    const int jj = __popc(past);
    const int before = jj > 0 ? __shfl_sync(kFull, incl, jj - 1) : 0;
    j = jj;
    y = r - before;
    seg = __shfl_sync(kFull, ot, jj);
    member(jj);
  }
  __device__ __forceinline__ void next(const DecodeParams& p, int upb, int nwin) {
    const int lane = threadIdx.x & 31;
    ++x;
    if (++y < seg) return;
    if (x < tiles) {  // the next member with own tiles
      const unsigned more = __ballot_sync(kFull, lane > j && lane < m && own_tiles_lane() > 0);
      const int jj = __ffs(more) - 1;
      j = jj;
      y = 0;
      seg = __shfl_sync(kFull, own_tiles_lane(), jj & 31);
      member(jj & 31);
      return;
    }
    x = 0;
    if (++k < upb) {
      seek(0);
      return;
    }
    k = 0;
    do {
      ++w;
      window(p);
    } while (tiles == 0 && w < nwin);
    if (w < nwin) seek(0);
  }
  // the tile's blocks: [bstart, bend) of table row `row`
  __device__ __forceinline__ int row() const { return b0 + (j < 0 ? 0 : j); }
  __device__ __forceinline__ int bstart() const { return (j < 0 ? 0 : lo) + kTileBlocks * y; }
  __device__ __forceinline__ int bend() const { return j < 0 ? P : nblk; }
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

// kWin: the plan has a sliding window (its own instance, so plans without one run none of
// the window's per-tile work).
template <int N, bool kWin>
__global__ void __launch_bounds__(tcm::kThreads, 1)
decode_tcm_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmap_k,
                  const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ CUtensorMap tmap_q) {
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
    if (p.q_box > 0) tma_prefetch_desc(&tmap_q);
  }
  grid_dependency_wait();

  // ---- this CTA's group, kv-head set and range [t0, t1) of the Wc cost units every group
  // walks: prefix sums over the windows. In cost units, unit u of a window spans kCostUnit +
  // kCostTile * tiles positions: its tile 0 the first kCostUnit + kCostTile, every later tile
  // kCostTile. A group takes the tiles from the one whose span holds t0 to the one before
  // the one whose span holds t1 (all tiles past the last position when t1 = Wc).
  const int S = p.tc_group;
  const int li = c % S;
  const int NG = static_cast<int>(gridDim.x) / S;
  const int upb = (p.num_kv_heads / S) * p.row_chunks;  // units per window of one CTA
  const int cap = p.share_cap > 1 ? p.share_cap : 1;
  const int nwin = (p.num_seqs + cap - 1) / cap;
  const int rpm = p.rows;  // query rows of one member (sequence)
  long long* wsum = reinterpret_cast<long long*>(smem + L::offScan);
  int* start = reinterpret_cast<int*>(smem + L::offScan + 96);
  long long* tpos = reinterpret_cast<long long*>(smem + L::offScan + 104);  // T0, T1, UE
  constexpr long long kUnitsMask = (1ll << tcm::kPackShift) - 1;
  auto cost_of = [](long long pk) {  // cost units of a packed (tiles, units) sum
    return tcm::kCostTile * (pk >> tcm::kPackShift) + tcm::kCostUnit * (pk & kUnitsMask);
  };
  long long Wc, t0, t1;
  int NGe;  // groups that take part: each range spans at least one tile's cost, so none is empty
  int n;    // tiles of this CTA
  {
    const int chunk = (nwin + tcm::kThreads - 1) / tcm::kThreads;
    const int s0 = min(nwin, static_cast<int>(threadIdx.x) * chunk), s1 = min(nwin, s0 + chunk);
    long long local = 0;
    for (int ww = s0; ww < s1; ++ww) {
      const long long tw = tcm::window_tiles<kWin>(p, ww);
      if (tw > 0) local += ((tw * upb) << tcm::kPackShift) + upb;
    }
    long long v = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long nv = __shfl_up_sync(kFull, v, o);
      if (lane >= o) v += nv;
    }
    if (lane == 31) wsum[warp] = v;
    __syncthreads();
    long long base = 0, Wpk = 0;
    for (int w2 = 0; w2 < tcm::kThreads / 32; ++w2) {
      if (w2 < warp) base += wsum[w2];
      Wpk += wsum[w2];
    }
    Wc = cost_of(Wpk);
    NGe = static_cast<int>(min(static_cast<long long>(NG), Wc / (tcm::kCostTile + tcm::kCostUnit)));
    const int gi = c / S;
    t0 = gi < NGe ? static_cast<long long>(gi) * Wc / NGe : 0;
    t1 = gi < NGe ? static_cast<long long>(gi + 1) * Wc / NGe : 0;
    const long long excl = base + v - local;  // packed sums of the windows before s0
    const long long ec = cost_of(excl), lc = cost_of(local);
    if (gi < NGe && t1 == Wc && threadIdx.x == 0) tpos[1] = Wpk >> tcm::kPackShift;
    // the tile whose span holds position `pos` of this thread's windows: window, tile of the
    // window, global tile index, and the cost end of its unit
    for (int e = 0; e < 2; ++e) {
      const long long pos = e == 0 ? t0 : t1;
      if (gi >= NGe || pos >= Wc || pos < ec || pos >= ec + lc) continue;
      long long acc = ec, acct = excl >> tcm::kPackShift;
      for (int ww = s0; ww < s1; ++ww) {
        const int tw = tcm::window_tiles<kWin>(p, ww);
        const long long uc = tcm::kCostUnit + static_cast<long long>(tcm::kCostTile) * tw;
        const long long cw = tw > 0 ? uc * upb : 0;
        if (pos < acc + cw) {
          const int k = static_cast<int>((pos - acc) / uc);
          const long long within = pos - acc - k * uc;
          const int x = within < tcm::kCostUnit + tcm::kCostTile
                            ? 0 : static_cast<int>((within - tcm::kCostUnit) / tcm::kCostTile);
          if (e == 0) {
            start[0] = ww;
            start[1] = k * tw + x;
            tpos[0] = acct + static_cast<long long>(k) * tw + x;
          } else {
            tpos[1] = acct + static_cast<long long>(k) * tw + x;
            tpos[2] = acc + (k + 1) * uc;
          }
          break;
        }
        acc += cw;
        acct += static_cast<long long>(tw) * upb;
      }
    }
    __syncthreads();
    n = gi < NGe ? static_cast<int>(tpos[1] - tpos[0]) : 0;
  }
  if (n <= 0) {  // uniform: no tiles for this CTA
    if (threadIdx.x == 0) p.tc_desc[c] = make_int4(-1, 0, 0, 0);
    grid_launch_dependents();
    return;
  }
  // unit k of a sequence -> kv head and row chunk of this CTA
  auto unit_kvh = [&](int k) { return li + S * (k / p.row_chunks); };
  auto unit_rc = [&](int k) { return k % p.row_chunks; };
  tcm::Walk<kWin> w0;
  w0.w = start[0];
  w0.window(p);  // every warp: its lanes hold the window's members
  w0.k = start[1] / w0.tiles;
  w0.seek(start[1] - w0.k * w0.tiles);

  if (warp == tcm::kMmaWarp) {
    tmem_alloc(&tmem_base_s, 4 * N < 32 ? 32 : 4 * N);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  // Q rows past a box (a shared-prefix window of fewer than N rows) stay zero: no box
  // writes them, and the async proxy (the MMA) reads them
  if (p.q_box > 0 && p.q_box * p.group < N) {
    for (int i = threadIdx.x; i < 2 * L::kQ / 16; i += tcm::kThreads)
      reinterpret_cast<uint4*>(smem + L::offQ)[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
    __syncthreads();
  }
  const uint32_t tmem = tmem_base_s;
  const uint32_t sm = smem_u32(smem);

  if (warp == tcm::kProducerWarp || warp == tcm::kVProducerWarp) {
    // ------------------------------------------------------------ TMA producers
    // Lanes 0..15 issue a tile's 16 boxes (half = lane / 8, block = lane % 8) of K (warp 8)
    // or V (warp 10); lanes 0..7 load the next tile's block ids while this one is issued.
    const bool is_k = warp == tcm::kProducerWarp;
    const CUtensorMap* tmap = is_k ? &tmap_k : &tmap_v;
    uint64_t* full = is_k ? bars.k_full : bars.v_full;
    uint64_t* empty = is_k ? bars.k_empty : bars.v_empty;
    const int stage_off = is_k ? L::offK : L::offV;
    tcm::Walk<kWin> w = w0;
    const int oob = static_cast<int>(p.num_blocks);  // block id past the pool: TMA fills zeros
    auto block_id = [&](const tcm::Walk<kWin>& at) {
      const int blk = at.bstart() + lane;
      return (lane < kTileBlocks && blk < at.bend())
                 ? __ldg(p.block_tables + static_cast<size_t>(at.row()) * p.max_blocks + blk)
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
        uint8_t* qb = smem + L::offQ + (j & 1) * L::kQ;
        if (p.q_box > 0) {
          // the unit's rows as two boxes (the halves of D), in flight with its first K tile:
          // tokens of row chunk rc (rc = 0 for a shared-prefix window), heads of kv head kvh
          if (lane == 0) {
            const int tok0 = w.b0 * p.q_per_seq + rc * p.q_box;
            mbar_arrive_expect_tx(&bars.q_full[j & 1], 2 * p.q_box * p.group * 128);
            tma_load_3d(qb, &tmap_q, &bars.q_full[j & 1], 0, kvh * p.group, tok0);
            tma_load_3d(qb + N * 128, &tmap_q, &bars.q_full[j & 1], 64, kvh * p.group, tok0);
          }
          __syncwarp();
        } else {
        if (lane < N) {
          const int r = lane;
          const int cg = rc * N + r;  // row of the window: member cg / rpm, row cg % rpm of it
          const bool valid = cg < w.m * rpm;
          const int mem = valid ? cg / rpm : 0;
          const int rr = cg - mem * rpm;
          const int i = valid ? rr / p.group : 0;
          const int gg = valid ? rr - i * p.group : 0;
          const uint4* src = reinterpret_cast<const uint4*>(
              p.query +
              (static_cast<size_t>((w.b0 + mem) * p.q_per_seq + i) * p.num_q_heads + kvh * p.group + gg) * D);
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
      }
      const int stages = is_k ? kKStages : kVStages;
      const int s = g % stages;
      const int kvh = unit_kvh(w.k);
      const int ph = __shfl_sync(kFull, phys_next, lane & (kTileBlocks - 1));
      tcm::Walk<kWin> wn = w;
      wn.next(p, upb, nwin);
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
    // The whole warp walks (its lanes hold the window's members); lane 0 tests the barriers
    // and issues, and its decisions are broadcast so that the warp stays converged.
    {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, N, 0, 0);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, N, 1, 1);
      tcm::Walk<kWin> w = w0;      // position of the next S
      int js = -1;           // unit counter of the S issued last
      int gs = 0, gp = 0;    // next tile to issue S for / PV for (gp <= gs <= gp + 3)
      int ring = 0;          // per tile in flight: bit 2(g&3) O buffer, bit 2(g&3)+1 first of unit
      int zring = 0;         // per tile in flight, byte g&3: V rows to clear (bit 0 on, block, row)
      int hring = 0;         // per tile in flight, byte g&3: sliding window, rows 0 .. r-1 of the
                             // tile's first block to clear (bit 0 on, r)
      const int win = kWin ? p.window : 0;
      bool ok = true;
      unsigned long long idle_since = 0;
      unsigned idle_polls = 0;
      while (gp < n) {
        bool progressed = false;
        bool pv_ready = false;
        if (lane == 0)
          pv_ready = gp < gs && mbar_test_wait(&bars.p_full[gp & 1], (gp >> 1) & 1) &&
                     mbar_test_wait(&bars.v_full[gp % kVStages], (gp / kVStages) & 1);
        if (__shfl_sync(kFull, pv_ready, 0)) {
          const int z = (zring >> (8 * (gp & 3))) & 0xFF;
          const int zh = (hring >> (8 * (gp & 3))) & 0xFF;
          if (zh & 1) {
            // Sliding window: the slots of a member's first block before its first row's
            // window start are seen by no row and may hold any bits; cleared like the tail.
            mbar_test_wait(&bars.v_full[gp % kVStages], (gp / kVStages) & 1);  // every lane sees the data
            const int nrow = zh >> 1;
            uint8_t* vblk = smem + L::offV + (gp % kVStages) * tcm::kStageBytes;
            for (int idx = lane; idx < 2 * nrow * 8; idx += 32) {
              const int hf = idx / (nrow * 8);
              const int rem = idx - hf * (nrow * 8);
              *reinterpret_cast<uint4*>(vblk + hf * tcm::kHalfBytes + (rem >> 3) * 128 + (rem & 7) * 16) =
                  make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
            __syncwarp();
          }
          if (z & 1) {
            // A member's last block is partly filled: its slots past the context may hold any
            // bits (NaN too), and although their p is 0, 0 * NaN is NaN, so those V rows are
            // cleared before the PV reads them.
            mbar_test_wait(&bars.v_full[gp % kVStages], (gp / kVStages) & 1);  // every lane sees the data
            const int jj = (z >> 1) & 7, r0 = z >> 4, nrow = kBlockSize - r0;
            uint8_t* vblk = smem + L::offV + (gp % kVStages) * tcm::kStageBytes + jj * kHalfTileBytes;
            for (int idx = lane; idx < 2 * nrow * 8; idx += 32) {
              const int hf = idx / (nrow * 8);
              const int rem = idx - hf * (nrow * 8);
              *reinterpret_cast<uint4*>(vblk + hf * tcm::kHalfBytes + (r0 + (rem >> 3)) * 128 + (rem & 7) * 16) =
                  make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
            __syncwarp();
          }
          if (lane == 0) {
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
          }
          __syncwarp();
          ++gp;
          progressed = true;
        }
        if (gs < n && gs - gp < 3) {
          const bool first = gs == 0 || w.x == 0;
          const int jn = first ? js + 1 : js;
          const int s = gs % kKStages;
          bool s_ready = false;
          if (lane == 0)
            s_ready = (!first || mbar_test_wait(&bars.q_full[jn & 1], (jn >> 1) & 1)) &&
                      mbar_test_wait(&bars.k_full[s], (gs / kKStages) & 1) &&
                      (gs < 2 || mbar_test_wait(&bars.s_free[gs & 1], ((gs >> 1) - 1) & 1));
          if (__shfl_sync(kFull, s_ready, 0)) {
            js = jn;
            const int obuf = js & 1;
            const bool last = gs == n - 1 || w.x == w.tiles - 1;
            if (lane == 0) {
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
            }
            __syncwarp();
            const int sh = 2 * (gs & 3);
            ring = (ring & ~(3 << sh)) | (obuf << sh) | ((first ? 1 : 0) << (sh + 1));
            int z = 0;
            if (w.j >= 0 && w.y == w.seg - 1 && (w.ctx & (kBlockSize - 1)))
              z = 1 | (((w.nblk - 1) - w.bstart()) << 1) | ((w.ctx & (kBlockSize - 1)) << 4);
            zring = (zring & ~(0xFF << (8 * (gs & 3)))) | (z << (8 * (gs & 3)));
            int zh = 0;
            if (win > 0 && w.j >= 0 && w.y == 0) {
              const int r1 = max(0, w.ctx - p.q_per_seq - win + 1) - w.lo * kBlockSize;
              if (r1 > 0) zh = 1 | (r1 << 1);
            }
            hring = (hring & ~(0xFF << (8 * (gs & 3)))) | (zh << (8 * (gs & 3)));
            w.next(p, upb, nwin);
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
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    constexpr int NC = N / 2;  // columns of this warpgroup
    const int wg = warp >> 2;
    const int cb = wg * NC;    // first column of this warpgroup
    const int t = (warp & 3) * 32 + lane;  // token of the tile = TMEM lane = head-dim index in O^T
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    float* red = reinterpret_cast<float*>(smem + L::offRed) + wg * L::kRedWg;
    int* votes = reinterpret_cast<int*>(red + 3 * 4 * NC);  // [2][4 warps]
    const float cs = p.scale_log2;
    const int win = kWin ? p.window : 0;  // sliding window (keys lim - win + 1 .. lim of a row), 0 = none
    tcm::Walk<kWin> w = w0;
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
    // Complete outputs leave through shared memory and bulk copies at N = 32; at N = 16 (8 rows
    // a warpgroup) element stores measured faster.
    constexpr bool kStagedOut = N == 32;
    // A unit piece whose output is written one tile later: by then its last PV is done.
    struct Pending {
      bool on, complete;
      int g, obuf, b0, kvh, rc, nrows, slot;
      float L_c, m_c;  // l and the reference maximum of column cb + (lane % NC)
    } pend;
    pend.on = false;
    bool bulk_pending = false;  // this thread has output copies whose shared-memory reads may be running
    auto flush = [&](Pending& e) {
      e.on = false;
      wait(&bars.pv_done[e.g & 1], (e.g >> 1) & 1);
      tc_fence_after_sync();
      uint32_t ov[NC];
      tmem_ld<NC>(tmem + lane_off + 2 * N + e.obuf * N + cb, ov);
      tc_wait_ld();
      tc_fence_before_sync();
      if (kStagedOut && e.complete) {
        // The rows leave through shared memory and bulk copies: element stores from these
        // threads stall for microseconds behind the kernel's own load traffic. Staging area:
        // this warpgroup's half of the P^T buffer of the piece's last tile (its PV is done;
        // the next P^T written there follows this warpgroup's next vote barrier, before which
        // the copies have finished reading), bf16 [NC rows][D].
        uint16_t* stg =
            reinterpret_cast<uint16_t*>(smem + L::offP + (e.g & 1) * L::kP + (cb / 8) * tcm::kPGroupBytes);
        if (ok) {
          const float inv_c = e.L_c > 0.f ? 1.f / e.L_c : 0.f;  // 1 / l of column cb + (lane % NC)
#pragma unroll
          for (int r = 0; r < NC; ++r) {
            const float inv = __shfl_sync(kFull, inv_c, r);
            stg[r * D + t] = static_cast<uint16_t>(pack_bf16x2(__uint_as_float(ov[r]) * inv, 0.f) & 0xFFFFu);
          }
          fence_proxy_async_smem();
        }
        tcm::named_sync_softmax(wg);  // every warp passes it, also after a timeout
        if (ok && (warp & 3) == 0 && lane == 0) {
          // column cb + r = row cg of the window: member cg / rpm, (i, g) of its row cg % rpm; the
          // rows of one query token's G heads are contiguous in the output: one copy per run
          const int cg = e.rc * N + cb;
          int mem = cg / rpm, i = (cg - mem * rpm) / p.group;
          int gg = cg - mem * rpm - i * p.group;
          const int rend = min(NC, e.nrows - cb);
          for (int r = 0; r < rend;) {
            const int len = min(rend - r, p.group - gg);
            bulk_store(p.out + (static_cast<size_t>((e.b0 + mem) * p.q_per_seq + i) * p.num_q_heads +
                                e.kvh * p.group + gg) * D,
                       stg + r * D, static_cast<uint32_t>(len * D * 2));
            r += len;
            gg += len;
            if (gg == p.group) {
              gg = 0;
              if (++i == p.q_per_seq) {
                i = 0;
                ++mem;
              }
            }
          }
          bulk_commit();
          bulk_pending = true;
        }
        return;
      }
      if (!ok) return;  // nothing is written after a timeout
      if (e.complete) {
        // column cb + r = row cg of the window: member cg / rpm, (i, g) of its row cg % rpm
        int cg = e.rc * N + cb;
        int mem = cg / rpm, i = (cg - mem * rpm) / p.group;
        int gg = cg - mem * rpm - i * p.group;
        const float inv_c = e.L_c > 0.f ? 1.f / e.L_c : 0.f;  // 1 / l of column cb + (lane % NC)
#pragma unroll
        for (int r = 0; r < NC; ++r) {
          const float inv = __shfl_sync(kFull, inv_c, r);
          if (cb + r < e.nrows)
            p.out[(static_cast<size_t>((e.b0 + mem) * p.q_per_seq + i) * p.num_q_heads + e.kvh * p.group + gg) * D +
                  t] = static_cast<uint16_t>(pack_bf16x2(__uint_as_float(ov[r]) * inv, 0.f) & 0xFFFFu);
          if (++gg == p.group) {
            gg = 0;
            if (++i == p.q_per_seq) {
              i = 0;
              ++mem;
            }
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
        nrows = min(N, w.m * rpm - rc * N);
        // the last visible token of each column's row (member mem of the window, query i);
        // padded columns see everything (their Q is zero and their output unused)
        int cg = rc * N + cb;
        int mem = cg / rpm, i = (cg - mem * rpm) / p.group;
        int gg = cg - mem * rpm - i * p.group;
        auto ctx_of = [&](int mm) { return __shfl_sync(kFull, w.lctx, mm & 31); };  // lane mm: member mm
        int cm = ctx_of(mem);
        minlim = (cap == 1) ? cm - p.q_per_seq + (rc * N) / p.group : 0;
#pragma unroll
        for (int r = 0; r < NC; ++r) {
          lim[r] = cb + r < nrows ? cm - p.q_per_seq + i : INT_MAX;
          if (++gg == p.group) {
            gg = 0;
            if (++i == p.q_per_seq) {
              i = 0;
              ++mem;
              cm = ctx_of(mem);
            }
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
      // visible: the shared prefix for every column below P*16; a member's own tile for
      // that member's columns up to their causal limit
      const int tok0 = w.bstart() * kBlockSize;
      const int tok = tok0 + t;
      bool edge;
      int lo = 0, hi = NC, tok_hi = INT_MAX;
      bool use_lim = true;
      if (w.j < 0) {
        tok_hi = w.P * kBlockSize;
        edge = tok0 + kTileTokens > tok_hi;
        use_lim = false;
      } else if (cap > 1) {
        edge = true;
        lo = max(0, w.j * rpm - rc * N - cb);
        hi = min(NC, (w.j + 1) * rpm - rc * N - cb);
      } else {
        // past the first row's last key, or (sliding window) before the last row's first key
        edge = tok0 + kTileTokens - 1 > minlim || (win > 0 && tok0 + win <= w.ctx - 1);
      }
      float x[NC], tmp[NC];
#pragma unroll
      for (int r = 0; r < NC; ++r) {
        float v = __uint_as_float(sv[r]) * cs;
        if (edge && (r < lo || r >= hi || tok >= tok_hi ||
                     (use_lim && (tok > lim[r] || (win > 0 && tok + win <= lim[r])))))
          v = -INFINITY;
        x[r] = v;
        tmp[r] = v;
      }
      // ---- do the references still hold (every score within 2^8 of its column's reference)?
      // Only then can the column maxima be skipped; a vote of the four warps decides.
      bool over = false;
#pragma unroll
      for (int r = 0; r < NC; ++r) over |= x[r] > mref[r] + tcm::kRescaleLog2;
      const int* vb = votes + (g & 1) * 4;
      const bool wover = __any_sync(kFull, over);
      if (lane == 0) votes[(g & 1) * 4 + (warp & 3)] = wover ? 1 : 0;
      if (bulk_pending) {  // a staged output is read out before its buffer takes a P^T again
        bulk_wait_read();
        bulk_pending = false;
      }
      tcm::named_sync_softmax(wg);
      const int jc = lane % NC;
      if ((vb[0] | vb[1] | vb[2] | vb[3]) != 0) {
      // ---- column maxima over the 128 tokens
      const float wmax = tcm::column_reduce<NC, true>(tmp, lane);
      float* rb = red + (g & 1) * 4 * NC;
      if (lane < NC) rb[(warp & 3) * NC + lane] = wmax;
      tcm::named_sync_softmax(wg);
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
        Pending& pe = pend;
        pe.on = true;
        pe.g = g;
        pe.obuf = j & 1;
        pe.b0 = w.b0;
        pe.kvh = kvh;
        pe.rc = rc;
        pe.nrows = nrows;
        pe.complete = first_x == 0 && w.x == w.tiles - 1;
        pe.slot = j == 0 ? 2 * c : 2 * c + 1;
        pe.L_c = (rl[jc] + rl[NC + jc]) + (rl[2 * NC + jc] + rl[3 * NC + jc]);
        pe.m_c = mref_c;
        if (g == n - 1 && wg == 0 && t == 0) {
          // the merge descriptor: this CTA's last unit continues in the next CTAs and
          // started here, so this CTA holds its first piece
          int4 dsc = make_int4(-1, 0, 0, 0);
          if (w.x != w.tiles - 1 && (j > 0 || first_x == 0)) {
            // the unit ends at cost position UE past t1: the last group whose t0 is below it
            // holds its last tile
            const long long UE = tpos[2];
            dsc = make_int4(j == 0 ? 2 * c : 2 * c + 1, static_cast<int>((UE * NGe - 1) / Wc) * S + li, w.w, w.k);
          }
          p.tc_desc[c] = dsc;
        }
      }
      w.next(p, upb, nwin);
    }
    if (pend.on) flush(pend);
    if (bulk_pending) bulk_wait_all();  // the last output copies complete before the CTA exits
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

// Combines the partial records of every unit (window, kv head, row chunk) cut by a range
// boundary (one CTA per
// decode CTA; the descriptor of CTA c names the unit whose first piece c holds and the
// last CTA c1 with a piece of it: the pieces are in record slots desc.x, then 2c' for
// c' = c+S, c+2S, ..., c1 (the same CTA of the following groups), in that order), then
// writes zeros for sequences with no keys.
template <int N>
__global__ void __launch_bounds__(tcm::kMergeThreads) tcm_merge_kernel(const DecodeParams p) {
  constexpr int D = tcm::kD;
  grid_dependency_wait();
  const int c = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int4 dsc = p.tc_desc[c];
  if (dsc.x >= 0) {
    const int cap = p.share_cap > 1 ? p.share_cap : 1;
    const int rpm = p.rows;
    const int b0 = dsc.z * cap;  // the window's first sequence
    const int m = min(cap, p.num_seqs - b0);
    const int S = p.tc_group;
    const int kvh = c % S + S * (dsc.w / p.row_chunks);
    const int rc = dsc.w % p.row_chunks;
    const int nrows = min(N, m * rpm - rc * N);
    const int pieces = 1 + (dsc.y - c) / S;
    const float* recs = p.records;
    const int rs = p.rec_stride, slot0 = dsc.x;
    auto rec_of = [=](int k) {
      return recs + static_cast<size_t>(k == 0 ? slot0 : 2 * (c + k * S)) * rs;
    };
    // one row per warp, 32 pieces at a time: lane k takes piece k's (m, l), and the output
    // slices of the first four pieces are loaded with them (nothing waits for the maximum);
    // each lane accumulates 4 of the D columns over the pieces in order, 4 pieces' loads at
    // a time, against a running maximum
    for (int r = warp; r < nrows; r += tcm::kMergeThreads / 32) {
      float M = -INFINITY, l = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int k0 = 0; k0 < pieces; k0 += 32) {
        const int kn = min(32, pieces - k0);
        const float2 ml = lane < kn ? reinterpret_cast<const float2*>(rec_of(k0 + lane) + N * D)[r]
                                    : make_float2(-INFINITY, 0.f);
        float4 o4[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
          o4[u] = u < kn ? reinterpret_cast<const float4*>(rec_of(k0 + u) + r * D)[lane]
                         : make_float4(0.f, 0.f, 0.f, 0.f);
        float Mb = ml.x;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) Mb = fmaxf(Mb, __shfl_xor_sync(kFull, Mb, o));
        const float Mn = fmaxf(M, Mb);
        if (Mn == -INFINITY) continue;  // uniform: no key in these pieces yet
        const float rs = M == -INFINITY ? 0.f : fast_exp2(M - Mn);  // what is folded in so far
        acc.x *= rs;
        acc.y *= rs;
        acc.z *= rs;
        acc.w *= rs;
        l *= rs;
        M = Mn;
        const float wk = ml.x == -INFINITY ? 0.f : fast_exp2(ml.x - M);
        float lk = ml.y * wk;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) lk += __shfl_xor_sync(kFull, lk, o);
        l += lk;
        for (int kk = 0; kk < kn; kk += 4) {
          if (kk > 0) {
#pragma unroll
            for (int u = 0; u < 4; ++u)
              o4[u] = kk + u < kn ? reinterpret_cast<const float4*>(rec_of(k0 + kk + u) + r * D)[lane]
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float wb = __shfl_sync(kFull, wk, (kk + u) & 31);
            if (kk + u < kn) {
              acc.x = fmaf(o4[u].x, wb, acc.x);
              acc.y = fmaf(o4[u].y, wb, acc.y);
              acc.z = fmaf(o4[u].z, wb, acc.z);
              acc.w = fmaf(o4[u].w, wb, acc.w);
            }
          }
        }
      }
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const int cg = rc * N + r;
      const int mem = cg / rpm, i = (cg - mem * rpm) / p.group;
      const int gg = cg - mem * rpm - i * p.group;
      uint2 packed;
      packed.x = pack_bf16x2(acc.x * inv, acc.y * inv);
      packed.y = pack_bf16x2(acc.z * inv, acc.w * inv);
      reinterpret_cast<uint2*>(p.out + (static_cast<size_t>((b0 + mem) * p.q_per_seq + i) * p.num_q_heads +
                                        kvh * p.group + gg) * D)[lane] = packed;
    }
  }
  // sequences without a visible key (context length 0) get zero rows
  const int rq = p.q_per_seq * p.num_q_heads;
  for (int b = c; b < p.num_seqs; b += gridDim.x) {
    if (num_blocks_of(p, __ldg(p.context_lens + b)) != 0) continue;
    uint16_t* o = p.out + static_cast<size_t>(b) * rq * D;
    for (int e = threadIdx.x; e < rq * D; e += blockDim.x) o[e] = 0;
  }
}

// Prefix sharing: the shared prefix of each window of `cap` consecutive sequences, in
// blocks: the longest run of table entries from position 0 on that all members share,
// at most the blocks every member sees whole from every query row
// (floor((ctx - q + 1) / 16)); 0 for a window of one sequence. One CTA per window.
__global__ void __launch_bounds__(256) tcm_share_prepass(const DecodeParams p) {
  grid_dependency_wait();
  __shared__ int first_diff;
  const int cap = p.share_cap;
  const int w = blockIdx.x;
  const int b0 = w * cap;
  const int m = min(cap, p.num_seqs - b0);
  __shared__ int pcap_s;
  if (threadIdx.x == 0) {
    first_diff = INT_MAX;
    pcap_s = m >= 2 ? INT_MAX : 0;
  }
  __syncthreads();
  if (m >= 2 && static_cast<int>(threadIdx.x) < m) {  // thread jj: member jj (cap <= 32)
    const int cx = __ldg(p.context_lens + b0 + threadIdx.x);
    atomicMin(&pcap_s, min(max(cx - p.q_per_seq + 1, 0) / kBlockSize, num_blocks_of(p, cx)));
  }
  __syncthreads();
  const int pcap = pcap_s;
  // every (position, member) pair is one independent comparison with the first member
  const int32_t* lead = p.block_tables + static_cast<size_t>(b0) * p.max_blocks;
  const int pairs = m >= 2 ? pcap * (m - 1) : 0;
  int mine = INT_MAX;
#pragma unroll 4
  for (int idx = threadIdx.x; idx < pairs; idx += blockDim.x) {
    const int x = idx / (m - 1);
    const int jj = 1 + (idx - x * (m - 1));
    if (__ldg(lead + static_cast<size_t>(jj) * p.max_blocks + x) != __ldg(lead + x)) mine = min(mine, x);
  }
  if (mine != INT_MAX) atomicMin(&first_diff, mine);
  __syncthreads();
  if (threadIdx.x == 0) p.win_prefix[w] = min(pcap, first_diff);
  grid_launch_dependents();
}

}  // namespace pa
