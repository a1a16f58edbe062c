// PagedAttention oracle: plain, slow, fp64 CPU restatement of what the paged
// KV-cache hot path computes (cache write, paged decode), and of the copy-on-write
// block copy.
//
// TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the CPU-baseline
// leg of the benchmark may load this library. The CUDA library never includes,
// links or calls it, and it shares no header, helper or constant with the CUDA
// sources.
//
// Sources (web pages; cited by title and section):
//   [DS] "vLLM 深度实战：从 PagedAttention 到 Speculative Decoding"
//        (chenxutan.com/d/2880), §3.2 KV Cache Block, §3.3 PagedAttention 的实现细节
//   [VS] vLLM study notes (zihan-zhang.net/vLLM-study), §1.1.1 (attention with a
//        causal mask), §1.2.1-1.2.2 (KV cache, size formula), §3.2 (block table,
//        page-wise read of K/V), §3.2.2 (sharing and copy-on-write), §4.3.1 (online
//        softmax)
//   [DP] "vLLM 深度解析：连续批处理与内存高效推理" (plumephp.com/ai-vllm-system),
//        §1.2 (KV size formula), §2.1 (block table, copy on write), §4.1 (block count
//        example), §4.2 (reference counts and sharing)
//
// Readings taken where the pages are silent or disagree (all stated here so the
// code can be checked against them by eye):
//   * Pool layout is [num_blocks][block_size][num_kv_heads][head_dim], token-major
//     with head_dim innermost ([VS] §3.2 gives K_pool[phys] as
//     [16, kv_heads, head_dim]; [DS] §3.3 prints a different, garbled order).
//   * slot = physical_block * block_size + offset ([DS] §3.3 address mapping);
//     a negative slot means "skip this token".
//   * A sequence with context length ctx owns ceil(ctx / block_size) blocks.
//   * GQA: query head h reads kv head h / (num_q_heads / num_kv_heads).
//   * The q_per_seq query tokens of a sequence sit at the last q_per_seq
//     positions: query token i is at position ctx - q_per_seq + i and sees keys
//     at positions 0..ctx - q_per_seq + i ([VS] §1.1.1 causal mask).
//   * A query row with no visible key has output 0.
//   * Sliding window W ([VS] §3.6.3: only the most recent W tokens are attended):
//     query token i sees keys max(0, pos - W + 1) .. pos, pos = ctx - q_per_seq + i.
//     Table entries wholly before every row's window are never read ([VS] §5.5 points
//     them at the null block 0).
//   * bf16 is widened to fp64 exactly (bit pattern << 16 is the fp32 value).
//   * FP8 KV cache ([VS] §4.2 names --kv-cache-dtype fp8 only): the E4M3 format, one fp32
//     scale per pool passed by the caller; stored code = nearest E4M3 (ties to even,
//     saturating at +-448) of the fp32 quotient x / scale; read value = code's value * scale.
//
// Parity pins for every function here live in the CPU test-suite (brute force
// contiguous attention, a library attention routine, closed forms, invariants,
// and the pages' worked numbers).
//
// ORACLE_MUTANT (compile-time, default 0) plants one plausible mistake; it
// exists only so the test-suite can show that its pins catch such mistakes.

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

namespace {

// Exact bf16 -> fp64 widening: a bf16 value is the upper 16 bits of an fp32.
double bf16_to_f64(uint16_t bits) {
#if ORACLE_MUTANT == 11
  uint32_t w = static_cast<uint32_t>(bits) << 15;  // planted: wrong shift
#else
  uint32_t w = static_cast<uint32_t>(bits) << 16;
#endif
  float f;
  std::memcpy(&f, &w, sizeof f);
  return static_cast<double>(f);
}

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Index of element (block, offset, kv_head, d) in the pool.
int64_t pool_index(int64_t block, int64_t offset, int64_t kv_head, int64_t d,
                   int64_t block_size, int64_t num_kv_heads, int64_t head_dim) {
#if ORACLE_MUTANT == 12
  // planted: head-major inside a block
  return ((block * num_kv_heads + kv_head) * block_size + offset) * head_dim + d;
#else
  return ((block * block_size + offset) * num_kv_heads + kv_head) * head_dim + d;
#endif
}

struct Shape {
  int num_seqs, q_per_seq, num_q_heads, num_kv_heads, head_dim, block_size;
  int max_blocks_per_seq;
  int64_t num_blocks;
  int window;  // sliding window in tokens; 0 = none
  // FP8 pools (E4M3 codes) and their per-pool scales; null: the bf16 pools
  const uint8_t* k8 = nullptr;
  const uint8_t* v8 = nullptr;
  double k_scale = 1.0, v_scale = 1.0;
};

// ---- FP8 E4M3 ([VS] §4.2: an FP8 KV cache, --kv-cache-dtype fp8) ----
// The 8-bit floating-point format E4M3: 1 sign bit, 4 exponent bits with bias 7, 3 mantissa
// bits; exponent field 0 holds the subnormals m * 2^-9; no infinities; S.1111.111 is NaN; the
// largest finite value is 1.75 * 2^8 = 448.
double fp8_e4m3_decode(uint8_t c) {
  const int e = (c >> 3) & 0xF, m = c & 7;
  double v;
  if (e == 15 && m == 7) {
    v = std::nan("");
  } else if (e == 0) {
    v = std::ldexp(static_cast<double>(m), -9);
  } else {
#if ORACLE_MUTANT == 42
    v = std::ldexp(1.0 + m / 8.0, e - 8);  // planted: exponent bias 8
#else
    v = std::ldexp(1.0 + m / 8.0, e - 7);
#endif
  }
  return (c & 0x80) ? -v : v;
}

// Nearest E4M3 code of x, ties to the even code; finite values above 448 in magnitude and
// infinities saturate to +-448; NaN gives 0x7F.
uint8_t fp8_e4m3_encode(float x) {
  if (std::isnan(x)) return 0x7F;
  const uint8_t sign = std::signbit(x) ? 0x80 : 0x00;
  const double a = std::fabs(static_cast<double>(x));
#if ORACLE_MUTANT == 43
  if (a >= 448.0) return sign | 0x7F;  // planted: out-of-range values become NaN
#else
  if (a >= 448.0) return sign | 0x7E;
#endif
  // the grid spacing of a's binade: 2^-9 below the smallest normal 2^-6, else 2^(e-3)
  int e2 = 0;
  std::frexp(a, &e2);                   // a = f * 2^e2, f in [0.5, 1)
  const int e = a < std::ldexp(1.0, -6) ? -6 : e2 - 1;   // a in [2^e, 2^(e+1))
  const double spacing = std::ldexp(1.0, e - 3);
  const double units = a / spacing;     // exact: a power-of-two scaling
  double q = std::floor(units);
#if ORACLE_MUTANT == 41
  (void)0;  // planted: truncation instead of rounding to nearest
#else
  const double frac = units - q;
  if (frac > 0.5 || (frac == 0.5 && std::fmod(q, 2.0) != 0.0)) q += 1.0;
#endif
  // q * 2^(e-3): subnormal (e = -6, q < 8), or 1.mmm * 2^e with q in [8, 16]
  int code;
  if (e == -6 && q < 8.0) {
    code = static_cast<int>(q);
  } else {
    int ee = e, mq = static_cast<int>(q);
    if (mq == 16) {
      mq = 8;
      ++ee;
    }
    code = ((ee + 7) << 3) | (mq - 8);
  }
  if (code >= 0x7F) code = 0x7E;  // not reached for a < 448; kept as a guard
  return static_cast<uint8_t>(sign | code);
}

// Gather the keys and values of one (sequence, kv head) into contiguous fp64
// arrays [ctx][head_dim], walking the block table as [DS] §3.3 and [VS] §3.2 do:
// token i lives in physical block block_table[i / block_size] at offset
// i % block_size. Positions before `from` are not read (they stay 0): no query row
// sees them, and their table entries may name the null block. Returns false if the
// table points outside the pool.
bool gather_kv(const uint16_t* key_cache, const uint16_t* value_cache,
               const int32_t* table_row, int ctx, int kv_head, const Shape& s,
               std::vector<double>& k_out, std::vector<double>& v_out, int from = 0) {
  k_out.assign(static_cast<size_t>(ctx) * s.head_dim, 0.0);
  v_out.assign(static_cast<size_t>(ctx) * s.head_dim, 0.0);
  for (int i = from; i < ctx; ++i) {
    int64_t logical_block = i / s.block_size;
#if ORACLE_MUTANT == 1
    int64_t offset = (i / s.block_size) % s.block_size;  // planted: wrong offset
#else
    int64_t offset = i % s.block_size;
#endif
    int64_t phys = table_row[logical_block];
    if (phys < 0 || phys >= s.num_blocks) return false;
    for (int d = 0; d < s.head_dim; ++d) {
      int64_t idx = pool_index(phys, offset, kv_head, d, s.block_size,
                               s.num_kv_heads, s.head_dim);
      if (s.k8) {  // FP8 pools: the code's value times the pool's scale (exact in fp64)
        k_out[static_cast<size_t>(i) * s.head_dim + d] = fp8_e4m3_decode(s.k8[idx]) * s.k_scale;
        v_out[static_cast<size_t>(i) * s.head_dim + d] = fp8_e4m3_decode(s.v8[idx]) * s.v_scale;
      } else {
        k_out[static_cast<size_t>(i) * s.head_dim + d] = bf16_to_f64(key_cache[idx]);
        v_out[static_cast<size_t>(i) * s.head_dim + d] = bf16_to_f64(value_cache[idx]);
      }
    }
  }
  return true;
}

// Attention of one query row against contiguous K/V, by the definition
// softmax(q K^T * scale) V over the visible keys first_visible..last_visible
// ([VS] §1.1.1; first_visible > 0 only under a sliding window). Two passes: first
// the maximum score, then the weights; no online rescaling.
void attend_row(const double* q, const std::vector<double>& k,
                const std::vector<double>& v, int first_visible, int last_visible,
                int head_dim, double scale, double* out) {
  for (int d = 0; d < head_dim; ++d) out[d] = 0.0;
  if (last_visible < first_visible) return;  // no visible key: output defined as 0
  const int n = last_visible - first_visible + 1;
  std::vector<double> score(n);
  for (int j = 0; j < n; ++j) {
    const size_t t = static_cast<size_t>(first_visible + j);
    double dot = 0.0;
    for (int d = 0; d < head_dim; ++d) {
#if ORACLE_MUTANT == 8
      dot += q[d] * v[t * head_dim + d];  // planted: V for K
#else
      dot += q[d] * k[t * head_dim + d];
#endif
    }
#if ORACLE_MUTANT == 5
    score[j] = dot;  // planted: scale dropped
#else
    score[j] = dot * scale;
#endif
  }
  double m = score[0];
  for (int j = 1; j < n; ++j) m = std::max(m, score[j]);
  double denom = 0.0;
  for (int j = 0; j < n; ++j) {
    const size_t t = static_cast<size_t>(first_visible + j);
    double w = std::exp(score[j] - m);
    denom += w;
    for (int d = 0; d < head_dim; ++d) out[d] += w * v[t * head_dim + d];
  }
#if ORACLE_MUTANT == 6
  (void)denom;  // planted: missing normalisation
#else
  for (int d = 0; d < head_dim; ++d) out[d] /= denom;
#endif
}

// Last key position visible to query token i of a sequence with ctx tokens.
int last_visible_position(int ctx, int q_per_seq, int i) {
#if ORACLE_MUTANT == 3
  return ctx - q_per_seq + i - 1;  // planted: strict causal inequality
#elif ORACLE_MUTANT == 7
  (void)q_per_seq; (void)i;
  return ctx - 1;  // planted: no causal window for speculative rows
#else
  return ctx - q_per_seq + i;
#endif
}

// First key position visible to a query whose last visible key is `last`. A sliding
// window of W tokens ([VS] §3.6.3: a Mistral-style window attends to the most recent W
// tokens only) starts at last - W + 1 (at least 0); without a window (W <= 0), at 0.
int first_visible_position(int last, int window) {
  if (window <= 0) return 0;
#if ORACLE_MUTANT == 13
  return std::max(0, last - window);  // planted: one key too many
#else
  return std::max(0, last - window + 1);
#endif
}

int kv_head_of(int q_head, int num_q_heads, int num_kv_heads) {
#if ORACLE_MUTANT == 2
  (void)num_q_heads;
  return q_head % num_kv_heads;  // planted: interleaved grouping
#else
  return q_head / (num_q_heads / num_kv_heads);
#endif
}

const int32_t* table_row_of(const int32_t* block_tables, int b, const Shape& s,
                            const int32_t* context_lens) {
#if ORACLE_MUTANT == 9
  // planted: rows packed by used length instead of max_blocks_per_seq
  int64_t off = 0;
  for (int j = 0; j < b; ++j) off += ceil_div(context_lens[j], s.block_size);
  return block_tables + off;
#else
  (void)context_lens;
  return block_tables + static_cast<int64_t>(b) * s.max_blocks_per_seq;
#endif
}

int g_threads_used = 0;

int resolve_threads(int requested) {
  if (requested > 0) return requested;
  unsigned hc = std::thread::hardware_concurrency();
  return hc == 0 ? 1 : static_cast<int>(hc);
}

// Computes the rows listed in `rows` ((b, i, h) triples) into out[r][head_dim].
// Work is split over (sequence, kv head) pairs so each gather is done once.
int decode_rows_impl(double* out, const uint16_t* query, const uint16_t* key_cache,
                     const uint16_t* value_cache, const int32_t* block_tables,
                     const int32_t* context_lens, const Shape& s, double scale,
                     const int32_t* rows, int64_t n_rows, int num_threads) {
  if (s.num_q_heads % s.num_kv_heads != 0) return 1;
  // Bucket requested rows by (b, kv_head).
  const int64_t units = static_cast<int64_t>(s.num_seqs) * s.num_kv_heads;
  std::vector<std::vector<int64_t>> by_unit(units);
  for (int64_t r = 0; r < n_rows; ++r) {
    int b = rows[3 * r], i = rows[3 * r + 1], h = rows[3 * r + 2];
    if (b < 0 || b >= s.num_seqs || i < 0 || i >= s.q_per_seq || h < 0 ||
        h >= s.num_q_heads)
      return 2;
    int kvh = kv_head_of(h, s.num_q_heads, s.num_kv_heads);
    by_unit[static_cast<int64_t>(b) * s.num_kv_heads + kvh].push_back(r);
  }
  for (int b = 0; b < s.num_seqs; ++b) {
    int ctx = context_lens[b];
    if (ctx < 0 || ceil_div(ctx, s.block_size) > s.max_blocks_per_seq) return 3;
  }
  std::atomic<int64_t> next{0};
  std::atomic<int> err{0};
  auto worker = [&]() {
    std::vector<double> k, v, qrow(s.head_dim);
    for (;;) {
      int64_t u = next.fetch_add(1);
      if (u >= units) break;
      if (by_unit[u].empty()) continue;
      int b = static_cast<int>(u / s.num_kv_heads);
      int kvh = static_cast<int>(u % s.num_kv_heads);
      int ctx = context_lens[b];
      // the lowest first-visible position of the sequence's query rows (row 0's)
      const int from = std::max(0, first_visible_position(last_visible_position(ctx, s.q_per_seq, 0), s.window));
      if (!gather_kv(key_cache, value_cache, table_row_of(block_tables, b, s, context_lens),
                     ctx, kvh, s, k, v, std::min(from, ctx))) {
        err.store(4);
        continue;
      }
      for (int64_t r : by_unit[u]) {
        int i = rows[3 * r + 1], h = rows[3 * r + 2];
        const uint16_t* qsrc =
            query + ((static_cast<int64_t>(b) * s.q_per_seq + i) * s.num_q_heads + h) * s.head_dim;
        for (int d = 0; d < s.head_dim; ++d) qrow[d] = bf16_to_f64(qsrc[d]);
        const int last = last_visible_position(ctx, s.q_per_seq, i);
        attend_row(qrow.data(), k, v, first_visible_position(last, s.window), last,
                   s.head_dim, scale, out + r * s.head_dim);
      }
    }
  };
  int nt = static_cast<int>(std::min<int64_t>(resolve_threads(num_threads), std::max<int64_t>(units, 1)));
  g_threads_used = nt;
  std::vector<std::thread> pool;
  for (int t = 1; t < nt; ++t) pool.emplace_back(worker);
  worker();
  for (auto& th : pool) th.join();
  return err.load();
}

}  // namespace

extern "C" {

// bf16 bit pattern -> fp64 (exact).
double oracle_bf16_to_f64(uint16_t bits) { return bf16_to_f64(bits); }

// Number of blocks a sequence of n tokens occupies ([DS] §3.2, [DP] §4.1).
int64_t oracle_blocks_for_tokens(int64_t n_tokens, int64_t block_size) {
  return ceil_div(n_tokens, block_size);
}

// KV-cache bytes per token of a whole model: 2 (K and V) x layers x kv heads x
// head_dim x bytes per value ([VS] §1.2.2, [DP] §1.2).
int64_t oracle_kv_bytes_per_token(int64_t layers, int64_t kv_heads, int64_t head_dim,
                                  int64_t bytes_per_value) {
  return 2 * layers * kv_heads * head_dim * bytes_per_value;
}

// Cache write: for every token t with slot_mapping[t] >= 0, copy the bf16 bit
// patterns of key[t] and value[t] ([num_kv_heads][head_dim], rows `key_stride` /
// `value_stride` elements apart) into pool row slot = block * block_size + offset.
// Every other pool element is left untouched. Returns 0, or 1 for an
// out-of-range slot (nothing is written for that token).
int oracle_reshape_and_cache(const uint16_t* key, const uint16_t* value,
                             int64_t key_stride, int64_t value_stride,
                             uint16_t* key_cache, uint16_t* value_cache,
                             const int64_t* slot_mapping, int64_t num_tokens,
                             int num_kv_heads, int head_dim, int64_t num_blocks,
                             int block_size) {
  int status = 0;
  for (int64_t t = 0; t < num_tokens; ++t) {
    int64_t slot = slot_mapping[t];
    if (slot < 0) continue;
    int64_t block = slot / block_size;
    int64_t offset = slot % block_size;
#if ORACLE_MUTANT == 10
    offset = (offset + 1) % block_size;  // planted: off-by-one slot
#endif
    if (block >= num_blocks) {
      status = 1;
      continue;
    }
    for (int h = 0; h < num_kv_heads; ++h) {
      for (int d = 0; d < head_dim; ++d) {
        int64_t dst = pool_index(block, offset, h, d, block_size, num_kv_heads, head_dim);
        key_cache[dst] = key[t * key_stride + static_cast<int64_t>(h) * head_dim + d];
        value_cache[dst] = value[t * value_stride + static_cast<int64_t>(h) * head_dim + d];
      }
    }
  }
  return status;
}

// Paged decode attention, every row: out[b][i][h][d] (fp64) for b < num_seqs,
// i < q_per_seq, h < num_q_heads. block_tables is [num_seqs][max_blocks_per_seq],
// context_lens[b] counts all tokens of sequence b including its q_per_seq new
// ones. window > 0: a sliding window of that many tokens ending at each query's
// position (table entries wholly before the window are not read; the pages point them
// at the null block 0, [VS] §5.5); window <= 0: none. num_threads <= 0 uses every
// hardware thread. Returns 0 on success.
int oracle_decode_window(double* out, const uint16_t* query, const uint16_t* key_cache,
                         const uint16_t* value_cache, const int32_t* block_tables,
                         const int32_t* context_lens, int num_seqs, int q_per_seq,
                         int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                         int max_blocks_per_seq, int64_t num_blocks, double scale,
                         int window, int num_threads) {
  Shape s{num_seqs, q_per_seq, num_q_heads, num_kv_heads, head_dim, block_size,
          max_blocks_per_seq, num_blocks, window};
  const int64_t n_rows = static_cast<int64_t>(num_seqs) * q_per_seq * num_q_heads;
  std::vector<int32_t> rows(3 * n_rows);
  int64_t r = 0;
  for (int b = 0; b < num_seqs; ++b)
    for (int i = 0; i < q_per_seq; ++i)
      for (int h = 0; h < num_q_heads; ++h, ++r) {
        rows[3 * r] = b;
        rows[3 * r + 1] = i;
        rows[3 * r + 2] = h;
      }
  return decode_rows_impl(out, query, key_cache, value_cache, block_tables, context_lens,
                          s, scale, rows.data(), n_rows, num_threads);
}

// Same as oracle_decode_window for a chosen list of rows: rows holds n_rows (b, i, h)
// triples and out receives n_rows x head_dim values in that order. Used to
// check sampled outputs of full-size problems.
int oracle_decode_rows_window(double* out, const uint16_t* query, const uint16_t* key_cache,
                              const uint16_t* value_cache, const int32_t* block_tables,
                              const int32_t* context_lens, int num_seqs, int q_per_seq,
                              int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                              int max_blocks_per_seq, int64_t num_blocks, double scale,
                              const int32_t* rows, int64_t n_rows, int window, int num_threads) {
  Shape s{num_seqs, q_per_seq, num_q_heads, num_kv_heads, head_dim, block_size,
          max_blocks_per_seq, num_blocks, window};
  return decode_rows_impl(out, query, key_cache, value_cache, block_tables, context_lens,
                          s, scale, rows, n_rows, num_threads);
}

// Copy-on-write block copy ([VS] §3.2.2 写时复制: a sequence about to write into a block
// that other sequences still reference first gets a private copy of it; [DP] §2.1 and
// §4.2: the same at the forks of parallel sampling and beam search). Each pair p of
// `mapping` ([num_pairs][2] = {source block, destination block}) copies every element of
// the source block (block_elems = block_size x num_kv_heads x head_dim values, in the key
// pool and in the value pool) onto the destination block; every other block is left as it
// was. A pair with a negative entry is padding and is skipped. Returns 0; 1 if an id is
// past the pool, 2 if a destination repeats or is also a source (the result would then
// depend on the order of the copies); nothing is copied in either error case.
int oracle_copy_blocks(uint16_t* key_cache, uint16_t* value_cache, int64_t num_blocks,
                       int64_t block_elems, const int64_t* mapping, int64_t num_pairs) {
  for (int64_t p = 0; p < num_pairs; ++p) {
    const int64_t src = mapping[2 * p], dst = mapping[2 * p + 1];
    if (src < 0 || dst < 0) continue;
    if (src >= num_blocks || dst >= num_blocks) return 1;
    for (int64_t o = 0; o < num_pairs; ++o) {
      const int64_t os = mapping[2 * o], od = mapping[2 * o + 1];
      if (os < 0 || od < 0) continue;
      if (od == dst && o != p) return 2;
      if (os == dst) return 2;
    }
  }
  for (int64_t p = 0; p < num_pairs; ++p) {
#if ORACLE_MUTANT == 33
    const int64_t src = mapping[2 * p + 1], dst = mapping[2 * p];  // planted: pair reversed
#else
    const int64_t src = mapping[2 * p], dst = mapping[2 * p + 1];
#endif
    if (src < 0 || dst < 0) continue;
#if ORACLE_MUTANT == 32
    const int64_t n = block_elems - block_elems / 16;  // planted: the last token left behind
#else
    const int64_t n = block_elems;
#endif
    for (int64_t e = 0; e < n; ++e) {
      key_cache[dst * block_elems + e] = key_cache[src * block_elems + e];
#if ORACLE_MUTANT != 31  // planted (31): the value pool is not copied
      value_cache[dst * block_elems + e] = value_cache[src * block_elems + e];
#endif
    }
  }
  return 0;
}

// Without a sliding window: every key up to the query's position is visible.
int oracle_decode(double* out, const uint16_t* query, const uint16_t* key_cache,
                  const uint16_t* value_cache, const int32_t* block_tables,
                  const int32_t* context_lens, int num_seqs, int q_per_seq,
                  int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                  int max_blocks_per_seq, int64_t num_blocks, double scale,
                  int num_threads) {
  return oracle_decode_window(out, query, key_cache, value_cache, block_tables, context_lens,
                              num_seqs, q_per_seq, num_q_heads, num_kv_heads, head_dim,
                              block_size, max_blocks_per_seq, num_blocks, scale, 0, num_threads);
}

int oracle_decode_rows(double* out, const uint16_t* query, const uint16_t* key_cache,
                       const uint16_t* value_cache, const int32_t* block_tables,
                       const int32_t* context_lens, int num_seqs, int q_per_seq,
                       int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                       int max_blocks_per_seq, int64_t num_blocks, double scale,
                       const int32_t* rows, int64_t n_rows, int num_threads) {
  return oracle_decode_rows_window(out, query, key_cache, value_cache, block_tables,
                                   context_lens, num_seqs, q_per_seq, num_q_heads,
                                   num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                                   num_blocks, scale, rows, n_rows, 0, num_threads);
}

// FP8 E4M3 codes of n fp32 values, and the values of n codes (for the format's pins).
void oracle_fp8_encode(const float* x, uint8_t* codes, int64_t n) {
  for (int64_t i = 0; i < n; ++i) codes[i] = fp8_e4m3_encode(x[i]);
}
void oracle_fp8_decode(const uint8_t* codes, double* x, int64_t n) {
  for (int64_t i = 0; i < n; ++i) x[i] = fp8_e4m3_decode(codes[i]);
}

// Cache write into FP8 pools ([VS] §4.2). Each bf16 element x of key[t] is stored as the
// E4M3 code of the fp32 quotient x / k_scale (value: / v_scale), at the same pool position as
// oracle_reshape_and_cache; every other pool byte is left untouched. Returns 0, or 1 for an
// out-of-range slot.
int oracle_reshape_and_cache_fp8(const uint16_t* key, const uint16_t* value, int64_t key_stride,
                                 int64_t value_stride, uint8_t* key_cache, uint8_t* value_cache,
                                 const int64_t* slot_mapping, int64_t num_tokens, int num_kv_heads,
                                 int head_dim, int64_t num_blocks, int block_size, float k_scale,
                                 float v_scale) {
  int status = 0;
  for (int64_t t = 0; t < num_tokens; ++t) {
    const int64_t slot = slot_mapping[t];
    if (slot < 0) continue;
    const int64_t block = slot / block_size, offset = slot % block_size;
    if (block >= num_blocks) {
      status = 1;
      continue;
    }
    for (int h = 0; h < num_kv_heads; ++h) {
      for (int d = 0; d < head_dim; ++d) {
        const int64_t dst = pool_index(block, offset, h, d, block_size, num_kv_heads, head_dim);
        const float k = static_cast<float>(bf16_to_f64(key[t * key_stride + static_cast<int64_t>(h) * head_dim + d]));
        const float v =
            static_cast<float>(bf16_to_f64(value[t * value_stride + static_cast<int64_t>(h) * head_dim + d]));
        key_cache[dst] = fp8_e4m3_encode(k / k_scale);
        value_cache[dst] = fp8_e4m3_encode(v / v_scale);
      }
    }
  }
  return status;
}

// Paged decode over FP8 pools: oracle_decode_window's definition with every key and value
// element read as its E4M3 code's value times the pool's scale.
int oracle_decode_fp8(double* out, const uint16_t* query, const uint8_t* key_cache,
                      const uint8_t* value_cache, const int32_t* block_tables,
                      const int32_t* context_lens, int num_seqs, int q_per_seq, int num_q_heads,
                      int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq,
                      int64_t num_blocks, double scale, double k_scale, double v_scale, int window,
                      int num_threads) {
  Shape s{num_seqs, q_per_seq, num_q_heads, num_kv_heads, head_dim, block_size,
          max_blocks_per_seq, num_blocks, window};
  s.k8 = key_cache;
  s.v8 = value_cache;
  s.k_scale = k_scale;
  s.v_scale = v_scale;
  const int64_t n_rows = static_cast<int64_t>(num_seqs) * q_per_seq * num_q_heads;
  std::vector<int32_t> rows(3 * n_rows);
  int64_t r = 0;
  for (int b = 0; b < num_seqs; ++b)
    for (int i = 0; i < q_per_seq; ++i)
      for (int h = 0; h < num_q_heads; ++h, ++r) {
        rows[3 * r] = b;
        rows[3 * r + 1] = i;
        rows[3 * r + 2] = h;
      }
  return decode_rows_impl(out, query, nullptr, nullptr, block_tables, context_lens, s, scale, rows.data(),
                          n_rows, num_threads);
}

// Threads the last decode call ran on.
int oracle_threads_used() { return g_threads_used; }

int oracle_mutant_id() { return ORACLE_MUTANT; }

}  // extern "C"
