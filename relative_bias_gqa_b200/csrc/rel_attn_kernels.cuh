// rel_attn_kernels.cuh -- sm_100a kernels of relative-bias GQA decode.
//
// Partial kernel, one CTA per (KV split, KV head, sequence):
//   warp 0      TMA producer: walks the split's pages through the block table
//               and streams K/V page tiles (and relative-table row chunks)
//               into a ring of 64 KB shared-memory stages.
//   warp 1      S / X issuer, and after the softmax warps a P.V issuer (one
//               thread each): tcgen05.mma with fp32 accumulators
//               in tensor memory, "swap-AB" orientation so that keys (and
//               head-dim for P.V) fill the 128-row M side and the GQA
//               group's G heads x T tokens are the N side:
//                 S^T = K . Q^T           (128 keys x N)
//                 X^T = R_chunk . Q^T     (136 relative rows x N)
//                 O^T = V^T . P^T         (128 dims x N)
//   softmax     NG groups of 4 warps (one key / one head-dim lane per thread).
//               One token: two groups, group g takes the tiles i with
//               i % 2 == g, so two tiles' softmax run at once (each group
//               keeps its own running max / sum / output and its own
//               relative-row chunk; the two partial states are merged by LSE
//               at the end).  Several tokens: every group takes every tile
//               and its own block of the query rows (two groups up to five
//               tokens, four beyond).  Per tile: tcgen05.ld of S^T, relative term sheared into place
//               through a shared-memory table indexed by bucket(distance),
//               masks, fp32 online softmax in the log2 domain, P to shared
//               memory (bf16 hi + lo, 128B-swizzled), O^T tile accumulated in
//               registers.
// Combine kernel: LSE-merge of the per-split partial results.
//
// The dense relative product followed by a distance-indexed gather is the
// "sheared-bias" idea of "vLLM TML Inkling 지원", section "저지연 컬렉티브 및
// 커널" (FA4 bullet); packing the GQA group's heads into one MMA tile is the
// idea of "vLLM、Inkling 2 Smallを初日サポート GB200で630 tok/s", section
// "vLLMの最適化と性能" (Gluon decode-kernel bullet).  Both are re-laid out
// here for tcgen05: keys on the 128-row side, the group (6 heads x T tokens,
// padded to 16/32/48) on the N side.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "sm100_ptx.cuh"


namespace relattn {

constexpr int kHeadDim = 128;
constexpr int kPage = 64;
constexpr int kMaxQTokens = 9;                 // query tokens per sequence (speculative verify)
constexpr int kTileKeys = 128;                 // two pages per tile
constexpr int kMaxTailBuckets = 512;           // log buckets supported
constexpr int kSoftmaxThreads = 128;           // one softmax group
// named barriers: 1 .. NG one per softmax group, then these two
constexpr int kBarSoftmaxAll = 5;              // every softmax thread (epilogue)
constexpr int kBarSetup = 6;                   // every warp but the producer (prologue)
// Softmax groups of the instance for G heads per KV head and T query tokens:
// four from six tokens on where each group then carries at most 12 rows of
// S^T (a thread's per-tile work halves and every SM sub-partition runs four
// softmax warps to hide each other's latencies), and always past 48 query
// rows (the 64-wide instances); else two.
__host__ __device__ constexpr int softmax_groups(int G, int T, bool f8 = false) {
  // E4M3 cache (the softmax warps also widen the codes): four groups from
  // four tokens on spread that work over 16 warps; measured on the 256K
  // verify step at G = 6, 4 tokens 257 against 298 us, 5 tokens 328 against
  // 341; 100K keys at G = 8, 4 tokens 119 against 135, but 5 tokens 169
  // against 158 (that instance spills), so G = 8 keeps two groups there.
  if (f8 && (T == 4 || (T == 5 && G <= 6))) return 4;
  // Six and nine tokens: three groups of two / three tokens.  On the 256K
  // verify step at G = 6: 221 against 265 us (four groups, 1 / 2 / 1 / 2
  // tokens) and 374 against 501 us (2 / 2 / 2 / 3); on 100K keys at G = 8
  // with six tokens 118 against 130 us (two groups), at G = 4 with six and
  // nine 159 and 177 against 171 and 197 us (four groups).  Uneven thirds
  // lose: 7 and 8 tokens at G = 6 took 368 and 377 us with three groups
  // against 258 and 247 with four, 7 at G = 8 205 against 199.
  if (T >= 6 && T % 3 == 0) return 3;
  return (T >= 6 && ((T + 3) / 4 * G <= 12 || G * T > 48)) ? 4 : 2;
}
constexpr int kVSlotBytes = 32768;             // V tile: 128 keys x 128 dims bf16
constexpr int kHalfTileBytes = 16384;          // 128 rows x 128 B (one 64-dim half)
constexpr int kPageHalfBytes = 8192;           // 64 rows x 128 B
constexpr unsigned kStatusTimeout = 1u;
constexpr unsigned kStatusBadSeq = 2u;
constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;  // 2 s
// Bound of the waits that let work already issued (TMA copies, MMAs) finish
// before a CTA releases its memory.  Fixed, whatever limit the caller sets
// for the other waits: such work always completes, and giving up on it
// early would free shared or tensor memory that it still writes.
constexpr unsigned long long kDrainLimitNs = 2000000000ull;        // 2 s
// Lazy-max slack (log2 units): p = exp2(x - m_ref) may reach 2^64, far
// inside fp32 / bf16 range even summed over 2^31 keys.
constexpr float kLazyLog2 = 64.f;
// Reference max of a row before its first valid logit: finite, so that
// exp2(x - m) and exp2(m_old - m_new) need no special case (any finite
// logit exceeds it by more than kLazyLog2 and sets a real reference).
constexpr float kNoMax = -1.0e30f;

struct alignas(64) DecodeParams {
  CUtensorMap tmap_k;   // K pool viewed as [num_pages*Hkv*P rows, 128] bf16
  CUtensorMap tmap_v;   // V pool, same view
  CUtensorMap tmap_r;   // relative table [Hkv][NB][128] bf16
  const __nv_bfloat16* q;
  const int* block_table;
  const int* seq_lens;
  void* out;
  float* lse;
  float* ws_lse;        // [S][rows]
  float* ws_o;          // [S][rows][128]
  unsigned* status;
  unsigned long long timeout_ns;
  int B, T, Hq, Hkv, num_pages, max_pages, num_splits, window, out_fp32;
  // Row mapping.  Grid z-index b is chunk (b % cps) of sequence (b / cps);
  // its T query tokens are rows tok(b) .. tok(b) + T - 1 of q / out / lse
  // (rows of Hq heads), tok(b) = (b / cps) * seq_stride + tok_off +
  // (b % cps) * T, and its context length is seq_lens[b / cps] - len_off -
  // (cps - 1 - b % cps) * T.  A decode step is cps = 1, seq_stride = T,
  // tok_off = len_off = 0; a chunked prefill runs cps chunks of T tokens of
  // one sequence, each attending causally to everything before it.
  int cps, seq_stride, tok_off, len_off;
  int rows_total;       // rows of the partial buffers: all query tokens x Hq
  int ex;               // distances d < ex are their own bucket
  int cost_exact;       // split weights of an exact-range and a narrow-bucket
  int cost_near;        // page (see split_pages)
  int nl;               // tail buckets: bucket = ex + max{k < nl : edges[k] <= d}
  float scale_log2;     // log2(e) / sqrt(D)
  float log2_ex, log_scale;  // tail-bucket guess: (log2(d) - log2_ex) * log_scale
  const float* k_scale;  // E4M3 KV cache only: per-KV-head scales
  const float* v_scale;
  int edges[kMaxTailBuckets + 1];
};

__host__ __device__ constexpr int align_up(int x, int a) { return (x + a - 1) / a * a; }

// Compile-time configuration of one kernel instance: N = padded group width
// (G heads x T tokens rounded up to the MMA N step), NG = softmax groups,
// G = query heads per KV head, T = query tokens, F8 = the KV cache holds E4M3
// codes (widened to bf16 in shared memory by the softmax warps).
// K tiles and relative-row chunks share one ring of slots (each slot is
// released as soon as its MMA has read it); V tiles have their own, deeper
// ring (a V slot is held until the P.V product of its tile).
template <int N, int NG, int G, int T, bool F8 = false>
struct KernelConfig {
  // N = 16 (one token): the softmax groups alternate tiles, each with all the
  // rows.  N = 32 / 48 / 64 (2..9 tokens): every group takes every tile, each
  // with its own block of rows (a column split of S^T, X^T and O^T).
  static constexpr bool kAlt = (N == 16);
  // warp 0 producer, warp 1 S / X issuer, the softmax warps, then the P.V
  // issuer.  Measured on B200 against one thread issuing both (256K-key
  // verify step): 4 tokens 210 -> 189 us, 6 tokens 222 -> 206, 8 tokens 238
  // -> 237; 100K keys at G = 8 with 8 tokens 146 -> 134; batched_32 1,945 ->
  // 1,702 (before the split heuristic changed).
  static constexpr int kPvWarp = 2 + 4 * NG;
  static constexpr int kThreads = 64 + kSoftmaxThreads * NG + 32;
  static constexpr int kConsumers = kAlt ? kSoftmaxThreads : kSoftmaxThreads * NG;  // arrivals per tile
  static constexpr int kXTables = kAlt ? NG : 1;               // relative chunks in flight (X, Y)
  // row capacity of a group: N / NG, or more when the tokens do not split
  // evenly (nine tokens over four groups: one group takes three)
  static constexpr int kGR = kAlt ? N : ((T + NG - 1) / NG * G > N / NG ? (T + NG - 1) / NG * G : N / NG);
  // relative rows per chunk: 128 cover one 128-key tile for one token; with
  // T tokens a tile needs 127 + T rows
  static constexpr int kRows = (N == 16) ? 128 : 136;
  static constexpr int kRHalfBytes = kRows * 128;
  static constexpr int kKSlotBytes = 2 * kRHalfBytes;          // >= one K tile (32 KB)
  // K slots turn over fast (freed by the S MMA), V slots slowly (held until
  // P.V), so the one-token instance gives V four of its six 32 KB slots.
  static constexpr int kKSlots = 2;
  static constexpr int kVSlots = (N == 16) ? 4 : (N == 32 ? 3 : 2);
  // P buffers: two, so that the softmax writes P(i+1) while P.V(i) still
  // reads P(i); the 64-wide instances keep one to fit shared memory (their
  // softmax then takes O(i-1), which proves P.V(i-1) done, before writing P(i))
  static constexpr int kPBufs = (N == 64) ? 1 : 2;
  static constexpr int kVLag = 0;                               // V issued this many tiles after K
  // Relative-table gather stride: odd for conflict-free gathers.  The N = 16
  // instance serves G live rows (one token).
  static constexpr int kYStride = (N == 16) ? (G % 2 == 0 ? G + 1 : G + 2) : N + 1;
  static constexpr int kOperandBytes = 2 * N * 128;            // N rows x 128 dims, two 64-dim halves
  static constexpr int kPBufBytes = 2 * kOperandBytes;         // [P_hi; P_lo]: 128 keys x 2N rows
  static constexpr int kYBytes = align_up(kRows * kYStride * 4, 16);
  static constexpr int oK = 0;
  static constexpr int oV = kKSlots * kKSlotBytes;
  static constexpr int oQ = oV + kVSlots * kVSlotBytes;
  static constexpr int oP = oQ + kOperandBytes;                // kPBufs P buffers
  static constexpr int oY = oP + kPBufs * kPBufBytes;          // one table per relative chunk in flight
  static constexpr int oRed = oY + kXTables * kYBytes;         // [NG][2][4][kGR]
  static constexpr int oAlpha = oRed + NG * 2 * 4 * kGR * 4;   // [NG][2][kGR]
  static constexpr int oEdges = oAlpha + NG * 2 * kGR * 4;
  static constexpr int oBar = align_up(oEdges + (kMaxTailBuckets + 1) * 4, 8);
  // barriers: kfull[KS], kempty[KS], vfull[VS], vempty[VS], s_full[2],
  //           s_empty[2], p_full[2], o_full[2], o_empty[2], x_full[kXTables],
  //           x_empty[kXTables], drain (S issuer), drain (P.V issuer),
  //           plan_full[kPlanSlots], plan_empty[kPlanSlots], and with an
  //           E4M3 cache kconv[KS] (the slot's item passed by every softmax
  //           warp: a K tile widened, a relative chunk let by)
  // Tile plans (column-split instances): the producer, which plans every
  // tile for its own loads, hands each plan to the softmax groups through a
  // ring of kPlanSlots records instead of every softmax thread re-planning.
  static constexpr int kPlanSlots = kAlt ? 0 : 4;
  static constexpr int kNumBars = 2 * kKSlots + 2 * kVSlots + 12 + 2 * kXTables + 2 * kPlanSlots +
                                  (F8 ? kKSlots : 0);
  // tmem base, abort flag, bad-page flag, K-ring and V-ring items issued
  static constexpr int oMisc = oBar + kNumBars * 8;
  // per K slot: 1 if its item is a relative-row chunk, 0 a K tile (producer
  // -> S issuer, published by the slot's full barrier)
  static constexpr int oItemFlag = oMisc + 32;
  static constexpr int oPlan = align_up(oItemFlag + kKSlots, 16);   // int4 {k_hi, c0, chunk, 0}
  static constexpr int kBytes = oPlan + 16 * kPlanSlots;
  static_assert(oPlan % 16 == 0, "16-byte plan records");
  static constexpr int kAllocBytes = kBytes + 1024;            // 1024-byte alignment slack
  // TMEM columns: S[2] (N each), O[2] (2N each: the P_hi and P_lo halves),
  // per group X0 (and X1 for 136-row chunks)
  static constexpr int kXCols = (kRows > 128) ? 2 * N : N;
  static constexpr int kTmemUsed = 6 * N + kXCols * kXTables;
  static constexpr int kTmemCols = (kTmemUsed <= 128) ? 128 : (kTmemUsed <= 256 ? 256 : 512);
  static_assert(kAllocBytes <= 232448, "shared memory budget exceeded");
  static_assert(kKSlotBytes >= 2 * kHalfTileBytes && oV % 1024 == 0 && oQ % 1024 == 0,
                "slot layout");
  // the epilogue exchanges the groups' rows through the K and V rings (idle
  // by then)
  static_assert(oQ >= NG * kGR * 128 * 4 * 2 + NG * kGR * 4 * 2, "epilogue exchange area");
};

// Column split of the query rows among NG softmax groups (T >= 2): group q
// takes tokens [tok_begin(q), tok_begin(q+1)) and the query slots from
// slot(q, A) on, slots packed with alignment A = 8 where that fits in N, else
// 4 (a 4-aligned group reads its tensor-memory columns from the 8-aligned
// column below and shifts by four).
__host__ __device__ constexpr int cs_tok_begin(int T, int NG, int q) { return q * T / NG; }
__host__ __device__ constexpr int cs_rows(int T, int G, int NG, int q) {
  return (cs_tok_begin(T, NG, q + 1) - cs_tok_begin(T, NG, q)) * G;
}
__host__ __device__ constexpr int cs_slot(int T, int G, int NG, int q, int a) {
  int s = 0;
  for (int u = 0; u < q; ++u) s = align_up(s + cs_rows(T, G, NG, u), a);
  return s;
}
__host__ __device__ constexpr int cs_end(int T, int G, int NG, int a) {
  return align_up(cs_slot(T, G, NG, NG - 1, a) + cs_rows(T, G, NG, NG - 1), a);
}

template <int T, int G, int NG>
struct ColSplit {
  __host__ __device__ static constexpr int tok_begin(int q) { return cs_tok_begin(T, NG, q); }
  __host__ __device__ static constexpr int rows(int q) { return cs_rows(T, G, NG, q); }
  __host__ __device__ static constexpr int slot(int q, int a) { return cs_slot(T, G, NG, q, a); }
  __host__ __device__ static constexpr int end(int a) { return cs_end(T, G, NG, a); }
  __host__ __device__ static constexpr int align(int n) { return end(8) <= n ? 8 : 4; }
  static constexpr int kMaxRows = (T + NG - 1) / NG * G;
};

// Group width N of the instance for G heads per KV head and T tokens (0: not
// supported): 16 for one token (the alternating-group instance, G <= 8);
// otherwise the smallest of 32 and 48 whose query slots hold every softmax
// group's row block 8-aligned, then (four groups) 64 8-aligned, then the
// smallest of 32 and 48 that holds them 4-aligned, then 64 4-aligned (past 48
// rows: G = 6 with 9 tokens).
__host__ __device__ constexpr int group_width_for(int G, int T, bool f8 = false) {
  if (G < 1 || G > 8 || T < 1 || T > kMaxQTokens) return 0;
  if (T == 1) return 16;
  const int NG = softmax_groups(G, T, f8);
  if (cs_end(T, G, NG, 8) <= 32) return 32;
  if (cs_end(T, G, NG, 8) <= 48) return 48;
  // four groups: 8-aligned blocks in a 64-wide tile beat 4-aligned ones in
  // a 48-wide tile (no shifted tensor-memory reads, 16-byte P stores;
  // measured on the 256K verify step: 261 against 286 us)
  if (NG == 4 && cs_end(T, G, NG, 8) <= 64) return 64;
  if (cs_end(T, G, NG, 4) <= 32) return 32;
  if (cs_end(T, G, NG, 4) <= 48) return 48;
  if (G * T > 48 && cs_end(T, G, NG, 4) <= 64) return 64;
  return 0;
}

// Per-CTA geometry shared by the three roles.
struct SplitGeom {
  int L, T, p0, W, lo, sp_begin, sp_end, ntiles;
};

struct TilePlan {
  int j0;       // first key of the tile
  int npg;      // pages loaded (1 or 2)
  int k_hi;     // tail-bucket index of the tile's largest distance (-1: exact region)
  bool chunk;   // a new relative-row chunk must be loaded before this tile
};

// Cursor state carried from tile to tile (one per softmax group: a group's
// tiles are planned against its own relative-row chunk).  Distances only
// shrink as the walk moves to later keys, so the tail-bucket indices are found
// by moving the cursors down the edge table.
struct PlanState {
  int c0 = 0;
  bool have = false;
  int k_hi, k_lo;
  __device__ explicit PlanState(int nl) : k_hi(nl - 1), k_lo(nl - 1) {}
};

// Largest k' <= k with edges[k'] <= d (edges[0] <= d is guaranteed).  The
// edges grow geometrically, so (log2(d) - log2_ex) * log_scale names the
// bucket up to rounding: the guess is checked against the table (one round of
// independent loads) and a binary search settles anything it does not pin.
__device__ __forceinline__ int seek_bucket(int k, int d, const int* edges, float log2_ex,
                                           float log_scale) {
  const float t = (__log2f((float)d) - log2_ex) * log_scale;
  int g = (t > 0.f) ? (int)fminf(t, 65536.f) : 0;         // NaN and negatives give 0
  g = min(g, k);
  const int em = edges[max(g - 1, 0)], e0 = edges[g];
  const int e1 = edges[min(g + 1, k)], e2 = edges[min(g + 2, k)];
  if (e0 <= d) {
    if (g == k || e1 > d) return g;
    if (g + 1 == k || e2 > d) return g + 1;
  } else if (g > 0 && em <= d) {
    return g - 1;
  }
  int lo = 0, hi = k;
#pragma unroll 1
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (edges[mid] <= d) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Out-of-line seek for the rare key whose bucket lies more than a few
// below its tile's largest (keeps the unrolled per-token code small).
__device__ __noinline__ int seek_bucket_far(int k, int d, const int* edges, float log2_ex,
                                            float log_scale) {
  return seek_bucket(k, d, edges, log2_ex, log_scale);
}

// Moves cursor k down to the tail bucket of d (d never lies above the
// cursor's bucket): usually no move or one step, else a seek.
__device__ __forceinline__ int step_down(int k, int d, const int* edges, float log2_ex,
                                         float log_scale) {
  if (k == 0 || edges[k] <= d) return k;
  if (edges[k - 1] <= d) return k - 1;
  return seek_bucket(k - 1, d, edges, log2_ex, log_scale);
}

// Pages [*begin, *end) of split s among S over the pages [first, last] a
// sequence's queries can see.  Splits are balanced by cost, not by page
// count: a page near the queries costs more than a far one (inside the
// exact-distance range every tile needs its own relative-row chunk, and up
// to a few thousand keys out the tail buckets are narrow), so the page at
// distance rank q from the query end is weighted 8 + cost_exact [q < QE] +
// cost_near [q < QN] eighths.  The cumulative cost from the query end is
// piecewise linear and is inverted per boundary; interior boundaries are
// rounded to an even page offset so that tiles stay two pages long.  The
// exact-range weight depends on the cache type: an exact-range tile also
// reads a 32 KB bf16 relative-row chunk, half again a bf16 tile's K and V
// bytes but twice an E4M3 tile's, and the E4M3 kernel keeps one chunk slot.
// Chosen on B200 by timing 100K-key batch-1 decode at 48/8 and 64/8 heads
// over 18 splits: bf16 3, 4 and 5 time alike; E4M3 8 / 11 / 14 / 17 / 21
// give 55.4 / 54.3 / 52.5 / 51.5 / 51.8 us per call at 48/8 heads (21 and
// more lose at 64/8); an E4M3 narrow-bucket weight of 2 then brings 64/8
// from 52.1 to 50.2 us (48/8 unchanged).
constexpr int kCostExactBf16 = 5, kCostNearBf16 = 1;
constexpr int kCostExactE4m3 = 17, kCostNearE4m3 = 2;
__host__ __device__ __forceinline__ void split_pages(int first, int last, int S, int s, int ex,
                                                     int cost_exact, int cost_near, int* begin,
                                                     int* end) {
  const int n = last - first + 1;
  const int qe = min(n, (ex + 128 + kPage - 1) / kPage + 1);   // pages holding exact-range keys
  const int qn = min(n, max(qe, 8 * ex / kPage));              // pages of the narrow tail buckets
  const int s1 = 8 + cost_exact + cost_near, s2 = 8 + cost_near;
  const int ce = s1 * qe;                                      // cost of the first qe pages
  const int cn = ce + s2 * (qn - qe);                          // ... of the first qn pages
  const int total = cn + 8 * (n - qn);                         // < 2^31 for n < 2^27 pages
  const int tq = total / S, tr = total % S;
  auto boundary = [&](int j) -> int {                           // page index of boundary j
    if (j <= 0) return last + 1;
    if (j >= S) return first;
    const int c = tq * j + tr * j / S;                         // floor(total * j / S)
    int q;
    if (c <= ce) q = (c + s1 - 1) / s1;
    else if (c <= cn) q = qe + (c - ce + s2 - 1) / s2;
    else q = qn + (c - cn + 7) / 8;
    const int b = last + 1 - min(q, n);
    return min(first + ((b - first + 1) & ~1), last + 1); // nearest even offset, ties toward the query
  };
  *begin = boundary(S - s);
  *end = boundary(S - 1 - s);
}

// Decides, for tile ti, the loaded pages and whether the relative-row chunk
// [c0, c0+ROWS) must move so that it covers every bucket the tile needs.
// All roles call it with identical arguments, so they agree on the sequence.
template <int ROWS>
__device__ __forceinline__ TilePlan plan_tile(const SplitGeom& g, int ti, int ex, float log2_ex,
                                              float log_scale, const int* edges, PlanState& st) {
  TilePlan t;
  const int pg = g.sp_begin + 2 * ti;
  t.j0 = pg * kPage;
  t.npg = min(2, g.sp_end - pg);
  const int ja = max(t.j0, g.lo);                          // first key anyone may see
  const int jb = min(t.j0 + t.npg * kPage, g.L) - 1;       // last key anyone may see
  int d_hi = (g.L - 1) - ja;
  if (g.W > 0) d_hi = min(d_hi, g.W - 1);
  const int d_lo = max(0, g.p0 - jb);
  int b_hi = d_hi, b_lo = d_lo;
  t.k_hi = -1;
  if (d_hi >= ex) {
    st.k_hi = step_down(st.k_hi, d_hi, edges, log2_ex, log_scale);
    t.k_hi = st.k_hi;
    b_hi = ex + st.k_hi;
  }
  if (d_lo >= ex) {
    st.k_lo = step_down(st.k_lo, d_lo, edges, log2_ex, log_scale);
    b_lo = ex + st.k_lo;
  }
  t.chunk = !(st.have && b_lo >= st.c0 && b_hi < st.c0 + ROWS);
  if (t.chunk) {
    st.c0 = max(0, b_hi - (ROWS - 1));
    st.have = true;
  }
  return t;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// First query-token row of grid z-index b (see DecodeParams).
__device__ __forceinline__ int first_token_row(const DecodeParams& p, int b) {
  const int bs = b / p.cps;
  return bs * p.seq_stride + p.tok_off + (b - bs * p.cps) * p.T;
}
// Context length of grid z-index b's query chunk, given its sequence's
// length L_seq.
__device__ __forceinline__ int chunk_seq_len(const DecodeParams& p, int b, int L_seq) {
  const int bs = b / p.cps;
  return L_seq - p.len_off - (p.cps - 1 - (b - bs * p.cps)) * p.T;
}

// Write this CTA's rows (all NQ rows of the group, every head-dim) with a
// constant value; used for empty splits and rejected sequences.  tok0 =
// the first query token's row.
template <int G>
__device__ void fill_rows(const DecodeParams& p, int tok0, int h, int s, float o_val, float lse_val) {
  const int rows = p.rows_total;
  const int NQ = p.T * G;
  for (int e = threadIdx.x; e < NQ * kHeadDim; e += blockDim.x) {
    const int n = e / kHeadDim, d = e % kHeadDim;
    const int t = n / G, gg = n % G;
    const int row = (tok0 + t) * p.Hq + h * G + gg;
    if (p.num_splits == 1) {
      if (p.out_fp32) reinterpret_cast<float*>(p.out)[(size_t)row * kHeadDim + d] = o_val;
      else reinterpret_cast<__nv_bfloat16*>(p.out)[(size_t)row * kHeadDim + d] = __float2bfloat16_rn(o_val);
      if (p.lse && d == 0) p.lse[row] = lse_val;
    } else {
      p.ws_o[((size_t)s * rows + row) * kHeadDim + d] = o_val;
      if (d == 0) p.ws_lse[(size_t)s * rows + row] = lse_val;
    }
  }
}

// Two E4M3 codes of w (the bytes `sel` picks, with their sign bytes) as a
// bf16 pair, exactly.  A code's exponent and mantissa bits, placed in a bf16's
// exponent-field low bits and mantissa top bits, read as 2^-120 times the
// code's value (subnormal codes become bf16 subnormals of the same scaled
// value); one bf16 multiply by 2^120 rebiases.  The NaN codes 0x7f / 0xff
// read as +-480 (a saturating quantiser never writes them).
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t w, uint32_t sel) {
  uint32_t x, r;
  asm("prmt.b32 %0, %1, 0, %2;" : "=r"(x) : "r"(w), "r"(sel));
  x = (x << 4) & 0x87f087f0u;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(0x7b807b80u));
  return r;
}

// Widens this warp's share of one tile (128 keys x 128 dims) of E4M3 codes
// in place into the bf16 layout of a ring slot: two 64-dim halves of 128 rows
// x 128 B, 16-byte chunks 128B-swizzled.  The codes sit in the upper half,
// key r's 128 codes in row r (chunk c = dims 16c..16c+15, swizzled the same
// way).  Key r's dims 0..63 go to the lower half's row r and dims 64..127 to
// the upper half's row r, which is the key's own code row, so the warp reads
// whole rows before it writes them.  Warp w of nw takes the 4-row quads w,
// w + nw, ... (two per pass); lanes 8i..8i+7 take chunks 0..3 of one row and
// 4..7 of its neighbour (row ^ 1), so that neither the loads nor the stores
// of a quarter-warp share a bank.  Rows for which zero_row(r) holds are
// written as zeros.  `slot` is the slot's shared-window address: explicit
// 32-bit ld/st.shared (measured against generic accesses through a pointer:
// 349 against 359 us on the 8-token 256K verify).
template <class ZeroRow>
__device__ __forceinline__ void widen_e4m3_rows(uint32_t slot, int w, int nw, int lane,
                                                ZeroRow zero_row) {
  const int c = lane & 7;
  const int rr = (lane >> 3) ^ (c >> 2);
  const uint32_t src = slot + kHalfTileBytes;
  const uint32_t dst = slot + (uint32_t)(c >> 2) * kHalfTileBytes;
  const int j0 = 2 * (c & 3);                     // bf16 chunks j0, j0 + 1 of the half row
  auto ld = [&](int r) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(src + (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4))));
    return v;
  };
  auto st = [&](int r, const uint4& in) {
    uint4 lo = make_uint4(0, 0, 0, 0), hi = lo;   // dims 16c..16c+7, 16c+8..16c+15
    if (!zero_row(r)) {
      lo.x = e4m3x2_to_bf16x2(in.x, 0x9180u);
      lo.y = e4m3x2_to_bf16x2(in.x, 0xb3a2u);
      lo.z = e4m3x2_to_bf16x2(in.y, 0x9180u);
      lo.w = e4m3x2_to_bf16x2(in.y, 0xb3a2u);
      hi.x = e4m3x2_to_bf16x2(in.z, 0x9180u);
      hi.y = e4m3x2_to_bf16x2(in.z, 0xb3a2u);
      hi.z = e4m3x2_to_bf16x2(in.w, 0x9180u);
      hi.w = e4m3x2_to_bf16x2(in.w, 0xb3a2u);
    }
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                 ::"r"(dst + (uint32_t)(r * 128 + ((j0 ^ (r & 7)) << 4))),
                 "r"(lo.x), "r"(lo.y), "r"(lo.z), "r"(lo.w) : "memory");
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                 ::"r"(dst + (uint32_t)(r * 128 + (((j0 + 1) ^ (r & 7)) << 4))),
                 "r"(hi.x), "r"(hi.y), "r"(hi.z), "r"(hi.w) : "memory");
  };
  constexpr int kQuads = kTileKeys / 4;
#pragma unroll 1
  for (int qd = w; qd < kQuads; qd += 2 * nw) {
    const int r1 = 4 * qd + rr, r2 = 4 * (qd + nw) + rr;
    const bool two = qd + nw < kQuads;             // the same for the whole warp
    const uint4 in1 = ld(r1);
    const uint4 in2 = two ? ld(r2) : in1;
    __syncwarp();
    st(r1, in1);
    if (two) st(r2, in2);
    __syncwarp();
  }
}

// E4M3 cache: the softmax warps pass the K-ring items on in order (kc counts
// them): a relative-row chunk is let by, a K tile widened (each warp its
// share of the rows), and every warp's pass is counted on the slot's kconv
// barrier.  Passes items until one K tile has been passed (returns 1); with
// `block` false it returns 0 at the first item whose copy has not landed
// (the next call resumes there); -1 when a wait gave up.
template <int KS, int kSlotBytes>
__device__ __forceinline__ int f8_pass_k(int& kc, bool block, uint32_t kfull0, uint32_t kconv0,
                                         const uint8_t* item_flag, uint32_t kring, int w, int nw,
                                         int lane, volatile int* abort_flag,
                                         unsigned long long tlim) {
  while (true) {
    const uint32_t fb = kfull0 + 8u * (uint32_t)(kc % KS);
    const uint32_t par = (uint32_t)(kc / KS) & 1u;
    if (block) {
      if (!__all_sync(0xffffffffu, ptx::mbar_wait(fb, par, abort_flag, tlim))) return -1;
    } else if (!__all_sync(0xffffffffu, ptx::mbar_test_wait(fb, par))) {
      return 0;
    }
    const bool chunk = item_flag[kc % KS] != 0;
    if (!chunk) widen_e4m3_rows(kring + (uint32_t)((kc % KS) * kSlotBytes), w, nw, lane, [](int) { return false; });
    ptx::fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(kconv0 + 8u * (uint32_t)(kc % KS));
    ++kc;
    if (!chunk) return 1;
  }
}

// T (query tokens) is a template parameter: every per-row loop below runs
// over the NQ = T*G live rows only, fully unrolled.
template <int N, int G, int NG, int T, bool F8 = false>
__global__ void __launch_bounds__(KernelConfig<N, NG, G, T, F8>::kThreads, 1)
rel_attn_partial_kernel(const __grid_constant__ DecodeParams p) {
  using KC = KernelConfig<N, NG, G, T, F8>;
  constexpr int KS = KC::kKSlots;
  constexpr int VS = KC::kVSlots;
  constexpr int ROWS = KC::kRows;
  constexpr int YS = KC::kYStride;

  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned, by pointer arithmetic on the shared array so that the
  // compiler keeps every access through smem in the shared window
  uint8_t* smem = smem_raw + ((1024u - (ptx::smem_addr(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = ptx::smem_addr(smem);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int s_idx = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  constexpr int NQ = T * G;
  // rows per softmax group: all NQ when the groups alternate tiles, else the
  // group's block of the column split (at most RG rows, TG tokens)
  using CSp = ColSplit<T, G, NG>;
  constexpr int kAlign = KC::kAlt ? 8 : CSp::align(N);
  constexpr int RG = KC::kAlt ? NQ : CSp::kMaxRows;
  constexpr int TG = RG / G;
  constexpr int RG8 = (RG + 7) / 8;
  constexpr int RGL8 = (kAlign == 8) ? RG8 : (RG + 4 + 7) / 8;   // 8-column loads per row block
  constexpr bool kEvenSplit = KC::kAlt || T % NG == 0;
  static_assert(KC::kAlt ? (NG == 2 && NQ <= N) : (NG == softmax_groups(G, T, F8) && CSp::end(kAlign) <= N &&
                                                   RG <= KC::kGR), "group width");

  // ------------------------------------------------------------ geometry
  const int row0 = first_token_row(p, b);      // q / out row of query token 0
  const int b_seq = b / p.cps;                 // the sequence (block-table row)
  // the block-table row towards L2 while the length is read: the split's
  // entries follow from it, and the producer's first load then hits L2
  if (warp == 0)
    ptx::prefetch_l2_range(p.block_table + (size_t)b_seq * p.max_pages, (size_t)p.max_pages * 4, 128, lane);
  SplitGeom g;
  // the sequence must hold all of its query tokens (seq_stride of them: T
  // for a decode step, C for a prefill) and fit its block-table row
  const int L_seq = __ldg(p.seq_lens + b_seq);
  g.L = chunk_seq_len(p, b, L_seq);
  g.T = T;
  if (L_seq < p.seq_stride || L_seq > p.max_pages * kPage) {
    if (tid == 0) atomicOr(p.status, kStatusBadSeq);
    fill_rows<G>(p, row0, h, s_idx, __int_as_float(0x7fc00000), __int_as_float(0x7fc00000));
    return;
  }
  g.p0 = g.L - T;
  g.W = p.window;
  g.lo = (g.W > 0) ? max(0, g.p0 - g.W + 1) : 0;
  split_pages(g.lo / kPage, (g.L - 1) / kPage, p.num_splits, s_idx, p.ex, p.cost_exact, p.cost_near, &g.sp_begin,
              &g.sp_end);
  g.ntiles = (g.sp_end > g.sp_begin) ? (g.sp_end - g.sp_begin + 1) / 2 : 0;
  if (g.ntiles == 0) {                       // a trailing split with no page
    fill_rows<G>(p, row0, h, s_idx, 0.f, -INFINITY);
    return;
  }

  // --------------------------------------------------------- smem carve-up
  const uint32_t sQ = sbase + KC::oQ;
  const uint32_t sP0 = sbase + KC::oP;
  int* s_edges = reinterpret_cast<int*>(smem + KC::oEdges);
  const uint32_t bar0 = sbase + KC::oBar;
  // K ring (K tiles and relative-row chunks) and V ring, each a full/empty pair
  auto kfull = [&](int s) { return bar0 + 8u * s; };
  auto kempty = [&](int s) { return bar0 + 8u * (KS + s); };
  auto vfull = [&](int s) { return bar0 + 8u * (2 * KS + s); };
  auto vempty = [&](int s) { return bar0 + 8u * (2 * KS + VS + s); };
  constexpr int kB = 2 * KS + 2 * VS;
  const uint32_t s_full = bar0 + 8u * (kB + 0);    // +8*buf
  const uint32_t s_empty = bar0 + 8u * (kB + 2);
  const uint32_t p_full = bar0 + 8u * (kB + 4);
  const uint32_t o_full = bar0 + 8u * (kB + 6);
  const uint32_t o_empty = bar0 + 8u * (kB + 8);
  const uint32_t x_full = bar0 + 8u * (kB + 10);   // +8*group
  const uint32_t x_empty = bar0 + 8u * (kB + 10 + KC::kXTables);
  const uint32_t drain_bar = bar0 + 8u * (kB + 10 + 2 * KC::kXTables);
  const uint32_t drain_pv = drain_bar + 8u;
  auto plan_full = [&](int s) { return drain_pv + 8u * (1 + s); };
  auto plan_empty = [&](int s) { return drain_pv + 8u * (1 + KC::kPlanSlots + s); };
  auto kconv = [&](int s) { return drain_pv + 8u * (1 + 2 * KC::kPlanSlots + s); };
  uint8_t* item_flag = smem + KC::oItemFlag;
  int4* plan_rec = reinterpret_cast<int4*>(smem + KC::oPlan);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + KC::oMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + KC::oMisc + 4);
  volatile int* bad_page_flag = reinterpret_cast<volatile int*>(smem + KC::oMisc + 8);
  int* issued = reinterpret_cast<int*>(smem + KC::oMisc + 12);   // [K-ring items, V tiles]
  auto kslot = [&](int k) { return sbase + KC::oK + (uint32_t)((k % KS) * KC::kKSlotBytes); };
  auto vslot = [&](int i) { return sbase + KC::oV + (uint32_t)((i % VS) * kVSlotBytes); };
  const unsigned long long tlim = p.timeout_ns;

  // -------------------------------------------------------------- prologue
  // Barriers first, by the lanes of warp 0 (in index order: the rings' full /
  // empty pairs, s_full[2], s_empty[2], p_full[2], o_full[2], o_empty[2],
  // x_full[X], x_empty[X], the two drains, plan_full / plan_empty[kPlanSlots],
  // then kconv[KS]; arrival counts 1, one per consumer thread for the
  // barriers the softmax threads arrive on, one per softmax warp for kconv).  The
  // producer's first block-table entries are requested before the CTA-wide
  // barrier; the other warps then allocate tensor memory and stage Q and the
  // bucket edges.
  if (warp == 0) {
    auto init_bar = [&](int i) {
      const int r = i - kB;
      const uint32_t cnt =
          (r < 0) ? 1u
          : (r < 2) ? 1u                                      // s_full
          : (r < 6) ? (uint32_t)KC::kConsumers                // s_empty, p_full
          : (r < 8) ? 1u                                      // o_full
          : (r < 10) ? (uint32_t)KC::kConsumers               // o_empty
          : (r < 10 + KC::kXTables) ? 1u                      // x_full
          : (r < 10 + 2 * KC::kXTables) ? (uint32_t)KC::kConsumers   // x_empty
          : (r < 12 + 2 * KC::kXTables + KC::kPlanSlots) ? 1u        // drains, plan_full
          : (r < 12 + 2 * KC::kXTables + 2 * KC::kPlanSlots) ? (uint32_t)KC::kConsumers  // plan_empty
          : (uint32_t)(KC::kConsumers / 32);                  // kconv
      ptx::mbar_init(bar0 + 8u * i, cnt);
    };
    if constexpr (KC::kNumBars <= 32) {
      if (lane < KC::kNumBars) init_bar(lane);
    } else {
      for (int i = lane; i < KC::kNumBars; i += 32) init_bar(i);
    }
    ptx::fence_mbar_init();
    if (lane == 0) {
      *abort_flag = 0;
      *bad_page_flag = 0;
      issued[0] = issued[1] = 0;
      ptx::prefetch_tmap(&p.tmap_k);
      ptx::prefetch_tmap(&p.tmap_v);
      ptx::prefetch_tmap(&p.tmap_r);
    }
  }
  const int* bt_row = p.block_table + (size_t)b_seq * p.max_pages;
  auto bt_load = [&](int grp) -> int {
    const int pg = g.sp_begin + 32 * grp + lane;
    return (pg < g.sp_end) ? __ldg(bt_row + pg) : 0;
  };
  int bt_cur = 0, bt_next = 0;
  if (warp == 0) {
    bt_cur = bt_load(0);
    bt_next = bt_load(1);
  }
  __syncthreads();
  uint32_t tmem = 0;
  if (warp != 0) {
    if (warp == 1) {
      ptx::tmem_alloc(ptx::smem_addr(tmem_holder), KC::kTmemCols);
      ptx::tmem_relinquish();
    } else if (warp != KC::kPvWarp) {
      const int st = tid - 64;
      const int nst = kSoftmaxThreads * NG;
      // Q group tile, 128B-swizzled K-major: query slot n holds (token t,
      // head gg) with n = t*G + gg, except that column-split groups start
      // their tokens at their own slots; other slots are zero.
      for (int u = st; u < N * 16; u += nst) {
        const int n = u >> 4, half = (u >> 3) & 1, w16 = u & 7;
        uint4 v = make_uint4(0, 0, 0, 0);
        int nl = -1;                                      // row t*G + gg of slot n
        if constexpr (KC::kAlt) {
          nl = n < NQ ? n : -1;
        } else {
#pragma unroll
          for (int q = 0; q < NG; ++q) {
            const int s0 = CSp::slot(q, kAlign);
            if (n >= s0 && n < s0 + CSp::rows(q)) nl = CSp::tok_begin(q) * G + n - s0;
          }
        }
        if (nl >= 0) {
          const int t = nl / G, gg = nl % G;
          const __nv_bfloat16* src = p.q + ((size_t)(row0 + t) * p.Hq + h * G + gg) * kHeadDim
                                     + half * 64 + w16 * 8;
          v = __ldg(reinterpret_cast<const uint4*>(src));
        }
        uint8_t* dst = smem + KC::oQ + half * (N * 128) + n * 128 + ((w16 ^ (n & 7)) << 4);
        *reinterpret_cast<uint4*>(dst) = v;
      }
      for (int e = st; e <= p.nl; e += nst) s_edges[e] = p.edges[e];
      ptx::fence_proxy_async_smem();
    }
    ptx::tc_fence_before();
    ptx::bar_sync_or(kBarSetup, KC::kThreads - 32, false);   // every warp but the producer
    ptx::tc_fence_after();
    tmem = *tmem_holder;
  }
  const uint32_t tS = tmem, tO = tmem + 2 * N;                         // O buffer b at +2N*b
  auto tX = [&](int gq) { return tmem + 6 * N + KC::kXCols * gq; };   // X0; X1 at +N

  // ------------------------------------------------------------- producer
  if (warp == 0) {
    const uint64_t pol = ptx::l2_policy_evict_first();
    int k = 0;                                // K-ring items issued
    int i_v = 0;                              // V-ring items (= tiles) issued
    int rows0[2] = {0, 0}, rows1[2] = {0, 0}, npgs[2] = {0, 0};
    PlanState ps0(p.nl), ps1(p.nl);
    bool ok = true, bad_page = false;
    // V of tile t is issued kVLag tiles after K of tile t, so a V slot is not
    // held while the tile's S and softmax run.
    for (int ti = 0; ti < g.ntiles + KC::kVLag; ++ti) {
      if (ti < g.ntiles) {
        if (ti > 0 && (ti & 15) == 0) {
          bt_cur = bt_next;
          bt_next = bt_load((ti >> 4) + 1);
        }
        const bool odd = KC::kAlt && (ti & 1);
        const TilePlan tp = plan_tile<ROWS>(g, ti, p.ex, p.log2_ex, p.log_scale, p.edges, odd ? ps1 : ps0);
        const int c0 = odd ? ps1.c0 : ps0.c0;
        if constexpr (KC::kPlanSlots > 0) {
          constexpr int PS = KC::kPlanSlots;
          ok = __all_sync(0xffffffffu,
                          ptx::mbar_wait(plan_empty(ti % PS), ((ti / PS) & 1) ^ 1, abort_flag, tlim));
          if (!ok) break;
          if (lane == 0) {
            plan_rec[ti % PS] = make_int4(tp.k_hi, c0, tp.chunk ? 1 : 0, 0);
            ptx::mbar_arrive(plan_full(ti % PS));
          }
        }
        if (tp.chunk) {
          ok = __all_sync(0xffffffffu,
                          ptx::mbar_wait(kempty(k % KS), ((k / KS) & 1) ^ 1, abort_flag, tlim));
          if (!ok) break;
          if (lane == 0) {
            const uint32_t st = kslot(k);
            item_flag[k % KS] = 1;
            ptx::mbar_arrive_expect_tx(kfull(k % KS), 2 * KC::kRHalfBytes);
            ptx::tma_load_3d(st, &p.tmap_r, kfull(k % KS), 0, c0, h);
            ptx::tma_load_3d(st + KC::kRHalfBytes, &p.tmap_r, kfull(k % KS), 64, c0, h);
          }
          ++k;
        }
        int e0 = __shfl_sync(0xffffffffu, bt_cur, (2 * ti) & 31);
        int e1 = __shfl_sync(0xffffffffu, bt_cur, (2 * ti + 1) & 31);
        if (e0 < 0 || e0 >= p.num_pages) { bad_page = true; e0 = 0; }
        if (tp.npg > 1 && (e1 < 0 || e1 >= p.num_pages)) { bad_page = true; e1 = 0; }
        rows0[ti & 1] = (e0 * p.Hkv + h) * kPage;
        rows1[ti & 1] = (e1 * p.Hkv + h) * kPage;
        npgs[ti & 1] = tp.npg;
        // K tile into the K ring
        ok = __all_sync(0xffffffffu,
                        ptx::mbar_wait(kempty(k % KS), ((k / KS) & 1) ^ 1, abort_flag, tlim));
        if (!ok) break;
        if (lane == 0) {
          const uint32_t st = kslot(k);
          const uint32_t fb = kfull(k % KS);
          item_flag[k % KS] = 0;
          if constexpr (F8) {
            // E4M3 codes, one 128-byte row per key, into the slot's upper
            // half (where the widened dims 64..127 of the same key go)
            ptx::mbar_arrive_expect_tx(fb, tp.npg * kPageHalfBytes);
            for (int pi = 0; pi < tp.npg; ++pi) {
              const int row = pi ? rows1[ti & 1] : rows0[ti & 1];
              ptx::tma_load_2d(st + kHalfTileBytes + pi * kPageHalfBytes, &p.tmap_k, fb, 0, row, pol);
            }
          } else {
            ptx::mbar_arrive_expect_tx(fb, tp.npg * 2 * kPageHalfBytes);
            for (int pi = 0; pi < tp.npg; ++pi) {
              const int row = pi ? rows1[ti & 1] : rows0[ti & 1];
              ptx::tma_load_2d(st + pi * kPageHalfBytes, &p.tmap_k, fb, 0, row, pol);
              ptx::tma_load_2d(st + kHalfTileBytes + pi * kPageHalfBytes, &p.tmap_k, fb, 64, row, pol);
            }
          }
        }
        ++k;
      }
      const int tv = ti - KC::kVLag;
      if (tv >= 0 && tv < g.ntiles) {
        // V tile into the V ring
        ok = __all_sync(0xffffffffu,
                        ptx::mbar_wait(vempty(tv % VS), ((tv / VS) & 1) ^ 1, abort_flag, tlim));
        if (!ok) break;
        if (lane == 0) {
          const uint32_t st = vslot(tv);
          const uint32_t fb = vfull(tv % VS);
          if constexpr (F8) {
            ptx::mbar_arrive_expect_tx(fb, npgs[tv & 1] * kPageHalfBytes);
            for (int pi = 0; pi < npgs[tv & 1]; ++pi) {
              const int row = pi ? rows1[tv & 1] : rows0[tv & 1];
              ptx::tma_load_2d(st + kHalfTileBytes + pi * kPageHalfBytes, &p.tmap_v, fb, 0, row, pol);
            }
          } else {
            ptx::mbar_arrive_expect_tx(fb, npgs[tv & 1] * 2 * kPageHalfBytes);
            for (int pi = 0; pi < npgs[tv & 1]; ++pi) {
              const int row = pi ? rows1[tv & 1] : rows0[tv & 1];
              ptx::tma_load_2d(st + pi * kPageHalfBytes, &p.tmap_v, fb, 0, row, pol);
              ptx::tma_load_2d(st + kHalfTileBytes + pi * kPageHalfBytes, &p.tmap_v, fb, 64, row, pol);
            }
          }
        }
        i_v = tv + 1;
      }
    }
    if (lane == 0) {
      if (bad_page) *bad_page_flag = 1;
      issued[0] = k;                         // for the drain at teardown
      issued[1] = i_v;
    }
  }
  // ------------------------------------------------------- S and X issuer
  // S / X and P.V are issued by two warps side by side: one issuing thread
  // spends most of a microsecond per tile on its waits, descriptors and MMA
  // issues, close to what the tile's bytes take at the HBM rate.
  else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t kIdescQK = ptx::idesc_bf16(128, N, false, false);
      // Base descriptors; every MMA operand below is one of these plus a
      // constant byte offset (the address field is the low 14 bits, >> 4).
      const uint64_t kdesc0 = ptx::sdesc_sw128(sbase + KC::oK, 16, 1024);          // K / R chunk, K-major
      const uint64_t qdesc0 = ptx::sdesc_sw128(sQ, 16, 1024);                      // Q, K-major
      int k = 0;                               // K-ring items taken
      int cg[2] = {0, 0};                      // chunks issued per group
      // an item is ready once its copy has landed and, with an E4M3 cache,
      // every softmax warp has passed it (widened a K tile, or let a chunk by)
      auto k_ready = [&](int kk) {
        return ptx::mbar_wait(kfull(kk % KS), (kk / KS) & 1, abort_flag, tlim) &&
               (!F8 || ptx::mbar_wait(kconv(kk % KS), (kk / KS) & 1, abort_flag, tlim));
      };
      for (int ti = 0; ti < g.ntiles; ++ti) {
        const int gq = KC::kAlt ? (ti & 1) : 0;
        if (!k_ready(k)) break;
        if (item_flag[k % KS]) {
          // the tile's new relative-row chunk came first: X = R_chunk . Q
          const int c = cg[gq];
          if (!ptx::mbar_wait(x_empty + 8u * gq, (c & 1) ^ 1, abort_flag, tlim)) break;
          ptx::tc_fence_after();
          const uint64_t kd = kdesc0 + (uint64_t)(((k % KS) * KC::kKSlotBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t ra = kd + (uint64_t)(((kk >> 2) * KC::kRHalfBytes + (kk & 3) * 32) >> 4);
            const uint64_t bq = qdesc0 + (uint64_t)(((kk >> 2) * (N * 128) + (kk & 3) * 32) >> 4);
            ptx::umma_bf16(tX(gq), ra, bq, kIdescQK, kk > 0);
            if constexpr (ROWS > 128)
              ptx::umma_bf16(tX(gq) + N, ra + (uint64_t)(1024 >> 4), bq, kIdescQK, kk > 0);
          }
          ptx::umma_commit(x_full + 8u * gq);
          ptx::umma_commit(kempty(k % KS));
          ++k;
          cg[gq] = c + 1;
          if (!k_ready(k)) break;
        }
        if (!ptx::mbar_wait(s_empty + 8u * (ti & 1), ((ti >> 1) & 1) ^ 1, abort_flag, tlim)) break;
        ptx::tc_fence_after();
        const uint64_t kd = kdesc0 + (uint64_t)(((k % KS) * KC::kKSlotBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          ptx::umma_bf16(tS + (ti & 1) * N, kd + (uint64_t)(((kk >> 2) * kHalfTileBytes + (kk & 3) * 32) >> 4),
                         qdesc0 + (uint64_t)(((kk >> 2) * (N * 128) + (kk & 3) * 32) >> 4), kIdescQK, kk > 0);
        }
        ptx::umma_commit(s_full + 8u * (ti & 1));
        ptx::umma_commit(kempty(k % KS));        // the K slot is free once S is done
        ++k;
      }
      // every MMA issued so far must finish before tensor memory is released
      ptx::umma_commit(drain_bar);
      volatile int never = 0;
      ptx::mbar_wait(drain_bar, 0, &never, kDrainLimitNs);
    }
    __syncwarp();
  }
  // ----------------------------------------------------------- P.V issuer
  else if (warp == KC::kPvWarp) {
    if (lane == 0) {
      constexpr uint32_t kIdescPV = ptx::idesc_bf16(128, 2 * N, true, true);
      const uint64_t vdesc0 = ptx::sdesc_sw128(sbase + KC::oV, kHalfTileBytes, 1024);  // V^T, MN-major
      const uint64_t pdesc0 = ptx::sdesc_noswz(sP0, 16 * 2 * N, 128);              // [P_hi; P_lo], MN-major
      for (int j = 0; j < g.ntiles; ++j) {
        if (!ptx::mbar_wait(p_full + 8u * (j & 1), (j >> 1) & 1, abort_flag, tlim) ||
            !ptx::mbar_wait(o_empty + 8u * (j & 1), ((j >> 1) & 1) ^ 1, abort_flag, tlim) ||
            !ptx::mbar_wait(vfull(j % VS), (j / VS) & 1, abort_flag, tlim))
          break;
        ptx::tc_fence_after();
        const uint64_t va = vdesc0 + (uint64_t)(((j % VS) * kVSlotBytes) >> 4);
        const uint64_t pbd = pdesc0 + (uint64_t)(((j % KC::kPBufs) * KC::kPBufBytes) >> 4);
        // B = [P_hi; P_lo] (2N rows): one pass over V gives O^T for both parts
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          ptx::umma_bf16(tO + (j & 1) * 2 * N, va + (uint64_t)((kk * 2048) >> 4),
                         pbd + (uint64_t)((kk * (2 * 16 * 2 * N)) >> 4), kIdescPV, kk > 0);
        }
        ptx::umma_commit(o_full + 8u * (j & 1));
        ptx::umma_commit(vempty(j % VS));
      }
      ptx::umma_commit(drain_pv);
      volatile int never = 0;
      ptx::mbar_wait(drain_pv, 0, &never, kDrainLimitNs);
    }
    __syncwarp();
  }
  // --------------------------------------------------------------- softmax
  else {
    const int grp = (warp - 2) >> 2;          // softmax group of this warp
    const int sp = warp & 3;                  // TMEM sub-partition of this warp
    const int kl = sp * 32 + lane;            // key lane (S^T) / head-dim lane (O^T)
    const int wsm = (warp - 2) & 3;           // warp index inside the group
    const int bar_id = 1 + grp;
    const uint32_t lane_off = (uint32_t)(sp * 32) << 16;
    // this group's rows: query slots [slot0, slot0 + RG), tokens from tok0;
    // `nrows` of them are live (fewer than RG only when T % NG != 0)
    int slot0 = 0, tok0 = 0, nrows = NQ;
    if constexpr (!KC::kAlt) {
      slot0 = CSp::slot(0, kAlign);
      tok0 = CSp::tok_begin(0);
      nrows = CSp::rows(0);
#pragma unroll
      for (int q = 1; q < NG; ++q) {
        if (grp == q) {
          slot0 = CSp::slot(q, kAlign);
          tok0 = CSp::tok_begin(q);
          nrows = CSp::rows(q);
        }
      }
    }
    auto live = [&](int r) { return r < RG && (kEvenSplit || r < nrows); };
    float* Y = reinterpret_cast<float*>(smem + KC::oY + (KC::kAlt ? grp : 0) * KC::kYBytes);
    float* red = reinterpret_cast<float*>(smem + KC::oRed) + grp * 2 * 4 * KC::kGR;
    float* alpha_buf = reinterpret_cast<float*>(smem + KC::oAlpha) + grp * 2 * KC::kGR;
    const uint32_t tXg = tX(KC::kAlt ? grp : 0) + lane_off;
    // This group's RG columns of a tensor-memory block whose query slot 0 is
    // at column `ta`, for this thread's lane.  A 4-aligned block is read from
    // the 8-aligned column below it and shifted down by four.
    const int cbase = slot0 & ~7;
    const bool sh4 = (kAlign == 4) && (slot0 & 4);
    auto ld_rows = [&](uint32_t ta, float (&v)[RG8 * 8]) {
      if constexpr (kAlign == 8) {
#pragma unroll
        for (int q8 = 0; q8 < RG8; ++q8) ptx::tmem_ld8(ta + slot0 + q8 * 8, v + q8 * 8);
        ptx::tmem_wait_ld();
      } else {
        float raw[RGL8 * 8];
#pragma unroll
        for (int q8 = 0; q8 < RGL8; ++q8) ptx::tmem_ld8(ta + cbase + q8 * 8, raw + q8 * 8);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int r = 0; r < RG8 * 8; ++r) v[r] = (r + 4 < RGL8 * 8 && sh4) ? raw[r + 4] : raw[r];
      }
    };
    // per-row running state: l (this thread's keys), O (this thread's head-dim
    // lane), reference max; alpha_r carries this tile's rescale factors when
    // O is taken right away (alternating groups)
    float l_part[RG], o_acc[RG], m_ref[RG];
    float alpha_r[KC::kAlt ? RG : 1];
#pragma unroll
    for (int r = 0; r < RG; ++r) { l_part[r] = 0.f; o_acc[r] = 0.f; m_ref[r] = kNoMax; }
#pragma unroll
    for (int r = 0; r < (KC::kAlt ? RG : 1); ++r) alpha_r[r] = 1.f;
    int c = 0, li = 0;                        // own chunks, own tiles
    PlanState ps(p.nl);                       // planned over this group's tiles
    // E4M3 cache: multiplier of the K.Q product with the K scale folded in
    // (the relative term is not scaled by it)
    float s_mul_f8 = 0.f;
    if constexpr (F8) s_mul_f8 = p.scale_log2 * __ldg(p.k_scale + h);
    bool failed = false, aborted = false;
    // E4M3 cache: K-ring items this warp has passed on, K tiles among them.
    // Tile t + 1's K is passed at the start of tile t if its copy has landed
    // (its S product then runs during tile t's softmax), else right after
    // tile t's P is handed on; tile t's V is widened just before that.
    int kc = 0, k_passed = 0;
    if constexpr (F8) {
      if (f8_pass_k<KS, KC::kKSlotBytes>(kc, true, kfull(0), kconv(0), item_flag, sbase + KC::oK, warp - 2,
                                         4 * NG, lane, abort_flag, tlim) < 0)
        failed = true;
      else
        k_passed = 1;
    }

    // Accumulate the O^T tile of tile j (this thread's head-dim lane, this
    // group's columns) with the rescale factors `al` of that tile.
    // `rescaled` false: the tile kept every reference max (alpha = 1), and
    // the factors are not read.
    auto process_o = [&](int j, const float* al, bool rescaled) {
      float ov[RG8 * 8];
      const bool okw = ptx::mbar_wait(o_full + 8u * (j & 1), (j >> 1) & 1, abort_flag, tlim);
      if (okw) {
        ptx::tc_fence_after();
        const uint32_t ob = tO + lane_off + (j & 1) * 2 * N;
        ld_rows(ob, ov);                                 // O^T from P_hi
        if (rescaled) {
#pragma unroll
          for (int r = 0; r < RG; ++r)
            if (live(r)) o_acc[r] = fmaf(o_acc[r], al[r], ov[r]);
        } else {
#pragma unroll
          for (int r = 0; r < RG; ++r)
            if (live(r)) o_acc[r] += ov[r];
        }
        ld_rows(ob + N, ov);                             // then from P_lo
#pragma unroll
        for (int r = 0; r < RG; ++r)
          if (live(r)) o_acc[r] += ov[r];
        ptx::tc_fence_before();
      }
      ptx::mbar_arrive(o_empty + 8u * (j & 1));
      if (!okw) failed = true;
    };

    int last_tile = -1;
    bool resc_prev = false;                   // tile last_tile moved some reference max
    // This group's tiles: every other one (alternating groups) or all.  With
    // alternating groups the plan of the group's next tile is made while P.V
    // of the current one runs (elsewhere the registers are scarcer).
    constexpr int kStep = KC::kAlt ? 2 : 1;
    const int t_first = KC::kAlt ? grp : 0;
    TilePlan tp_next{};
    int c0_next = 0;
    if (KC::kAlt && t_first < g.ntiles) {
      tp_next = plan_tile<ROWS>(g, t_first, p.ex, p.log2_ex, p.log_scale, s_edges, ps);
      c0_next = ps.c0;
    }
    for (int ti = t_first; ti < g.ntiles; ti += kStep) {
      TilePlan tp = tp_next;
      int c0 = c0_next;
      if constexpr (F8) {
        if (k_passed == ti + 1 && ti + 1 < g.ntiles &&
            f8_pass_k<KS, KC::kKSlotBytes>(kc, false, kfull(0), kconv(0), item_flag, sbase + KC::oK,
                                           warp - 2, 4 * NG, lane, abort_flag, tlim) > 0)
          ++k_passed;
      }
      if constexpr (KC::kPlanSlots > 0) {
        // the producer's plan of this tile (all threads of the group agree on
        // whether it arrived before any of them acts on it)
        constexpr int PS = KC::kPlanSlots;
        const bool okp = ptx::mbar_wait(plan_full(ti % PS), (ti / PS) & 1, abort_flag, tlim);
        const int4 rec = okp ? plan_rec[ti % PS] : make_int4(0, 0, 0, 0);
        ptx::mbar_arrive(plan_empty(ti % PS));
        if (ptx::bar_sync_or(bar_id, kSoftmaxThreads, !okp || failed)) { aborted = true; break; }
        const int pg = g.sp_begin + 2 * ti;
        tp.j0 = pg * kPage;
        tp.npg = min(2, g.sp_end - pg);
        tp.k_hi = rec.x;
        tp.chunk = rec.z != 0;
        c0 = rec.y;
      }
      if (tp.chunk) {
        {
          // ---- new relative-row chunk: this group's columns of X^T (128 or
          //      136 relative rows) -> gather table Y, already multiplied by
          //      the logit scale so that each logit is one fma
          const int xb = KC::kAlt ? grp : 0;
          const bool okw = ptx::mbar_wait(x_full + 8u * xb, c & 1, abort_flag, tlim);
          if (okw) {
            float xv[RG8 * 8];
            ptx::tc_fence_after();
            ld_rows(tXg, xv);
#pragma unroll
            for (int r = 0; r < RG; ++r)
              if (live(r)) Y[kl * YS + slot0 + r] = xv[r] * p.scale_log2;
            if (ROWS > 128 && sp == 3) {         // rows 128..135 come from lanes 120..127 of X1
              ld_rows(tXg + N, xv);
              if (lane >= 24) {
#pragma unroll
                for (int r = 0; r < RG; ++r)
                  if (live(r)) Y[(kl + 8) * YS + slot0 + r] = xv[r] * p.scale_log2;
              }
            }
            ptx::tc_fence_before();
          }
          ptx::mbar_arrive(x_empty + 8u * xb);
          ++c;
          if (ptx::bar_sync_or(bar_id, kSoftmaxThreads, !okw || failed)) { aborted = true; break; }
        }
      }
      const int i = ti;                       // buffers and phases follow the tile index

      // ---- S^T tile: this thread owns key j, this group's columns
      float s[RG8 * 8];
      const bool okw = ptx::mbar_wait(s_full + 8u * (i & 1), (i >> 1) & 1, abort_flag, tlim);
      if (okw) {
        ptx::tc_fence_after();
        ld_rows(tS + lane_off + (i & 1) * N, s);
        ptx::tc_fence_before();
      }
      ptx::mbar_arrive(s_empty + 8u * (i & 1));

      const int j = tp.j0 + kl;
      const bool loaded = kl < tp.npg * kPage;
      const int d0 = g.p0 - j;                    // distance from token 0
      // The tile's tail buckets lie just below k_hi (log buckets are at least
      // 28 keys wide, so a 128-key tile spans at most a few): the four edges
      // below it, loaded once per tile, place almost every key by compares.
      int e_hi[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) e_hi[m] = s_edges[max(tp.k_hi - m, 0)];
#pragma unroll
      for (int tt = 0; tt < TG; ++tt) {
        if (!kEvenSplit && tt * G >= nrows) break;
        const int d = d0 + tok0 + tt;
        const bool v = loaded && d >= 0 && (g.W <= 0 || d < g.W);
        int bk = d;                               // exact region: the distance itself
        if (v && d >= p.ex) {
          int k = tp.k_hi - (int)(e_hi[0] > d) - (int)(e_hi[1] > d) - (int)(e_hi[2] > d) -
                  (int)(e_hi[3] > d);
          k = max(k, 0);
          if (k > 0 && s_edges[k] > d) k = seek_bucket_far(k, d, s_edges, p.log2_ex, p.log_scale);
          bk = p.ex + k;
        }
        const float* yrow = Y + (v ? bk - c0 : 0) * YS + slot0;
#pragma unroll
        for (int gg = 0; gg < G; ++gg) {
          const int r = tt * G + gg;
          s[r] = v ? fmaf(s[r], F8 ? s_mul_f8 : p.scale_log2, yrow[r]) : -INFINITY;
        }
      }
      // ---- lazy max: p = exp2(x - m_ref) with the row's reference max
      //      m_ref.  Only when some logit exceeds it by more than kLazyLog2
      //      (the first tile, or a jump) does the group take the tile max
      //      and rescale; otherwise alpha = 1 and no reduction is needed.
      //      Results stay exact: lse = m_ref + log2(l) for any m_ref.
      bool over = false;
#pragma unroll
      for (int r = 0; r < RG; ++r)
        if (live(r)) over |= s[r] > m_ref[r] + kLazyLog2;
      float* al_buf = alpha_buf + (li & 1) * KC::kGR;
      bool resc_now = false;                  // this tile moved some reference max
      if (ptx::bar_sync_or(bar_id, kSoftmaxThreads, over || !okw || failed)) {
        resc_now = true;
        if (ptx::bar_sync_or(bar_id, kSoftmaxThreads, !okw || failed)) { aborted = true; break; }
        float* redb = red + (li & 1) * 4 * KC::kGR;
#pragma unroll
        for (int r = 0; r < RG; ++r) {
          if (live(r)) {
            const float mx = warp_max(s[r]);
            if (lane == 0) redb[wsm * KC::kGR + r] = mx;
          }
        }
        ptx::bar_sync_or(bar_id, kSoftmaxThreads, false);
#pragma unroll
        for (int r = 0; r < RG; ++r) {
          if (live(r)) {
            const float tmax = fmaxf(fmaxf(redb[r], redb[KC::kGR + r]),
                                     fmaxf(redb[2 * KC::kGR + r], redb[3 * KC::kGR + r]));
            const float mn = fmaxf(m_ref[r], tmax);
            const float alpha = exp2f(m_ref[r] - mn);
            l_part[r] *= alpha;
            if constexpr (KC::kAlt) alpha_r[r] = alpha;
            else if (kl == 0) al_buf[r] = alpha;
            m_ref[r] = mn;
          }
        }
      } else if constexpr (KC::kAlt) {
#pragma unroll
        for (int r = 0; r < RG; ++r) alpha_r[r] = 1.f;
      }
      // ---- P = exp2(x - m_ref) as bf16 hi + lo parts (~16 significant bits in
      //      the P.V product), stacked [P_hi; P_lo] = 2N rows, MN-major without
      //      swizzle: 8-row x 16-byte core matrices, row blocks 128 B apart,
      //      8-key groups 32*N B apart.  Each thread writes its key for its
      //      group's rows, in units of kAlign rows (16- or 8-byte stores; a
      //      group's units end before the next group's slots).  Rows past the
      //      group's live ones get zeros; slots no group owns are never read
      //      back, as O^T column n depends on P row n only.
      if constexpr (KC::kPBufs == 1) {
        // one P buffer: P.V(i-1) must have read it before P(i) goes in, and
        // taking O(i-1) waits for exactly that
        if (last_tile >= 0) process_o(last_tile, alpha_buf + ((li - 1) & 1) * KC::kGR, resc_prev);
      }
      {
        constexpr int U = kAlign;                              // rows per store
        constexpr int NU = (RG + U - 1) / U;
        const int nu = kEvenSplit ? NU : (nrows + U - 1) / U;
        const uint32_t pbuf = sP0 + (uint32_t)((i % KC::kPBufs) * KC::kPBufBytes);
        const uint32_t pkey = pbuf + (uint32_t)((kl >> 3) * (16 * 2 * N) + (kl & 7) * 16);
#pragma unroll
        for (int cb = 0; cb < NU; ++cb) {
          if (!kEvenSplit && cb >= nu) break;
          uint32_t hi[U / 2], lo[U / 2];
#pragma unroll
          for (int q2 = 0; q2 < U / 2; ++q2) {
            const int r0 = cb * U + 2 * q2, r1 = r0 + 1;
            float p0 = 0.f, p1 = 0.f;
            if (live(r0)) p0 = exp2f(s[r0] - m_ref[r0]);
            if (live(r1)) p1 = exp2f(s[r1] - m_ref[r1]);
            if (live(r0)) l_part[r0] += p0;
            if (live(r1)) l_part[r1] += p1;
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
            const __nv_bfloat162 l2 = __floats2bfloat162_rn(p0 - __low2float(h2), p1 - __high2float(h2));
            hi[q2] = *reinterpret_cast<const uint32_t*>(&h2);
            lo[q2] = *reinterpret_cast<const uint32_t*>(&l2);
          }
          const int row = slot0 + cb * U;
          const uint32_t addr = pkey + (uint32_t)((row >> 3) * 128 + (row & 7) * 2);   // rows of P_hi
          if constexpr (U == 8) {
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                         ::"r"(addr), "r"(hi[0]), "r"(hi[1]), "r"(hi[2]), "r"(hi[3]) : "memory");
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"    // rows N.. of P_lo
                         ::"r"(addr + N * 16), "r"(lo[0]), "r"(lo[1]), "r"(lo[2]), "r"(lo[3]) : "memory");
          } else {
            asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(addr), "r"(hi[0]), "r"(hi[1]) : "memory");
            asm volatile("st.shared.v2.b32 [%0], {%1, %2};"            // rows N.. of P_lo
                         ::"r"(addr + N * 16), "r"(lo[0]), "r"(lo[1]) : "memory");
          }
        }
      }
      // ---- keys no token may see: clear their V rows (stale or poisoned data
      //      must not reach the P.V product, where 0 * NaN = NaN); with both
      //      groups on the tile, group 0 does it.  E4M3 cache: every softmax
      //      warp widens its share of the V tile, writing those rows as zeros.
      if constexpr (F8) {
        if (__all_sync(0xffffffffu, ptx::mbar_wait(vfull(i % VS), (i / VS) & 1, abort_flag, tlim))) {
          const int jt = tp.j0, nload = tp.npg * kPage;
          widen_e4m3_rows(sbase + KC::oV + (uint32_t)((i % VS) * kVSlotBytes), warp - 2, 4 * NG, lane, [&](int r) {
            const int jr = jt + r;
            return !(r < nload && jr <= g.L - 1 && (g.W <= 0 || g.p0 - jr < g.W));
          });
        } else {
          failed = true;
        }
      } else if (KC::kAlt || grp == 0) {
        const bool any_valid = loaded && j <= g.L - 1 && (g.W <= 0 || g.p0 - j < g.W);
        if (!any_valid) {
          // The row is cleared after its copy has landed.  If the wait gives
          // up (the CTA is aborting) the row is left alone: the CTA's rows
          // are then written as NaN whatever P.V computes.
          if (ptx::mbar_wait(vfull(i % VS), (i / VS) & 1, abort_flag, tlim)) {
            uint8_t* vrow = smem + KC::oV + (i % VS) * kVSlotBytes + kl * 128;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              reinterpret_cast<uint4*>(vrow)[q] = make_uint4(0, 0, 0, 0);
              reinterpret_cast<uint4*>(vrow + kHalfTileBytes)[q] = make_uint4(0, 0, 0, 0);
            }
          } else {
            failed = true;
          }
        }
      }
      ptx::fence_proxy_async_smem();
      ptx::mbar_arrive(p_full + 8u * (i & 1));
      if constexpr (F8) {
        // (skipped by the whole warp once any lane has given up a wait)
        if (k_passed == ti + 1 && ti + 1 < g.ntiles && !__any_sync(0xffffffffu, failed)) {
          if (f8_pass_k<KS, KC::kKSlotBytes>(kc, true, kfull(0), kconv(0), item_flag, sbase + KC::oK,
                                             warp - 2, 4 * NG, lane, abort_flag, tlim) < 0)
            failed = true;
          else
            ++k_passed;
        }
      }
      if (KC::kAlt && ti + kStep < g.ntiles) {
        tp_next = plan_tile<ROWS>(g, ti + kStep, p.ex, p.log2_ex, p.log_scale, s_edges, ps);
        c0_next = ps.c0;
      }
      if constexpr (KC::kAlt) {
        // this group's next tile is i + 2: take O(i) now
        process_o(i, alpha_r, true);
      } else if constexpr (KC::kPBufs == 2) {
        // every group is on every tile: take O(i-1) while P.V(i) runs
        if (last_tile >= 0) {
          process_o(last_tile, alpha_buf + ((li - 1) & 1) * KC::kGR, resc_prev);
        }
      }
      resc_prev = resc_now;
      last_tile = i;
      ++li;
    }
    if constexpr (!KC::kAlt) {
      if (!aborted) {
        if (ptx::bar_sync_or(bar_id, kSoftmaxThreads, failed)) aborted = true;
        else if (last_tile >= 0) process_o(last_tile, alpha_buf + ((li - 1) & 1) * KC::kGR, resc_prev);
      }
    }
    ptx::pdl_launch_dependents();

    // ---- epilogue: each group's unnormalised O, per-lane l and reference
    //      max go to shared memory (the K ring, idle once every S has been
    //      read); then all softmax threads finish the rows in short loops.
    //      Alternating groups hold the same rows (merged by LSE); column-split
    //      groups hold disjoint rows.
    bool bad = ptx::bar_sync_or(kBarSoftmaxAll, kSoftmaxThreads * NG, aborted || failed);
    float* eo = reinterpret_cast<float*>(smem);             // [NG][RG][128]
    float* el = eo + NG * RG * kHeadDim;                    // [NG][RG][128]
    float* em = el + NG * RG * kHeadDim;                    // [NG][RG]
    float* es = em + NG * RG;                               // [NG][RG]
    if (!bad) {
#pragma unroll
      for (int r = 0; r < RG; ++r) {
        eo[(grp * RG + r) * kHeadDim + kl] = o_acc[r];
        el[(grp * RG + r) * kHeadDim + kl] = l_part[r];
      }
      if (kl == 0) {
#pragma unroll
        for (int r = 0; r < RG; ++r) em[grp * RG + r] = m_ref[r];
      }
    }
    bad = ptx::bar_sync_or(kBarSoftmaxAll, kSoftmaxThreads * NG, bad);
    if (!bad) {
      const int et = tid - 64, ew = et >> 5;               // softmax thread / warp index
      // row sums of l: one warp per (group, row)
      for (int q = ew; q < NG * RG; q += 4 * NG) {
        const float* src = el + q * kHeadDim;
        const float v = warp_sum(src[lane] + src[lane + 32] + src[lane + 64] + src[lane + 96]);
        if (lane == 0) es[q] = v;
      }
      ptx::bar_sync_or(kBarSoftmaxAll, kSoftmaxThreads * NG, false);
      const int rows = p.rows_total;
      // output rows: (token t, head gg) <- entries (group, local row)
      for (int e = et; e < NQ * kHeadDim; e += kSoftmaxThreads * NG) {
        const int n = e / kHeadDim, d = e % kHeadDim;
        const int t = n / G, gg = n - t * G;
        float m = -INFINITY, o = 0.f, l = 0.f;
        if constexpr (KC::kAlt) {
#pragma unroll
          for (int q = 0; q < NG; ++q) m = fmaxf(m, em[q * RG + n]);
          const float mu = (m == -INFINITY) ? 0.f : m;
#pragma unroll
          for (int q = 0; q < NG; ++q) {
            const float sc = exp2f(em[q * RG + n] - mu);
            o = fmaf(eo[(q * RG + n) * kHeadDim + d], sc, o);
            l = fmaf(es[q * RG + n], sc, l);
          }
        } else {
          int q = 0, tq = 0;                        // the group of token t, its first token
#pragma unroll
          for (int u = 1; u < NG; ++u) {
            if (t >= CSp::tok_begin(u)) {
              q = u;
              tq = CSp::tok_begin(u);
            }
          }
          const int idx = q * RG + (t - tq) * G + gg;
          m = em[idx];
          o = eo[idx * kHeadDim + d];
          l = es[idx];
        }
        o = (l > 0.f) ? o / l : 0.f;
        if constexpr (F8) o *= __ldg(p.v_scale + h);
        const float lse_v = (l > 0.f) ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
        const int row = (row0 + t) * p.Hq + h * G + gg;
        if (p.num_splits == 1) {
          if (p.out_fp32) reinterpret_cast<float*>(p.out)[(size_t)row * kHeadDim + d] = o;
          else reinterpret_cast<__nv_bfloat16*>(p.out)[(size_t)row * kHeadDim + d] = __float2bfloat16_rn(o);
          if (p.lse && d == 0) p.lse[row] = lse_v;
        } else {
          p.ws_o[((size_t)s_idx * rows + row) * kHeadDim + d] = o;
          if (d == 0) p.ws_lse[(size_t)s_idx * rows + row] = lse_v;
        }
      }
    }
  }

  // -------------------------------------------------------------- teardown
  ptx::tc_fence_before();
  __syncthreads();
  // A CTA that gave up on a wait, or met a block-table entry outside the
  // pool, overwrites its rows (final output, or this split's partials, which
  // the combine kernel then propagates) with NaN: callers of the entry
  // point without a workspace see the problem even though they cannot read
  // the status word.
  const bool aborted_cta = *abort_flag != 0, bad_cta = *bad_page_flag != 0;
  if (tid == 0) {
    if (aborted_cta) {
      atomicOr(p.status, kStatusTimeout);
      // The consumers stopped early: let the copies already issued land
      // before the CTA's shared memory is released (in a normal run every
      // copy has been waited for by its consumer).  Only the last KS / VS
      // items can still be in flight: issuing item k waited for item k - KS
      // to be consumed, hence landed.
      volatile int never = 0;
      const int k = issued[0], i_v = issued[1];
      for (int kk = max(0, k - KS); kk < k; ++kk)
        ptx::mbar_wait(kfull(kk % KS), (kk / KS) & 1, &never, kDrainLimitNs);
      for (int iv = max(0, i_v - VS); iv < i_v; ++iv)
        ptx::mbar_wait(vfull(iv % VS), (iv / VS) & 1, &never, kDrainLimitNs);
    }
    if (bad_cta) atomicOr(p.status, kStatusBadSeq);
  }
  if (aborted_cta || bad_cta)
    fill_rows<G>(p, row0, h, s_idx, __int_as_float(0x7fc00000), __int_as_float(0x7fc00000));
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, KC::kTmemCols);
  }
}

// LSE merge of per-split partial results: one CTA per (b, t, hq) row; its
// 8 warps take every 8th split, so the merge costs about two dependent memory
// round trips (the lse values, then the outputs) whatever the split count.
constexpr int kCombineThreads = 256;

__global__ void __launch_bounds__(kCombineThreads)
rel_attn_combine_kernel(const float* __restrict__ ws_lse, const float* __restrict__ ws_o,
                        int num_splits, int rows, void* out, float* lse, int out_fp32) {
  ptx::pdl_wait_primary();
  __shared__ float w_s[256];
  __shared__ float red[8];
  __shared__ float4 part[8][32];
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int row = blockIdx.x;
  const float l = (t < num_splits) ? __ldg(ws_lse + (size_t)t * rows + row) : -INFINITY;
  // this warp's first kPre splits' partial outputs, in flight while the
  // weights are formed (the workspace holds every split's row, empty splits
  // included, so these loads stay inside it)
  constexpr int kPre = 4;
  float4 opre[kPre];
#pragma unroll
  for (int k = 0; k < kPre; ++k) {
    const int s = warp + 8 * k;
    opre[k] = (s < num_splits)
                  ? __ldg(reinterpret_cast<const float4*>(ws_o + ((size_t)s * rows + row) * kHeadDim) + lane)
                  : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  if (__syncthreads_or(l != l)) {                  // a rejected sequence: propagate NaN
    if (t < 32) {
      const float qnan = __int_as_float(0x7fc00000);
      if (out_fp32) {
        reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + (size_t)row * kHeadDim)[lane] =
            make_float4(qnan, qnan, qnan, qnan);
      } else {
        reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(out) + (size_t)row * kHeadDim)[lane] =
            make_uint2(0x7fc07fc0u, 0x7fc07fc0u);
      }
      if (lse && lane == 0) lse[row] = qnan;
    }
    return;
  }
  float mx = warp_max(l);
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  mx = red[0];
#pragma unroll
  for (int q = 1; q < 8; ++q) mx = fmaxf(mx, red[q]);
  const float w = (mx == -INFINITY || l == -INFINITY) ? 0.f : expf(l - mx);
  w_s[t] = w;
  float sum = warp_sum(w);
  __syncthreads();                                   // w_s complete, red[] reads done
  if (lane == 0) red[warp] = sum;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int k = 0; k < kPre; ++k) {
    const int s = warp + 8 * k;
    const float ws = (s < num_splits) ? w_s[s] : 0.f;
    if (ws != 0.f) {
      acc.x = fmaf(ws, opre[k].x, acc.x);
      acc.y = fmaf(ws, opre[k].y, acc.y);
      acc.z = fmaf(ws, opre[k].z, acc.z);
      acc.w = fmaf(ws, opre[k].w, acc.w);
    }
  }
  for (int s = warp + 8 * kPre; s < num_splits; s += 8) {
    const float ws = w_s[s];
    if (ws != 0.f) {
      const float4 o = __ldg(reinterpret_cast<const float4*>(ws_o + ((size_t)s * rows + row) * kHeadDim) + lane);
      acc.x = fmaf(ws, o.x, acc.x);
      acc.y = fmaf(ws, o.y, acc.y);
      acc.z = fmaf(ws, o.z, acc.z);
      acc.w = fmaf(ws, o.w, acc.w);
    }
  }
  part[warp][lane] = acc;
  __syncthreads();
  if (warp == 0) {
    sum = red[0];
#pragma unroll
    for (int q = 1; q < 8; ++q) sum += red[q];
#pragma unroll
    for (int q = 1; q < 8; ++q) {
      const float4 o = part[q][lane];
      acc.x += o.x; acc.y += o.y; acc.z += o.z; acc.w += o.w;
    }
    const float inv = (sum > 0.f) ? 1.f / sum : 0.f;
    acc.x *= inv; acc.y *= inv; acc.z *= inv; acc.w *= inv;
    if (out_fp32) {
      reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + (size_t)row * kHeadDim)[lane] = acc;
    } else {
      __nv_bfloat162 lo2 = __floats2bfloat162_rn(acc.x, acc.y);
      __nv_bfloat162 hi2 = __floats2bfloat162_rn(acc.z, acc.w);
      uint2 pk;
      pk.x = *reinterpret_cast<uint32_t*>(&lo2);
      pk.y = *reinterpret_cast<uint32_t*>(&hi2);
      reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(out) + (size_t)row * kHeadDim)[lane] = pk;
    }
    if (lse && lane == 0) lse[row] = (sum > 0.f) ? mx + logf(sum) : -INFINITY;
  }
}

}  // namespace relattn
