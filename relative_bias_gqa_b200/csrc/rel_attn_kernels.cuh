// rel_attn_kernels.cuh -- sm_100a kernels of relative-bias GQA decode.
//
// Partial kernel, one CTA per (KV split, KV head, sequence):
//   warp 0      TMA producer: walks the split's pages through the block table
//               and streams K/V page tiles (and relative-table row chunks)
//               into a ring of 64 KB shared-memory stages.
//   warp 1      MMA issuer (one thread): tcgen05.mma with fp32 accumulators
//               in tensor memory, "swap-AB" orientation so that keys (and
//               head-dim for P.V) fill the 128-row M side and the GQA
//               group's G heads x T tokens are the N side:
//                 S^T = K . Q^T           (128 keys x N)
//                 X^T = R_chunk . Q^T     (136 relative rows x N)
//                 O^T = V^T . P^T         (128 dims x N)
//   warps 2-5   softmax (128 threads, one key / one head-dim lane each):
//               tcgen05.ld of S^T, relative term sheared into place through a
//               shared-memory table indexed by bucket(distance), masks,
//               fp32 online softmax in the log2 domain, P to shared memory
//               (bf16, 128B-swizzled), O^T tiles accumulated in registers.
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
#include <cstdint>

#include "sm100_ptx.cuh"

// Optional timestamp hook for pipeline studies; expands to nothing unless a
// build defines it.
#ifndef RELATTN_TRACE
#define RELATTN_TRACE(event, tile)
#endif

namespace relattn {

constexpr int kHeadDim = 128;
constexpr int kPage = 64;
constexpr int kTileKeys = 128;                 // two pages per tile
constexpr int kRChunkRows = 136;               // relative-table rows per chunk
constexpr int kMaxTailBuckets = 512;           // log buckets supported
constexpr int kThreads = 192;
constexpr int kSoftmaxThreads = 128;
constexpr int kStageBytes = 65536;             // K (32 KB) + V (32 KB)
constexpr int kHalfTileBytes = 16384;          // 128 rows x 128 B (one 64-dim half)
constexpr int kPageHalfBytes = 8192;           // 64 rows x 128 B
constexpr int kRHalfBytes = kRChunkRows * 128; // 17408
constexpr unsigned kStatusTimeout = 1u;
constexpr unsigned kStatusBadSeq = 2u;
constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;  // 2 s

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
  int ex;               // distances d < ex are their own bucket
  int nl;               // tail buckets: bucket = ex + max{k < nl : edges[k] <= d}
  float scale_log2;     // log2(e) / sqrt(D)
  int edges[kMaxTailBuckets + 1];
};

__host__ __device__ constexpr int align_up(int x, int a) { return (x + a - 1) / a * a; }

// Shared-memory carve-up for an N-wide (padded group) tile.
template <int N>
struct SmemLayout {
  static constexpr int kStages = (N == 16) ? 3 : 2;
  static constexpr int kYStride = N + 1;                       // odd: conflict-free gathers
  static constexpr int kOperandBytes = 2 * N * 128;            // N rows x 128 dims, two 64-dim halves
  static constexpr int oQ = kStages * kStageBytes;
  static constexpr int oP = oQ + kOperandBytes;                // two P buffers, each hi + lo
  static constexpr int kPBufBytes = 2 * kOperandBytes;
  static constexpr int oY = oP + 2 * kPBufBytes;
  static constexpr int oRed = oY + align_up(kRChunkRows * kYStride * 4, 16);
  static constexpr int oLred = oRed + 2 * 4 * N * 4;
  static constexpr int oAlpha = oLred + 4 * N * 4;
  static constexpr int oM = oAlpha + 2 * N * 4;
  static constexpr int oEdges = oM + 2 * N * 4;
  static constexpr int oBar = align_up(oEdges + (kMaxTailBuckets + 1) * 4, 8);
  // barriers: full[S], empty[S], s_full[2], s_empty[2], p_full[2], o_full[2],
  //           o_empty[2], x_full, x_empty, drain
  static constexpr int kNumBars = 2 * kStages + 13;
  static constexpr int oMisc = oBar + kNumBars * 8;            // tmem base, abort flag
  static constexpr int kBytes = oMisc + 16;
  static constexpr int kAllocBytes = kBytes + 1024;            // 1024-byte alignment slack
  static constexpr int kTmemCols = (6 * N <= 128) ? 128 : (6 * N <= 256 ? 256 : 512);
  static_assert(kAllocBytes <= 232448, "shared memory budget exceeded");
};

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

// Cursor state carried from tile to tile.  Distances only shrink as the walk
// moves to later keys, so the tail-bucket indices are found by stepping the
// cursors down the edge table instead of searching it.
struct PlanState {
  int c0 = 0;
  bool have = false;
  int k_hi, k_lo;
  __device__ explicit PlanState(int nl) : k_hi(nl - 1), k_lo(nl - 1) {}
};

__device__ __forceinline__ int step_down(int k, int d, const int* edges) {
  while (k > 0 && edges[k] > d) --k;
  return k;
}

// Decides, for tile ti, the loaded pages and whether the relative-row chunk
// [c0, c0+136) must move so that it covers every bucket the tile needs.
// All roles call it with identical arguments, so they agree on the sequence.
__device__ __forceinline__ TilePlan plan_tile(const SplitGeom& g, int ti, int ex, const int* edges,
                                              PlanState& st) {
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
    st.k_hi = step_down(st.k_hi, d_hi, edges);
    t.k_hi = st.k_hi;
    b_hi = ex + st.k_hi;
  }
  if (d_lo >= ex) {
    st.k_lo = step_down(st.k_lo, d_lo, edges);
    b_lo = ex + st.k_lo;
  }
  t.chunk = !(st.have && b_lo >= st.c0 && b_hi < st.c0 + kRChunkRows);
  if (t.chunk) {
    st.c0 = max(0, b_hi - (kRChunkRows - 1));
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

// Write this CTA's rows (all NQ rows of the group, every head-dim) with a
// constant value; used for empty splits and rejected sequences.
template <int G>
__device__ void fill_rows(const DecodeParams& p, int b, int h, int s, float o_val, float lse_val) {
  const int rows = p.B * p.T * p.Hq;
  const int NQ = p.T * G;
  for (int e = threadIdx.x; e < NQ * kHeadDim; e += blockDim.x) {
    const int n = e / kHeadDim, d = e % kHeadDim;
    const int t = n / G, gg = n % G;
    const int row = (b * p.T + t) * p.Hq + h * G + gg;
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

template <int N, int G>
__global__ void __launch_bounds__(kThreads, 1)
rel_attn_partial_kernel(const __grid_constant__ DecodeParams p) {
  using SL = SmemLayout<N>;
  constexpr int STG = SL::kStages;
  constexpr int YS = SL::kYStride;
  constexpr int TMAX = (N + G - 1) / G;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_addr(smem);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int s_idx = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int T = p.T;
  const int NQ = T * G;

  // ------------------------------------------------------------ geometry
  SplitGeom g;
  g.L = __ldg(p.seq_lens + b);
  g.T = T;
  if (g.L < T || g.L > p.max_pages * kPage) {
    if (tid == 0) atomicOr(p.status, kStatusBadSeq);
    fill_rows<G>(p, b, h, s_idx, __int_as_float(0x7fc00000), __int_as_float(0x7fc00000));
    return;
  }
  g.p0 = g.L - T;
  g.W = p.window;
  g.lo = (g.W > 0) ? max(0, g.p0 - g.W + 1) : 0;
  {
    const int first = g.lo / kPage, last = (g.L - 1) / kPage;
    const int n_pages = last - first + 1;
    const int S = p.num_splits;
    const int pps = 2 * ((n_pages + 2 * S - 1) / (2 * S));
    g.sp_begin = first + s_idx * pps;
    g.sp_end = min(g.sp_begin + pps, last + 1);
    g.ntiles = (g.sp_end > g.sp_begin) ? (g.sp_end - g.sp_begin + 1) / 2 : 0;
  }
  if (g.ntiles == 0) {                       // a trailing split with no page
    fill_rows<G>(p, b, h, s_idx, 0.f, -INFINITY);
    return;
  }

  // --------------------------------------------------------- smem carve-up
  const uint32_t sQ = sbase + SL::oQ;
  const uint32_t sP0 = sbase + SL::oP;
  float* Y = reinterpret_cast<float*>(smem + SL::oY);
  float* red = reinterpret_cast<float*>(smem + SL::oRed);
  float* lred = reinterpret_cast<float*>(smem + SL::oLred);
  float* alpha_buf = reinterpret_cast<float*>(smem + SL::oAlpha);
  float* m_buf = reinterpret_cast<float*>(smem + SL::oM);
  int* s_edges = reinterpret_cast<int*>(smem + SL::oEdges);
  const uint32_t bar0 = sbase + SL::oBar;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STG + s); };
  const uint32_t s_full = bar0 + 8u * (2 * STG + 0);    // +8*buf
  const uint32_t s_empty = bar0 + 8u * (2 * STG + 2);
  const uint32_t p_full = bar0 + 8u * (2 * STG + 4);
  const uint32_t o_full = bar0 + 8u * (2 * STG + 6);
  const uint32_t o_empty = bar0 + 8u * (2 * STG + 8);
  const uint32_t x_full = bar0 + 8u * (2 * STG + 10);
  const uint32_t x_empty = bar0 + 8u * (2 * STG + 11);
  const uint32_t drain_bar = bar0 + 8u * (2 * STG + 12);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + SL::oMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SL::oMisc + 4);
  auto stage_addr = [&](int k) { return sbase + (uint32_t)((k % STG) * kStageBytes); };
  const unsigned long long tlim = p.timeout_ns;

  // -------------------------------------------------------------- prologue
  if (warp == 0) {
    if (lane == 0) {
      for (int s = 0; s < STG; ++s) {
        ptx::mbar_init(full_bar(s), 1);
        ptx::mbar_init(empty_bar(s), 1);
      }
      for (int i = 0; i < 2; ++i) {
        ptx::mbar_init(s_full + 8u * i, 1);
        ptx::mbar_init(s_empty + 8u * i, kSoftmaxThreads);
        ptx::mbar_init(p_full + 8u * i, kSoftmaxThreads);
        ptx::mbar_init(o_full + 8u * i, 1);
        ptx::mbar_init(o_empty + 8u * i, kSoftmaxThreads);
      }
      ptx::mbar_init(x_full, 1);
      ptx::mbar_init(x_empty, kSoftmaxThreads);
      ptx::mbar_init(drain_bar, 1);
      *abort_flag = 0;
      ptx::fence_mbar_init();
      ptx::prefetch_tmap(&p.tmap_k);
      ptx::prefetch_tmap(&p.tmap_v);
      ptx::prefetch_tmap(&p.tmap_r);
    }
  } else if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_addr(tmem_holder), SL::kTmemCols);
    ptx::tmem_relinquish();
  } else {
    const int st = tid - 64;
    // Q group tile: rows n = t*G + g (padding rows zero), 128B-swizzled K-major.
    for (int u = st; u < N * 16; u += kSoftmaxThreads) {
      const int n = u >> 4, half = (u >> 3) & 1, w16 = u & 7;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (n < NQ) {
        const int t = n / G, gg = n % G;
        const __nv_bfloat16* src = p.q + ((size_t)(b * T + t) * p.Hq + h * G + gg) * kHeadDim
                                   + half * 64 + w16 * 8;
        v = __ldg(reinterpret_cast<const uint4*>(src));
      }
      uint8_t* dst = smem + SL::oQ + half * (N * 128) + n * 128 + ((w16 ^ (n & 7)) << 4);
      *reinterpret_cast<uint4*>(dst) = v;
    }
    for (int e = st; e <= p.nl; e += kSoftmaxThreads) s_edges[e] = p.edges[e];
    for (int e = st; e < 2 * N; e += kSoftmaxThreads) m_buf[e] = -INFINITY;
    ptx::fence_proxy_async_smem();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  // ------------------------------------------------------------- producer
  if (warp == 0) {
    const uint64_t pol = ptx::l2_policy_evict_first();
    const int* bt_row = p.block_table + (size_t)b * p.max_pages;
    auto bt_load = [&](int grp) -> int {
      const int pg = g.sp_begin + 32 * grp + lane;
      return (pg < g.sp_end) ? __ldg(bt_row + pg) : 0;
    };
    int bt_cur = bt_load(0);
    int bt_next = bt_load(1);
    int k = 0;
    PlanState ps(p.nl);
    bool ok = true, bad_page = false;
    for (int ti = 0; ti < g.ntiles; ++ti) {
      if (ti > 0 && (ti & 15) == 0) {
        bt_cur = bt_next;
        bt_next = bt_load((ti >> 4) + 1);
      }
      const TilePlan tp = plan_tile(g, ti, p.ex, s_edges, ps);
      if (tp.chunk) {
        ok = __all_sync(0xffffffffu,
                        ptx::mbar_wait(empty_bar(k % STG), ((k / STG) & 1) ^ 1, abort_flag, tlim));
        if (!ok) break;
        if (lane == 0) {
          const uint32_t st = stage_addr(k);
          ptx::mbar_arrive_expect_tx(full_bar(k % STG), 2 * kRHalfBytes);
          ptx::tma_load_3d(st, &p.tmap_r, full_bar(k % STG), 0, ps.c0, h);
          ptx::tma_load_3d(st + kRHalfBytes, &p.tmap_r, full_bar(k % STG), 64, ps.c0, h);
        }
        ++k;
      }
      ok = __all_sync(0xffffffffu,
                      ptx::mbar_wait(empty_bar(k % STG), ((k / STG) & 1) ^ 1, abort_flag, tlim));
      if (!ok) break;
      const int e0 = __shfl_sync(0xffffffffu, bt_cur, (2 * ti) & 31);
      const int e1 = __shfl_sync(0xffffffffu, bt_cur, (2 * ti + 1) & 31);
      if (lane == 0) {
        const uint32_t st = stage_addr(k);
        const uint32_t fb = full_bar(k % STG);
        ptx::mbar_arrive_expect_tx(fb, tp.npg * 4 * kPageHalfBytes);
        for (int pi = 0; pi < tp.npg; ++pi) {
          int phys = pi ? e1 : e0;
          if (phys < 0 || phys >= p.num_pages) { bad_page = true; phys = 0; }
          const int row = (phys * p.Hkv + h) * kPage;
          ptx::tma_load_2d(st + pi * kPageHalfBytes, &p.tmap_k, fb, 0, row, pol);
          ptx::tma_load_2d(st + kHalfTileBytes + pi * kPageHalfBytes, &p.tmap_k, fb, 64, row, pol);
          ptx::tma_load_2d(st + 2 * kHalfTileBytes + pi * kPageHalfBytes, &p.tmap_v, fb, 0, row, pol);
          ptx::tma_load_2d(st + 3 * kHalfTileBytes + pi * kPageHalfBytes, &p.tmap_v, fb, 64, row, pol);
        }
        RELATTN_TRACE(0, ti);
      }
      ++k;
    }
    if (lane == 0) {
      if (bad_page) atomicOr(p.status, kStatusBadSeq);
      if (!ok) {
        // Let the copies already issued land before the CTA's memory is released.
        volatile int never = 0;
        for (int kk = max(0, k - STG); kk < k; ++kk)
          ptx::mbar_wait(full_bar(kk % STG), (kk / STG) & 1, &never, tlim);
      }
    }
  }
  // ------------------------------------------------------------ MMA issuer
  else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t kIdescQK = ptx::idesc_bf16(128, N, false, false);
      constexpr uint32_t kIdescPV = ptx::idesc_bf16(128, N, true, false);
      const uint32_t tS = tmem, tX0 = tmem + 2 * N, tX1 = tmem + 3 * N, tO = tmem + 4 * N;
      int k = 0, c = 0, i = 0, stage_prev = 0;
      PlanState ps(p.nl);
      bool ok = true;
      auto issue_pv = [&](int j, int stg) -> bool {
        if (!ptx::mbar_wait(p_full + 8u * (j & 1), (j >> 1) & 1, abort_flag, tlim)) return false;
        if (!ptx::mbar_wait(o_empty + 8u * (j & 1), ((j >> 1) & 1) ^ 1, abort_flag, tlim)) return false;
        ptx::tc_fence_after();
        RELATTN_TRACE(3, j);
        const uint32_t v = sbase + (uint32_t)(stg * kStageBytes) + 2 * kHalfTileBytes;
        const uint32_t pb = sP0 + (uint32_t)((j & 1) * SL::kPBufBytes);
        // P = P_hi + P_lo (two bf16 parts): O^T += V^T P_hi^T + V^T P_lo^T
#pragma unroll
        for (int part = 0; part < 2; ++part) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t a = ptx::sdesc_sw128(v + kk * 2048, kHalfTileBytes, 1024);
            const uint64_t bd = ptx::sdesc_sw128(pb + part * SL::kOperandBytes + (kk >> 2) * (N * 128) +
                                                 (kk & 3) * 32, 16, 1024);
            ptx::umma_bf16(tO + (j & 1) * N, a, bd, kIdescPV, (part | kk) > 0);
          }
        }
        ptx::umma_commit(o_full + 8u * (j & 1));
        ptx::umma_commit(empty_bar(stg));
        return true;
      };
      for (int ti = 0; ti < g.ntiles; ++ti) {
        const TilePlan tp = plan_tile(g, ti, p.ex, s_edges, ps);
        // P.V of the previous tile releases its stage.  Issue it first unless
        // this tile's data has already landed: a stage must never wait on a
        // load that itself waits for that stage.
        bool pv_pending = i > 0;
        if (pv_pending) {
          const int kt = k + (tp.chunk ? 1 : 0);
          if (!ptx::mbar_try_wait(full_bar(kt % STG), (kt / STG) & 1)) {
            if (!(ok = issue_pv(i - 1, stage_prev))) break;
            pv_pending = false;
          }
        }
        if (tp.chunk) {
          ok = ptx::mbar_wait(full_bar(k % STG), (k / STG) & 1, abort_flag, tlim) &&
               ptx::mbar_wait(x_empty, (c & 1) ^ 1, abort_flag, tlim);
          if (!ok) break;
          ptx::tc_fence_after();
          const uint32_t st = stage_addr(k);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t koff = (kk >> 2) * kRHalfBytes + (kk & 3) * 32;
            const uint64_t bq = ptx::sdesc_sw128(sQ + (kk >> 2) * (N * 128) + (kk & 3) * 32, 16, 1024);
            ptx::umma_bf16(tX0, ptx::sdesc_sw128(st + koff, 16, 1024), bq, kIdescQK, kk > 0);
            ptx::umma_bf16(tX1, ptx::sdesc_sw128(st + 1024 + koff, 16, 1024), bq, kIdescQK, kk > 0);
          }
          ptx::umma_commit(x_full);
          ptx::umma_commit(empty_bar(k % STG));
          ++k;
          ++c;
        }
        ok = ptx::mbar_wait(full_bar(k % STG), (k / STG) & 1, abort_flag, tlim) &&
             ptx::mbar_wait(s_empty + 8u * (i & 1), ((i >> 1) & 1) ^ 1, abort_flag, tlim);
        if (!ok) break;
        ptx::tc_fence_after();
        RELATTN_TRACE(1, i);
        {
          const uint32_t st = stage_addr(k);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t a = ptx::sdesc_sw128(st + (kk >> 2) * kHalfTileBytes + (kk & 3) * 32, 16, 1024);
            const uint64_t bq = ptx::sdesc_sw128(sQ + (kk >> 2) * (N * 128) + (kk & 3) * 32, 16, 1024);
            ptx::umma_bf16(tS + (i & 1) * N, a, bq, kIdescQK, kk > 0);
          }
          ptx::umma_commit(s_full + 8u * (i & 1));
        }
        if (pv_pending && !(ok = issue_pv(i - 1, stage_prev))) break;
        stage_prev = k % STG;
        ++k;
        ++i;
      }
      if (ok && i > 0) ok = issue_pv(i - 1, stage_prev);
      // every MMA issued so far must finish before tensor memory is released
      ptx::umma_commit(drain_bar);
      volatile int never = 0;
      ptx::mbar_wait(drain_bar, 0, &never, tlim);
    }
    __syncwarp();
  }
  // --------------------------------------------------------------- softmax
  else {
    const int sp = warp & 3;                  // TMEM sub-partition of this warp
    const int kl = sp * 32 + lane;            // key lane (S^T) / head-dim lane (O^T)
    const int wsm = warp - 2;
    const uint32_t lane_off = (uint32_t)(sp * 32) << 16;
    const uint32_t tS = tmem + lane_off, tX0 = tmem + 2 * N + lane_off,
                   tX1 = tmem + 3 * N + lane_off, tO = tmem + 4 * N + lane_off;
    float l_part[N], o_acc[N];
#pragma unroll
    for (int n = 0; n < N; ++n) { l_part[n] = 0.f; o_acc[n] = 0.f; }
    int k = 0, c = 0, i = 0;
    PlanState ps(p.nl);
    bool failed = false, aborted = false;

    auto process_o = [&](int j) {
      float ov[N];
      const bool okw = ptx::mbar_wait(o_full + 8u * (j & 1), (j >> 1) & 1, abort_flag, tlim);
      if (okw) {
        ptx::tc_fence_after();
#pragma unroll
        for (int q16 = 0; q16 < N / 16; ++q16) ptx::tmem_ld16(tO + (j & 1) * N + q16 * 16, ov + q16 * 16);
        ptx::tmem_wait_ld();
        ptx::tc_fence_before();
      }
      ptx::mbar_arrive(o_empty + 8u * (j & 1));
      if (!okw) { failed = true; return; }
      const float* al = alpha_buf + (j & 1) * N;
#pragma unroll
      for (int n = 0; n < N; ++n)
        if (n < NQ) o_acc[n] = fmaf(o_acc[n], al[n], ov[n]);
    };

    for (int ti = 0; ti < g.ntiles; ++ti) {
      const TilePlan tp = plan_tile(g, ti, p.ex, s_edges, ps);
      if (tp.chunk) {
        const bool okw = ptx::mbar_wait(x_full, c & 1, abort_flag, tlim);
        if (okw) {
          float xv[N];
          ptx::tc_fence_after();
#pragma unroll
          for (int q16 = 0; q16 < N / 16; ++q16) ptx::tmem_ld16(tX0 + q16 * 16, xv + q16 * 16);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int n = 0; n < N; ++n)
            if (n < NQ) Y[kl * YS + n] = xv[n];
          if (sp == 3) {                       // rows 128..135 come from lanes 120..127 of X1
#pragma unroll
            for (int q16 = 0; q16 < N / 16; ++q16) ptx::tmem_ld16(tX1 + q16 * 16, xv + q16 * 16);
            ptx::tmem_wait_ld();
            if (lane >= 24) {
#pragma unroll
              for (int n = 0; n < N; ++n)
                if (n < NQ) Y[(kl + 8) * YS + n] = xv[n];
            }
          }
          ptx::tc_fence_before();
        }
        ptx::mbar_arrive(x_empty);
        ++k;
        ++c;
        if (ptx::bar_sync_or(1, kSoftmaxThreads, !okw || failed)) { aborted = true; break; }
      }

      // ---- S^T tile: this thread owns key j
      float s[N];
      const bool okw = ptx::mbar_wait(s_full + 8u * (i & 1), (i >> 1) & 1, abort_flag, tlim);
      if (okw) {
        ptx::tc_fence_after();
        RELATTN_TRACE(4, i);
#pragma unroll
        for (int q16 = 0; q16 < N / 16; ++q16) ptx::tmem_ld16(tS + (i & 1) * N + q16 * 16, s + q16 * 16);
        ptx::tmem_wait_ld();
        ptx::tc_fence_before();
      }
      ptx::mbar_arrive(s_empty + 8u * (i & 1));

      const int j = tp.j0 + kl;
      const bool loaded = kl < tp.npg * kPage;
      const int d0 = g.p0 - j;                    // distance from token 0
#pragma unroll
      for (int t = 0; t < TMAX; ++t) {
        if (t < T) {
          const int d = d0 + t;
          const bool v = loaded && d >= 0 && (g.W <= 0 || d < g.W);
          // bucket: the distance itself below ex, else step down from the
          // tile's largest tail bucket (a tile spans only a few of them)
          const int r = !v ? 0 : (d < p.ex ? d : p.ex + step_down(tp.k_hi, d, s_edges)) - ps.c0;
          const float* yrow = Y + r * YS;
#pragma unroll
          for (int gg = 0; gg < G; ++gg) {
            const int n = t * G + gg;
            if (n < N) s[n] = v ? (s[n] + yrow[n]) * p.scale_log2 : -INFINITY;
          }
        } else {
#pragma unroll
          for (int gg = 0; gg < G; ++gg) {
            const int n = t * G + gg;
            if (n < N) s[n] = -INFINITY;
          }
        }
      }
      // ---- tile max over the 128 keys
      float* redb = red + (i & 1) * 4 * N;
#pragma unroll
      for (int n = 0; n < N; ++n) {
        if (n < NQ) {
          const float mx = warp_max(s[n]);
          if (lane == 0) redb[wsm * N + n] = mx;
        }
      }
      if (ptx::bar_sync_or(1, kSoftmaxThreads, !okw || failed)) { aborted = true; break; }
      RELATTN_TRACE(5, i);
      const float* m_old = m_buf + ((i & 1) ^ 1) * N;
      float* m_new_buf = m_buf + (i & 1) * N;
      float* al_buf = alpha_buf + (i & 1) * N;
      const uint32_t pbuf = sP0 + (uint32_t)((i & 1) * SL::kPBufBytes);
      const uint32_t p_row_base = pbuf + (uint32_t)((kl >> 6) * (N * 128));
      const uint32_t u = (uint32_t)((kl & 63) >> 3), byte_in = (uint32_t)((kl & 7) * 2);
#pragma unroll
      for (int n = 0; n < N; ++n) {
        if (n < NQ) {
          const float tmax = fmaxf(fmaxf(redb[n], redb[N + n]), fmaxf(redb[2 * N + n], redb[3 * N + n]));
          const float mo = m_old[n];
          const float mn = fmaxf(mo, tmax);
          const float mu = (mn == -INFINITY) ? 0.f : mn;
          const float alpha = exp2f(mo - mu);
          const float pv = exp2f(s[n] - mu);
          l_part[n] = fmaf(l_part[n], alpha, pv);
          if (kl == 0) { m_new_buf[n] = mn; al_buf[n] = alpha; }
          // bf16 hi/lo split keeps ~16 significant bits of p in the P.V product
          const __nv_bfloat16 ph = __float2bfloat16_rn(pv);
          const __nv_bfloat16 pl = __float2bfloat16_rn(pv - __bfloat162float(ph));
          const uint32_t addr = p_row_base + n * 128 + ((u ^ (n & 7)) << 4) + byte_in;
          asm volatile("st.shared.b16 [%0], %1;" ::"r"(addr), "h"(__bfloat16_as_ushort(ph)) : "memory");
          asm volatile("st.shared.b16 [%0], %1;" ::"r"(addr + SL::kOperandBytes), "h"(__bfloat16_as_ushort(pl)) : "memory");
        }
      }
      // ---- keys no token may see: clear their V rows (stale or poisoned data
      //      must not reach the P.V product, where 0 * NaN = NaN)
      {
        const bool any_valid = loaded && j <= g.L - 1 && (g.W <= 0 || g.p0 - j < g.W);
        if (!any_valid) {
          volatile int never = 0;
          ptx::mbar_wait(full_bar(k % STG), (k / STG) & 1, &never, tlim);
          uint8_t* vrow = smem + (k % STG) * kStageBytes + 2 * kHalfTileBytes + kl * 128;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            reinterpret_cast<uint4*>(vrow)[q] = make_uint4(0, 0, 0, 0);
            reinterpret_cast<uint4*>(vrow + kHalfTileBytes)[q] = make_uint4(0, 0, 0, 0);
          }
        }
      }
      ptx::fence_proxy_async_smem();
      ptx::mbar_arrive(p_full + 8u * (i & 1));
      RELATTN_TRACE(6, i);
      if (i > 0) {
        process_o(i - 1);
        RELATTN_TRACE(7, i - 1);
      }
      ++k;
      ++i;
    }
    if (!aborted) {
      if (ptx::bar_sync_or(1, kSoftmaxThreads, failed)) aborted = true;
      else process_o(i - 1);
    }
    ptx::pdl_launch_dependents();
    if (!aborted) {
      // ---- epilogue: finish l, normalise, write this split's rows
#pragma unroll
      for (int n = 0; n < N; ++n) {
        if (n < NQ) {
          const float sum = warp_sum(l_part[n]);
          if (lane == 0) lred[wsm * N + n] = sum;
        }
      }
      if (ptx::bar_sync_or(1, kSoftmaxThreads, failed)) aborted = true;
      if (!aborted) {
        const float* m_fin = m_buf + ((i - 1) & 1) * N;
        const int rows = p.B * T * p.Hq;
        const int d = kl;
#pragma unroll
        for (int n = 0; n < N; ++n) {
          if (n < NQ) {
            const int t = n / G, gg = n % G;
            const int row = (b * T + t) * p.Hq + h * G + gg;
            const float lt = lred[n] + lred[N + n] + lred[2 * N + n] + lred[3 * N + n];
            const float o = (lt > 0.f) ? o_acc[n] / lt : 0.f;
            const float lse_v = (lt > 0.f) ? (m_fin[n] + log2f(lt)) * 0.69314718055994531f : -INFINITY;
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
    }
  }

  // -------------------------------------------------------------- teardown
  ptx::tc_fence_before();
  __syncthreads();
  if (tid == 0 && *abort_flag) atomicOr(p.status, kStatusTimeout);
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, SL::kTmemCols);
  }
}

// LSE merge of per-split partial results: one warp per (b, t, hq) row.
__global__ void __launch_bounds__(128)
rel_attn_combine_kernel(const float* __restrict__ ws_lse, const float* __restrict__ ws_o,
                        int num_splits, int rows, void* out, float* lse, int out_fp32) {
  ptx::pdl_wait_primary();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 4 + warp;
  if (row >= rows) return;
  float w[8];
  float mx = -INFINITY;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int s = q * 32 + lane;
    w[q] = (s < num_splits) ? __ldg(ws_lse + (size_t)s * rows + row) : -INFINITY;
    mx = fmaxf(mx, w[q]);
  }
  bool nan_seen = false;
#pragma unroll
  for (int q = 0; q < 8; ++q) nan_seen |= (w[q] != w[q]);
  if (__any_sync(0xffffffffu, nan_seen)) {       // a rejected sequence: propagate NaN
    const float qnan = __int_as_float(0x7fc00000);
    if (out_fp32) {
      reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + (size_t)row * kHeadDim)[lane] =
          make_float4(qnan, qnan, qnan, qnan);
    } else {
      reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(out) + (size_t)row * kHeadDim)[lane] =
          make_uint2(0x7fc07fc0u, 0x7fc07fc0u);
    }
    if (lse && lane == 0) lse[row] = qnan;
    return;
  }
  mx = warp_max(mx);
  float sum = 0.f;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    w[q] = (mx == -INFINITY || w[q] == -INFINITY) ? 0.f : expf(w[q] - mx);
    sum += w[q];
  }
  sum = warp_sum(sum);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    if (q * 32 >= num_splits) break;
    const int cnt = min(32, num_splits - q * 32);
    for (int sl = 0; sl < cnt; ++sl) {
      const float ws = __shfl_sync(0xffffffffu, w[q], sl);
      if (ws != 0.f) {
        const float4 o = __ldg(reinterpret_cast<const float4*>(
            ws_o + ((size_t)(q * 32 + sl) * rows + row) * kHeadDim) + lane);
        acc.x = fmaf(ws, o.x, acc.x);
        acc.y = fmaf(ws, o.y, acc.y);
        acc.z = fmaf(ws, o.z, acc.z);
        acc.w = fmaf(ws, o.w, acc.w);
      }
    }
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

}  // namespace relattn
