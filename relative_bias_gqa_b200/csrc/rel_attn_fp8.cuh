// rel_attn_fp8.cuh -- partial kernel over an FP8 (E4M3) KV cache, one query
// token per sequence.
//
// The FP8 KV cache is the next step the Inkling page plans for its global
// attention layers ("vLLM TML Inkling 지원", section "미래 로드맵"): it halves
// the bytes of the bandwidth-bound decode.  Codes are OFP8 E4M3, one fp32
// scale per KV head for K and one for V (k = e4m3(code) * k_scale[h]).
//
// Tensor-core MMAs take both operands in the same 16-bit type, and the
// query must not lose precision, so the tiles are widened on chip:
//   warp 0        TMA producer: E4M3 K and V page tiles (8 KB per page) into
//                 two staging rings, relative-row chunks into their own slot.
//   warp 1        MMA issuer: S^T = K16 . Qh^T and O^T = V16^T . [P_hi; P_lo]^T
//                 in f16 (E4M3 -> f16 is exact; Qh is the query in f16),
//                 X^T = R_chunk . Q^T in bf16 as in the bf16 kernel.
//   warps 2..9    two softmax groups alternating tiles (as the one-token bf16
//                 kernel), P in f16 hi + lo parts.
//   warps 10..13  converter: one thread per key row widens the staged E4M3 K
//                 and V rows to f16 (cvt.rn.f16x2.e4m3x2, exact) into the
//                 MMA's 128B-swizzled layouts, zeroing V rows no query may see.
// The K scale multiplies the S logits, the V scale the final output.  The
// softmax's lazy reference max lets P grow to 2^14 here (f16 range).
#pragma once

namespace relattn {

struct Fp8Config {
  static constexpr int N = 16, NG = 2, NQ = 6, RG = 6, ROWS = 128;
  static constexpr int kThreads = 64 + kSoftmaxThreads * NG + 128;
  static constexpr int kK8Slots = 3, kV8Slots = 3;
  static constexpr int k8TileBytes = 128 * 128;                 // 128 keys x 128 B
  static constexpr int k8PageBytes = 64 * 128;
  static constexpr int kF16TileBytes = 2 * kHalfTileBytes;      // 128 keys x 256 B
  static constexpr int kRHalfBytes = ROWS * 128;
  static constexpr int kYStride = 7;
  static constexpr int kGR = 8;
  static constexpr int kPBufBytes = 2 * (2 * N * 128);          // [P_hi; P_lo]: 128 keys x 2N rows f16
  static constexpr int kYBytes = align_up(ROWS * kYStride * 4, 16);
  static constexpr int oK8 = 0;
  static constexpr int oV8 = oK8 + kK8Slots * k8TileBytes;
  static constexpr int oXR = oV8 + kV8Slots * k8TileBytes;      // relative-row chunk (bf16)
  static constexpr int oKF = oXR + 2 * kRHalfBytes;             // K tile widened to f16
  static constexpr int oVF = oKF + kF16TileBytes;               // V tile widened to f16
  static constexpr int oQ = oVF + kF16TileBytes;                // Q bf16 (for X)
  static constexpr int oQh = oQ + 2 * N * 128;                  // Q f16 (for S)
  static constexpr int oP = oQh + 2 * N * 128;                  // two P buffers
  static constexpr int oY = oP + 2 * kPBufBytes;                // one table per group
  static constexpr int oRed = oY + NG * kYBytes;                // [NG][2][4][kGR]
  static constexpr int oAlpha = oRed + NG * 2 * 4 * kGR * 4;    // [NG][2][kGR] (unused slack)
  static constexpr int oEdges = oAlpha + NG * 2 * kGR * 4;
  static constexpr int oBar = align_up(oEdges + (kMaxTailBuckets + 1) * 4, 8);
  // k8full[3] k8empty[3] v8full[3] v8empty[3] kf_full kf_empty vf_full vf_empty
  // xr_full xr_empty s_full[2] s_empty[2] p_full[2] o_full[2] o_empty[2]
  // x_full[2] x_empty[2] drain
  static constexpr int kNumBars = 2 * kK8Slots + 2 * kV8Slots + 6 + 14 + 1;
  static constexpr int oMisc = oBar + kNumBars * 8;
  static constexpr int kBytes = oMisc + 16;
  static constexpr int kAllocBytes = kBytes + 1024;
  static constexpr int kTmemCols = 128;                         // S[2] 32 + O[2] 64 + X[2] 32
  static_assert(kAllocBytes <= 232448, "shared memory budget exceeded");
  static_assert(oKF % 1024 == 0 && oVF % 1024 == 0 && oXR % 1024 == 0 && oQ % 1024 == 0 &&
                oQh % 1024 == 0 && oV8 % 1024 == 0, "slot alignment");
  static_assert(oXR >= NG * RG * 128 * 4 * 2 + NG * RG * 4 * 2, "epilogue exchange area");
};

// E4M3 pair (low 16 bits) -> f16x2, exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t v) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"((uint16_t)v));
  return r;
}

template <int G>
__global__ void __launch_bounds__(Fp8Config::kThreads, 1)
rel_attn_partial_fp8_kernel(const __grid_constant__ DecodeParams p) {
  using FC = Fp8Config;
  constexpr int N = FC::N, NG = FC::NG, NQ = FC::NQ, RG = FC::RG, ROWS = FC::ROWS;
  constexpr int YS = FC::kYStride;
  constexpr int K8S = FC::kK8Slots, V8S = FC::kV8Slots;
  constexpr int T = 1;
  static_assert(NQ == G * T, "one token, six heads");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_addr(smem);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int s_idx = blockIdx.x, h = blockIdx.y, b = blockIdx.z;

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
  split_pages(g.lo / kPage, (g.L - 1) / kPage, p.num_splits, s_idx, p.ex, &g.sp_begin, &g.sp_end);
  g.ntiles = (g.sp_end > g.sp_begin) ? (g.sp_end - g.sp_begin + 1) / 2 : 0;
  if (g.ntiles == 0) {
    fill_rows<G>(p, b, h, s_idx, 0.f, -INFINITY);
    return;
  }

  // --------------------------------------------------------- smem carve-up
  int* s_edges = reinterpret_cast<int*>(smem + FC::oEdges);
  const uint32_t bar0 = sbase + FC::oBar;
  auto k8full = [&](int s) { return bar0 + 8u * s; };
  auto k8empty = [&](int s) { return bar0 + 8u * (K8S + s); };
  auto v8full = [&](int s) { return bar0 + 8u * (2 * K8S + s); };
  auto v8empty = [&](int s) { return bar0 + 8u * (2 * K8S + V8S + s); };
  constexpr int kB = 2 * K8S + 2 * V8S;
  const uint32_t kf_full = bar0 + 8u * (kB + 0), kf_empty = bar0 + 8u * (kB + 1);
  const uint32_t vf_full = bar0 + 8u * (kB + 2), vf_empty = bar0 + 8u * (kB + 3);
  const uint32_t xr_full = bar0 + 8u * (kB + 4), xr_empty = bar0 + 8u * (kB + 5);
  const uint32_t s_full = bar0 + 8u * (kB + 6);     // +8*buf
  const uint32_t s_empty = bar0 + 8u * (kB + 8);
  const uint32_t p_full = bar0 + 8u * (kB + 10);
  const uint32_t o_full = bar0 + 8u * (kB + 12);
  const uint32_t o_empty = bar0 + 8u * (kB + 14);
  const uint32_t x_full = bar0 + 8u * (kB + 16);    // +8*group
  const uint32_t x_empty = bar0 + 8u * (kB + 18);
  const uint32_t drain_bar = bar0 + 8u * (kB + 20);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + FC::oMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + FC::oMisc + 4);
  volatile int* bad_page_flag = reinterpret_cast<volatile int*>(smem + FC::oMisc + 8);
  const unsigned long long tlim = p.timeout_ns;

  // -------------------------------------------------------------- prologue
  if (tid == 0) {
    for (int s = 0; s < K8S; ++s) { ptx::mbar_init(k8full(s), 1); ptx::mbar_init(k8empty(s), 128); }
    for (int s = 0; s < V8S; ++s) { ptx::mbar_init(v8full(s), 1); ptx::mbar_init(v8empty(s), 128); }
    ptx::mbar_init(kf_full, 128);
    ptx::mbar_init(kf_empty, 1);
    ptx::mbar_init(vf_full, 128);
    ptx::mbar_init(vf_empty, 1);
    ptx::mbar_init(xr_full, 1);
    ptx::mbar_init(xr_empty, 1);
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(s_full + 8u * i, 1);
      ptx::mbar_init(s_empty + 8u * i, kSoftmaxThreads);
      ptx::mbar_init(p_full + 8u * i, kSoftmaxThreads);
      ptx::mbar_init(o_full + 8u * i, 1);
      ptx::mbar_init(o_empty + 8u * i, kSoftmaxThreads);
      ptx::mbar_init(x_full + 8u * i, 1);
      ptx::mbar_init(x_empty + 8u * i, kSoftmaxThreads);
    }
    ptx::mbar_init(drain_bar, 1);
    *abort_flag = 0;
    *bad_page_flag = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&p.tmap_k);
    ptx::prefetch_tmap(&p.tmap_v);
    ptx::prefetch_tmap(&p.tmap_r);
  }
  __syncthreads();
  uint32_t tmem = 0;
  if (warp != 0) {
    if (warp == 1) {
      ptx::tmem_alloc(ptx::smem_addr(tmem_holder), FC::kTmemCols);
      ptx::tmem_relinquish();
    } else if (warp < 10) {
      // Q group tile, twice (bf16 for the relative product, f16 for S):
      // rows n = g (padding rows zero), 128B-swizzled K-major.
      const int st = tid - 64;
      for (int u = st; u < N * 16; u += kSoftmaxThreads * NG) {
        const int n = u >> 4, half = (u >> 3) & 1, w16 = u & 7;
        uint4 v = make_uint4(0, 0, 0, 0), vh = make_uint4(0, 0, 0, 0);
        if (n < NQ) {
          const __nv_bfloat16* src = p.q + ((size_t)b * p.Hq + h * G + n) * kHeadDim + half * 64 + w16 * 8;
          v = __ldg(reinterpret_cast<const uint4*>(src));
          const __nv_bfloat162* q2 = reinterpret_cast<const __nv_bfloat162*>(&v);
          __half2* h2 = reinterpret_cast<__half2*>(&vh);
#pragma unroll
          for (int e = 0; e < 4; ++e) h2[e] = __float22half2_rn(__bfloat1622float2(q2[e]));
        }
        const int off = half * (N * 128) + n * 128 + ((w16 ^ (n & 7)) << 4);
        *reinterpret_cast<uint4*>(smem + FC::oQ + off) = v;
        *reinterpret_cast<uint4*>(smem + FC::oQh + off) = vh;
      }
      ptx::fence_proxy_async_smem();
    } else {
      // converter warps copy the bucket edges
      for (int e = tid - 320; e <= p.nl; e += 128) s_edges[e] = p.edges[e];
    }
    ptx::tc_fence_before();
    ptx::bar_sync_or(6, FC::kThreads - 32, false);   // every warp but the producer
    ptx::tc_fence_after();
    tmem = *tmem_holder;
  }
  const uint32_t tS = tmem, tO = tmem + 2 * N;
  auto tX = [&](int gq) { return tmem + 6 * N + N * gq; };

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
    int nchunks = 0, nk = 0, nv = 0;           // chunks, K tiles, V tiles issued
    PlanState ps0(p.nl), ps1(p.nl);
    bool ok = true, bad_page = false;
    int ti = 0;
    for (; ti < g.ntiles; ++ti) {
      if (ti > 0 && (ti & 15) == 0) {
        bt_cur = bt_next;
        bt_next = bt_load((ti >> 4) + 1);
      }
      const bool odd = ti & 1;
      const TilePlan tp = plan_tile<ROWS>(g, ti, p.ex, p.log2_ex, p.log_scale, p.edges, odd ? ps1 : ps0);
      const int c0 = odd ? ps1.c0 : ps0.c0;
      int e0 = __shfl_sync(0xffffffffu, bt_cur, (2 * ti) & 31);
      int e1 = __shfl_sync(0xffffffffu, bt_cur, (2 * ti + 1) & 31);
      if (e0 < 0 || e0 >= p.num_pages) { bad_page = true; e0 = 0; }
      if (tp.npg > 1 && (e1 < 0 || e1 >= p.num_pages)) { bad_page = true; e1 = 0; }
      const int row0 = (e0 * p.Hkv + h) * kPage, row1 = (e1 * p.Hkv + h) * kPage;
      // E4M3 K tile
      ok = __all_sync(0xffffffffu, ptx::mbar_wait(k8empty(ti % K8S), ((ti / K8S) & 1) ^ 1, abort_flag, tlim));
      if (!ok) break;
      if (lane == 0) {
        const uint32_t st = sbase + FC::oK8 + (ti % K8S) * FC::k8TileBytes;
        ptx::mbar_arrive_expect_tx(k8full(ti % K8S), tp.npg * FC::k8PageBytes);
        ptx::tma_load_2d(st, &p.tmap_k, k8full(ti % K8S), 0, row0, pol);
        if (tp.npg > 1) ptx::tma_load_2d(st + FC::k8PageBytes, &p.tmap_k, k8full(ti % K8S), 0, row1, pol);
      }
      ++nk;
      // relative-row chunk
      if (tp.chunk) {
        ok = __all_sync(0xffffffffu, ptx::mbar_wait(xr_empty, (nchunks & 1) ^ 1, abort_flag, tlim));
        if (!ok) break;
        if (lane == 0) {
          const uint32_t st = sbase + FC::oXR;
          ptx::mbar_arrive_expect_tx(xr_full, 2 * FC::kRHalfBytes);
          ptx::tma_load_3d(st, &p.tmap_r, xr_full, 0, c0, h);
          ptx::tma_load_3d(st + FC::kRHalfBytes, &p.tmap_r, xr_full, 64, c0, h);
        }
        ++nchunks;
      }
      // E4M3 V tile
      ok = __all_sync(0xffffffffu, ptx::mbar_wait(v8empty(ti % V8S), ((ti / V8S) & 1) ^ 1, abort_flag, tlim));
      if (!ok) break;
      if (lane == 0) {
        const uint32_t st = sbase + FC::oV8 + (ti % V8S) * FC::k8TileBytes;
        ptx::mbar_arrive_expect_tx(v8full(ti % V8S), tp.npg * FC::k8PageBytes);
        ptx::tma_load_2d(st, &p.tmap_v, v8full(ti % V8S), 0, row0, pol);
        if (tp.npg > 1) ptx::tma_load_2d(st + FC::k8PageBytes, &p.tmap_v, v8full(ti % V8S), 0, row1, pol);
      }
      ++nv;
    }
    if (lane == 0) {
      if (bad_page) *bad_page_flag = 1;
      // Let the copies already issued land before the CTA's memory is
      // released, on every exit (the consumers may have stopped early).
      volatile int never = 0;
      for (int t = max(0, nk - K8S); t < nk; ++t)
        ptx::mbar_wait(k8full(t % K8S), (t / K8S) & 1, &never, kDrainLimitNs);
      for (int t = max(0, nv - V8S); t < nv; ++t)
        ptx::mbar_wait(v8full(t % V8S), (t / V8S) & 1, &never, kDrainLimitNs);
      if (nchunks > 0) ptx::mbar_wait(xr_full, (nchunks - 1) & 1, &never, kDrainLimitNs);
    }
  }
  // ------------------------------------------------------------ converter
  // Order K(0), then per tile K(i+1) before V(i): K(i+1) needs only S(i) to
  // have read the K16 slot, V(i) needs P.V(i-1) to have read the V16 slot,
  // so the K side runs a tile ahead and S(i+1) and its softmax never wait
  // behind the P.V chain.
  else if (warp >= 10) {
    const int kc = tid - 320;                     // key row of the tile
    const int sw = kc & 7;
    // one E4M3 row (128 B, 8 swizzled 16-byte chunks) -> f16 row (two 128 B
    // halves of the K-major / MN-major 128B-swizzled tile)
    auto widen = [&](uint32_t src_slot, uint8_t* dst_tile, bool zero) {
      const uint8_t* src = smem + (src_slot - sbase) + kc * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint4 lo4 = make_uint4(0, 0, 0, 0), hi4 = make_uint4(0, 0, 0, 0);
        if (!zero) {
          const uint4 w = *reinterpret_cast<const uint4*>(src + ((c ^ sw) << 4));
          lo4 = make_uint4(e4m3x2_to_f16x2(w.x & 0xffffu), e4m3x2_to_f16x2(w.x >> 16),
                           e4m3x2_to_f16x2(w.y & 0xffffu), e4m3x2_to_f16x2(w.y >> 16));
          hi4 = make_uint4(e4m3x2_to_f16x2(w.z & 0xffffu), e4m3x2_to_f16x2(w.z >> 16),
                           e4m3x2_to_f16x2(w.w & 0xffffu), e4m3x2_to_f16x2(w.w >> 16));
        }
        // 16 dims 16c..16c+15 -> half c/4, 16-byte chunks 2(c%4), 2(c%4)+1
        uint8_t* row = dst_tile + (c >> 2) * kHalfTileBytes + kc * 128;
        *reinterpret_cast<uint4*>(row + (((2 * (c & 3)) ^ sw) << 4)) = lo4;
        *reinterpret_cast<uint4*>(row + (((2 * (c & 3) + 1) ^ sw) << 4)) = hi4;
      }
    };
    auto tile_pages = [&](int ti) { return min(2, g.sp_end - (g.sp_begin + 2 * ti)); };
    auto convert_k = [&](int ti) -> bool {
      if (!ptx::mbar_wait(k8full(ti % K8S), (ti / K8S) & 1, abort_flag, tlim) ||
          !ptx::mbar_wait(kf_empty, (ti & 1) ^ 1, abort_flag, tlim))
        return false;
      if (kc < tile_pages(ti) * kPage) widen(sbase + FC::oK8 + (ti % K8S) * FC::k8TileBytes, smem + FC::oKF, false);
      ptx::fence_proxy_async_smem();
      ptx::mbar_arrive(kf_full);
      ptx::mbar_arrive(k8empty(ti % K8S));
      return true;
    };
    auto convert_v = [&](int ti) -> bool {
      // rows no query may see are zeroed: 0 * NaN must not reach P.V
      const int j = (g.sp_begin + 2 * ti) * kPage + kc;
      const bool any_valid = kc < tile_pages(ti) * kPage && j <= g.L - 1 && (g.W <= 0 || g.p0 - j < g.W);
      if (!ptx::mbar_wait(v8full(ti % V8S), (ti / V8S) & 1, abort_flag, tlim) ||
          !ptx::mbar_wait(vf_empty, (ti & 1) ^ 1, abort_flag, tlim))
        return false;
      widen(sbase + FC::oV8 + (ti % V8S) * FC::k8TileBytes, smem + FC::oVF, !any_valid);
      ptx::fence_proxy_async_smem();
      ptx::mbar_arrive(vf_full);
      ptx::mbar_arrive(v8empty(ti % V8S));
      return true;
    };
    bool ok = convert_k(0);
    for (int ti = 0; ti < g.ntiles && ok; ++ti) {
      if (ti + 1 < g.ntiles) ok = convert_k(ti + 1);
      ok = ok && convert_v(ti);
    }
  }
  // ------------------------------------------------------------ MMA issuer
  else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t kIdescQKh = ptx::idesc_f16(128, N, false, false);    // K16 . Qh
      constexpr uint32_t kIdescXR = ptx::idesc_bf16(128, N, false, false);    // R . Q
      constexpr uint32_t kIdescPV = ptx::idesc_f16(128, 2 * N, true, true);   // V16^T . P
      const uint64_t kfdesc = ptx::sdesc_sw128(sbase + FC::oKF, 16, 1024);
      const uint64_t xrdesc = ptx::sdesc_sw128(sbase + FC::oXR, 16, 1024);
      const uint64_t qdesc = ptx::sdesc_sw128(sbase + FC::oQ, 16, 1024);
      const uint64_t qhdesc = ptx::sdesc_sw128(sbase + FC::oQh, 16, 1024);
      const uint64_t vdesc = ptx::sdesc_sw128(sbase + FC::oVF, kHalfTileBytes, 1024);
      const uint64_t pdesc = ptx::sdesc_noswz(sbase + FC::oP, 16 * 2 * N, 128);
      int i = 0, nx = 0;                       // tiles, chunks issued
      int cg[2] = {0, 0};                      // chunks per group
      PlanState ps0(p.nl), ps1(p.nl);
      bool ok = true;
      auto issue_pv = [&](int j) -> bool {
        if (!ptx::mbar_wait(p_full + 8u * (j & 1), (j >> 1) & 1, abort_flag, tlim)) return false;
        if (!ptx::mbar_wait(o_empty + 8u * (j & 1), ((j >> 1) & 1) ^ 1, abort_flag, tlim)) return false;
        if (!ptx::mbar_wait(vf_full, j & 1, abort_flag, tlim)) return false;
        ptx::tc_fence_after();
        const uint64_t pbd = pdesc + (uint64_t)(((j & 1) * FC::kPBufBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          ptx::umma_bf16(tO + (j & 1) * 2 * N, vdesc + (uint64_t)((kk * 2048) >> 4),
                         pbd + (uint64_t)((kk * (2 * 16 * 2 * N)) >> 4), kIdescPV, kk > 0);
        ptx::umma_commit(o_full + 8u * (j & 1));
        ptx::umma_commit(vf_empty);
        return true;
      };
      for (int ti = 0; ti < g.ntiles; ++ti) {
        const int gq = ti & 1;
        const TilePlan tp = plan_tile<ROWS>(g, ti, p.ex, p.log2_ex, p.log_scale, s_edges, gq ? ps1 : ps0);
        // S(i) first, then P.V(i-1): the converter widens K(i) before
        // V(i-1), so S(i) never waits on the P.V chain.
        const bool pv_pending = i > 0;
        if (tp.chunk) {
          ok = ptx::mbar_wait(xr_full, nx & 1, abort_flag, tlim) &&
               ptx::mbar_wait(x_empty + 8u * gq, (cg[gq] & 1) ^ 1, abort_flag, tlim);
          if (!ok) break;
          ptx::tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t ko = (kk >> 2) * FC::kRHalfBytes + (kk & 3) * 32;
            const uint32_t qo = (kk >> 2) * (N * 128) + (kk & 3) * 32;
            ptx::umma_bf16(tX(gq), xrdesc + (uint64_t)(ko >> 4), qdesc + (uint64_t)(qo >> 4), kIdescXR, kk > 0);
          }
          ptx::umma_commit(x_full + 8u * gq);
          ptx::umma_commit(xr_empty);
          ++nx;
          ++cg[gq];
        }
        ok = ptx::mbar_wait(kf_full, i & 1, abort_flag, tlim) &&
             ptx::mbar_wait(s_empty + 8u * (i & 1), ((i >> 1) & 1) ^ 1, abort_flag, tlim);
        if (!ok) break;
        ptx::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t ko = (kk >> 2) * kHalfTileBytes + (kk & 3) * 32;
          const uint32_t qo = (kk >> 2) * (N * 128) + (kk & 3) * 32;
          ptx::umma_bf16(tS + (i & 1) * N, kfdesc + (uint64_t)(ko >> 4), qhdesc + (uint64_t)(qo >> 4),
                         kIdescQKh, kk > 0);
        }
        ptx::umma_commit(s_full + 8u * (i & 1));
        ptx::umma_commit(kf_empty);              // the K16 slot is free once S is done
        if (pv_pending && !(ok = issue_pv(i - 1))) break;
        ++i;
      }
      if (ok && i > 0) ok = issue_pv(i - 1);
      ptx::umma_commit(drain_bar);
      volatile int never = 0;
      ptx::mbar_wait(drain_bar, 0, &never, kDrainLimitNs);
    }
    __syncwarp();
  }
  // --------------------------------------------------------------- softmax
  else {
    constexpr float kLazy = 14.f;             // P = exp2(x - m_ref) < 2^14 stays in f16 range
    const int grp = (warp - 2) >> 2;          // group g takes the tiles i with i % 2 == g
    const int sp = warp & 3;
    const int kl = sp * 32 + lane;            // key lane (S^T) / head-dim lane (O^T)
    const int wsm = (warp - 2) & 3;
    const int bar_id = 1 + grp;
    const uint32_t lane_off = (uint32_t)(sp * 32) << 16;
    float* Y = reinterpret_cast<float*>(smem + FC::oY + grp * FC::kYBytes);
    float* red = reinterpret_cast<float*>(smem + FC::oRed) + grp * 2 * 4 * FC::kGR;
    const uint32_t tXg = tX(grp) + lane_off;
    const float sl = p.scale_log2;
    const float ksl = __ldg(p.k_scale + h) * sl;
    float l_part[RG], o_acc[RG], m_ref[RG], alpha_r[RG];
#pragma unroll
    for (int r = 0; r < RG; ++r) { l_part[r] = 0.f; o_acc[r] = 0.f; m_ref[r] = kNoMax; alpha_r[r] = 1.f; }
    int c = 0, li = 0;
    PlanState ps0(p.nl), ps1(p.nl);
    bool failed = false, aborted = false;

    auto process_o = [&](int j) {
      float ov[8];
      const bool okw = ptx::mbar_wait(o_full + 8u * (j & 1), (j >> 1) & 1, abort_flag, tlim);
      if (okw) {
        ptx::tc_fence_after();
        const uint32_t ob = tO + lane_off + (j & 1) * 2 * N;
#pragma unroll
        for (int part = 0; part < 2; ++part) {          // O^T from P_hi, then from P_lo
          ptx::tmem_ld8(ob + part * N, ov);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int r = 0; r < RG; ++r) o_acc[r] = part ? o_acc[r] + ov[r] : fmaf(o_acc[r], alpha_r[r], ov[r]);
        }
        ptx::tc_fence_before();
      }
      ptx::mbar_arrive(o_empty + 8u * (j & 1));
      if (!okw) failed = true;
    };

    for (int ti = 0; ti < g.ntiles; ++ti) {
      const int owner = ti & 1;
      const TilePlan tp = plan_tile<ROWS>(g, ti, p.ex, p.log2_ex, p.log_scale, s_edges, owner ? ps1 : ps0);
      const int c0 = owner ? ps1.c0 : ps0.c0;
      if (owner != grp) continue;
      if (tp.chunk) {
        // ---- new relative-row chunk: X^T (128 rows x N) -> gather table Y
        const bool okw = ptx::mbar_wait(x_full + 8u * grp, c & 1, abort_flag, tlim);
        if (okw) {
          float xv[8];
          ptx::tc_fence_after();
          ptx::tmem_ld8(tXg, xv);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int r = 0; r < RG; ++r) Y[kl * YS + r] = xv[r];
          ptx::tc_fence_before();
        }
        ptx::mbar_arrive(x_empty + 8u * grp);
        ++c;
        if (ptx::bar_sync_or(bar_id, kSoftmaxThreads, !okw || failed)) { aborted = true; break; }
      }
      const int i = ti;

      // ---- S^T tile: this thread owns key j
      float s[8];
      const bool okw = ptx::mbar_wait(s_full + 8u * (i & 1), (i >> 1) & 1, abort_flag, tlim);
      if (okw) {
        ptx::tc_fence_after();
        ptx::tmem_ld8(tS + lane_off + (i & 1) * N, s);
        ptx::tmem_wait_ld();
        ptx::tc_fence_before();
      }
      ptx::mbar_arrive(s_empty + 8u * (i & 1));

      const int j = tp.j0 + kl;
      const bool loaded = kl < tp.npg * kPage;
      const int d = g.p0 - j;
      const bool v = loaded && d >= 0 && (g.W <= 0 || d < g.W);
      int bk = d;
      if (v && d >= p.ex) {
        int k = tp.k_hi;
#pragma unroll
        for (int m = 0; m < 4; ++m) k -= (int)(s_edges[max(tp.k_hi - m, 0)] > d);
        k = max(k, 0);
        if (k > 0 && s_edges[k] > d) k = seek_bucket_far(k, d, s_edges, p.log2_ex, p.log_scale);
        bk = p.ex + k;
      }
      const float* yrow = Y + (v ? bk - c0 : 0) * YS;
#pragma unroll
      for (int r = 0; r < RG; ++r) s[r] = v ? fmaf(s[r], ksl, yrow[r] * sl) : -INFINITY;

      // ---- lazy max (as the bf16 kernel, threshold 2^14)
      bool over = false;
#pragma unroll
      for (int r = 0; r < RG; ++r) over |= s[r] > m_ref[r] + kLazy;
      if (ptx::bar_sync_or(bar_id, kSoftmaxThreads, over || !okw || failed)) {
        if (ptx::bar_sync_or(bar_id, kSoftmaxThreads, !okw || failed)) { aborted = true; break; }
        float* redb = red + (li & 1) * 4 * FC::kGR;
#pragma unroll
        for (int r = 0; r < RG; ++r) {
          const float mx = warp_max(s[r]);
          if (lane == 0) redb[wsm * FC::kGR + r] = mx;
        }
        ptx::bar_sync_or(bar_id, kSoftmaxThreads, false);
#pragma unroll
        for (int r = 0; r < RG; ++r) {
          const float tmax = fmaxf(fmaxf(redb[r], redb[FC::kGR + r]),
                                   fmaxf(redb[2 * FC::kGR + r], redb[3 * FC::kGR + r]));
          const float mn = fmaxf(m_ref[r], tmax);
          alpha_r[r] = exp2f(m_ref[r] - mn);
          l_part[r] *= alpha_r[r];
          m_ref[r] = mn;
        }
      } else {
#pragma unroll
        for (int r = 0; r < RG; ++r) alpha_r[r] = 1.f;
      }
      // ---- P = exp2(x - m_ref) as f16 hi + lo parts, stacked [P_hi; P_lo],
      //      MN-major without swizzle (8-row x 16-byte core matrices)
      {
        const uint32_t pbuf = sbase + FC::oP + (uint32_t)((i & 1) * FC::kPBufBytes);
        const uint32_t prow = pbuf + (uint32_t)((kl >> 3) * (16 * 2 * N) + (kl & 7) * 16);
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int q2 = 0; q2 < 4; ++q2) {
          const int r0 = 2 * q2, r1 = r0 + 1;
          float p0 = 0.f, p1 = 0.f;
          if (r0 < RG) { p0 = exp2f(s[r0] - m_ref[r0]); l_part[r0] += p0; }
          if (r1 < RG) { p1 = exp2f(s[r1] - m_ref[r1]); l_part[r1] += p1; }
          const __half2 h2 = __floats2half2_rn(p0, p1);
          const __half2 l2 = __floats2half2_rn(p0 - __low2float(h2), p1 - __high2float(h2));
          hi[q2] = *reinterpret_cast<const uint32_t*>(&h2);
          lo[q2] = *reinterpret_cast<const uint32_t*>(&l2);
        }
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                     ::"r"(prow), "r"(hi[0]), "r"(hi[1]), "r"(hi[2]), "r"(hi[3]) : "memory");
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                     ::"r"(prow + N * 16), "r"(lo[0]), "r"(lo[1]), "r"(lo[2]), "r"(lo[3]) : "memory");
      }
      ptx::fence_proxy_async_smem();
      ptx::mbar_arrive(p_full + 8u * (i & 1));
      process_o(i);                            // this group's next tile is i + 2
      ++li;
    }
    ptx::pdl_launch_dependents();

    // ---- epilogue: the two groups hold the same rows; merge them by LSE
    //      through the idle staging ring, scale by the V scale, write
    bool bad = ptx::bar_sync_or(3, kSoftmaxThreads * NG, aborted || failed);
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
    bad = ptx::bar_sync_or(3, kSoftmaxThreads * NG, bad);
    if (!bad) {
      const int et = tid - 64, ew = et >> 5;
      for (int q = ew; q < NG * RG; q += 4 * NG) {
        const float* src = el + q * kHeadDim;
        const float vsum = warp_sum(src[lane] + src[lane + 32] + src[lane + 64] + src[lane + 96]);
        if (lane == 0) es[q] = vsum;
      }
      ptx::bar_sync_or(3, kSoftmaxThreads * NG, false);
      const float vsc = __ldg(p.v_scale + h);
      const int rows = p.B * p.Hq;
      for (int e = et; e < NQ * kHeadDim; e += kSoftmaxThreads * NG) {
        const int n = e / kHeadDim, dd = e % kHeadDim;
        const float m = fmaxf(em[n], em[RG + n]);
        const float sc0 = exp2f(em[n] - m), sc1 = exp2f(em[RG + n] - m);
        const float l = es[n] * sc0 + es[RG + n] * sc1;
        float o = eo[n * kHeadDim + dd] * sc0 + eo[(RG + n) * kHeadDim + dd] * sc1;
        o = (l > 0.f) ? o * vsc / l : 0.f;
        const float lse_v = (l > 0.f) ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
        const int row = b * p.Hq + h * G + n;
        if (p.num_splits == 1) {
          if (p.out_fp32) reinterpret_cast<float*>(p.out)[(size_t)row * kHeadDim + dd] = o;
          else reinterpret_cast<__nv_bfloat16*>(p.out)[(size_t)row * kHeadDim + dd] = __float2bfloat16_rn(o);
          if (p.lse && dd == 0) p.lse[row] = lse_v;
        } else {
          p.ws_o[((size_t)s_idx * rows + row) * kHeadDim + dd] = o;
          if (dd == 0) p.ws_lse[(size_t)s_idx * rows + row] = lse_v;
        }
      }
    }
  }

  // -------------------------------------------------------------- teardown
  ptx::tc_fence_before();
  __syncthreads();
  // an aborted CTA, or one that met a block-table entry outside the pool,
  // writes its rows as NaN (see the bf16 kernel)
  const bool aborted_cta = *abort_flag != 0, bad_cta = *bad_page_flag != 0;
  if (tid == 0) {
    if (aborted_cta) atomicOr(p.status, kStatusTimeout);
    if (bad_cta) atomicOr(p.status, kStatusBadSeq);
  }
  if (aborted_cta || bad_cta)
    fill_rows<G>(p, b, h, s_idx, __int_as_float(0x7fc00000), __int_as_float(0x7fc00000));
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, FC::kTmemCols);
  }
}

}  // namespace relattn
