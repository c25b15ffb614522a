// rel_attn_fp8.cuh -- partial kernel over an FP8 (E4M3) KV cache, one query
// token per sequence.
//
// The FP8 KV cache is the next step the Inkling page plans for its global
// attention layers ("vLLM TML Inkling 지원", section "미래 로드맵"): it halves
// the bytes of the bandwidth-bound decode.  Codes are OFP8 E4M3, one fp32
// scale per KV head for K and one for V (k = e4m3(code) * k_scale[h]).
//
// The E4M3 page tiles are the tensor-core operands themselves
// (tcgen05.mma kind::f8f6f4, both operands E4M3): nothing is widened on
// chip.  Neither the query nor P may lose precision, so each is carried as
// a short sum of E4M3 terms, each term scaled into E4M3 range and given its
// own rows of the MMA's N side:
//   S^T = K8 . [Q_hi; Q_lo]^T       q * 2^e_r = Q_hi + Q_lo / 16, exact for a
//                                   bf16 query (8 significant bits = 4 + 4)
//   O^T = V8^T . [P_hi; P_mid; P_lo]^T   P = P_hi + P_mid / 16 + P_lo / 256,
//                                   12 significant bits
//   X^T = R_chunk . Q^T             bf16 (kind::f16) as in the bf16 kernel
// Roles: warp 0 TMA producer of K8 page tiles (8 KB per page) and
// relative-row chunks, warp 11 of V8 page tiles (each in its own ring), warp
// 1 issues S and X, warp 10 issues P.V, two softmax groups of 4 warps (2..9)
// alternate tiles.  The two
// MMA issuers run side by side: a single issuing thread spends about a
// microsecond per tile on its waits, descriptors and eight MMA issues, more
// than the tile's bytes take to arrive at the HBM rate.
// The K scale and the query's per-row power of two fold into the logit
// scale, the V scale into the output.  The lazy reference max keeps
// P <= 2^8 here, inside E4M3 range.
#pragma once

namespace relattn {

template <int G>
struct Fp8Config {
  static constexpr int N = 16;                                  // S^T / X^T columns
  static constexpr int NP = 32;                                 // P.V columns: 3 terms x G rows
  static constexpr int NG = 2, RG = G;
  static_assert(2 * G <= N && 3 * G <= NP && G % 2 == 0, "group size");
  static constexpr int kPvWarp = 2 + 4 * NG;                   // after the softmax warps
  static constexpr int kVWarp = kPvWarp + 1;                    // V-tile producer
  static constexpr int kThreads = 64 + kSoftmaxThreads * NG + 64;
  static constexpr int kKSlots = 4, kVSlots = 6, kRSlots = 1;
  static constexpr int kTile8 = 128 * 128;                      // 128 keys x 128 B
  static constexpr int kPage8 = 64 * 128;
  static constexpr int kRHalf = 128 * 128;                      // 128 rows x 64 dims bf16
  static constexpr int kRBytes = 2 * kRHalf;
  static constexpr int kYStride = G + 1;
  static constexpr int kGR = 8;
  static constexpr int kPBufBytes = 128 * NP;                   // 128 keys x 32 B
  static constexpr int kYBytes = align_up(128 * kYStride * 4, 16);
  static constexpr int oK = 0;
  static constexpr int oV = oK + kKSlots * kTile8;
  static constexpr int oR = oV + kVSlots * kTile8;
  static constexpr int oQ8 = oR + kRSlots * kRBytes;            // [Q_hi; Q_lo; 0]: 16 rows x 128 B
  static constexpr int oQ = oQ8 + N * 128;                      // bf16 Q for X: 16 rows x 256 B
  static constexpr int oP = oQ + 2 * N * 128;                   // two P buffers
  static constexpr int oY = oP + 2 * kPBufBytes;                // one table per group
  static constexpr int oRed = oY + NG * kYBytes;                // [NG][2][4][kGR]
  static constexpr int oQf = oRed + NG * 2 * 4 * kGR * 4;       // per-row logit factors [G]
  static constexpr int oEdges = oQf + 64;
  static constexpr int oBar = align_up(oEdges + (kMaxTailBuckets + 1) * 4, 8);
  // kfull/kempty[KS] vfull/vempty[VS] rfull/rempty[RS] s_full/s_empty[2]
  // p_full[2] o_full/o_empty[2] x_full/x_empty[2] drain (S issuer) drain (P.V issuer)
  static constexpr int kNumBars = 2 * (kKSlots + kVSlots + kRSlots) + 4 + 2 + 4 + 4 + 2;
  // tmem base, abort flag, bad-page flag, K / V tiles and relative chunks issued
  static constexpr int oMisc = oBar + kNumBars * 8;
  // per K slot: 1 if its tile starts a new relative-row chunk (producer ->
  // S issuer, published by the slot's full barrier)
  static constexpr int oChunkFlag = oMisc + 32;
  static constexpr int kBytes = oChunkFlag + align_up(kKSlots, 16);
  static constexpr int kAllocBytes = kBytes + 1024;
  static constexpr int kTmemCols = 128;                         // S[2] 32 + O[2] 64 + X[2] 32
  static_assert(kAllocBytes <= 232448, "shared memory budget exceeded");
  static_assert(oV % 1024 == 0 && oR % 1024 == 0 && oQ8 % 1024 == 0 && oQ % 1024 == 0,
                "operand alignment");
  static_assert(oV >= NG * RG * 128 * 4 * 2 + NG * RG * 4 * 2, "epilogue exchange area");
};

// E4M3 codes of (lo, hi), round to nearest even, saturating; lo in the low byte.
__device__ __forceinline__ uint32_t e4m3x2_rn(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}
// The two values of an E4M3 pair (low byte first), exactly.
__device__ __forceinline__ float2 e4m3x2_value(uint32_t v) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"((uint16_t)v));
  return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

template <int G>
__global__ void __launch_bounds__(Fp8Config<G>::kThreads, 1)
rel_attn_partial_fp8_kernel(const __grid_constant__ DecodeParams p) {
  using FC = Fp8Config<G>;
  constexpr int N = FC::N, NP = FC::NP, NG = FC::NG, RG = FC::RG;
  constexpr int YS = FC::kYStride;
  constexpr int KS = FC::kKSlots, VS = FC::kVSlots, RS = FC::kRSlots;
  constexpr int T = 1;
  constexpr float kLazy8 = 8.f;               // P = exp2(x - m_ref) <= 2^8 < 448

  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned, by pointer arithmetic on the shared array so that the
  // compiler keeps every access through smem in the shared window
  uint8_t* smem = smem_raw + ((1024u - (ptx::smem_addr(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = ptx::smem_addr(smem);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  // Several query tokens run as one-token chunks (DecodeParams::cps of them
  // per sequence), the chunk index fastest in x so that the CTAs of one
  // (split, KV head) read the same pages at about the same time.
  const int chunk = (int)blockIdx.x % p.cps;
  const int s_idx = (int)blockIdx.x / p.cps, h = blockIdx.y;
  const int b_seq = blockIdx.z;                    // the sequence (block-table row)
  const int b = b_seq * p.cps + chunk;             // grid z-index of this chunk
  const int row0 = first_token_row(p, b);          // q / out row of its token

  // ------------------------------------------------------------ geometry
  SplitGeom g;
  // the block-table row towards L2 while the length is read
  if (warp == 0)
    ptx::prefetch_l2_range(p.block_table + (size_t)b_seq * p.max_pages, (size_t)p.max_pages * 4, 128, lane);
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
  if (g.ntiles == 0) {
    fill_rows<G>(p, row0, h, s_idx, 0.f, -INFINITY);
    return;
  }

  // --------------------------------------------------------- smem carve-up
  int* s_edges = reinterpret_cast<int*>(smem + FC::oEdges);
  float* qf = reinterpret_cast<float*>(smem + FC::oQf);
  const uint32_t bar0 = sbase + FC::oBar;
  auto kfull = [&](int s) { return bar0 + 8u * s; };
  auto kempty = [&](int s) { return bar0 + 8u * (KS + s); };
  auto vfull = [&](int s) { return bar0 + 8u * (2 * KS + s); };
  auto vempty = [&](int s) { return bar0 + 8u * (2 * KS + VS + s); };
  auto rfull = [&](int s) { return bar0 + 8u * (2 * KS + 2 * VS + s); };
  auto rempty = [&](int s) { return bar0 + 8u * (2 * KS + 2 * VS + RS + s); };
  constexpr int kB = 2 * (KS + VS + RS);
  const uint32_t s_full = bar0 + 8u * (kB + 0);     // +8*buf
  const uint32_t s_empty = bar0 + 8u * (kB + 2);
  const uint32_t p_full = bar0 + 8u * (kB + 4);
  const uint32_t o_full = bar0 + 8u * (kB + 6);
  const uint32_t o_empty = bar0 + 8u * (kB + 8);
  const uint32_t x_full = bar0 + 8u * (kB + 10);    // +8*group
  const uint32_t x_empty = bar0 + 8u * (kB + 12);
  const uint32_t drain_bar = bar0 + 8u * (kB + 14);
  const uint32_t drain_pv = bar0 + 8u * (kB + 15);
  uint8_t* chunk_flag = smem + FC::oChunkFlag;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + FC::oMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + FC::oMisc + 4);
  volatile int* bad_page_flag = reinterpret_cast<volatile int*>(smem + FC::oMisc + 8);
  int* issued = reinterpret_cast<int*>(smem + FC::oMisc + 12);   // [K tiles, V tiles, chunks]
  auto kslot = [&](int i) { return sbase + FC::oK + (uint32_t)((i % KS) * FC::kTile8); };
  auto vslot = [&](int i) { return sbase + FC::oV + (uint32_t)((i % VS) * FC::kTile8); };
  auto rslot = [&](int c) { return sbase + FC::oR + (uint32_t)((c % RS) * FC::kRBytes); };
  const unsigned long long tlim = p.timeout_ns;

  // -------------------------------------------------------------- prologue
  if (tid == 0) {
    for (int s = 0; s < KS; ++s) { ptx::mbar_init(kfull(s), 1); ptx::mbar_init(kempty(s), 1); }
    for (int s = 0; s < VS; ++s) { ptx::mbar_init(vfull(s), 1); ptx::mbar_init(vempty(s), 1); }
    for (int s = 0; s < RS; ++s) { ptx::mbar_init(rfull(s), 1); ptx::mbar_init(rempty(s), 1); }
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
    ptx::mbar_init(drain_pv, 1);
    *abort_flag = 0;
    *bad_page_flag = 0;
    issued[0] = issued[1] = issued[2] = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&p.tmap_k);
    ptx::prefetch_tmap(&p.tmap_v);
    ptx::prefetch_tmap(&p.tmap_r);
  }
  __syncthreads();
  uint32_t tmem = 0;
  if (warp != 0 && warp != FC::kVWarp) {
    if (warp == 1) {
      ptx::tmem_alloc(ptx::smem_addr(tmem_holder), FC::kTmemCols);
      ptx::tmem_relinquish();
    } else if (warp != FC::kPvWarp) {
      const int st = tid - 64;                  // softmax thread 0..255
      const int sw = st >> 5;                   // its warp 0..7
      // bf16 Q for X: rows 0..G-1 the group's heads, other rows zero,
      // 128B-swizzled K-major in two 64-dim halves
      for (int u = st; u < N * 16; u += kSoftmaxThreads * NG) {
        const int n = u >> 4, half = (u >> 3) & 1, w16 = u & 7;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (n < G)
          v = __ldg(reinterpret_cast<const uint4*>(
              p.q + ((size_t)row0 * p.Hq + h * G + n) * kHeadDim + half * 64 + w16 * 8));
        *reinterpret_cast<uint4*>(smem + FC::oQ + half * (N * 128) + n * 128 + ((w16 ^ (n & 7)) << 4)) = v;
      }
      // E4M3 Q: warp w < G splits head row w.  q * 2^e (e puts the row's
      // largest |q| in [128, 256)) = Q_hi + Q_lo / 16: Q_hi the nearest E4M3
      // value, Q_lo the E4M3 code of 16 x the remainder (at most four
      // significant bits of a bf16 query remain, so the sum is exact down to
      // 2^-10 x the row maximum).  Rows G..2G-1 hold Q_lo, the rest zero.
      if (sw < G) {
        const uint2 raw = __ldg(reinterpret_cast<const uint2*>(
            p.q + ((size_t)row0 * p.Hq + h * G + sw) * kHeadDim + lane * 4));
        const __nv_bfloat162* q2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
        const float2 a = __bfloat1622float2(q2[0]), c = __bfloat1622float2(q2[1]);
        float mx = fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(c.x), fabsf(c.y)));
        mx = warp_max(mx);
        int e = 0;
        if (mx > 0.f) {
          int ex;
          frexpf(mx, &ex);                      // mx = m 2^ex, m in [0.5, 1)
          e = 8 - ex;                           // mx 2^e in [128, 256)
        }
        const float sc = ldexpf(1.f, e);
        const float x0 = a.x * sc, x1 = a.y * sc, x2 = c.x * sc, x3 = c.y * sc;
        const uint32_t h01 = e4m3x2_rn(x0, x1), h23 = e4m3x2_rn(x2, x3);
        const float2 v01 = e4m3x2_value(h01), v23 = e4m3x2_value(h23);
        const uint32_t l01 = e4m3x2_rn((x0 - v01.x) * 16.f, (x1 - v01.y) * 16.f);
        const uint32_t l23 = e4m3x2_rn((x2 - v23.x) * 16.f, (x3 - v23.y) * 16.f);
        const int chunk = lane >> 2, sub = (lane & 3) * 4;
        auto put = [&](int n, uint32_t w) {
          *reinterpret_cast<uint32_t*>(smem + FC::oQ8 + n * 128 + ((chunk ^ (n & 7)) << 4) + sub) = w;
        };
        put(sw, h01 | (h23 << 16));
        put(G + sw, l01 | (l23 << 16));
        // logit factor of this row: the K scale, the 2^-e of the split and
        // log2(e) / sqrt(D)
        if (lane == 0) qf[sw] = __ldg(p.k_scale + h) * ldexpf(1.f, -e) * p.scale_log2;
      } else {
        // rows 2G..15 are zero
        for (int u = (sw - G) * 32 + lane; u < (N - 2 * G) * 32; u += (8 - G) * 32)
          *reinterpret_cast<uint32_t*>(smem + FC::oQ8 + (2 * G + u / 32) * 128 + (u % 32) * 4) = 0u;
      }
      for (int e = st; e <= p.nl; e += kSoftmaxThreads * NG) s_edges[e] = p.edges[e];
      ptx::fence_proxy_async_smem();
    }
    ptx::tc_fence_before();
    ptx::bar_sync_or(kBarSetup, FC::kThreads - 64, false);   // every warp but the producers
    ptx::tc_fence_after();
    tmem = *tmem_holder;
  }
  const uint32_t tS = tmem;                        // S buffer i at +N*i
  const uint32_t tO = tmem + 2 * N;                // O buffer i at +NP*i
  auto tX = [&](int gq) { return tmem + 2 * N + 2 * NP + N * gq; };

  // ------------------------------------------------------------- producer
  if (warp == 0) {
    const uint64_t pol = ptx::l2_policy_evict_first();
    const int* bt_row = p.block_table + (size_t)b_seq * p.max_pages;
    auto bt_load = [&](int grp) -> int {
      const int pg = g.sp_begin + 32 * grp + lane;
      return (pg < g.sp_end) ? __ldg(bt_row + pg) : 0;
    };
    int bt_cur = bt_load(0);
    int bt_next = bt_load(1);
    int nk = 0, nr = 0;                        // K tiles, relative chunks issued
    PlanState ps0(p.nl), ps1(p.nl);
    bool ok = true, bad_page = false;
    for (int ti = 0; ti < g.ntiles; ++ti) {
      if (ti > 0 && (ti & 15) == 0) {
        bt_cur = bt_next;
        bt_next = bt_load((ti >> 4) + 1);
      }
      const bool odd = ti & 1;
      const TilePlan tp = plan_tile<128>(g, ti, p.ex, p.log2_ex, p.log_scale, p.edges, odd ? ps1 : ps0);
      const int c0 = odd ? ps1.c0 : ps0.c0;
      if (tp.chunk) {
        ok = __all_sync(0xffffffffu, ptx::mbar_wait(rempty(nr % RS), ((nr / RS) & 1) ^ 1, abort_flag, tlim));
        if (!ok) break;
        if (lane == 0) {
          const uint32_t st = rslot(nr);
          ptx::mbar_arrive_expect_tx(rfull(nr % RS), FC::kRBytes);
          ptx::tma_load_3d(st, &p.tmap_r, rfull(nr % RS), 0, c0, h);
          ptx::tma_load_3d(st + FC::kRHalf, &p.tmap_r, rfull(nr % RS), 64, c0, h);
        }
        ++nr;
      }
      int e0 = __shfl_sync(0xffffffffu, bt_cur, (2 * ti) & 31);
      int e1 = __shfl_sync(0xffffffffu, bt_cur, (2 * ti + 1) & 31);
      if (e0 < 0 || e0 >= p.num_pages) { bad_page = true; e0 = 0; }
      if (tp.npg > 1 && (e1 < 0 || e1 >= p.num_pages)) { bad_page = true; e1 = 0; }
      const int row0 = (e0 * p.Hkv + h) * kPage, row1 = (e1 * p.Hkv + h) * kPage;
      ok = __all_sync(0xffffffffu, ptx::mbar_wait(kempty(ti % KS), ((ti / KS) & 1) ^ 1, abort_flag, tlim));
      if (!ok) break;
      if (lane == 0) {
        chunk_flag[ti % KS] = tp.chunk ? 1 : 0;
        ptx::mbar_arrive_expect_tx(kfull(ti % KS), tp.npg * FC::kPage8);
        ptx::tma_load_2d(kslot(ti), &p.tmap_k, kfull(ti % KS), 0, row0, pol);
        if (tp.npg > 1) ptx::tma_load_2d(kslot(ti) + FC::kPage8, &p.tmap_k, kfull(ti % KS), 0, row1, pol);
      }
      ++nk;
    }
    if (lane == 0) {
      if (bad_page) *bad_page_flag = 1;
      issued[0] = nk;                        // for the drain at teardown
      issued[2] = nr;
    }
  }
  // ------------------------------------------------------- V-tile producer
  // V tiles come from a warp of their own: one warp issuing K, V and the
  // relative chunks, with the tile plan in between, took longer per tile than
  // the tile's bytes take to arrive.
  else if (warp == FC::kVWarp) {
    const uint64_t pol = ptx::l2_policy_evict_first();
    const int* bt_row = p.block_table + (size_t)b_seq * p.max_pages;
    auto bt_load = [&](int grp) -> int {
      const int pg = g.sp_begin + 32 * grp + lane;
      return (pg < g.sp_end) ? __ldg(bt_row + pg) : 0;
    };
    int bt_cur = bt_load(0);
    int bt_next = bt_load(1);
    int nv = 0;                                // V tiles issued
    bool bad_page = false;
    for (int ti = 0; ti < g.ntiles; ++ti) {
      if (ti > 0 && (ti & 15) == 0) {
        bt_cur = bt_next;
        bt_next = bt_load((ti >> 4) + 1);
      }
      const int npg = min(2, g.sp_end - (g.sp_begin + 2 * ti));
      int e0 = __shfl_sync(0xffffffffu, bt_cur, (2 * ti) & 31);
      int e1 = __shfl_sync(0xffffffffu, bt_cur, (2 * ti + 1) & 31);
      if (e0 < 0 || e0 >= p.num_pages) { bad_page = true; e0 = 0; }
      if (npg > 1 && (e1 < 0 || e1 >= p.num_pages)) { bad_page = true; e1 = 0; }
      const int row0 = (e0 * p.Hkv + h) * kPage, row1 = (e1 * p.Hkv + h) * kPage;
      if (!__all_sync(0xffffffffu, ptx::mbar_wait(vempty(ti % VS), ((ti / VS) & 1) ^ 1, abort_flag, tlim)))
        break;
      if (lane == 0) {
        ptx::mbar_arrive_expect_tx(vfull(ti % VS), npg * FC::kPage8);
        ptx::tma_load_2d(vslot(ti), &p.tmap_v, vfull(ti % VS), 0, row0, pol);
        if (npg > 1) ptx::tma_load_2d(vslot(ti) + FC::kPage8, &p.tmap_v, vfull(ti % VS), 0, row1, pol);
      }
      ++nv;
    }
    if (lane == 0) {
      if (bad_page) *bad_page_flag = 1;
      issued[1] = nv;                        // for the drain at teardown
    }
  }
  // ------------------------------------------------------- S and X issuer
  else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t kIdescS = ptx::idesc_e4m3(128, N, false, false);    // K8 . [Q_hi; Q_lo]
      constexpr uint32_t kIdescX = ptx::idesc_bf16(128, N, false, false);    // R . Q
      const uint64_t kdesc0 = ptx::sdesc_sw128(sbase + FC::oK, 16, 1024);    // K8, K-major
      const uint64_t q8desc = ptx::sdesc_sw128(sbase + FC::oQ8, 16, 1024);   // Q8, K-major
      const uint64_t rdesc0 = ptx::sdesc_sw128(sbase + FC::oR, 16, 1024);    // R chunk, K-major
      const uint64_t qdesc = ptx::sdesc_sw128(sbase + FC::oQ, 16, 1024);     // bf16 Q, K-major
      int nr = 0;                              // chunks issued
      int cg[2] = {0, 0};                      // chunks per group
      for (int ti = 0; ti < g.ntiles; ++ti) {
        const int gq = ti & 1;
        if (!ptx::mbar_wait(kfull(ti % KS), (ti / KS) & 1, abort_flag, tlim)) break;
        if (chunk_flag[ti % KS]) {
          const int c = cg[gq];
          if (!ptx::mbar_wait(rfull(nr % RS), (nr / RS) & 1, abort_flag, tlim) ||
              !ptx::mbar_wait(x_empty + 8u * gq, (c & 1) ^ 1, abort_flag, tlim))
            break;
          ptx::tc_fence_after();
          const uint64_t rd = rdesc0 + (uint64_t)(((nr % RS) * FC::kRBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t ra = rd + (uint64_t)(((kk >> 2) * FC::kRHalf + (kk & 3) * 32) >> 4);
            const uint64_t bq = qdesc + (uint64_t)(((kk >> 2) * (N * 128) + (kk & 3) * 32) >> 4);
            ptx::umma_bf16(tX(gq), ra, bq, kIdescX, kk > 0);
          }
          ptx::umma_commit(x_full + 8u * gq);
          ptx::umma_commit(rempty(nr % RS));
          ++nr;
          cg[gq] = c + 1;
        }
        if (!ptx::mbar_wait(s_empty + 8u * gq, ((ti >> 1) & 1) ^ 1, abort_flag, tlim)) break;
        ptx::tc_fence_after();
        const uint64_t kd = kdesc0 + (uint64_t)(((ti % KS) * FC::kTile8) >> 4);
        // K = 32 dims (32 B of each 128 B row) per MMA
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          ptx::umma_e4m3(tS + gq * N, kd + (uint64_t)((kk * 32) >> 4),
                         q8desc + (uint64_t)((kk * 32) >> 4), kIdescS, kk > 0);
        ptx::umma_commit(s_full + 8u * gq);
        ptx::umma_commit(kempty(ti % KS));
      }
      ptx::umma_commit(drain_bar);
      volatile int never = 0;
      ptx::mbar_wait(drain_bar, 0, &never, kDrainLimitNs);
    }
    __syncwarp();
  }
  // ----------------------------------------------------------- P.V issuer
  else if (warp == FC::kPvWarp) {
    if (lane == 0) {
      constexpr uint32_t kIdescPV = ptx::idesc_e4m3(128, NP, true, true);    // V8^T . [P terms]
      const uint64_t vdesc0 = ptx::sdesc_sw128(sbase + FC::oV, 16, 1024);    // V8^T, MN-major
      const uint64_t pdesc0 = ptx::sdesc_noswz(sbase + FC::oP, 256, 128);    // P terms, MN-major
      for (int j = 0; j < g.ntiles; ++j) {
        if (!ptx::mbar_wait(p_full + 8u * (j & 1), (j >> 1) & 1, abort_flag, tlim) ||
            !ptx::mbar_wait(o_empty + 8u * (j & 1), ((j >> 1) & 1) ^ 1, abort_flag, tlim) ||
            !ptx::mbar_wait(vfull(j % VS), (j / VS) & 1, abort_flag, tlim))
          break;
        ptx::tc_fence_after();
        const uint64_t va = vdesc0 + (uint64_t)(((j % VS) * FC::kTile8) >> 4);
        const uint64_t pb = pdesc0 + (uint64_t)(((j & 1) * FC::kPBufBytes) >> 4);
        // K = 32 keys per MMA: 32 rows of the V tile (4 KB), four 8-key
        // core-matrix groups of P (1 KB)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          ptx::umma_e4m3(tO + (j & 1) * NP, va + (uint64_t)((kk * 4096) >> 4),
                         pb + (uint64_t)((kk * 1024) >> 4), kIdescPV, kk > 0);
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
    float fq[RG];
#pragma unroll
    for (int r = 0; r < RG; ++r) fq[r] = qf[r];
    float l_part[RG], o_acc[RG], m_ref[RG], alpha_r[RG];
#pragma unroll
    for (int r = 0; r < RG; ++r) { l_part[r] = 0.f; o_acc[r] = 0.f; m_ref[r] = kNoMax; alpha_r[r] = 1.f; }
    int c = 0, li = 0;
    PlanState ps(p.nl);                       // this group's tiles only
    bool failed = false, aborted = false;

    // O^T of tile j: columns 0..G-1 from P_hi, G..2G-1 from P_mid, 2G..3G-1
    // from P_lo
    auto process_o = [&](int j) {
      float ov[24];
      const bool okw = ptx::mbar_wait(o_full + 8u * (j & 1), (j >> 1) & 1, abort_flag, tlim);
      if (okw) {
        ptx::tc_fence_after();
        const uint32_t ob = tO + lane_off + (j & 1) * NP;
        ptx::tmem_ld16(ob, ov);
        ptx::tmem_ld8(ob + 16, ov + 16);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int r = 0; r < RG; ++r)
          o_acc[r] = fmaf(o_acc[r], alpha_r[r],
                          ov[r] + fmaf(ov[G + r], 0.0625f, ov[2 * G + r] * 0.00390625f));
        ptx::tc_fence_before();
      }
      ptx::mbar_arrive(o_empty + 8u * (j & 1));
      if (!okw) failed = true;
    };

    // Group g takes the tiles g, g + 2, ...; the plan of its next tile is
    // made while P.V of the current one runs.
    TilePlan tp_next{};
    int c0_next = 0;
    if (grp < g.ntiles) {
      tp_next = plan_tile<128>(g, grp, p.ex, p.log2_ex, p.log_scale, s_edges, ps);
      c0_next = ps.c0;
    }
    for (int ti = grp; ti < g.ntiles; ti += 2) {
      const TilePlan tp = tp_next;
      const int c0 = c0_next;
      if (tp.chunk) {
        // ---- new relative-row chunk: X^T (128 rows x G) -> gather table Y
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

      // ---- S^T tile: this thread owns key j; columns r (Q_hi) and G + r (Q_lo)
      float sv[16];
      const bool okw = ptx::mbar_wait(s_full + 8u * (i & 1), (i >> 1) & 1, abort_flag, tlim);
      if (okw) {
        ptx::tc_fence_after();
        ptx::tmem_ld16(tS + lane_off + (i & 1) * N, sv);
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
      float s[RG];
#pragma unroll
      for (int r = 0; r < RG; ++r)
        s[r] = v ? fmaf(fmaf(sv[G + r], 0.0625f, sv[r]), fq[r], yrow[r] * sl) : -INFINITY;

      // ---- lazy max (threshold 2^8: P stays inside E4M3 range)
      bool over = false;
#pragma unroll
      for (int r = 0; r < RG; ++r) over |= s[r] > m_ref[r] + kLazy8;
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
      // ---- P = exp2(x - m_ref) in [0, 2^8] as P_hi + P_mid / 16 + P_lo / 256
      //      (each the E4M3 code of 2^(4k) x what the earlier terms left;
      //      the remainders are exact in fp32), one 32-byte row per key:
      //      bytes 0..G-1 P_hi, G..2G-1 P_mid, 2G..3G-1 P_lo, the rest zero;
      //      MN-major without swizzle (8-key x 16-byte core matrices, 8-key
      //      groups 256 B apart, the two 16-row halves 128 B apart)
      {
        uint32_t hi[RG / 2], mid[RG / 2], low[RG / 2];
#pragma unroll
        for (int q2 = 0; q2 < RG / 2; ++q2) {
          const int r0 = 2 * q2, r1 = r0 + 1;
          const float p0 = exp2f(s[r0] - m_ref[r0]), p1 = exp2f(s[r1] - m_ref[r1]);
          l_part[r0] += p0;
          l_part[r1] += p1;
          hi[q2] = e4m3x2_rn(p0, p1);
          const float2 vh = e4m3x2_value(hi[q2]);
          const float a0 = p0 - vh.x, a1 = p1 - vh.y;
          mid[q2] = e4m3x2_rn(a0 * 16.f, a1 * 16.f);
          const float2 vm = e4m3x2_value(mid[q2]);
          low[q2] = e4m3x2_rn(fmaf(vm.x, -0.0625f, a0) * 256.f, fmaf(vm.y, -0.0625f, a1) * 256.f);
        }
        // the row of bytes [hi | mid | lo | 0...] as 8 little-endian words
        uint32_t w[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) w[q] = 0u;
#pragma unroll
        for (int q2 = 0; q2 < RG / 2; ++q2) {
          const int bh = 2 * q2, bm = G + 2 * q2, bl = 2 * G + 2 * q2;   // byte offsets
          w[bh >> 2] |= hi[q2] << ((bh & 3) * 8);
          w[bm >> 2] |= mid[q2] << ((bm & 3) * 8);
          w[bl >> 2] |= low[q2] << ((bl & 3) * 8);
        }
        const uint32_t prow = sbase + FC::oP + (uint32_t)((i & 1) * FC::kPBufBytes) +
                              (uint32_t)((kl >> 3) * 256 + (kl & 7) * 16);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                     ::"r"(prow), "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]) : "memory");
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                     ::"r"(prow + 128), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]) : "memory");
      }
      // ---- keys no token may see: clear their V rows (stale or poisoned
      //      codes must not reach P.V, where 0 * NaN = NaN)
      {
        const bool any_valid = loaded && j <= g.L - 1 && (g.W <= 0 || g.p0 - j < g.W);
        if (!any_valid) {
          if (ptx::mbar_wait(vfull(i % VS), (i / VS) & 1, abort_flag, tlim)) {
            uint4* vrow = reinterpret_cast<uint4*>(smem + FC::oV + (i % VS) * FC::kTile8 + kl * 128);
#pragma unroll
            for (int q = 0; q < 8; ++q) vrow[q] = make_uint4(0, 0, 0, 0);
          } else {
            failed = true;
          }
        }
      }
      ptx::fence_proxy_async_smem();
      ptx::mbar_arrive(p_full + 8u * (i & 1));
      if (ti + 2 < g.ntiles) {
        tp_next = plan_tile<128>(g, ti + 2, p.ex, p.log2_ex, p.log_scale, s_edges, ps);
        c0_next = ps.c0;
      }
      process_o(i);                            // this group's next tile is i + 2
      ++li;
    }
    ptx::pdl_launch_dependents();

    // ---- epilogue: the two groups hold the same rows; merge them by LSE
    //      through the idle K ring, scale by the V scale, write
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
      const int et = tid - 64, ew = et >> 5;
      for (int q = ew; q < NG * RG; q += 4 * NG) {
        const float* src = el + q * kHeadDim;
        const float vsum = warp_sum(src[lane] + src[lane + 32] + src[lane + 64] + src[lane + 96]);
        if (lane == 0) es[q] = vsum;
      }
      ptx::bar_sync_or(kBarSoftmaxAll, kSoftmaxThreads * NG, false);
      const float vsc = __ldg(p.v_scale + h);
      const int rows = p.rows_total;
      for (int e = et; e < RG * kHeadDim; e += kSoftmaxThreads * NG) {
        const int n = e / kHeadDim, dd = e % kHeadDim;
        const float m = fmaxf(em[n], em[RG + n]);
        const float sc0 = exp2f(em[n] - m), sc1 = exp2f(em[RG + n] - m);
        const float l = es[n] * sc0 + es[RG + n] * sc1;
        float o = eo[n * kHeadDim + dd] * sc0 + eo[(RG + n) * kHeadDim + dd] * sc1;
        o = (l > 0.f) ? o * vsc / l : 0.f;
        const float lse_v = (l > 0.f) ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
        const int row = row0 * p.Hq + h * G + n;
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
    if (aborted_cta) {
      atomicOr(p.status, kStatusTimeout);
      // the consumers stopped early: let the copies already issued land
      // before the CTA's memory is released (see the bf16 kernel)
      volatile int never = 0;
      const int nk = issued[0], nv = issued[1], nr = issued[2];
      for (int t = max(0, nk - KS); t < nk; ++t)
        ptx::mbar_wait(kfull(t % KS), (t / KS) & 1, &never, kDrainLimitNs);
      for (int t = max(0, nv - VS); t < nv; ++t)
        ptx::mbar_wait(vfull(t % VS), (t / VS) & 1, &never, kDrainLimitNs);
      for (int c = max(0, nr - RS); c < nr; ++c)
        ptx::mbar_wait(rfull(c % RS), (c / RS) & 1, &never, kDrainLimitNs);
    }
    if (bad_cta) atomicOr(p.status, kStatusBadSeq);
  }
  if (aborted_cta || bad_cta)
    fill_rows<G>(p, row0, h, s_idx, __int_as_float(0x7fc00000), __int_as_float(0x7fc00000));
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, FC::kTmemCols);
  }
}

}  // namespace relattn
