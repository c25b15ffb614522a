// rel_attn_kvwrite.cuh -- the KV-cache producer step that feeds the decode
// kernels: short convolution over the new tokens' K and V, the paged
// KV-cache write, and (optionally) E4M3 quantisation, in one kernel.
//
// "vLLM TML Inkling 지원", section "TML Inkling 모델 아키텍처": every layer
// applies short convolutions (window 4) to the attention keys and values;
// section "Sconv 캐시 및 TP 샤딩": the sconv state lives in the unified
// KV-cache manager as the cache of a virtual sliding-window layer, and the
// convolution works per channel.  "A vLLM már az első napon támogatja a
// Reflection Beam modellt" names a fused KV-cache update.  Reading taken:
//   k~[p][h][c] = sum_{i=0..3} w_k[h][c][i] * k[p-i][h][c]   (k[q<0] = 0)
// and likewise for V; the raw (pre-convolution) K/V of every position are
// kept in a paged sconv cache laid out and addressed like the KV cache.
//
// One thread per (new token, KV head, 8 channels): eight 16-byte loads of
// the raw K and V vectors at p, p-1, p-2, p-3 (from the new tokens, or from
// the sconv cache for positions before them; neighbouring tokens share them
// through L1), all issued before any arithmetic (K then V one at a time
// measured 37.0 against 34.3 us for 8,192 tokens, 12.1 against 8.2 us for
// one), a 64-byte load of each tap set, fp32 accumulation with taps in the
// order 0, 1, 2, 3, then a 16-byte raw store and a 16-byte bf16 (or 8-byte
// E4M3) cache store per K and V.  Positions written (the new ones) and positions
// read from the sconv cache (the older ones) never meet, so a launch has no
// read-after-write hazard of its own.  HBM-bound: per new token and KV head
// 256 B in, 256 B raw out, 256 B (or 128 B) cache out.
#pragma once

namespace relattn {

struct KvWriteParams {
  const __nv_bfloat16* k_new;   // [B, T, Hkv, D]
  const __nv_bfloat16* v_new;
  const __nv_bfloat16* conv_w;  // [2, Hkv, D, 4]: K taps, then V taps
  __nv_bfloat16* k_raw;         // sconv cache [num_pages, Hkv, P, D]
  __nv_bfloat16* v_raw;
  void* k_cache;                // KV cache [num_pages, Hkv, P, D]: bf16, or E4M3 codes
  void* v_cache;
  const float* k_scale;         // E4M3 only: per-KV-head scales
  const float* v_scale;
  const int* block_table;       // [B, max_pages]
  const int* seq_lens;          // [B], including the T new tokens
  unsigned* status;             // status word, or null
  int B, T, Hkv, num_pages, max_pages;
};

constexpr int kKvwThreads = 128;                 // 8 tokens x 16 groups of 8 channels
constexpr int kKvwTokensPerCta = kKvwThreads / (kHeadDim / 8);

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float* f) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 x = __bfloat1622float2(h[e]);
    f[2 * e] = x.x;
    f[2 * e + 1] = x.y;
  }
}

// E4M3 codes of (lo, hi), round to nearest even, saturating at +-448; lo in
// the low byte.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

template <bool E4M3>
__global__ void __launch_bounds__(kKvwThreads)
rel_attn_kv_write_kernel(const __grid_constant__ KvWriteParams p) {
  // a following kernel launched as a programmatic dependent may start its
  // prologue now; it waits for this grid's writes before reading them
  ptx::pdl_launch_dependents();
  const int b = blockIdx.z, h = blockIdx.y;
  const int t = blockIdx.x * kKvwTokensPerCta + (threadIdx.x >> 4);
  const int c0 = (threadIdx.x & 15) * 8;
  if (t >= p.T) return;
  const int L = __ldg(p.seq_lens + b);
  if (L < p.T || L > p.max_pages * kPage) {
    if (p.status && t == 0 && c0 == 0) atomicOr(p.status, kStatusBadSeq);
    return;
  }
  const int first_new = L - p.T;
  const int pos = first_new + t;
  const int* bt = p.block_table + (size_t)b * p.max_pages;
  // pages of positions pos, pos-1, pos-2, pos-3 (the older ones only where
  // they come from the sconv cache), all checked before anything is written
  int qpage[4];
  bool bad = false;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int q = pos - i;
    qpage[i] = -1;
    if (i == 0 || (q >= 0 && q < first_new)) {
      qpage[i] = __ldg(bt + q / kPage);
      bad |= qpage[i] < 0 || qpage[i] >= p.num_pages;
    }
  }
  if (bad) {
    if (p.status) atomicOr(p.status, kStatusBadSeq);
    return;
  }
  const size_t dst = (((size_t)qpage[0] * p.Hkv + h) * kPage + pos % kPage) * kHeadDim + c0;
  // all eight raw vectors (K and V at pos, pos-1, pos-2, pos-3) first
  uint4 xs[2][4];
#pragma unroll
  for (int kv = 0; kv < 2; ++kv) {
    const __nv_bfloat16* src_new = kv ? p.v_new : p.k_new;
    const __nv_bfloat16* raw = kv ? p.v_raw : p.k_raw;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int q = pos - i;
      uint4 xv = make_uint4(0, 0, 0, 0);
      if (q >= first_new) {
        xv = __ldg(reinterpret_cast<const uint4*>(
            src_new + (((size_t)b * p.T + (q - first_new)) * p.Hkv + h) * kHeadDim + c0));
      } else if (q >= 0) {
        xv = *reinterpret_cast<const uint4*>(
            raw + (((size_t)qpage[i] * p.Hkv + h) * kPage + q % kPage) * kHeadDim + c0);
      }
      xs[kv][i] = xv;
    }
  }
#pragma unroll
  for (int kv = 0; kv < 2; ++kv) {
    __nv_bfloat16* raw = kv ? p.v_raw : p.k_raw;
    const uint4* wp = reinterpret_cast<const uint4*>(p.conv_w + (((size_t)kv * p.Hkv + h) * kHeadDim + c0) * 4);
    float w[32];
#pragma unroll
    for (int u = 0; u < 4; ++u) bf16x8_to_f32(__ldg(wp + u), w + 8 * u);
    float acc[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float x[8];
      bf16x8_to_f32(xs[kv][i], x);
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] = (i == 0) ? w[4 * c] * x[c] : fmaf(w[4 * c + i], x[c], acc[c]);
    }
    *reinterpret_cast<uint4*>(raw + dst) = xs[kv][0];
    if constexpr (!E4M3) {
      uint4 o;
      __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
      for (int e = 0; e < 4; ++e) o2[e] = __floats2bfloat162_rn(acc[2 * e], acc[2 * e + 1]);
      *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(kv ? p.v_cache : p.k_cache) + dst) = o;
    } else {
      const float sc = __ldg((kv ? p.v_scale : p.k_scale) + h);
      uint32_t pk[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) pk[e] = f32x2_to_e4m3x2(acc[2 * e] / sc, acc[2 * e + 1] / sc);
      const uint2 o = make_uint2(pk[0] | (pk[1] << 16), pk[2] | (pk[3] << 16));
      *reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(kv ? p.v_cache : p.k_cache) + dst) = o;
    }
  }
}

}  // namespace relattn
