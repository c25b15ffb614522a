// rel_attn.cu -- host side of the C ABI declared in include/rel_attn.h:
// argument validation, the split heuristic, the bucket edge table, TMA
// tensor-map encoding and the launches of the partial and combine kernels.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <numeric>
#include <vector>

#include "rel_attn.h"
#include "rel_attn_kernels.cuh"
#include "rel_attn_fp8.cuh"
#include "rel_attn_kvwrite.cuh"

namespace relattn {
namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxSplits = 256;
constexpr size_t kHeaderBytes = 256;   // status word lives here

// Bound of each device-side wait of later launches (0: kDefaultTimeoutNs);
// set by rel_attn_set_wait_limit.
std::atomic<unsigned long long> g_wait_limit_ns{0};

struct DeviceInfo {
  bool probed = false;
  bool sm100 = false;
  int sm_count = 0;
  bool attr_set[3][kMaxQTokens] = {};     // [G = 4, 6, 8][T - 1]
  bool attr_set_f8[3][kMaxQTokens] = {};  // the same, E4M3 cache (T >= 2)
  bool attr_fp8[3] = {};                   // [G = 4, 6, 8]
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool encode_fn_ready() {
  static std::once_flag once;
  std::call_once(once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000,
                                         cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode != nullptr;
}

// GQA group sizes with kernel instances: 48/8 heads (Inkling 2 Small, every
// layer) and the 64/8 full / 64/16 sliding layers of the previous Inkling.
bool group_supported(int G) { return G == 4 || G == 6 || G == 8; }

// E4M3 cache, T query tokens: up to three run as T one-token chunks of the
// FP8 kernel (E4M3 tensor-core MMAs), four and more through the multi-token
// kernel with the codes widened to bf16 in shared memory.  Measured on B200
// (256K-key verify step, 48/8 heads, us per call, chunks / widened): 2 tokens
// 167 / 282, 3: 244 / 323, 4: 320 / 320, 5: 396 / 364, 6: 472 / 337, 8: 624 /
// 359, 9: 701 / 419; 32 sequences of 16K-128K keys with 4 tokens 2,921 /
// 2,860, with 8 tokens 5,790 / 3,237.
constexpr int kE4m3WidenMinTokens = 4;
bool e4m3_widened(int q_tokens) { return q_tokens >= kE4m3WidenMinTokens; }

int validate_shape(const rel_attn_shape* s) {
  if (!s) return REL_ATTN_ERR_INVALID_ARG;
  if (s->batch < 1 || s->batch > 65535) return REL_ATTN_ERR_INVALID_ARG;
  if (s->q_tokens < 1 || s->q_tokens > kMaxQTokens) return REL_ATTN_ERR_INVALID_ARG;
  if (s->num_kv_heads < 1 || s->num_kv_heads > 65535) return REL_ATTN_ERR_INVALID_ARG;
  if (s->num_q_heads < 1 || s->num_q_heads % s->num_kv_heads) return REL_ATTN_ERR_INVALID_ARG;
  const int G = s->num_q_heads / s->num_kv_heads;
  if (!group_supported(G) || group_width_for(G, s->q_tokens) == 0) return REL_ATTN_ERR_INVALID_ARG;
  if (s->head_dim != kHeadDim || s->page_size != kPage) return REL_ATTN_ERR_INVALID_ARG;
  if (s->num_pages < 1 || s->max_pages_per_seq < 1) return REL_ATTN_ERR_INVALID_ARG;
  if ((long long)s->num_pages * s->num_kv_heads * kPage >= (1ll << 31)) return REL_ATTN_ERR_INVALID_ARG;
  if ((long long)s->max_pages_per_seq * kPage >= (1ll << 31)) return REL_ATTN_ERR_INVALID_ARG;
  if (s->num_buckets < 1 || s->exact_buckets < 1) return REL_ATTN_ERR_INVALID_ARG;
  if (s->num_buckets > s->exact_buckets) {
    if (s->num_buckets - s->exact_buckets > kMaxTailBuckets) return REL_ATTN_ERR_INVALID_ARG;
    if (s->max_distance <= s->exact_buckets) return REL_ATTN_ERR_INVALID_ARG;
  }
  if (s->max_seq_len < 0) return REL_ATTN_ERR_INVALID_ARG;
  if (s->out_fp32 != 0 && s->out_fp32 != 1) return REL_ATTN_ERR_INVALID_ARG;
  return REL_ATTN_OK;
}

// Unsigned integer of arbitrary size (32-bit limbs, least significant
// first): just enough to compare two products of powers exactly.
struct BigUint {
  std::vector<uint32_t> limb{1};
  void mul(uint32_t m) {
    uint64_t carry = 0;
    for (auto& x : limb) {
      const uint64_t v = (uint64_t)x * m + carry;
      x = (uint32_t)v;
      carry = v >> 32;
    }
    if (carry) limb.push_back((uint32_t)carry);
  }
  void mul_pow(uint32_t m, int e) { for (int i = 0; i < e; ++i) mul(m); }
  int compare(const BigUint& o) const {
    if (limb.size() != o.limb.size()) return limb.size() < o.limb.size() ? -1 : 1;
    for (size_t i = limb.size(); i-- > 0;)
      if (limb[i] != o.limb[i]) return limb[i] < o.limb[i] ? -1 : 1;
    return 0;
  }
};

// x >= E * (Dmax/E)^(k/n), decided exactly: with k/n = a/c in lowest terms
// (c >= 1), the inequality is x^c >= E^(c-a) * Dmax^a between integers.
bool at_or_above_edge(long long x, int E, int Dmax, int k, int n) {
  if (x <= 0) return false;
  const int g = std::gcd(k, n);
  const int a = k / g, c = n / g;
  BigUint lhs, rhs;
  lhs.mul_pow((uint32_t)x, c);
  rhs.mul_pow((uint32_t)E, c - a);
  rhs.mul_pow((uint32_t)Dmax, a);
  return lhs.compare(rhs) >= 0;
}

// Lower edges of the tail buckets, e_k = ceil(E * (Dmax/E)^(k/NL)), exact:
// long double names the edge to well under one unit, and where it lies
// within 1e-6 of an integer the integer comparison above settles it.
// `log_scale` = NL / log2(Dmax/E): (log2(d) - log2(E)) * log_scale is the
// tail bucket of d up to rounding, a starting guess the kernels correct
// against the table (0 when there is a single tail bucket).
void bucket_table(const rel_attn_shape* s, int* ex, int* nl, int* edges, float* log2_ex,
                  float* log_scale) {
  const int NB = s->num_buckets, E = s->exact_buckets;
  if (NB <= E) {
    *ex = NB - 1;
    *nl = 1;
    edges[0] = NB - 1;
    *log2_ex = 0.f;
    *log_scale = 0.f;
    return;
  }
  const int n = NB - E;
  *ex = E;
  *nl = n;
  const long double lr = log2l((long double)s->max_distance / (long double)E);
  *log2_ex = (float)log2l((long double)E);
  *log_scale = (float)((long double)n / lr);
  for (int k = 0; k <= n; ++k) {
    const long double x = (long double)E * exp2l(lr * (long double)k / (long double)n);
    const long double r = nearbyintl(x);
    long long e;
    if (fabsl(x - r) > 1e-6L) {
      e = (long long)ceill(x);
    } else {
      e = (long long)r;
      if (!at_or_above_edge(e, E, s->max_distance, k, n)) ++e;
      else if (at_or_above_edge(e - 1, E, s->max_distance, k, n)) --e;
    }
    edges[k] = (int)e;
  }
}

// Small caches: the edge table depends only on (NB, E, Dmax) and a tensor
// map only on (base pointer, extents); both are rebuilt otherwise per call.
struct EdgeEntry {
  int nb = -1, e = -1, dmax = -1, ex = 0, nl = 0;
  float log2_ex = 0.f, log_scale = 0.f;
  int edges[kMaxTailBuckets + 1];
  // largest number of bucket indices that 127 + T consecutive distances
  // span (index T = 1..kMaxQTokens), see bucket_span_fits
  int max_span[kMaxQTokens + 1];
};
struct MapEntry { const void* base = nullptr; uint64_t a = 0, b = 0; int kind = -1; CUtensorMap map; };
constexpr int kEdgeCache = 4, kMapCache = 16;
EdgeEntry g_edge_cache[kEdgeCache];
MapEntry g_map_cache[kMapCache];
int g_edge_next = 0, g_map_next = 0;
std::mutex g_cache_mu;

int bucket_host(int d, int ex, int nl, const int* edges);

// Bucket indices spanned by the distances [d, d + W - 1], maximised over d.
// bucket() is non-decreasing, so the maximum is taken at a distance where a
// bucket starts: every exact distance and every tail edge.
void fill_max_spans(EdgeEntry& e) {
  for (int T = 1; T <= kMaxQTokens; ++T) {
    const long long W = 127 + T;
    int best = 0;
    auto span_at = [&](long long d) {
      const long long d1 = std::min<long long>(d + W - 1, INT32_MAX);
      const int sp = bucket_host((int)d1, e.ex, e.nl, e.edges) - bucket_host((int)d, e.ex, e.nl, e.edges) + 1;
      best = std::max(best, sp);
    };
    for (int d = 0; d <= e.ex; ++d) span_at(d);
    for (int k = 0; k <= e.nl && e.nl > 0; ++k) span_at(e.edges[k]);
    e.max_span[T] = best;
  }
}

void bucket_table_cached(const rel_attn_shape* s, int* ex, int* nl, int* edges,
                         float* log2_ex = nullptr, float* log_scale = nullptr) {
  std::lock_guard<std::mutex> lk(g_cache_mu);
  const EdgeEntry* hit = nullptr;
  for (auto& e : g_edge_cache) {
    if (e.nb == s->num_buckets && e.e == s->exact_buckets && e.dmax == s->max_distance) {
      hit = &e;
      break;
    }
  }
  if (!hit) {
    EdgeEntry& e = g_edge_cache[g_edge_next++ % kEdgeCache];
    bucket_table(s, &e.ex, &e.nl, e.edges, &e.log2_ex, &e.log_scale);
    e.nb = s->num_buckets; e.e = s->exact_buckets; e.dmax = s->max_distance;
    fill_max_spans(e);
    hit = &e;
  }
  *ex = hit->ex;
  *nl = hit->nl;
  if (log2_ex) *log2_ex = hit->log2_ex;
  if (log_scale) *log_scale = hit->log_scale;
  memcpy(edges, hit->edges, sizeof(int) * (hit->nl + 1));
}

// Whether one relative-row chunk holds every bucket a tile can need: the
// 127 + T distances of a 128-key tile (T query tokens) must span at most
// 128 bucket indices for one token and 136 for several (the chunk's rows).
// A table whose tail buckets are narrower than a distance near the exact
// range can span more; such tables are rejected.  kernel_tokens is the T the
// partial kernel runs with (1 for the E4M3 kernel, whose tokens are chunks).
bool bucket_span_fits(const rel_attn_shape* s, int kernel_tokens) {
  int ex, nl;
  static thread_local int edges[kMaxTailBuckets + 1];
  bucket_table_cached(s, &ex, &nl, edges);
  int span = 0;
  {
    std::lock_guard<std::mutex> lk(g_cache_mu);
    for (auto& e : g_edge_cache)
      if (e.nb == s->num_buckets && e.e == s->exact_buckets && e.dmax == s->max_distance) {
        span = e.max_span[kernel_tokens];
        break;
      }
  }
  return span >= 1 && span <= (kernel_tokens == 1 ? 128 : 136);
}

int bucket_host(int d, int ex, int nl, const int* edges) {
  if (d < ex) return d;
  int lo = 0, hi = nl - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (edges[mid] <= d) lo = mid; else hi = mid - 1;
  }
  return ex + lo;
}

int splits_heuristic(const rel_attn_shape* s, int window, int sm_count) {
  const long long cap = (long long)s->max_pages_per_seq * kPage;
  long long max_len = (s->max_seq_len > 0) ? std::min<long long>(s->max_seq_len, cap) : cap;
  long long visible = (window > 0) ? std::min<long long>(max_len, (long long)window + s->q_tokens - 1)
                                   : max_len;
  // a window may straddle one more page than it has keys for, but never more
  // pages than the whole context: full attention bounds every window
  const long long pages = std::min<long long>((visible + kPage - 1) / kPage + (window > 0 ? 1 : 0),
                                              (max_len + kPage - 1) / kPage);
  const long long tiles = (pages + 1) / 2;
  const long long units = (long long)s->batch * s->num_kv_heads;
  long long S;
  // Several waves: about twelve CTAs per SM in all, so that CTAs of unequal
  // length (sequences of different lengths) even out and the last wave is
  // short.  Measured on batched_32 (256 units, 148 SMs), us per call for
  // S = 2 / 4 / 6 / 8 / 10 / 12 / 16: bf16 1,700 / 1,508 / 1,455 / 1,439 /
  // 1,431 / 1,456 / 1,478, E4M3 938 (S 2) / 814 / 820 / 830 / 855 / 899 (S 6..16).
  if (units >= sm_count) S = (12LL * sm_count + units - 1) / units;
  else S = sm_count / units;                                          // one full wave
  S = std::max<long long>(1, std::min<long long>(S, std::min<long long>(tiles, 256)));
  return (int)S;
}

size_t workspace_for(const rel_attn_shape* s, int S) {
  if (S <= 1) return kHeaderBytes;
  const size_t rows = (size_t)s->batch * s->q_tokens * s->num_q_heads;
  return kHeaderBytes + align256((size_t)S * rows * sizeof(float)) +
         (size_t)S * rows * kHeadDim * sizeof(float);
}

int probe_device(int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return REL_ATTN_ERR_NO_DEVICE;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& di = g_dev[dev];
  if (!di.probed) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) {
      cudaGetLastError();
      return REL_ATTN_ERR_NO_DEVICE;
    }
    di.sm100 = (prop.major == 10 && prop.minor == 0);
    di.sm_count = prop.multiProcessorCount;
    di.probed = true;
  }
  *dev_out = dev;
  return di.sm100 ? REL_ATTN_OK : REL_ATTN_ERR_NO_DEVICE;
}

bool make_map_2d(CUtensorMap* m, const void* base, uint64_t rows) {
  cuuint64_t dims[2] = {(cuuint64_t)kHeadDim, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kHeadDim * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)kPage};
  cuuint32_t estr[2] = {1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// E4M3 pool: one 128-byte row per (page, head, slot), a 64-row box per page.
bool make_map_2d_e4m3(CUtensorMap* m, const void* base, uint64_t rows) {
  cuuint64_t dims[2] = {(cuuint64_t)kHeadDim, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kHeadDim};
  cuuint32_t box[2] = {(cuuint32_t)kHeadDim, (cuuint32_t)kPage};
  cuuint32_t estr[2] = {1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_rel(CUtensorMap* m, const void* base, int NB, int Hkv, int box_rows) {
  cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)NB, (cuuint64_t)Hkv};
  cuuint64_t strides[2] = {(cuuint64_t)kHeadDim * 2, (cuuint64_t)NB * kHeadDim * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool cached_map(CUtensorMap* out, int kind, const void* base, uint64_t a, uint64_t b) {
  {
    std::lock_guard<std::mutex> lk(g_cache_mu);
    for (auto& e : g_map_cache)
      if (e.kind == kind && e.base == base && e.a == a && e.b == b) { *out = e.map; return true; }
  }
  CUtensorMap m;
  // kinds: 0 = K pool, 1 = V pool, 2 / 3 = relative table with 136- / 128-row
  // boxes, 4 / 5 = E4M3 K / V pool
  const bool ok = (kind >= 4) ? make_map_2d_e4m3(&m, base, a)
                  : (kind >= 2) ? make_map_rel(&m, base, (int)a, (int)b, kind == 2 ? 136 : 128)
                                : make_map_2d(&m, base, a);
  if (!ok) return false;
  std::lock_guard<std::mutex> lk(g_cache_mu);
  MapEntry& e = g_map_cache[g_map_next++ % kMapCache];
  e.kind = kind; e.base = base; e.a = a; e.b = b; e.map = m;
  *out = m;
  return true;
}

template <int G, int T, bool F8>
int launch_partial(const DecodeParams& prm, int S, int B, int Hkv, cudaStream_t st, DeviceInfo& di) {
  constexpr int N = group_width_for(G, T, F8);
  if constexpr (N == 0 || (F8 && T == 1)) {
    return REL_ATTN_ERR_INVALID_ARG;                  // no instance for this shape
  } else {
    constexpr int NG = softmax_groups(G, T, F8);
    using KC = KernelConfig<N, NG, G, T, F8>;
    auto kern = rel_attn_partial_kernel<N, G, NG, T, F8>;
    constexpr int smem = KC::kAllocBytes;
    bool& attr = F8 ? di.attr_set_f8[G / 2 - 2][T - 1] : di.attr_set[G / 2 - 2][T - 1];
    if (!attr) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return REL_ATTN_ERR_CUDA;
      attr = true;
    }
    dim3 grid(S, Hkv, B);
    kern<<<grid, KC::kThreads, smem, st>>>(prm);
    return cudaGetLastError() == cudaSuccess ? REL_ATTN_OK : REL_ATTN_ERR_CUDA;
  }
}

template <int G, bool F8>
int launch_partial_group(const DecodeParams& prm, int T, int S, int B, int Hkv, cudaStream_t st,
                         DeviceInfo& di) {
  switch (T) {
    case 1: return launch_partial<G, 1, F8>(prm, S, B, Hkv, st, di);
    case 2: return launch_partial<G, 2, F8>(prm, S, B, Hkv, st, di);
    case 3: return launch_partial<G, 3, F8>(prm, S, B, Hkv, st, di);
    case 4: return launch_partial<G, 4, F8>(prm, S, B, Hkv, st, di);
    case 5: return launch_partial<G, 5, F8>(prm, S, B, Hkv, st, di);
    case 6: return launch_partial<G, 6, F8>(prm, S, B, Hkv, st, di);
    case 7: return launch_partial<G, 7, F8>(prm, S, B, Hkv, st, di);
    case 8: return launch_partial<G, 8, F8>(prm, S, B, Hkv, st, di);
    case 9: return launch_partial<G, 9, F8>(prm, S, B, Hkv, st, di);
    default: return REL_ATTN_ERR_INVALID_ARG;
  }
}

}  // namespace
}  // namespace relattn

using namespace relattn;

extern "C" {

const char* rel_attn_version(void) { return "rel_attn 0.1.0 sm_100a"; }

const char* rel_attn_error_string(int code) {
  switch (code) {
    case REL_ATTN_OK: return "success";
    case REL_ATTN_ERR_INVALID_ARG: return "invalid argument";
    case REL_ATTN_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case REL_ATTN_ERR_CUDA: return "CUDA runtime or launch failure";
    case REL_ATTN_ERR_TIMEOUT: return "device-side bounded wait expired";
    case REL_ATTN_ERR_BAD_SEQ: return "sequence length or block-table entry out of range";
    case REL_ATTN_ERR_NO_DEVICE: return "no sm_100 device is current";
    default: return "unknown error";
  }
}

size_t rel_attn_workspace_bytes(const rel_attn_shape* shape, int num_splits) {
  if (validate_shape(shape) != REL_ATTN_OK || num_splits > 256) return 0;
  int S = num_splits;
  if (S <= 0) {
    int dev;
    const int sms = (probe_device(&dev) == REL_ATTN_OK) ? g_dev[dev].sm_count : 148;
    S = splits_heuristic(shape, 0, sms);   // full attention bounds every window
  }
  return workspace_for(shape, S);
}

int rel_attn_choose_splits(const rel_attn_shape* shape, int window, int sm_count) {
  const int rc = validate_shape(shape);
  if (rc != REL_ATTN_OK) return rc;
  if (sm_count <= 0) {
    int dev;
    const int prc = probe_device(&dev);
    if (prc != REL_ATTN_OK) return prc;
    sm_count = g_dev[dev].sm_count;
  }
  return splits_heuristic(shape, window, sm_count);
}

int rel_attn_bucket(const rel_attn_shape* shape, int distance) {
  if (validate_shape(shape) != REL_ATTN_OK || distance < 0) return -1;
  int ex, nl;
  static thread_local int edges[kMaxTailBuckets + 1];
  bucket_table_cached(shape, &ex, &nl, edges);
  return bucket_host(distance, ex, nl, edges);
}

static int split_pages_api(const rel_attn_shape* shape, int seq_len, int window, int num_splits,
                           int split, int cost_exact, int cost_near, int* first_page,
                           int* end_page) {
  if (validate_shape(shape) != REL_ATTN_OK || !first_page || !end_page) return REL_ATTN_ERR_INVALID_ARG;
  if (seq_len < shape->q_tokens || seq_len > shape->max_pages_per_seq * kPage)
    return REL_ATTN_ERR_INVALID_ARG;
  if (num_splits < 1 || num_splits > kMaxSplits || split < 0 || split >= num_splits)
    return REL_ATTN_ERR_INVALID_ARG;
  int ex, nl;
  static thread_local int edges[kMaxTailBuckets + 1];
  bucket_table_cached(shape, &ex, &nl, edges);
  const int p0 = seq_len - shape->q_tokens;
  const int lo = (window > 0) ? std::max(0, p0 - window + 1) : 0;
  split_pages(lo / kPage, (seq_len - 1) / kPage, num_splits, split, ex, cost_exact, cost_near,
              first_page, end_page);
  return REL_ATTN_OK;
}

int rel_attn_split_pages(const rel_attn_shape* shape, int seq_len, int window, int num_splits,
                         int split, int* first_page, int* end_page) {
  return split_pages_api(shape, seq_len, window, num_splits, split, kCostExactBf16, kCostNearBf16,
                         first_page, end_page);
}

int rel_attn_split_pages_e4m3(const rel_attn_shape* shape, int seq_len, int window, int num_splits,
                              int split, int* first_page, int* end_page) {
  return split_pages_api(shape, seq_len, window, num_splits, split, kCostExactE4m3, kCostNearE4m3,
                         first_page, end_page);
}

int rel_attn_set_wait_limit(unsigned long long limit_ns) {
  g_wait_limit_ns.store(limit_ns, std::memory_order_relaxed);
  return REL_ATTN_OK;
}

int rel_attn_workspace_init(void* workspace, size_t workspace_bytes, void* stream) {
  if (!workspace || workspace_bytes < kHeaderBytes) return REL_ATTN_ERR_INVALID_ARG;
  return cudaMemsetAsync(workspace, 0, kHeaderBytes, (cudaStream_t)stream) == cudaSuccess
             ? REL_ATTN_OK : REL_ATTN_ERR_CUDA;
}

int rel_attn_read_status(void* workspace, void* stream) {
  if (!workspace) return REL_ATTN_ERR_INVALID_ARG;
  unsigned st = 0;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemcpyAsync(&st, workspace, sizeof(st), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return REL_ATTN_ERR_CUDA;
  if (st == 0) return REL_ATTN_OK;
  if (cudaMemsetAsync(workspace, 0, sizeof(st), s) != cudaSuccess) return REL_ATTN_ERR_CUDA;
  if (st & kStatusTimeout) return REL_ATTN_ERR_TIMEOUT;
  return REL_ATTN_ERR_BAD_SEQ;
}

namespace {

// Validation and parameter set-up shared by the entry points.  Returns the
// resolved split count through *S.
int prepare(const rel_attn_shape* shape, const void* q, const void* k_cache, const void* v_cache,
            const int32_t* block_table, const int32_t* seq_lens, const void* rel_table, int window,
            int num_splits, void* out, float* lse, void* workspace, size_t workspace_bytes,
            DecodeParams* prm, int* S_out, DeviceInfo** di_out, const float* k_scale = nullptr,
            const float* v_scale = nullptr, bool kv_e4m3 = false) {
  // ---- validation (no CUDA call before this block passes)
  int rc = validate_shape(shape);
  if (rc != REL_ATTN_OK) return rc;
  // (one-token chunks need the one-token span)
  const bool e4m3_chunks = kv_e4m3 && shape->q_tokens > 1 && !e4m3_widened(shape->q_tokens);
  if (!bucket_span_fits(shape, e4m3_chunks ? 1 : shape->q_tokens)) return REL_ATTN_ERR_INVALID_ARG;
  if (kv_e4m3) {
    if (!k_scale || !v_scale ||
        (reinterpret_cast<uintptr_t>(k_scale) & 3) || (reinterpret_cast<uintptr_t>(v_scale) & 3))
      return REL_ATTN_ERR_INVALID_ARG;
  }
  if (!q || !k_cache || !v_cache || !block_table || !seq_lens || !rel_table || !out || !workspace)
    return REL_ATTN_ERR_INVALID_ARG;
  auto misaligned = [](const void* ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) & (a - 1)) != 0; };
  if (misaligned(q, 16) || misaligned(k_cache, 16) || misaligned(v_cache, 16) ||
      misaligned(rel_table, 16) || misaligned(out, 16) || misaligned(workspace, 256) ||
      misaligned(block_table, 4) || misaligned(seq_lens, 4) || (lse && misaligned(lse, 4)))
    return REL_ATTN_ERR_INVALID_ARG;
  if (num_splits > 256) return REL_ATTN_ERR_INVALID_ARG;
  if (workspace_bytes < kHeaderBytes) return REL_ATTN_ERR_WORKSPACE_TOO_SMALL;

  int dev;
  rc = probe_device(&dev);
  if (rc != REL_ATTN_OK) return rc;
  DeviceInfo& di = g_dev[dev];
  const int S = (num_splits > 0) ? num_splits : splits_heuristic(shape, window, di.sm_count);
  if (workspace_bytes < workspace_for(shape, S)) return REL_ATTN_ERR_WORKSPACE_TOO_SMALL;
  if (!encode_fn_ready()) return REL_ATTN_ERR_CUDA;

  const int B = shape->batch, T = shape->q_tokens, Hq = shape->num_q_heads, Hkv = shape->num_kv_heads;
  const size_t rows = (size_t)B * T * Hq;
  memset(prm, 0, sizeof(*prm));
  const uint64_t kv_rows = (uint64_t)shape->num_pages * Hkv * kPage;
  if (!cached_map(&prm->tmap_k, kv_e4m3 ? 4 : 0, k_cache, kv_rows, 0) ||
      !cached_map(&prm->tmap_v, kv_e4m3 ? 5 : 1, v_cache, kv_rows, 0) ||
      !cached_map(&prm->tmap_r, group_width_for(Hq / Hkv, e4m3_chunks ? 1 : T) == 16 ? 3 : 2, rel_table,
                  (uint64_t)shape->num_buckets, (uint64_t)Hkv))
    return REL_ATTN_ERR_CUDA;
  prm->q = reinterpret_cast<const __nv_bfloat16*>(q);
  prm->block_table = block_table;
  prm->seq_lens = seq_lens;
  prm->out = out;
  prm->lse = lse;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  prm->status = reinterpret_cast<unsigned*>(ws);
  prm->ws_lse = reinterpret_cast<float*>(ws + kHeaderBytes);
  prm->ws_o = reinterpret_cast<float*>(ws + kHeaderBytes + align256((size_t)S * rows * sizeof(float)));
  const unsigned long long wl = g_wait_limit_ns.load(std::memory_order_relaxed);
  prm->timeout_ns = wl ? wl : kDefaultTimeoutNs;
  prm->B = B; prm->T = T; prm->Hq = Hq; prm->Hkv = Hkv;
  prm->cps = 1; prm->seq_stride = T; prm->tok_off = 0; prm->len_off = 0;
  if (e4m3_chunks) {
    // T one-token chunks of the sequence in one launch, each attending
    // causally up to its own position
    prm->T = 1;
    prm->cps = T;
  }
  prm->rows_total = (int)rows;
  prm->num_pages = shape->num_pages;
  prm->max_pages = shape->max_pages_per_seq;
  prm->num_splits = S;
  prm->window = window;
  prm->out_fp32 = shape->out_fp32;
  bucket_table_cached(shape, &prm->ex, &prm->nl, prm->edges, &prm->log2_ex, &prm->log_scale);
  prm->cost_exact = kv_e4m3 ? kCostExactE4m3 : kCostExactBf16;
  prm->cost_near = kv_e4m3 ? kCostNearE4m3 : kCostNearBf16;
  prm->scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)kHeadDim));
  prm->k_scale = k_scale;
  prm->v_scale = v_scale;
  *S_out = S;
  *di_out = &di;
  return REL_ATTN_OK;
}

// bf16 cache, any token count; with e4m3 set, the E4M3 multi-token instances
// (T >= 2)
int launch_partial_any(const DecodeParams& prm, const rel_attn_shape* shape, int S, cudaStream_t st,
                       DeviceInfo& di, bool e4m3 = false) {
  const int B = shape->batch, Hkv = shape->num_kv_heads, T = shape->q_tokens;
  switch (shape->num_q_heads / Hkv) {
    case 4: return e4m3 ? launch_partial_group<4, true>(prm, T, S, B, Hkv, st, di)
                        : launch_partial_group<4, false>(prm, T, S, B, Hkv, st, di);
    case 6: return e4m3 ? launch_partial_group<6, true>(prm, T, S, B, Hkv, st, di)
                        : launch_partial_group<6, false>(prm, T, S, B, Hkv, st, di);
    case 8: return e4m3 ? launch_partial_group<8, true>(prm, T, S, B, Hkv, st, di)
                        : launch_partial_group<8, false>(prm, T, S, B, Hkv, st, di);
    default: return REL_ATTN_ERR_INVALID_ARG;
  }
}

// (templates cannot have C linkage; this block sits inside extern "C")
extern "C++" template <int G>
int launch_partial_e4m3_g(const DecodeParams& prm, int S, int B, int Hkv, cudaStream_t st, DeviceInfo& di) {
  using FC = Fp8Config<G>;
  auto kern = rel_attn_partial_fp8_kernel<G>;
  bool& attr = di.attr_fp8[G / 2 - 2];
  if (!attr) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, FC::kAllocBytes) != cudaSuccess)
      return REL_ATTN_ERR_CUDA;
    attr = true;
  }
  dim3 grid(S * prm.cps, Hkv, B);                  // chunk index fastest in x
  kern<<<grid, FC::kThreads, FC::kAllocBytes, st>>>(prm);
  return cudaGetLastError() == cudaSuccess ? REL_ATTN_OK : REL_ATTN_ERR_CUDA;
}

int launch_partial_e4m3(const DecodeParams& prm, const rel_attn_shape* shape, int S, cudaStream_t st,
                        DeviceInfo& di) {
  const int B = shape->batch, Hkv = shape->num_kv_heads;
  if (e4m3_widened(shape->q_tokens)) return launch_partial_any(prm, shape, S, st, di, true);
  switch (shape->num_q_heads / Hkv) {
    case 4: return launch_partial_e4m3_g<4>(prm, S, B, Hkv, st, di);
    case 6: return launch_partial_e4m3_g<6>(prm, S, B, Hkv, st, di);
    case 8: return launch_partial_e4m3_g<8>(prm, S, B, Hkv, st, di);
    default: return REL_ATTN_ERR_INVALID_ARG;
  }
}

// LSE-merge launch; programmatic dependent launch lets it start while the
// partial kernel drains (it waits on griddepcontrol before reading).
int launch_combine(const rel_attn_shape* shape, int S, void* out, float* lse, void* workspace,
                   cudaStream_t st) {
  const size_t rows = (size_t)shape->batch * shape->q_tokens * shape->num_q_heads;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  const float* ws_lse = reinterpret_cast<const float*>(ws + kHeaderBytes);
  const float* ws_o = reinterpret_cast<const float*>(ws + kHeaderBytes + align256((size_t)S * rows * sizeof(float)));
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3((unsigned)rows);
  cfg.blockDim = dim3(kCombineThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, rel_attn_combine_kernel, ws_lse, ws_o, S, (int)rows, out, lse,
                         shape->out_fp32) != cudaSuccess) {
    cudaGetLastError();
    return REL_ATTN_ERR_CUDA;
  }
  return REL_ATTN_OK;
}

}  // namespace

int rel_attn_decode(const rel_attn_shape* shape, const void* q, const void* k_cache,
                    const void* v_cache, const int32_t* block_table, const int32_t* seq_lens,
                    const void* rel_table, int window, int num_splits, void* out, float* lse,
                    void* workspace, size_t workspace_bytes, void* stream) {
  DecodeParams prm;
  int S = 0;
  DeviceInfo* di = nullptr;
  int rc = prepare(shape, q, k_cache, v_cache, block_table, seq_lens, rel_table, window, num_splits,
                   out, lse, workspace, workspace_bytes, &prm, &S, &di);
  if (rc != REL_ATTN_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  rc = launch_partial_any(prm, shape, S, st, *di);
  if (rc != REL_ATTN_OK || S == 1) return rc;
  return launch_combine(shape, S, out, lse, workspace, st);
}

int rel_attn_partial(const rel_attn_shape* shape, const void* q, const void* k_cache,
                     const void* v_cache, const int32_t* block_table, const int32_t* seq_lens,
                     const void* rel_table, int window, int num_splits, void* out, float* lse,
                     void* workspace, size_t workspace_bytes, void* stream) {
  if (num_splits < 1) return REL_ATTN_ERR_INVALID_ARG;
  DecodeParams prm;
  int S = 0;
  DeviceInfo* di = nullptr;
  int rc = prepare(shape, q, k_cache, v_cache, block_table, seq_lens, rel_table, window, num_splits,
                   out, lse, workspace, workspace_bytes, &prm, &S, &di);
  if (rc != REL_ATTN_OK) return rc;
  return launch_partial_any(prm, shape, S, reinterpret_cast<cudaStream_t>(stream), *di);
}

int rel_attn_decode_e4m3(const rel_attn_shape* shape, const void* q, const void* k_cache,
                         const void* v_cache, const float* k_scale, const float* v_scale,
                         const int32_t* block_table, const int32_t* seq_lens,
                         const void* rel_table, int window, int num_splits, void* out, float* lse,
                         void* workspace, size_t workspace_bytes, void* stream) {
  DecodeParams prm;
  int S = 0;
  DeviceInfo* di = nullptr;
  int rc = prepare(shape, q, k_cache, v_cache, block_table, seq_lens, rel_table, window, num_splits,
                   out, lse, workspace, workspace_bytes, &prm, &S, &di, k_scale, v_scale, true);
  if (rc != REL_ATTN_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  rc = launch_partial_e4m3(prm, shape, S, st, *di);
  if (rc != REL_ATTN_OK || S == 1) return rc;
  return launch_combine(shape, S, out, lse, workspace, st);
}

int rel_attn_partial_e4m3(const rel_attn_shape* shape, const void* q, const void* k_cache,
                          const void* v_cache, const float* k_scale, const float* v_scale,
                          const int32_t* block_table, const int32_t* seq_lens,
                          const void* rel_table, int window, int num_splits, void* out, float* lse,
                          void* workspace, size_t workspace_bytes, void* stream) {
  if (num_splits < 1) return REL_ATTN_ERR_INVALID_ARG;
  DecodeParams prm;
  int S = 0;
  DeviceInfo* di = nullptr;
  int rc = prepare(shape, q, k_cache, v_cache, block_table, seq_lens, rel_table, window, num_splits,
                   out, lse, workspace, workspace_bytes, &prm, &S, &di, k_scale, v_scale, true);
  if (rc != REL_ATTN_OK) return rc;
  return launch_partial_e4m3(prm, shape, S, reinterpret_cast<cudaStream_t>(stream), *di);
}

int rel_attn_combine(const rel_attn_shape* shape, int num_splits, void* out, float* lse,
                     void* workspace, size_t workspace_bytes, void* stream) {
  int rc = validate_shape(shape);
  if (rc != REL_ATTN_OK) return rc;
  if (num_splits < 1 || num_splits > 256 || !out || !workspace) return REL_ATTN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(out) & 15) || (reinterpret_cast<uintptr_t>(workspace) & 255) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3)))
    return REL_ATTN_ERR_INVALID_ARG;
  if (workspace_bytes < workspace_for(shape, num_splits)) return REL_ATTN_ERR_WORKSPACE_TOO_SMALL;
  if (num_splits == 1) return REL_ATTN_OK;
  int dev;
  rc = probe_device(&dev);
  if (rc != REL_ATTN_OK) return rc;
  return launch_combine(shape, num_splits, out, lse, workspace, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Chunked prefill: the C query tokens of each sequence run as chunks of
// kPrefillChunk tokens through the multi-token decode instances (each chunk a
// virtual batch entry on its sequence's block-table row, attending causally
// to everything before it), the first C % kPrefillChunk tokens as one more
// launch of the instance for that many tokens; then the combine kernel when
// the keys are split.
// ---------------------------------------------------------------------------
namespace {
constexpr int kPrefillChunk = 8;
}  // namespace

extern "C" int rel_attn_prefill(const rel_attn_shape* shape, const void* q, const void* k_cache,
                                const void* v_cache, const int32_t* block_table,
                                const int32_t* seq_lens, const void* rel_table, int window,
                                int num_splits, void* out, float* lse, void* workspace,
                                size_t workspace_bytes, void* stream) {
  if (!shape) return REL_ATTN_ERR_INVALID_ARG;
  const int C = shape->q_tokens;
  if (C < 1 || C > (1 << 20)) return REL_ATTN_ERR_INVALID_ARG;
  // validate everything else as for a decode step of one chunk (never more
  // rows than the whole prefill, so its workspace check is implied by ours)
  const int nfull = C / kPrefillChunk, rem = C % kPrefillChunk;
  rel_attn_shape chunk_shape = *shape;
  chunk_shape.q_tokens = nfull > 0 ? kPrefillChunk : rem;
  int rc = validate_shape(&chunk_shape);
  if (rc != REL_ATTN_OK) return rc;
  if ((long long)shape->batch * (nfull > 0 ? nfull : 1) > 65535) return REL_ATTN_ERR_INVALID_ARG;
  if (num_splits > 256) return REL_ATTN_ERR_INVALID_ARG;
  int dev;
  rc = probe_device(&dev);
  if (rc != REL_ATTN_OK) return rc;
  // one split per chunk unless the chunks do not fill the GPU
  int S = num_splits;
  if (S <= 0) {
    const long long units = (long long)shape->batch * shape->num_kv_heads * (nfull + (rem > 0));
    S = (units >= g_dev[dev].sm_count) ? 1 : (int)std::max<long long>(1, g_dev[dev].sm_count / units);
    const long long cap = (long long)shape->max_pages_per_seq * kPage;
    const long long len = shape->max_seq_len > 0 ? std::min<long long>(shape->max_seq_len, cap) : cap;
    S = (int)std::max<long long>(1, std::min<long long>(S, (len + 2 * kPage - 1) / (2 * kPage)));
  }
  // `shape` (q_tokens = C) sizes the workspace: all B * C * Hq rows' partials
  DecodeParams prm;
  int S_used = 0;
  DeviceInfo* di = nullptr;
  rc = prepare(&chunk_shape, q, k_cache, v_cache, block_table, seq_lens, rel_table, window, S,
               out, lse, workspace, workspace_bytes, &prm, &S_used, &di);
  if (rc != REL_ATTN_OK) return rc;
  const size_t rows = (size_t)shape->batch * C * shape->num_q_heads;
  if (workspace_bytes < workspace_for(shape, S)) return REL_ATTN_ERR_WORKSPACE_TOO_SMALL;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  prm.ws_lse = reinterpret_cast<float*>(ws + kHeaderBytes);
  prm.ws_o = reinterpret_cast<float*>(ws + kHeaderBytes + align256((size_t)S * rows * sizeof(float)));
  prm.rows_total = (int)rows;
  prm.seq_stride = C;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int B = shape->batch, Hkv = shape->num_kv_heads, G = shape->num_q_heads / Hkv;
  if (nfull > 0) {
    DecodeParams pf = prm;
    pf.T = kPrefillChunk;
    pf.cps = nfull;
    pf.tok_off = rem;
    pf.len_off = 0;
    if (!cached_map(&pf.tmap_r, group_width_for(G, kPrefillChunk) == 16 ? 3 : 2, rel_table,
                    (uint64_t)shape->num_buckets, (uint64_t)Hkv))
      return REL_ATTN_ERR_CUDA;
    rel_attn_shape sh = chunk_shape;
    sh.batch = B * nfull;
    sh.q_tokens = kPrefillChunk;
    rc = launch_partial_any(pf, &sh, S, st, *di);
    if (rc != REL_ATTN_OK) return rc;
  }
  if (rem > 0) {
    DecodeParams pr = prm;
    pr.T = rem;
    pr.cps = 1;
    pr.tok_off = 0;
    pr.len_off = C - rem;
    if (!cached_map(&pr.tmap_r, group_width_for(G, rem) == 16 ? 3 : 2, rel_table,
                    (uint64_t)shape->num_buckets, (uint64_t)Hkv))
      return REL_ATTN_ERR_CUDA;
    rel_attn_shape sh = chunk_shape;
    sh.q_tokens = rem;
    rc = launch_partial_any(pr, &sh, S, st, *di);
    if (rc != REL_ATTN_OK) return rc;
  }
  if (S == 1) return REL_ATTN_OK;
  return launch_combine(shape, S, out, lse, workspace, st);
}

// ---------------------------------------------------------------------------
// The KV-cache producer step: short convolution over the new tokens' K and V,
// paged KV-cache write, optional E4M3 quantisation (rel_attn_kvwrite.cuh).
// ---------------------------------------------------------------------------
extern "C" int rel_attn_kv_write(const rel_attn_shape* shape, const void* k_new, const void* v_new,
                                 const void* conv_w, void* k_raw, void* v_raw, void* k_cache,
                                 void* v_cache, const float* k_scale, const float* v_scale,
                                 const int32_t* block_table, const int32_t* seq_lens,
                                 void* workspace, void* stream) {
  const rel_attn_shape* s = shape;
  if (!s) return REL_ATTN_ERR_INVALID_ARG;
  if (s->batch < 1 || s->batch > 65535 || s->q_tokens < 1 || s->q_tokens > (1 << 24) ||
      s->num_kv_heads < 1 || s->num_kv_heads > 65535 || s->head_dim != kHeadDim ||
      s->page_size != kPage || s->num_pages < 1 || s->max_pages_per_seq < 1)
    return REL_ATTN_ERR_INVALID_ARG;
  if ((long long)s->num_pages * s->num_kv_heads * kPage >= (1ll << 31) ||
      (long long)s->max_pages_per_seq * kPage >= (1ll << 31))
    return REL_ATTN_ERR_INVALID_ARG;
  if (!k_new || !v_new || !conv_w || !k_raw || !v_raw || !k_cache || !v_cache || !block_table ||
      !seq_lens)
    return REL_ATTN_ERR_INVALID_ARG;
  const bool e4m3 = k_scale != nullptr;
  if (e4m3 != (v_scale != nullptr)) return REL_ATTN_ERR_INVALID_ARG;
  auto misaligned = [](const void* ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) & (a - 1)) != 0; };
  if (misaligned(k_new, 16) || misaligned(v_new, 16) || misaligned(conv_w, 16) ||
      misaligned(k_raw, 16) || misaligned(v_raw, 16) || misaligned(k_cache, 16) ||
      misaligned(v_cache, 16) || misaligned(block_table, 4) || misaligned(seq_lens, 4) ||
      (e4m3 && (misaligned(k_scale, 4) || misaligned(v_scale, 4))) ||
      (workspace && misaligned(workspace, 256)))
    return REL_ATTN_ERR_INVALID_ARG;
  int dev;
  int rc = probe_device(&dev);
  if (rc != REL_ATTN_OK) return rc;
  KvWriteParams prm;
  prm.k_new = reinterpret_cast<const __nv_bfloat16*>(k_new);
  prm.v_new = reinterpret_cast<const __nv_bfloat16*>(v_new);
  prm.conv_w = reinterpret_cast<const __nv_bfloat16*>(conv_w);
  prm.k_raw = reinterpret_cast<__nv_bfloat16*>(k_raw);
  prm.v_raw = reinterpret_cast<__nv_bfloat16*>(v_raw);
  prm.k_cache = k_cache;
  prm.v_cache = v_cache;
  prm.k_scale = k_scale;
  prm.v_scale = v_scale;
  prm.block_table = block_table;
  prm.seq_lens = seq_lens;
  prm.status = reinterpret_cast<unsigned*>(workspace);
  prm.B = s->batch;
  prm.T = s->q_tokens;
  prm.Hkv = s->num_kv_heads;
  prm.num_pages = s->num_pages;
  prm.max_pages = s->max_pages_per_seq;
  const dim3 grid((unsigned)((s->q_tokens + kKvwTokensPerCta - 1) / kKvwTokensPerCta),
                  (unsigned)s->num_kv_heads, (unsigned)s->batch);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (e4m3) rel_attn_kv_write_kernel<true><<<grid, kKvwThreads, 0, st>>>(prm);
  else rel_attn_kv_write_kernel<false><<<grid, kKvwThreads, 0, st>>>(prm);
  return cudaGetLastError() == cudaSuccess ? REL_ATTN_OK : REL_ATTN_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Allocation-free entry point.
//
// Some callers have no way to allocate device memory: a plugin that is handed
// only its input and output buffers by a host framework, or a serving engine
// that reserves all of HBM for its KV cache up front, so that an extra
// cudaMalloc fails.  rel_attn_decode_static lets them run the operation with
// the scratch space (device status word + per-split partial results) taken
// from a fixed array compiled into this library instead of a caller-owned
// workspace.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kStaticScratchBytes = size_t(4) << 20;   // 4 MiB on every device

// Every GPU that loads the library holds this array until the process exits.
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

void* g_static_scratch_addr[kMaxDevices];
std::mutex g_static_mu;

// Device address of the array on the current device, looked up once per
// device.  In host code the array's name is only a host-side stand-in, so the
// kernels must be given this address, never the symbol itself.
int static_scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return REL_ATTN_ERR_NO_DEVICE;
  }
  std::lock_guard<std::mutex> lk(g_static_mu);
  if (!g_static_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return REL_ATTN_ERR_CUDA;
    }
    g_static_scratch_addr[dev] = p;
  }
  *out = g_static_scratch_addr[dev];
  return REL_ATTN_OK;
}

}  // namespace

extern "C" int rel_attn_decode_static(const rel_attn_shape* shape, const void* q,
                                      const void* k_cache, const void* v_cache,
                                      const int32_t* block_table, const int32_t* seq_lens,
                                      const void* rel_table, int window, int num_splits,
                                      void* out, float* lse, void* stream) {
  int rc = validate_shape(shape);
  if (rc != REL_ATTN_OK) return rc;
  if (!q || !k_cache || !v_cache || !block_table || !seq_lens || !rel_table || !out)
    return REL_ATTN_ERR_INVALID_ARG;
  auto misaligned = [](const void* ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) & (a - 1)) != 0; };
  if (misaligned(q, 16) || misaligned(k_cache, 16) || misaligned(v_cache, 16) ||
      misaligned(rel_table, 16) || misaligned(out, 16) || misaligned(block_table, 4) ||
      misaligned(seq_lens, 4) || (lse && misaligned(lse, 4)))
    return REL_ATTN_ERR_INVALID_ARG;
  if (num_splits > 256) return REL_ATTN_ERR_INVALID_ARG;
  int dev;
  rc = probe_device(&dev);
  if (rc != REL_ATTN_OK) return rc;
  const int S = (num_splits > 0) ? num_splits : splits_heuristic(shape, window, g_dev[dev].sm_count);
  if (workspace_for(shape, S) > kStaticScratchBytes) return REL_ATTN_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = nullptr;
  rc = static_scratch_address(&scratch);
  if (rc != REL_ATTN_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // The array keeps whatever the previous call left there: the status word
  // must start at zero; the per-split partials are rewritten in full.
  if (cudaMemsetAsync(scratch, 0, kHeaderBytes, st) != cudaSuccess) {
    cudaGetLastError();
    return REL_ATTN_ERR_CUDA;
  }
  return rel_attn_decode(shape, q, k_cache, v_cache, block_table, seq_lens, rel_table, window, S,
                         out, lse, scratch, kStaticScratchBytes, stream);
}
