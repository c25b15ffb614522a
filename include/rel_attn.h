/*
 * rel_attn.h -- C ABI of the B200 (sm_100a) relative-bias GQA decode library.
 *
 * One operation: decode-time grouped-query attention over a paged bf16 KV
 * cache with a learned relative-position term added to the pre-softmax
 * logits.  For query token t of sequence b (position p = L_b - T + t) and
 * query head hq (KV head h = hq / (Hq/Hkv)):
 *
 *   s_j = ( q.k_j + q.R_h[bucket(p - j)] ) / sqrt(D),   j in J_t
 *   J_t = { j : 0 <= j <= p,  and p - j <= W - 1 when W > 0 }
 *   lse = ln sum_j exp(s_j),   out = sum_j exp(s_j - lse) v_j
 *
 * bucket(d): d for d < E (E = exact_buckets, 1024); beyond that NL = NB - E
 * log-spaced buckets with lower edges e_k = ceil(E (Dmax/E)^(k/NL)),
 * bucket = E + min(NL-1, max{k : e_k <= d}); when NB <= E, min(d, NB-1).
 * The kernels read the relative rows a 128-key tile needs as one contiguous
 * block of 128 rows (one query token per kernel) or 136 (several), so any
 * 127 + T consecutive distances must span at most that many bucket indices.
 * The standard table (NB 1,280, E 1,024, Dmax 2^20) spans 128 / 129..136;
 * a table whose tail buckets start narrower than one distance can span more
 * and is refused by the compute entry points with REL_ATTN_ERR_INVALID_ARG
 * (rel_attn_bucket still evaluates it).
 *
 * Sources: "vLLM TML Inkling 지원", section "TML Inkling 모델 아키텍처"
 * (learned relative term added to the pre-softmax logits instead of RoPE;
 * GQA with head size 128); "vLLM、Inkling 2 Smallを初日サポート GB200で630
 * tok/s", section "モデルの構成" (48 query / 8 KV heads, sliding window
 * 1,024; the previous Inkling: 64 / 8 heads on full-attention layers, 64 / 16
 * with window 512 on sliding ones, so G = 6, 8 and 4) and section
 * "vLLMの最適化と性能" (the GQA group's 6 heads packed into one 64-row tile
 * of a decode kernel); "vLLM TML Inkling 지원", section
 * "저지연 컬렉티브 및 커널" (sheared relative bias; num_splits chosen from
 * batch size and KV length).  The pages give no formula: the form and the
 * bucket function above are this library's reading.
 *
 * Conventions for every entry point:
 *   - Tensor arguments are DEVICE pointers owned by the caller; the library
 *     never allocates, frees or retains them.  Host-side arguments are the
 *     shape struct and scalars.  `out` and `lse` are written with plain
 *     stores only, so they may also be mapped pinned host memory (under
 *     unified addressing its host address is valid on the device): the
 *     result then reaches the host without a copy after the call.
 *   - Return value 0 on success, a negative REL_ATTN_ERR_* code otherwise.
 *     Arguments are validated before anything is launched: on an error
 *     nothing runs on the stream.
 *   - Launches are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  The caller synchronises.
 *   - One workspace must not be used by two calls that run concurrently.
 *   - Host threads: the library keeps process-wide caches (encoded tensor
 *     maps and bucket-edge tables, behind a mutex; per-device attributes,
 *     set on first use without one).  Issue calls from one host thread at a
 *     time (any number of streams); callers with several host threads
 *     serialise the calls.
 */
#ifndef REL_ATTN_H
#define REL_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define REL_ATTN_OK                       0
#define REL_ATTN_ERR_INVALID_ARG         -1  /* bad pointer, shape or scalar      */
#define REL_ATTN_ERR_WORKSPACE_TOO_SMALL -2  /* workspace_bytes below the query  */
#define REL_ATTN_ERR_CUDA                -3  /* CUDA runtime / launch failure     */
#define REL_ATTN_ERR_TIMEOUT             -4  /* a device-side bounded wait expired */
#define REL_ATTN_ERR_BAD_SEQ             -5  /* device saw seq_len or page out of range */
#define REL_ATTN_ERR_NO_DEVICE           -6  /* current device is not sm_100     */

/* Problem shape.  All fields are host integers. */
typedef struct rel_attn_shape {
  int batch;             /* B >= 1                                              */
  int q_tokens;          /* T, query tokens per sequence, 1..9 (verify steps)  */
  int num_q_heads;       /* Hq                                                  */
  int num_kv_heads;      /* Hkv, Hq % Hkv == 0, G = Hq/Hkv in {4, 6, 8};
                            T <= 9 for G = 4 and 6, T <= 8 for G = 8 (at most
                            64 query rows G*T per KV head)                     */
  int head_dim;          /* D, must be 128                                      */
  int page_size;         /* P, must be 64                                       */
  int num_pages;         /* pages in the K/V pool                               */
  int max_pages_per_seq; /* row stride (in entries) of block_table             */
  int num_buckets;       /* NB, rows of each KV head's relative table          */
  int exact_buckets;     /* E (1024); 1 <= E                                    */
  int max_distance;      /* Dmax (2^20); E < Dmax                               */
  int max_seq_len;       /* host upper bound on seq_lens (0: use the block-table
                            capacity); used only by the split heuristic        */
  int out_fp32;          /* 0: out is bf16, 1: out is fp32                     */
} rel_attn_shape;

/*
 * rel_attn_decode -- the whole hot path: split-KV partial kernel, then (when
 * num_splits > 1) the LSE-merge combine kernel.
 *
 *   q           bf16 [B, T, Hq, D], row-major.
 *   k_cache     bf16 [num_pages, Hkv, P, D]: one (page, KV head) is a
 *   v_cache     contiguous P x D block.  16-byte aligned.
 *   block_table int32 [B, max_pages_per_seq]: physical page of logical page
 *               i of sequence b.  Only entries that hold keys some query
 *               token can see are read (others may be anything, e.g. -1).
 *   seq_lens    int32 [B]: context length L_b including the T query tokens;
 *               T <= L_b <= max_pages_per_seq * P.  Device memory.
 *   rel_table   bf16 [Hkv, NB, D]: relative embeddings R_h.  16-byte aligned.
 *   window      W > 0: sliding window of W keys (self included); W <= 0: full.
 *   num_splits  KV splits per (sequence, KV head), 1..256; <= 0 picks the
 *               heuristic (rel_attn_choose_splits).
 *   out         [B, T, Hq, D], bf16 or fp32 per shape->out_fp32.
 *   lse         fp32 [B, T, Hq] natural-log LSE of the scaled logits, or NULL.
 *   workspace   device scratch of at least rel_attn_workspace_bytes(shape,
 *               num_splits) bytes, 256-byte aligned, prepared once with
 *               rel_attn_workspace_init (it holds the device status word).
 *
 * Device-side problems (seq_len out of range, a block-table entry outside
 * the pool, a wait that exceeded its bound) do not fault: they set bits in
 * the workspace status word, read with rel_attn_read_status, and the rows
 * they touch are written as NaN (out and lse): every row of a sequence whose
 * seq_len is out of range; the rows of each KV head whose walk met an entry
 * outside the pool or gave up a wait (through the combine kernel, a NaN
 * partial makes the whole merged row NaN).
 */
int rel_attn_decode(const rel_attn_shape* shape, const void* q,
                    const void* k_cache, const void* v_cache,
                    const int32_t* block_table, const int32_t* seq_lens,
                    const void* rel_table, int window, int num_splits,
                    void* out, float* lse, void* workspace,
                    size_t workspace_bytes, void* stream);

/*
 * Split-phase form of rel_attn_decode, for callers that schedule the two
 * kernels themselves (e.g. to time them apart, or to exchange per-split
 * partials between devices before merging).  rel_attn_partial +
 * rel_attn_combine with the same num_splits compute exactly what
 * rel_attn_decode computes.  num_splits must be explicit here (1..256; use
 * rel_attn_choose_splits).  With num_splits == 1 the partial call writes
 * out/lse itself and the combine call is a no-op.  With num_splits > 1 the
 * partial call writes the per-split (normalised output, lse) pairs into the
 * workspace -- fp32 [S][B*T*Hq] lse after the 256-byte header, then fp32
 * [S][B*T*Hq][D] outputs at the next 256-byte boundary; a split with no
 * visible key holds lse = -inf and zeros -- and the combine call merges them:
 *   lse = ln sum_s exp(lse_s),  out = sum_s exp(lse_s - lse) o_s.
 */
int rel_attn_partial(const rel_attn_shape* shape, const void* q,
                     const void* k_cache, const void* v_cache,
                     const int32_t* block_table, const int32_t* seq_lens,
                     const void* rel_table, int window, int num_splits,
                     void* out, float* lse, void* workspace,
                     size_t workspace_bytes, void* stream);
int rel_attn_combine(const rel_attn_shape* shape, int num_splits, void* out,
                     float* lse, void* workspace, size_t workspace_bytes,
                     void* stream);

/*
 * rel_attn_decode_e4m3 / rel_attn_partial_e4m3 -- the same operation over an
 * FP8 KV cache ("vLLM TML Inkling 지원", section "미래 로드맵", plans FP8 for
 * the full-context layers to relieve the KV-cache bottleneck; the pages fix
 * no format, so this library reads it as follows).
 *
 *   k_cache, v_cache  uint8 [num_pages, Hkv, 64, 128], OFP8 E4M3 codes
 *                     (1 sign, 4 exponent bits with bias 7, 3 mantissa bits;
 *                     0x7F / 0xFF are NaN), device memory, 16-byte aligned.
 *   k_scale, v_scale  fp32 [Hkv], device memory, 4-byte aligned: key j of KV
 *                     head h is e4m3(k_code) * k_scale[h], likewise for V.
 * Every other argument, the workspace and the outputs are as for
 * rel_attn_decode / rel_attn_partial (rel_attn_combine merges the splits of
 * either).  Token t of T attends to the keys before position L - T + t + 1
 * as in rel_attn_decode.  Two kernels serve the call:
 *   q_tokens 1..3  The E4M3 tiles go to the tensor cores as they are (E4M3 x
 *                  E4M3 MMAs, fp32 accumulation): the query is carried as
 *                  two E4M3 terms scaled per row by a power of two (exact
 *                  for a bf16 query), the softmax weights as three (12
 *                  significant bits); the relative term stays bf16.  Two or
 *                  three tokens run as one-token chunks of each sequence in
 *                  one launch (the chunks of one split and KV head side by
 *                  side, so that their page reads meet in L2).
 *   q_tokens 4..9  The multi-token kernel of rel_attn_decode with the codes
 *                  widened to bf16 in shared memory (exactly: every E4M3
 *                  value is a bf16 value), k_scale[h] folded into the logit
 *                  multiplier and v_scale[h] into the final normalisation;
 *                  with unit scales the result is bit for bit that of
 *                  rel_attn_decode on the codes' values for six tokens and
 *                  more and for five at Hq/Hkv = 8 (at four, and five for
 *                  Hq/Hkv <= 6, the rows are split over four softmax groups
 *                  instead of two, which agrees to rounding).  The NaN codes read
 *                  as +-480 on this path (a saturating quantiser, such as
 *                  rel_attn_kv_write, never writes them).
 * The bucket-density limit (see the top of this file) applies with T = 1 for
 * up to three tokens and with T itself from four on.
 * Limits: Hq/Hkv must be 4, 6 or 8 and the shape valid for rel_attn_decode
 * (else REL_ATTN_ERR_INVALID_ARG).
 */
int rel_attn_decode_e4m3(const rel_attn_shape* shape, const void* q,
                         const void* k_cache, const void* v_cache,
                         const float* k_scale, const float* v_scale,
                         const int32_t* block_table, const int32_t* seq_lens,
                         const void* rel_table, int window, int num_splits,
                         void* out, float* lse, void* workspace,
                         size_t workspace_bytes, void* stream);
int rel_attn_partial_e4m3(const rel_attn_shape* shape, const void* q,
                          const void* k_cache, const void* v_cache,
                          const float* k_scale, const float* v_scale,
                          const int32_t* block_table, const int32_t* seq_lens,
                          const void* rel_table, int window, int num_splits,
                          void* out, float* lse, void* workspace,
                          size_t workspace_bytes, void* stream);

/*
 * rel_attn_decode_static -- rel_attn_decode without a workspace argument.
 * (An addition of this library; the pages describe nothing like it.)
 *
 * For callers that cannot allocate device memory: for example a plugin that a
 * host framework hands only its input and output buffers, or a serving engine
 * that has reserved all of HBM for its KV cache so that another cudaMalloc
 * would fail.  The scratch space comes from a fixed array inside the library
 * (REL_ATTN_STATIC_SCRATCH_BYTES = 4 MiB, held on every GPU that loads the
 * library until the process exits); this entry point itself allocates nothing.
 *
 *   - Arguments are those of rel_attn_decode minus the workspace.
 *   - Shapes whose workspace (rel_attn_workspace_bytes(shape, num_splits))
 *     exceeds 4 MiB are rejected with REL_ATTN_ERR_WORKSPACE_TOO_SMALL before
 *     anything is launched; pass a smaller num_splits or use rel_attn_decode.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 *   - All calls on a device share the one array, and it keeps the previous
 *     call's contents (each call clears the status word it needs).  Calls that
 *     overlap on the GPU -- on different streams, or from different host
 *     threads -- race on it; serialise them.
 *   - Device-side status is not reported (there is no workspace to read it
 *     from), but the rows it concerns still come back as NaN, as described
 *     for rel_attn_decode.
 */
#define REL_ATTN_STATIC_SCRATCH_BYTES ((size_t)4 << 20)
int rel_attn_decode_static(const rel_attn_shape* shape, const void* q,
                           const void* k_cache, const void* v_cache,
                           const int32_t* block_table, const int32_t* seq_lens,
                           const void* rel_table, int window, int num_splits,
                           void* out, float* lse, void* stream);

/*
 * rel_attn_prefill -- the same attention for many query tokens per
 * sequence at once: a prefill, or a chunk of one ("vLLM、Inkling 2 Smallを
 * 初日サポート GB200で630 tok/s", section "vLLMの最適化と性能", and
 * "A vLLM már az első napon támogatja a Reflection Beam modellt" measure
 * 8K-token and 8 x 2,048-token prefills).  Query token t of sequence b sits
 * at position L_b - C + t and attends causally (and within the window) to
 * every key up to it, exactly as the tokens of a decode step do.
 *
 *   shape       as for rel_attn_decode except q_tokens = C, the query tokens
 *               per sequence, 1 .. 2^20 (batch * ceil(C / 8) <= 65535).
 *   q, out      [B, C, Hq, D]; lse [B, C, Hq] or NULL.
 *   seq_lens    L_b, counting the C query tokens (C <= L_b).
 *   workspace   rel_attn_workspace_bytes(shape, num_splits) bytes with this
 *               shape (q_tokens = C); num_splits <= 0 picks one split per
 *               chunk unless the chunks are too few to fill the GPU.
 * Every other argument, the error handling and the status word are as for
 * rel_attn_decode.  The tokens run as chunks of 8 through the decode
 * kernels (the first C mod 8 tokens as one more chunk), each chunk reading
 * the keys up to its last token.
 */
int rel_attn_prefill(const rel_attn_shape* shape, const void* q,
                     const void* k_cache, const void* v_cache,
                     const int32_t* block_table, const int32_t* seq_lens,
                     const void* rel_table, int window, int num_splits,
                     void* out, float* lse, void* workspace,
                     size_t workspace_bytes, void* stream);

/*
 * rel_attn_kv_write -- the producer step that fills the cache the decode
 * reads: a short convolution over the new tokens' K and V, written into the
 * paged KV cache (bf16, or E4M3 codes), with the raw K/V kept for the next
 * steps' convolutions.  One kernel.
 *
 * "vLLM TML Inkling 지원", section "TML Inkling 모델 아키텍처": every layer
 * applies a short convolution of window 4 to the attention keys and to the
 * attention values; section "Sconv 캐시 및 TP 샤딩": the convolution state
 * is kept by the unified KV-cache manager as the cache of a virtual
 * sliding-window layer, channel by channel.  The pages give no formula;
 * this library reads it as a causal depthwise convolution over positions:
 *   k~[p][h][c] = sum_{i=0..3} w[0][h][c][i] * k[p-i][h][c]   (k[q < 0] = 0)
 * and likewise for V with w[1].  The sum is formed in fp32 with the taps in
 * the order i = 0, 1, 2, 3, then rounded to nearest even (bf16), or divided
 * by the KV head's scale and rounded to nearest even E4M3 (saturating at
 * +-448).
 *
 * shape       reads batch, q_tokens (T = new tokens per sequence, 1..2^24),
 *             num_kv_heads, head_dim (128), page_size (64), num_pages and
 *             max_pages_per_seq; the other fields are ignored.
 *   k_new     bf16 [B, T, Hkv, D]: the new tokens' keys before the
 *   v_new     convolution (positions L_b - T .. L_b - 1), and values.
 *   conv_w    bf16 [2, Hkv, D, 4]: the K taps, then the V taps; tap i
 *             multiplies the vector at position p - i.
 *   k_raw     bf16 [num_pages, Hkv, P, D]: the sconv cache, the raw K and V
 *   v_raw     of every position, addressed by block_table like the KV
 *             cache.  Positions before L_b - T are read (the last three);
 *             the new positions are written.
 *   k_cache   [num_pages, Hkv, P, D]: the KV cache the decode reads; bf16,
 *   v_cache   or uint8 E4M3 codes when k_scale / v_scale are given.
 *   k_scale   fp32 [Hkv] per-KV-head scales (both, or both NULL for bf16).
 *   v_scale
 *   block_table, seq_lens   as for rel_attn_decode: seq_lens[b] = L_b
 *             counts the T new tokens (T <= L_b <= max_pages_per_seq * P).
 *   workspace NULL, or a workspace as for rel_attn_decode (256-byte
 *             aligned, initialised): a sequence whose length or block-table
 *             entries are out of range sets REL_ATTN_ERR_BAD_SEQ in its
 *             status word.  The new tokens of such a sequence that touch a
 *             bad entry are not written.
 * All device pointers are caller-owned, 16-byte aligned (4 for the int32
 * and fp32 arrays).  Asynchronous on `stream`; nothing is allocated.
 */
int rel_attn_kv_write(const rel_attn_shape* shape, const void* k_new, const void* v_new,
                      const void* conv_w, void* k_raw, void* v_raw, void* k_cache,
                      void* v_cache, const float* k_scale, const float* v_scale,
                      const int32_t* block_table, const int32_t* seq_lens,
                      void* workspace, void* stream);

/* Bytes of workspace rel_attn_decode needs for this shape and split count
 * (num_splits <= 0: the heuristic's choice).  0 when the shape is invalid. */
size_t rel_attn_workspace_bytes(const rel_attn_shape* shape, int num_splits);

/* Zero the workspace status word (asynchronous on `stream`).  Call once
 * after allocating a workspace and after reading a non-zero status. */
int rel_attn_workspace_init(void* workspace, size_t workspace_bytes, void* stream);

/* Bound, in nanoseconds, of each device-side wait in launches made after
 * this call, process-wide; 0 restores the default (2 s).  For failure-
 * detection tests: a short bound makes waits run out, and the kernels then
 * end with REL_ATTN_ERR_TIMEOUT in the status word and NaN rows instead of
 * hanging.  The waits that let copies and tensor-core operations already in
 * flight finish before a CTA exits keep a fixed 2 s bound whatever is set
 * here.  Always returns 0. */
int rel_attn_set_wait_limit(unsigned long long limit_ns);

/* Synchronise `stream`, read the workspace status word and clear it.
 * Returns 0, REL_ATTN_ERR_TIMEOUT, REL_ATTN_ERR_BAD_SEQ or REL_ATTN_ERR_CUDA. */
int rel_attn_read_status(void* workspace, void* stream);

/* The split heuristic: KV splits per (sequence, KV head) so that
 * batch * Hkv * splits fills `sm_count` SMs in one wave when batch * Hkv <
 * sm_count, and otherwise gives about twelve CTAs per SM in all (short
 * CTAs even out sequences of different lengths), bounded by the work
 * available (at least one 128-key tile per split) and by 256.  sm_count <= 0
 * queries the current device.  Returns >= 1, or a negative error code. */
int rel_attn_choose_splits(const rel_attn_shape* shape, int window, int sm_count);

/* bucket(distance) exactly as the kernels compute it (host copy of the same
 * edge table), for tests.  Returns -1 for an invalid shape or distance < 0. */
int rel_attn_bucket(const rel_attn_shape* shape, int distance);

/* The pages [*first_page, *end_page) of a sequence of `seq_len` keys (its
 * q_tokens queries at the end) that split `split` of `num_splits` walks:
 * the same cost-weighted partition the partial kernel computes on the
 * device (pages holding keys inside the exact-distance range weigh more
 * than far pages; interior boundaries fall on even page offsets).  For
 * tests and inspection; nothing is launched.  Returns 0, or
 * REL_ATTN_ERR_INVALID_ARG for an invalid shape, seq_len < q_tokens or
 * beyond the block-table row, or split outside [0, num_splits). */
int rel_attn_split_pages(const rel_attn_shape* shape, int seq_len, int window, int num_splits,
                         int split, int* first_page, int* end_page);

/* The same for calls over an E4M3 cache (rel_attn_decode_e4m3 /
 * rel_attn_partial_e4m3), whose partition weighs an exact-range page more:
 * such a tile also reads a 32 KB bf16 relative-row chunk, twice its E4M3 K
 * and V bytes.  Arguments, results and errors as rel_attn_split_pages. */
int rel_attn_split_pages_e4m3(const rel_attn_shape* shape, int seq_len, int window, int num_splits,
                              int split, int* first_page, int* end_page);

/* Static description of an error code. */
const char* rel_attn_error_string(int code);

/* Library version, e.g. "rel_attn 0.1.0 sm_100a". */
const char* rel_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* REL_ATTN_H */
