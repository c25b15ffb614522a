"""Plain definition of the KV-cache producer step (the oracle for it).

TEST INFRASTRUCTURE ONLY -- see the package docstring.

What the step computes
----------------------
"vLLM TML Inkling 지원", section "TML Inkling 모델 아키텍처", says every layer
applies short convolutions ("sconv", window 4) to the attention keys and the
attention values; section "Sconv 캐시 및 TP 샤딩" says vLLM keeps the sconv
state in its unified KV-cache manager as the KV cache of a virtual
sliding-window layer, and that sconv works channel by channel (the channels
can be sharded across GPUs).  "A vLLM már az első napon támogatja a
Reflection Beam modellt" lists a fused KV-cache update among its
optimisations.  The pages print no formula.  Reading taken:

  * the convolution is causal and depthwise over the sequence: for KV head
    h, channel c and position p,
        k~[p][h][c] = sum_{i=0..3} w_k[h][c][i] * k[p - i][h][c]
    with k[q] = 0 for q < 0 (and likewise for V with w_v);
  * the sconv cache holds the raw (pre-convolution) K and V of every
    position, in a paged pool laid out and addressed like the KV cache
    (same block table, page size 64): the convolution of a new token reads
    the raw vectors of the three positions before it from there;
  * one step takes the T new tokens of each sequence (positions L-T..L-1,
    L = seq_len including them), writes their raw K/V into the sconv cache
    and their convolved K/V into the KV cache: bf16, or OFP8 E4M3 codes of
    value / scale[h] (round to nearest even, saturating at +-448, the
    finite range) with the per-KV-head scales of the E4M3 decode path.

Precision: the definition (``short_conv_ref``) is exact (fp64).  The stored
bf16 value and the E4M3 code are roundings, decided from the sum as the GPU
accumulates it: in fp32, taps in the order i = 0, 1, 2, 3 (each product of
two bf16 values is exact in fp32, each addition rounds to nearest even).
``short_conv_fp32`` writes that order out and is pinned to the exact sum.
"""

from __future__ import annotations

import numpy as np

TAPS = 4


def short_conv_ref(raw, w) -> np.ndarray:
    """Exact causal depthwise convolution: raw [n, C] (positions 0..n-1),
    w [C, TAPS] -> out [n, C], out[p] = sum_i w[:, i] * raw[p - i]."""
    raw = np.asarray(raw, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    out = np.zeros_like(raw)
    for i in range(TAPS):
        if i == 0:
            out += w[:, 0] * raw
        else:
            out[i:] += w[:, i] * raw[:-i]
    return out


def short_conv_fp32(raw, w) -> np.ndarray:
    """The same sum as the kernel forms it: fp32, taps 0, 1, 2, 3 in order."""
    raw = np.asarray(raw, dtype=np.float32)
    w = np.asarray(w, dtype=np.float32)
    n = raw.shape[0]
    acc = (w[:, 0] * raw).astype(np.float32)
    for i in range(1, TAPS):
        shifted = np.zeros_like(raw)
        shifted[i:] = raw[:n - i]
        acc = (acc + (w[:, i] * shifted).astype(np.float32)).astype(np.float32)
    return acc


def bf16_rne(x) -> np.ndarray:
    """Round to the nearest bfloat16 (8 significant bits), ties to even;
    returned as float64 values.  Normal range only (no bf16 subnormals
    arise here)."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                      # x = m * 2^e, 0.5 <= |m| < 1
    r = np.rint(m * 256.0)                  # 8 significant bits; rint: ties to even
    return np.ldexp(r, e - 8)


def e4m3_rne_satfinite(x) -> np.ndarray:
    """OFP8 E4M3 byte code of each finite value: round to nearest even,
    magnitudes past 448 (the largest finite E4M3 value) saturate to 448."""
    x = np.asarray(x, dtype=np.float64)
    sign = np.where(np.signbit(x), 0x80, 0).astype(np.int64)
    a = np.minimum(np.abs(x), 448.0)
    codes = np.zeros(a.shape, dtype=np.int64)
    sub = a < 2.0 ** -6                     # subnormal range: quantum 2^-9
    codes[sub] = np.rint(a[sub] / 2.0 ** -9).astype(np.int64)    # 8 -> 0x08 = 2^-6 (continuous)
    nrm = ~sub
    m, e = np.frexp(a[nrm])                 # a = m 2^e, m in [0.5, 1)
    e = e - 1                               # a = (2m) 2^e, 2m in [1, 2)
    q = np.rint((2.0 * m - 1.0) * 8.0).astype(np.int64)
    carry = q == 8
    e = e + carry
    q = np.where(carry, 0, q)
    codes[nrm] = ((e + 7) << 3) | q
    return (codes | sign).astype(np.uint8)


def _np(x):
    if hasattr(x, "detach"):
        x = x.detach().cpu()
        if x.dtype.is_floating_point and x.element_size() == 2:
            x = x.float()
        return x.numpy()
    return np.asarray(x)


def kv_write_ref(k_new, v_new, conv_w, k_raw, v_raw, k_cache, v_cache, block_table,
                 seq_lens, k_scale=None, v_scale=None):
    """One producer step for a batch.

    k_new / v_new [B, T, Hkv, D] (bf16 values); conv_w [2, Hkv, D, TAPS]
    (index 0 for K, 1 for V; tap i multiplies position p - i); k_raw / v_raw
    [num_pages, Hkv, P, D] the sconv cache; k_cache / v_cache the KV cache,
    [num_pages, Hkv, P, D] bf16 values or uint8 E4M3 codes (then k_scale /
    v_scale [Hkv] are given); block_table [B, max_pages]; seq_lens [B].
    Returns new copies (k_raw, v_raw, k_cache, v_cache): the raw pools with
    the new tokens' K/V at their positions, the caches with their convolved
    K/V (float64 bf16 values, or uint8 codes).  Nothing else changes.
    """
    k_new, v_new, w = _np(k_new), _np(v_new), _np(conv_w)
    raws = [_np(k_raw).astype(np.float64).copy(), _np(v_raw).astype(np.float64).copy()]
    e4m3 = k_scale is not None
    caches = [_np(k_cache).copy(), _np(v_cache).copy()]
    if not e4m3:
        caches = [c.astype(np.float64) for c in caches]
    scales = [_np(k_scale), _np(v_scale)] if e4m3 else [None, None]
    bt = _np(block_table).astype(np.int64)
    lens = _np(seq_lens).astype(np.int64)
    B, T, Hkv, D = k_new.shape
    P = raws[0].shape[2]
    for b in range(B):
        L = int(lens[b])
        first_new = L - T
        lo = max(0, first_new - (TAPS - 1))
        pos = np.arange(lo, L)
        for kv, new in enumerate((k_new, v_new)):
            raw_pool, cache = raws[kv], caches[kv]
            for h in range(Hkv):
                # raw history of positions lo..L-1: old ones from the sconv
                # cache, new ones from the input
                hist = np.zeros((len(pos), D))
                old = pos < first_new
                pg = bt[b, pos[old] // P]
                hist[old] = raw_pool[pg, h, pos[old] % P]
                hist[~old] = new[b, :, h].astype(np.float64)
                # convolution over the history (positions before lo count as
                # zero: they are < 0, or not needed by the new tokens)
                conv32 = short_conv_fp32(hist, w[kv, h])[-T:]
                new_pos = np.arange(first_new, L)
                npg = bt[b, new_pos // P]
                raw_pool[npg, h, new_pos % P] = new[b, :, h]
                if e4m3:
                    q32 = (conv32 / np.float32(scales[kv][h])).astype(np.float32)
                    cache[npg, h, new_pos % P] = e4m3_rne_satfinite(q32)
                else:
                    cache[npg, h, new_pos % P] = bf16_rne(conv32)
    return raws[0], raws[1], caches[0], caches[1]
