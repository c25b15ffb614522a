"""Plain fp64 definition of relative-bias GQA decode attention (the oracle).

TEST INFRASTRUCTURE ONLY -- see the package docstring.  Nothing here is
tuned; every step is the definition written out so that it can be checked
by eye.

The operation
-------------
For sequence b with context length L (which already includes its T query
tokens), query token t sits at position p_t = L - T + t.  Query head hq
reads KV head h = hq // G with G = Hq / Hkv (contiguous grouping, the usual
GQA convention).  It attends to the keys

    J_t = { j : 0 <= j <= p_t  and  (W <= 0  or  p_t - j <= W - 1) }

(exactly W keys, itself included, when a window W > 0 is set).  Key j's
vectors live at slot j % P of physical page block_table[b][j // P].  The
logit of key j is

    s_j = ( q . k_j  +  q . R_h[ bucket(p_t - j) ] ) / sqrt(D)

with R_h the learned relative table of KV head h (NB rows), and

    lse = log sum_{j in J_t} exp(s_j)          (natural log)
    out = sum_{j in J_t} exp(s_j - lse) v_j.

Sources (the pages describe the method only loosely):
  * "vLLM TML Inkling 지원", section "TML Inkling 모델 아키텍처": instead of
    RoPE the model adds a learned relative-position term to the pre-softmax
    attention logits; every layer is GQA with head size 128; the English
    sentence of that section says the "qkvr" linears stay in BF16 (a fourth
    projection feeding the relative term).
  * "vLLM、Inkling 2 Smallを初日サポート GB200で630 tok/s", section
    "モデルの構成": 48/8 heads, sliding window 1,024; hybrid sliding-window
    and full-attention layers.
  * "vLLM TML Inkling 지원", section "저지연 컬렉티브 및 커널" (FA4 bullet):
    the relative logits are formed densely and sheared into place
    ("sheared-bias"), and the KV length is cut into num_splits pieces.
The pages print no formula.  The form above (query dotted with a per-KV-head
table indexed by a bucketed distance, both terms inside one 1/sqrt(D)) and
the bucket function below are the library's stated reading.

Bucket function
---------------
With E exact buckets (1024), NB rows and the log range up to Dmax (2^20):
  * NB <= E:              bucket(d) = min(d, NB - 1)
  * NB >  E and d <  E:   bucket(d) = d
  * NB >  E and d >= E:   bucket(d) = E + min(NL - 1, max{k : e_k <= d}),
    NL = NB - E log buckets with lower edges e_k = ceil(E * (Dmax/E)^(k/NL)),
    k = 0..NL.  Distances beyond Dmax fall in the last bucket.
"""

from __future__ import annotations

import math

import numpy as np

EXACT_BUCKETS = 1024
MAX_DISTANCE = 1 << 20


# --------------------------------------------------------------------------
# bucket function
# --------------------------------------------------------------------------
def log_bucket_edges(num_buckets: int, exact_buckets: int = EXACT_BUCKETS,
                     max_distance: int = MAX_DISTANCE) -> np.ndarray:
    """Lower edges e_0..e_NL of the log buckets, exact in integer arithmetic.

    e_k is the smallest integer e with e >= E * (Dmax/E)^(k/NL), i.e. with
    e^NL * E^k >= E^NL * Dmax^k; Python integers make that comparison exact,
    so no floating-point rounding can move an edge.
    """
    E, dmax = int(exact_buckets), int(max_distance)
    nl = int(num_buckets) - E
    if nl <= 0:
        return np.zeros(0, dtype=np.int64)
    edges = []
    for k in range(nl + 1):
        target = E ** nl * dmax ** k
        e = max(1, int(math.ceil(E * (dmax / E) ** (k / nl))) - 2)
        while e ** nl * E ** k < target:
            e += 1
        while e > 1 and (e - 1) ** nl * E ** k >= target:
            e -= 1
        edges.append(e)
    return np.asarray(edges, dtype=np.int64)


def bucket_of_distance(d, num_buckets: int, exact_buckets: int = EXACT_BUCKETS,
                       max_distance: int = MAX_DISTANCE, edges=None) -> np.ndarray:
    """bucket(d) for non-negative integer distances (vectorised)."""
    d = np.asarray(d, dtype=np.int64)
    if d.size and d.min() < 0:
        raise ValueError("distances must be >= 0")
    if num_buckets <= exact_buckets:
        return np.minimum(d, num_buckets - 1)
    if edges is None:
        edges = log_bucket_edges(num_buckets, exact_buckets, max_distance)
    nl = num_buckets - exact_buckets
    k = np.searchsorted(edges, d, side="right") - 1      # max{k : e_k <= d}
    k = np.clip(k, 0, nl - 1)
    return np.where(d < exact_buckets, d, exact_buckets + k)


# --------------------------------------------------------------------------
# attention at explicit positions
# --------------------------------------------------------------------------
def attend_at_positions(q_rows, q_pos, keys, values, key_pos, rel, window: int,
                        num_buckets: int, exact_buckets: int = EXACT_BUCKETS,
                        max_distance: int = MAX_DISTANCE):
    """Attention of one GQA group at explicit positions.

    q_rows [T, G, D], q_pos [T]; keys / values [n, D] at positions key_pos [n];
    rel [NB, D] is the group's relative table.  Returns out [T, G, D] and
    lse [T, G] in fp64.  Positions enter only through q_pos[t] - key_pos.
    """
    q_rows = np.asarray(q_rows, dtype=np.float64)
    keys = np.asarray(keys, dtype=np.float64)
    values = np.asarray(values, dtype=np.float64)
    rel = np.asarray(rel, dtype=np.float64)
    key_pos = np.asarray(key_pos, dtype=np.int64)
    T, G, D = q_rows.shape
    scale = 1.0 / math.sqrt(D)
    edges = log_bucket_edges(num_buckets, exact_buckets, max_distance)
    # q . R[r] for every table row r; the relative term of key j is then the
    # entry at r = bucket(p_t - j) (a dense q R^T product indexed by distance).
    q_dot_rel = q_rows @ rel.T                                   # [T, G, NB]
    out = np.zeros((T, G, D))
    lse = np.full((T, G), -np.inf)
    for t in range(T):
        dist = int(q_pos[t]) - key_pos
        sel = dist >= 0
        if window > 0:
            sel &= dist <= window - 1
        idx = np.nonzero(sel)[0]
        if idx.size == 0:
            continue
        buckets = bucket_of_distance(dist[idx], num_buckets, exact_buckets,
                                     max_distance, edges)
        logits = (q_rows[t] @ keys[idx].T + q_dot_rel[t][:, buckets]) * scale
        m = logits.max(axis=1, keepdims=True)
        lse_t = m[:, 0] + np.log(np.exp(logits - m).sum(axis=1))
        out[t] = np.exp(logits - lse_t[:, None]) @ values[idx]
        lse[t] = lse_t
    return out, lse


def _as_np(x):
    if hasattr(x, "detach"):                     # torch tensor (bf16 included)
        x = x.detach().cpu()
        if x.dtype.is_floating_point:
            x = x.float()
        return x.numpy()
    return np.asarray(x)


def _group_keys(k_cache, v_cache, block_table_row, key_pos, h, page_size):
    pages = np.asarray(block_table_row)[key_pos // page_size]
    slots = key_pos % page_size
    return (k_cache[pages, h, slots].astype(np.float64),
            v_cache[pages, h, slots].astype(np.float64))


def rel_attn_decode_ref(q, k_cache, v_cache, block_table, seq_lens, rel_table,
                        window: int, exact_buckets: int = EXACT_BUCKETS,
                        max_distance: int = MAX_DISTANCE, batch_indices=None):
    """The operation for a whole batch.

    q [B, T, Hq, D]; k_cache / v_cache [num_pages, Hkv, P, D];
    block_table [B, max_pages] (int); seq_lens [B]; rel_table [Hkv, NB, D].
    Inputs may be numpy arrays or CPU/GPU torch tensors (bf16 values are
    upcast exactly).  Returns (out [B, T, Hq, D], lse [B, T, Hq]) in fp64.
    ``batch_indices`` restricts the work to some sequences (others stay 0).
    """
    q = _as_np(q)
    k_cache = _as_np(k_cache)
    v_cache = _as_np(v_cache)
    block_table = _as_np(block_table)
    seq_lens = _as_np(seq_lens)
    rel_table = _as_np(rel_table)
    B, T, Hq, D = q.shape
    _, Hkv, P, _ = k_cache.shape
    NB = rel_table.shape[1]
    G = Hq // Hkv
    out = np.zeros((B, T, Hq, D))
    lse = np.zeros((B, T, Hq))
    for b in (range(B) if batch_indices is None else batch_indices):
        L = int(seq_lens[b])
        q_pos = L - T + np.arange(T)
        lo = 0 if window <= 0 else max(0, int(q_pos[0]) - window + 1)
        key_pos = np.arange(lo, L)
        for h in range(Hkv):
            keys, vals = _group_keys(k_cache, v_cache, block_table[b], key_pos, h, P)
            o, l = attend_at_positions(q[b, :, h * G:(h + 1) * G], q_pos, keys,
                                       vals, key_pos, rel_table[h], window, NB,
                                       exact_buckets, max_distance)
            out[b, :, h * G:(h + 1) * G] = o
            lse[b, :, h * G:(h + 1) * G] = l
    return out, lse


def rel_attn_decode_split_ref(q, k_cache, v_cache, block_table, seq_lens,
                              rel_table, window: int, num_splits: int,
                              exact_buckets: int = EXACT_BUCKETS,
                              max_distance: int = MAX_DISTANCE):
    """Split-KV form: partial results over contiguous page groups, then merge.

    The visible pages of each sequence are cut into ``num_splits`` contiguous
    groups of ceil(n_pages / num_splits) pages (trailing groups may be empty).
    Each group gives a normalised partial output o_s and its lse_s (0 and -inf
    when it holds no visible key); the merge is
        lse = log sum_s exp(lse_s),  out = sum_s exp(lse_s - lse) o_s.
    Mathematically equal to rel_attn_decode_ref for every split count.
    """
    q = _as_np(q)
    k_cache = _as_np(k_cache)
    v_cache = _as_np(v_cache)
    block_table = _as_np(block_table)
    seq_lens = _as_np(seq_lens)
    rel_table = _as_np(rel_table)
    B, T, Hq, D = q.shape
    _, Hkv, P, _ = k_cache.shape
    NB = rel_table.shape[1]
    G = Hq // Hkv
    out = np.zeros((B, T, Hq, D))
    lse = np.zeros((B, T, Hq))
    for b in range(B):
        L = int(seq_lens[b])
        q_pos = L - T + np.arange(T)
        lo = 0 if window <= 0 else max(0, int(q_pos[0]) - window + 1)
        first, last = lo // P, (L - 1) // P
        n_pages = last - first + 1
        per = -(-n_pages // num_splits)
        for h in range(Hkv):
            parts_o, parts_l = [], []
            for s in range(num_splits):
                pa = first + s * per
                pb = min(first + (s + 1) * per, last + 1)
                key_pos = np.arange(max(pa * P, lo), min(pb * P, L))
                if key_pos.size == 0:
                    parts_o.append(np.zeros((T, G, D)))
                    parts_l.append(np.full((T, G), -np.inf))
                    continue
                keys, vals = _group_keys(k_cache, v_cache, block_table[b],
                                         key_pos, h, P)
                o, l = attend_at_positions(q[b, :, h * G:(h + 1) * G], q_pos,
                                           keys, vals, key_pos, rel_table[h],
                                           window, NB, exact_buckets,
                                           max_distance)
                parts_o.append(o)
                parts_l.append(l)
            lse_s = np.stack(parts_l)                            # [S, T, G]
            m = lse_s.max(axis=0)
            tot = m + np.log(np.exp(lse_s - m).sum(axis=0))
            w = np.exp(lse_s - tot)                              # [S, T, G]
            out[b, :, h * G:(h + 1) * G] = (w[..., None] * np.stack(parts_o)).sum(axis=0)
            lse[b, :, h * G:(h + 1) * G] = tot
    return out, lse


# --------------------------------------------------------------------------
# brute force (pure Python, tiny inputs only)
# --------------------------------------------------------------------------
def rel_attn_decode_bruteforce(q, k_cache, v_cache, block_table, seq_lens,
                               rel_table, window: int,
                               exact_buckets: int = EXACT_BUCKETS,
                               max_distance: int = MAX_DISTANCE):
    """Triple loop in plain Python floats; shares no helper with the above.

    The bucket edges here come from floating-point pow + ceil and a linear
    scan, not from the exact-integer table, so the two bucket paths check
    each other.
    """
    q = _as_np(q).tolist()
    k_cache = _as_np(k_cache).tolist()
    v_cache = _as_np(v_cache).tolist()
    block_table = _as_np(block_table).tolist()
    seq_lens = [int(x) for x in _as_np(seq_lens).tolist()]
    rel_table = _as_np(rel_table).tolist()
    B, T, Hq, D = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    Hkv, P = len(k_cache[0]), len(k_cache[0][0])
    NB = len(rel_table[0])
    G = Hq // Hkv
    E = exact_buckets
    NL = NB - E
    float_edges = [math.ceil(E * (max_distance / E) ** (k / NL)) for k in range(NL + 1)] if NL > 0 else []

    def bucket(d):
        if NB <= E:
            return d if d < NB - 1 else NB - 1
        if d < E:
            return d
        best = 0
        for k in range(NL):
            if float_edges[k] <= d:
                best = k
        return E + best

    out = [[[[0.0] * D for _ in range(Hq)] for _ in range(T)] for _ in range(B)]
    lse = [[[0.0] * Hq for _ in range(T)] for _ in range(B)]
    for b in range(B):
        L = seq_lens[b]
        for t in range(T):
            p = L - T + t
            for hq in range(Hq):
                h = hq // G
                qv = q[b][t][hq]
                logits, vals = [], []
                for j in range(L):
                    if j > p:
                        continue
                    if window > 0 and p - j > window - 1:
                        continue
                    page = block_table[b][j // P]
                    kv = k_cache[page][h][j % P]
                    r = rel_table[h][bucket(p - j)]
                    dot_k = 0.0
                    dot_r = 0.0
                    for c in range(D):
                        dot_k += qv[c] * kv[c]
                        dot_r += qv[c] * r[c]
                    logits.append((dot_k + dot_r) / math.sqrt(D))
                    vals.append(v_cache[page][h][j % P])
                m = max(logits)
                z = sum(math.exp(x - m) for x in logits)
                lse_v = m + math.log(z)
                lse[b][t][hq] = lse_v
                for c in range(D):
                    out[b][t][hq][c] = sum(math.exp(x - lse_v) * v[c]
                                           for x, v in zip(logits, vals))
    return np.asarray(out), np.asarray(lse)


# --------------------------------------------------------------------------
# FP8 (e4m3) KV cache
# --------------------------------------------------------------------------
# "vLLM TML Inkling 지원", section "미래 로드맵", plans FP8 for the global
# (full-context) attention layers to cut the KV-cache bottleneck; the
# Reflection Beam page's serving example runs an FP8 KV cache.  Neither fixes
# the format or the scales.  Reading taken: the OFP8 E4M3 format (1 sign bit,
# 4 exponent bits with bias 7, 3 mantissa bits, no infinities, S.1111.111 is
# NaN) and one fp32 scale per KV head for K and one for V:
#     k_j = e4m3(k_code_j) * k_scale[h],   v_j = e4m3(v_code_j) * v_scale[h].
def e4m3_to_float(codes) -> np.ndarray:
    """Real value of each E4M3 byte code, from the bit fields."""
    c = np.asarray(codes).astype(np.int64) & 0xFF
    sign = np.where(c & 0x80, -1.0, 1.0)
    exp = (c >> 3) & 0xF
    man = (c & 0x7).astype(np.float64)
    normal = sign * np.ldexp(1.0 + man / 8.0, (exp - 7).astype(np.int64))
    subnormal = sign * np.ldexp(man / 8.0, -6)
    v = np.where(exp == 0, subnormal, normal)
    return np.where((c & 0x7F) == 0x7F, np.nan, v)


def dequant_kv(codes, scale) -> np.ndarray:
    """[num_pages, Hkv, P, D] byte codes times the per-KV-head scale."""
    v = e4m3_to_float(np.asarray(codes))
    sc = np.asarray(_as_np(scale), dtype=np.float64).reshape(1, -1, 1, 1)
    return v * sc


def rel_attn_decode_fp8kv_ref(q, k_codes, v_codes, k_scale, v_scale, block_table, seq_lens,
                              rel_table, window: int, exact_buckets: int = EXACT_BUCKETS,
                              max_distance: int = MAX_DISTANCE, batch_indices=None):
    """The operation over an E4M3 KV cache: dequantise exactly (fp64), then the
    same definition as rel_attn_decode_ref.  k_codes / v_codes are uint8
    [num_pages, Hkv, P, D] (numpy, or torch uint8 / float8_e4m3fn viewed as
    uint8); k_scale / v_scale are [Hkv]."""
    def codes_of(x):
        if hasattr(x, "detach"):
            x = x.detach().cpu()
            if x.element_size() == 1 and x.dtype.is_floating_point:
                x = x.view(__import__("torch").uint8)
            return x.numpy()
        return np.asarray(x)
    k = dequant_kv(codes_of(k_codes), k_scale)
    v = dequant_kv(codes_of(v_codes), v_scale)
    return rel_attn_decode_ref(q, k, v, block_table, seq_lens, rel_table, window,
                               exact_buckets, max_distance, batch_indices)
