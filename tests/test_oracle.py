"""Pins for the fp64 oracle (CPU only).

Each test checks the oracle against something other than itself: pure-Python
brute force, closed forms, invariants of the definition, a textbook library
routine (scaled-dot-product attention) and hand-derived bucket values.  The
last group plants plausible mistakes in the oracle and checks that the pins
catch them.
"""

import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import rel_attn_ref as ref
from relative_bias_gqa_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def small_case(*, L, T=1, Hq=4, Hkv=2, D=8, P=4, window=0, NB=1280, seed=0,
               B=1, rel_std=0.5, lens=None):
    lens = lens if lens is not None else [L] * B
    return W.make_case(seq_lens=lens, q_tokens=T, num_q_heads=Hq,
                       num_kv_heads=Hkv, head_dim=D, page_size=P,
                       window=window, num_buckets=NB, seed=seed,
                       rel_std=rel_std, extra_pages=3)


def run_ref(case, fn=None, **kw):
    fn = fn or oracle.rel_attn_decode_ref
    return fn(case.q, case.k_cache, case.v_cache, case.block_table,
              case.seq_lens, case.rel_table, case.window,
              exact_buckets=case.exact_buckets,
              max_distance=case.max_distance, **kw)


def key_set(L, T, t, window):
    p = L - T + t
    return [j for j in range(0, p + 1) if window <= 0 or p - j <= window - 1]


# ---------------------------------------------------------------- buckets
def test_bucket_golden_values():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "bucket_values.txt"))
            if l.strip() and not l.startswith("#")]
    for nb, d, want in rows:
        got = int(oracle.bucket_of_distance([int(d)], int(nb))[0])
        assert got == int(want), (nb, d, got, want)


def test_bucket_closed_form_exhaustive():
    # Every integer distance in [1024, 2^20) against the floor-log2 closed form.
    d = np.arange(1024, 1 << 20, dtype=np.int64)
    b = oracle.bucket_of_distance(d, 1280)
    closed = 1024 + np.minimum(255, np.floor(25.6 * np.log2(d / 1024.0))).astype(np.int64)
    assert np.array_equal(b, closed)
    d0 = np.arange(0, 1024)
    assert np.array_equal(oracle.bucket_of_distance(d0, 1280), d0)


def test_bucket_edges_properties():
    e = oracle.log_bucket_edges(1280)
    assert e.shape == (257,)
    assert e[0] == 1024 and e[-1] == 1 << 20
    assert np.all(np.diff(e) >= 28)          # strictly increasing, no empty bucket
    # the exact-integer edges agree with the plain floating-point evaluation
    fl = [math.ceil(1024 * (2 ** 20 / 1024) ** (k / 256)) for k in range(257)]
    assert list(e) == fl
    d = np.arange(0, 1 << 21)
    b = oracle.bucket_of_distance(d, 1280)
    assert np.all(np.diff(b) >= 0) and len(np.unique(b)) == 1280


def test_bucket_small_tables():
    # NB <= E clamps; NB slightly above E has a handful of wide log buckets
    assert list(oracle.bucket_of_distance([0, 5, 7, 8, 100], 8)) == [0, 5, 7, 7, 7]
    e = oracle.log_bucket_edges(1030)
    assert e[0] == 1024 and e[-1] == 1 << 20 and len(e) == 7
    for k in range(6):
        assert oracle.bucket_of_distance([int(e[k])], 1030)[0] == 1024 + k
        assert oracle.bucket_of_distance([int(e[k + 1]) - 1], 1030)[0] == 1024 + k


# ------------------------------------------------------------ brute force
BRUTE_CASES = [
    dict(L=37, T=1, D=4, P=4, window=0, NB=8),
    dict(L=37, T=3, D=4, P=4, window=5, NB=8),
    dict(L=64, T=8, D=4, P=4, window=1, NB=1030),
    dict(L=300, T=1, D=4, P=64, window=64, NB=1280),
    dict(L=300, T=8, D=4, P=64, window=0, NB=1030),
    dict(L=130, T=3, D=128, P=64, window=0, NB=1280, Hq=2, Hkv=1),
    dict(L=200, T=8, D=128, P=4, window=64, NB=8, Hq=2, Hkv=2),
]


@pytest.mark.parametrize("kw", BRUTE_CASES)
def test_bruteforce_matches_vectorised(kw):
    case = small_case(**kw)
    o1, l1 = run_ref(case)
    o2, l2 = run_ref(case, oracle.rel_attn_decode_bruteforce)
    assert np.abs(o1 - o2).max() <= 1e-12
    assert np.abs(l1 - l2).max() <= 1e-12


def test_bruteforce_long_distance_buckets():
    # distances past 1024 reach the log buckets: a long, cheap (D=2) sequence
    case = small_case(L=3000, T=2, Hq=2, Hkv=1, D=2, P=64, NB=1280, rel_std=1.0)
    o1, l1 = run_ref(case)
    o2, l2 = run_ref(case, oracle.rel_attn_decode_bruteforce)
    assert np.abs(o1 - o2).max() <= 1e-12 and np.abs(l1 - l2).max() <= 1e-12


# ---------------------------------------------- library special case (R = 0)
@pytest.mark.parametrize("T,window", [(1, 0), (3, 0), (8, 5), (2, 1)])
def test_zero_rel_is_sdpa(T, window):
    case = small_case(L=150, T=T, Hq=6, Hkv=2, D=16, P=8, window=window)
    case.rel_table.zero_()
    out, lse = run_ref(case)
    L = 150
    Hq, Hkv, G = 6, 2, 3
    pages = case.block_table[0].long()
    j = torch.arange(L)
    k = case.k_cache.double()[pages[j // 8], :, j % 8]          # [L, Hkv, D]
    v = case.v_cache.double()[pages[j // 8], :, j % 8]
    k = k.repeat_interleave(G, dim=1).permute(1, 0, 2)[None]    # [1, Hq, L, D]
    v = v.repeat_interleave(G, dim=1).permute(1, 0, 2)[None]
    q = case.q.double()[0].permute(1, 0, 2)[None]               # [1, Hq, T, D]
    p = torch.arange(L - T, L)[:, None]
    mask = (j[None] <= p)
    if window > 0:
        mask &= (p - j[None]) <= window - 1
    sd = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask)
    assert np.abs(out[0] - sd[0].permute(1, 0, 2).numpy()).max() <= 1e-12
    logits = (q @ k.transpose(-1, -2)) / math.sqrt(16)
    logits = logits.masked_fill(~mask, float("-inf"))
    l_t = torch.logsumexp(logits, dim=-1)[0].permute(1, 0)
    assert np.abs(lse[0] - l_t.numpy()).max() <= 1e-12


# ---------------------------------------------------------------- invariants
def test_constant_values_return_constant():
    case = small_case(L=500, T=4, Hq=4, Hkv=2, D=32, P=16, window=0)
    case.v_cache.fill_(0.375)
    out, _ = run_ref(case)
    assert np.abs(out - 0.375).max() <= 1e-12


def test_translation_invariance_explicit_positions():
    rng = np.random.default_rng(3)
    T, G, D, n = 3, 2, 16, 400
    q = rng.standard_normal((T, G, D))
    keys = rng.standard_normal((n, D))
    vals = rng.standard_normal((n, D))
    rel = rng.standard_normal((1280, D))
    key_pos = np.arange(n)
    q_pos = np.array([397, 398, 399])
    base = oracle.attend_at_positions(q, q_pos, keys, vals, key_pos, rel, 0, 1280)
    for delta in (1, 977, 300_000):
        o, l = oracle.attend_at_positions(q, q_pos + delta, keys, vals,
                                          key_pos + delta, rel, 0, 1280)
        assert np.abs(o - base[0]).max() <= 1e-12 and np.abs(l - base[1]).max() <= 1e-12
    # a far-away query (distances in the log buckets) is shift-invariant too
    far = oracle.attend_at_positions(q, q_pos + 50_000, keys, vals, key_pos, rel, 0, 1280)
    o, l = oracle.attend_at_positions(q, q_pos + 50_000 + 977, keys, vals,
                                      key_pos + 977, rel, 0, 1280)
    assert np.abs(o - far[0]).max() <= 1e-12 and np.abs(l - far[1]).max() <= 1e-12


def test_translation_invariance_sliding_window_api():
    # Same last W keys at context L and L + delta: same output.
    Wn, P, D = 16, 4, 8
    a = small_case(L=40, T=2, D=D, P=P, window=Wn, seed=5)
    delta = 24                                    # whole pages, so slots line up
    b = small_case(L=40 + delta, T=2, D=D, P=P, window=Wn, seed=6)
    b.q.copy_(a.q)
    b.rel_table.copy_(a.rel_table)
    for j in range(40):
        pa = int(a.block_table[0, j // P])
        pb = int(b.block_table[0, (j + delta) // P])
        b.k_cache[pb, :, (j + delta) % P] = a.k_cache[pa, :, j % P]
        b.v_cache[pb, :, (j + delta) % P] = a.v_cache[pa, :, j % P]
    oa, la = run_ref(a)
    ob, lb = run_ref(b)
    assert np.abs(oa - ob).max() <= 1e-12 and np.abs(la - lb).max() <= 1e-12


@pytest.mark.parametrize("L", [1, 7, 16])
def test_sliding_equals_full_when_context_fits(L):
    a = small_case(L=L, T=1, D=8, P=4, window=16)
    o_w, l_w = run_ref(a)
    a.window = 0
    o_f, l_f = run_ref(a)
    assert np.abs(o_w - o_f).max() == 0 and np.abs(l_w - l_f).max() == 0


def test_window_one_returns_own_value():
    case = small_case(L=50, T=3, D=8, P=4, window=1)
    out, _ = run_ref(case)
    for t in range(3):
        j = 50 - 3 + t
        pg = int(case.block_table[0, j // 4])
        v = case.v_cache[pg, :, j % 4].double().numpy()             # [Hkv, D]
        want = np.repeat(v, 2, axis=0)                              # G = 2
        assert np.abs(out[0, t] - want).max() <= 1e-12


@pytest.mark.parametrize("S", [1, 2, 3, 7, 64, 256])
def test_split_merge_equals_unsplit(S):
    case = small_case(L=700, T=3, Hq=4, Hkv=2, D=8, P=4, window=0, B=2,
                      lens=[700, 333])
    o, l = run_ref(case)
    os_, ls = run_ref(case, oracle.rel_attn_decode_split_ref, num_splits=S)
    assert np.abs(o - os_).max() <= 1e-12 and np.abs(l - ls).max() <= 1e-12
    case.window = 37
    o, l = run_ref(case)
    os_, ls = run_ref(case, oracle.rel_attn_decode_split_ref, num_splits=S)
    assert np.abs(o - os_).max() <= 1e-12 and np.abs(l - ls).max() <= 1e-12


@pytest.mark.parametrize("window", [0, 1, 9, 64])
def test_zero_logits_count_keys(window):
    case = small_case(L=301, T=5, D=8, P=8, window=window, B=2, lens=[301, 12])
    case.q.zero_()
    case.rel_table.zero_()
    _, lse = run_ref(case)
    for b, L in enumerate([301, 12]):
        for t in range(5):
            n = len(key_set(L, 5, t, window))
            assert np.abs(lse[b, t] - math.log(n)).max() <= 1e-12


def test_key_set_identity_bits():
    # V[j][c] = bit c of the logical position j: out * |J| counts selected keys.
    P, D, L, T, Wn = 8, 16, 1000, 4, 77
    case = small_case(L=L, T=T, D=D, P=P, window=Wn)
    case.q.zero_()
    case.rel_table.zero_()
    for j in range(L):
        pg = int(case.block_table[0, j // P])
        bits = torch.tensor([(j >> c) & 1 for c in range(D)], dtype=torch.bfloat16)
        case.v_cache[pg, :, j % P] = bits
    out, _ = run_ref(case)
    for t in range(T):
        J = key_set(L, T, t, Wn)
        want = np.array([sum((j >> c) & 1 for j in J) for c in range(D)], float)
        got = out[0, t] * len(J)
        assert np.abs(got - want[None]).max() <= 1e-9


def test_relative_probe_direction():
    # A table row aligned with q makes the key at distance d* dominate.
    L, T, D = 400, 1, 8
    for d_star in (0, 5, 63, 250):
        case = small_case(L=L, T=T, Hq=2, Hkv=1, D=D, P=4, NB=1280)
        case.q.zero_()
        case.q[..., 0] = 4.0
        case.rel_table.zero_()
        case.rel_table[0, d_star, 0] = 64.0        # logit 4*64/sqrt(8) ~ 90.5
        out, _ = run_ref(case)
        j = L - 1 - d_star
        pg = int(case.block_table[0, j // 4])
        want = case.v_cache[pg, 0, j % 4].double().numpy()
        assert np.abs(out[0, 0, 0] - want).max() <= 1e-9


def test_gqa_head_mapping():
    case = small_case(L=90, T=2, Hq=6, Hkv=3, D=8, P=8)
    for h in range(3):
        case.v_cache[:, h] = float(h + 1)
    out, _ = run_ref(case)
    for hq in range(6):
        assert np.abs(out[0, :, hq] - (hq // 2 + 1)).max() <= 1e-12


@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (16, 2), (16, 4)])
def test_gqa_head_mapping_other_group_sizes(Hq, Hkv):
    # G = 4 and 8 (the previous Inkling's 64/16 and 64/8 layers, scaled down)
    case = small_case(L=70, T=3, Hq=Hq, Hkv=Hkv, D=8, P=8)
    for h in range(Hkv):
        case.v_cache[:, h] = float(h + 1)
    out, _ = run_ref(case)
    G = Hq // Hkv
    for hq in range(Hq):
        assert np.abs(out[0, :, hq] - (hq // G + 1)).max() <= 1e-12


@pytest.mark.parametrize("Hq,Hkv,T,window", [(16, 2, 6, 0), (8, 2, 8, 7), (16, 4, 1, 0)])
def test_zero_rel_is_sdpa_other_group_sizes(Hq, Hkv, T, window):
    case = small_case(L=120, T=T, Hq=Hq, Hkv=Hkv, D=16, P=8, window=window)
    case.rel_table.zero_()
    out, lse = run_ref(case)
    L, G = 120, Hq // Hkv
    pages = case.block_table[0].long()
    j = torch.arange(L)
    k = case.k_cache.double()[pages[j // 8], :, j % 8].repeat_interleave(G, dim=1).permute(1, 0, 2)[None]
    v = case.v_cache.double()[pages[j // 8], :, j % 8].repeat_interleave(G, dim=1).permute(1, 0, 2)[None]
    q = case.q.double()[0].permute(1, 0, 2)[None]
    p = torch.arange(L - T, L)[:, None]
    mask = (j[None] <= p)
    if window > 0:
        mask &= (p - j[None]) <= window - 1
    sd = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask)
    assert np.abs(out[0] - sd[0].permute(1, 0, 2).numpy()).max() <= 1e-12
    logits = ((q @ k.transpose(-1, -2)) / math.sqrt(16)).masked_fill(~mask, float("-inf"))
    assert np.abs(lse[0] - torch.logsumexp(logits, dim=-1)[0].permute(1, 0).numpy()).max() <= 1e-12


# ------------------------------------------------- planted mistakes are caught
def _pins_fail(monkeypatch, name, bad):
    monkeypatch.setattr(ref, name, bad)
    failures = 0
    checks = [
        lambda: test_bruteforce_matches_vectorised(BRUTE_CASES[1]),
        lambda: test_bruteforce_matches_vectorised(BRUTE_CASES[3]),
        lambda: test_bruteforce_long_distance_buckets(),
        lambda: test_key_set_identity_bits(),
        lambda: test_relative_probe_direction(),
        lambda: test_gqa_head_mapping(),
        lambda: test_zero_logits_count_keys(9),
    ]
    for c in checks:
        try:
            c()
        except AssertionError:
            failures += 1
    return failures


def test_planted_bucket_off_by_one(monkeypatch):
    good = ref.bucket_of_distance
    bad = lambda d, nb, *a, **k: np.minimum(good(d, nb, *a, **k) + 1, nb - 1)
    assert _pins_fail(monkeypatch, "bucket_of_distance", bad) > 0


def test_planted_log_bucket_shift(monkeypatch):
    good = ref.bucket_of_distance

    def bad(d, nb, E=1024, *a, **k):
        b = good(d, nb, E, *a, **k)
        return np.where(b >= E, np.minimum(b + 1, nb - 1), b)
    assert _pins_fail(monkeypatch, "bucket_of_distance", bad) > 0


def test_planted_wrong_head(monkeypatch):
    good = ref._group_keys
    bad = lambda kc, vc, row, pos, h, P: good(kc, vc, row, pos, (h + 1) % kc.shape[1], P)
    assert _pins_fail(monkeypatch, "_group_keys", bad) > 0


def test_planted_wrong_slot(monkeypatch):
    def bad(kc, vc, row, pos, h, P):
        pages = np.asarray(row)[pos // P]
        slots = (P - 1) - pos % P
        return kc[pages, h, slots].astype(np.float64), vc[pages, h, slots].astype(np.float64)
    assert _pins_fail(monkeypatch, "_group_keys", bad) > 0


def test_planted_dropped_relative_term(monkeypatch):
    good = ref.attend_at_positions

    def bad(q, qp, k, v, kp, rel, *a, **kw):
        return good(q, qp, k, v, kp, np.zeros_like(np.asarray(rel, float)), *a, **kw)
    assert _pins_fail(monkeypatch, "attend_at_positions", bad) > 0


def test_planted_reversed_distance(monkeypatch):
    good = ref.attend_at_positions

    def bad(q, qp, k, v, kp, *a, **kw):
        # mirror key positions inside the visible range (distance sign mix-up)
        kp = np.asarray(kp)
        return good(q, qp, k[::-1], v[::-1], kp, *a, **kw)
    assert _pins_fail(monkeypatch, "attend_at_positions", bad) > 0


# ------------------------------------------------------- FP8 (E4M3) KV cache
def test_e4m3_known_codes():
    """Values fixed by the E4M3 bit layout (bias 7, 3 mantissa bits)."""
    v = oracle.e4m3_to_float(np.array([0x00, 0x80, 0x38, 0xB8, 0x7E, 0xFE, 0x01, 0x07, 0x08,
                                       0x3C, 0x40, 0x7F, 0xFF]))
    want = [0.0, -0.0, 1.0, -1.0, 448.0, -448.0, 2.0 ** -9, 7 * 2.0 ** -9, 2.0 ** -6,
            1.5, 2.0]
    assert np.array_equal(v[:11], want)
    assert math.copysign(1.0, v[1]) == -1.0
    assert np.isnan(v[11]) and np.isnan(v[12])


def test_e4m3_matches_library_decode():
    """Every code against torch's float8_e4m3fn decoding."""
    codes = torch.arange(256, dtype=torch.uint8)
    lib = codes.view(torch.float8_e4m3fn).double().numpy()
    mine = oracle.e4m3_to_float(codes.numpy())
    assert np.array_equal(np.isnan(mine), np.isnan(lib))
    ok = ~np.isnan(lib)
    assert np.array_equal(mine[ok], lib[ok])


def fp8_case(seed=0, L=37, T=1, window=0):
    case = small_case(L=L, T=T, window=window, seed=seed)
    g = np.random.default_rng(seed + 7)
    shape = tuple(case.k_cache.shape)
    codes = lambda: g.integers(0, 256, size=shape, dtype=np.uint8) & 0xF7 | 0x30  # exponent 6 or 14: finite
    kc, vc = codes(), codes()
    Hkv = shape[1]
    ks = g.uniform(0.01, 0.05, Hkv)
    vs = g.uniform(0.5, 2.0, Hkv)
    return case, kc, vc, ks, vs


def run_fp8(case, kc, vc, ks, vs):
    return oracle.rel_attn_decode_fp8kv_ref(case.q, kc, vc, ks, vs, case.block_table,
                                            case.seq_lens, case.rel_table, case.window,
                                            exact_buckets=case.exact_buckets,
                                            max_distance=case.max_distance)


def test_fp8kv_is_the_bf16_definition_on_decoded_values():
    """Dequantised by hand (code value x scale, built from the format's bit
    fields in the brute-force style) and fed to the pure-Python brute force."""
    case, kc, vc, ks, vs = fp8_case(seed=3, L=23, T=2)

    def decode(x):
        s = -1.0 if x & 0x80 else 1.0
        e, m = (x >> 3) & 0xF, x & 7
        return s * (m / 8.0) * 2.0 ** -6 if e == 0 else s * (1 + m / 8.0) * 2.0 ** (e - 7)

    dec = np.vectorize(decode, otypes=[np.float64])
    k = dec(kc) * ks.reshape(1, -1, 1, 1)
    v = dec(vc) * vs.reshape(1, -1, 1, 1)
    o1, l1 = run_fp8(case, kc, vc, ks, vs)
    o2, l2 = oracle.rel_attn_decode_bruteforce(case.q, k, v, case.block_table, case.seq_lens,
                                               case.rel_table, case.window,
                                               exact_buckets=case.exact_buckets,
                                               max_distance=case.max_distance)
    assert np.allclose(o1, o2, atol=1e-12) and np.allclose(l1, l2, atol=1e-12)


def test_fp8kv_v_scale_is_linear():
    case, kc, vc, ks, vs = fp8_case(seed=1)
    o1, l1 = run_fp8(case, kc, vc, ks, vs)
    o2, l2 = run_fp8(case, kc, vc, ks, vs * 3.0)
    assert np.allclose(o2, 3.0 * o1, atol=1e-12) and np.allclose(l1, l2, atol=1e-12)


def test_fp8kv_zero_k_scale_leaves_the_relative_term():
    """k_scale = 0 removes q.k: the result equals the definition with K = 0."""
    case, kc, vc, ks, vs = fp8_case(seed=2, L=41)
    o1, l1 = run_fp8(case, kc, vc, np.zeros_like(ks), vs)
    v = oracle.dequant_kv(vc, vs)
    o2, l2 = oracle.rel_attn_decode_ref(case.q, np.zeros_like(v), v, case.block_table,
                                        case.seq_lens, case.rel_table, case.window,
                                        exact_buckets=case.exact_buckets,
                                        max_distance=case.max_distance)
    assert np.allclose(o1, o2, atol=1e-12) and np.allclose(l1, l2, atol=1e-12)


def test_planted_e4m3_bias(monkeypatch):
    """An exponent bias of 8 instead of 7 must fail the known-code pin."""
    good = ref.e4m3_to_float

    def bad(codes):
        return good(codes) * 0.5
    monkeypatch.setattr(oracle, "e4m3_to_float", bad)
    with pytest.raises(AssertionError):
        test_e4m3_known_codes()
