"""Pins of the KV-cache producer oracle (CPU only).

Each function of oracle/kv_write_ref.py is checked against something other
than itself: closed forms (identity and delta taps, linearity, constant
inputs), a pure-Python brute force over explicit positions, the exact
fp64 sum within the fp32 error bound, hand-derived roundings, the E4M3
decoder of the decode oracle, and torch's own float8 / bfloat16 casts.
"""

import math
import random

import numpy as np
import pytest
import torch

import oracle
import importlib

K = importlib.import_module("oracle.kv_write_ref")


def _bf16(x):
    return torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).float().numpy().astype(np.float64)


# ----------------------------------------------------------- short conv
def test_identity_and_delta_taps():
    rng = np.random.default_rng(0)
    raw = rng.standard_normal((50, 16))
    for i in range(4):
        w = np.zeros((16, 4))
        w[:, i] = 1.0
        out = K.short_conv_ref(raw, w)
        want = np.zeros_like(raw)
        want[i:] = raw[:50 - i]                       # causal shift by i, zero fill
        assert np.array_equal(out, want)


def test_linearity_and_constant_input():
    rng = np.random.default_rng(1)
    a, b = rng.standard_normal((2, 40, 8))
    w = rng.standard_normal((8, 4))
    assert np.allclose(K.short_conv_ref(2 * a - 3 * b, w),
                       2 * K.short_conv_ref(a, w) - 3 * K.short_conv_ref(b, w), atol=1e-12)
    const = np.full((20, 8), 1.5)
    out = K.short_conv_ref(const, w)
    assert np.allclose(out[3:], 1.5 * w.sum(axis=1), atol=1e-12)   # full window from p = 3 on
    assert np.allclose(out[0], 1.5 * w[:, 0], atol=1e-12)          # zeros before position 0


def test_short_conv_bruteforce():
    rng = random.Random(2)
    n, C = 13, 3
    raw = [[rng.uniform(-2, 2) for _ in range(C)] for _ in range(n)]
    w = [[rng.uniform(-1, 1) for _ in range(4)] for _ in range(C)]
    out = K.short_conv_ref(np.array(raw), np.array(w))
    for p in range(n):
        for c in range(C):
            s = 0.0
            for i in range(4):
                if p - i >= 0:
                    s += w[c][i] * raw[p - i][c]
            assert abs(out[p, c] - s) < 1e-12


def test_fp32_order_within_rounding_of_exact_sum():
    rng = np.random.default_rng(3)
    raw = _bf16(rng.standard_normal((300, 64)))
    w = _bf16(rng.standard_normal((64, 4)) * 0.5)
    exact = K.short_conv_ref(raw, w)
    f32 = K.short_conv_fp32(raw, w).astype(np.float64)
    # three fp32 additions of exact products: |err| <= 3 * 2^-24 * sum |w x|
    mag = K.short_conv_ref(np.abs(raw), np.abs(w))
    assert np.all(np.abs(f32 - exact) <= 3 * 2.0 ** -24 * mag + 1e-300)
    # small integers sum exactly in fp32: the two agree bit for bit
    ri = rng.integers(-8, 8, (50, 8)).astype(np.float64)
    wi = rng.integers(-4, 4, (8, 4)).astype(np.float64)
    assert np.array_equal(K.short_conv_fp32(ri, wi).astype(np.float64), K.short_conv_ref(ri, wi))


def test_fp32_order_is_taps_in_sequence():
    """(2^24 + 1) cannot be held in fp32: the order of the additions shows.
    Taps 0 and 1 give 2^24 and 1 (sum rounds to 2^24, ties to even), tap 2
    adds 1 again (rounds to 2^24), tap 3 adds 2 (exact): 2^24 + 2."""
    raw = np.array([[2.0], [1.0], [1.0], [2.0 ** 24]])      # positions 0..3
    w = np.array([[1.0, 1.0, 1.0, 1.0]])
    # output at p = 3: w0 x3 + w1 x2 + w2 x1 + w3 x0 = 2^24, 1, 1, 2 in tap order
    assert K.short_conv_fp32(raw, w)[3, 0] == np.float32(2.0 ** 24 + 2)
    assert K.short_conv_ref(raw, w)[3, 0] == 2.0 ** 24 + 4


# --------------------------------------------------------------- roundings
def test_bf16_rne_hand_values():
    one = 1.0
    ulp = 2.0 ** -7                                   # bf16 spacing in [1, 2)
    assert K.bf16_rne(one + ulp / 2) == one           # tie -> even (1.0)
    assert K.bf16_rne(one + 3 * ulp / 2) == one + 2 * ulp   # tie -> even (1 + 2 ulp)
    assert K.bf16_rne(one + ulp / 2 + 2.0 ** -30) == one + ulp
    assert K.bf16_rne(-3.0) == -3.0 and K.bf16_rne(0.0) == 0.0
    assert K.bf16_rne(255.5) == 256.0                  # 255.5 needs 9 bits; tie -> 256 (even)


def test_bf16_rne_matches_torch_on_fp32():
    rng = np.random.default_rng(4)
    x = (rng.standard_normal(200_000) * np.exp(rng.uniform(-20, 20, 200_000))).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).float().numpy().astype(np.float64)
    assert np.array_equal(K.bf16_rne(x.astype(np.float64)), want)


def test_e4m3_encode_hand_values():
    enc = lambda v: int(K.e4m3_rne_satfinite(np.array([v]))[0])
    assert enc(0.0) == 0x00 and enc(-0.0) == 0x80
    assert enc(1.0) == 0x38                           # exponent 7 (bias 7), mantissa 0
    assert enc(448.0) == 0x7E and enc(1e6) == 0x7E and enc(-1e6) == 0xFE   # saturation
    assert enc(2.0 ** -6) == 0x08                     # smallest normal
    assert enc(2.0 ** -9) == 0x01                     # smallest subnormal
    assert enc(2.0 ** -10) == 0x00                    # half the smallest subnormal: tie -> 0
    assert enc(1.5 * 2.0 ** -9) == 0x02               # 1.5 quanta: tie -> even (2)
    assert enc(1.0625) == 0x38                        # 1 + 1/16: tie between 1 and 1.125 -> 1
    assert enc(1.1875) == 0x3A                        # 1 + 3/16: tie between 1.125, 1.25 -> 1.25
    assert enc(-2.5) == 0xC2


def test_e4m3_encode_roundtrips_every_finite_code():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = oracle.e4m3_to_float(codes)
    back = K.e4m3_rne_satfinite(vals)
    # +0 and -0 keep their sign bit; every other code comes back as itself
    assert np.array_equal(back, codes)


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(5)
    x = (rng.standard_normal(100_000) * np.exp(rng.uniform(-12, 6, 100_000))).astype(np.float32)
    x = x[np.abs(x) <= 448]
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(K.e4m3_rne_satfinite(x.astype(np.float64)), want)


# ------------------------------------------------------ the producer step
def _case(lens, T, Hkv=2, D=16, P=4, seed=0, extra=3):
    g = torch.Generator().manual_seed(seed)
    pages = sum(math.ceil(L / P) for L in lens) + extra
    bt = torch.full((len(lens), max(math.ceil(L / P) for L in lens)), -1, dtype=torch.int32)
    perm = torch.randperm(pages, generator=g)
    o = 0
    for b, L in enumerate(lens):
        n = math.ceil(L / P)
        bt[b, :n] = perm[o:o + n].int()
        o += n
    bf = lambda *s: torch.randn(*s, generator=g).to(torch.bfloat16)
    return dict(k_new=bf(len(lens), T, Hkv, D), v_new=bf(len(lens), T, Hkv, D),
                conv_w=(torch.randn(2, Hkv, D, 4, generator=g) * 0.5).to(torch.bfloat16),
                k_raw=bf(pages, Hkv, P, D), v_raw=bf(pages, Hkv, P, D),
                k_cache=bf(pages, Hkv, P, D), v_cache=bf(pages, Hkv, P, D),
                block_table=bt, seq_lens=torch.tensor(lens, dtype=torch.int32))


def test_kv_write_bruteforce_by_position():
    """Pure-Python per-element sum over explicit positions: the raw value of
    position q is looked up through the block table (old positions) or in
    the new tokens, zero before position 0."""
    c = _case([7, 3, 13], T=3, seed=6)
    kr, vr, kc, vc = oracle.kv_write_ref(**c)
    P = c["k_raw"].shape[2]
    bt, lens = c["block_table"].tolist(), c["seq_lens"].tolist()
    T = c["k_new"].shape[1]
    for kv, (new, raw, cache) in enumerate(((c["k_new"], c["k_raw"], kc), (c["v_new"], c["v_raw"], vc))):
        new, raw = new.float(), raw.float()
        for b, L in enumerate(lens):
            for t in range(T):
                p = L - T + t
                for h in range(new.shape[2]):
                    for ch in range(0, new.shape[3], 5):
                        s = 0.0
                        for i in range(4):
                            q = p - i
                            if q < 0:
                                x = 0.0
                            elif q >= L - T:
                                x = float(new[b, q - (L - T), h, ch])
                            else:
                                x = float(raw[bt[b][q // P], h, q % P, ch])
                            s += float(c["conv_w"][kv, h, ch, i]) * x
                        got = cache[bt[b][p // P], h, p % P, ch]
                        # the stored bf16 value: within half a bf16 unit of the
                        # exact sum, plus the fp32 accumulation's rounding
                        ulp = 2.0 ** (math.floor(math.log2(abs(s))) - 7) if s != 0 else 0.0
                        assert abs(got - s) <= ulp / 2 + 4 * 2.0 ** -24 * (abs(s) + 8), (b, t, h, ch)


def test_kv_write_untouched_elsewhere_and_raw_copied():
    c = _case([9, 5], T=2, seed=7)
    kr, vr, kc, vc = oracle.kv_write_ref(**c)
    P = c["k_raw"].shape[2]
    mask = np.zeros(c["k_raw"].shape[:3], dtype=bool)
    for b, L in enumerate(c["seq_lens"].tolist()):
        for p in range(L - 2, L):
            mask[int(c["block_table"][b, p // P]), :, p % P] = True
            for kv, (raw_new, new) in enumerate(((kr, c["k_new"]), (vr, c["v_new"]))):
                assert np.array_equal(raw_new[int(c["block_table"][b, p // P]), :, p % P],
                                      new[b, p - (L - 2)].float().numpy())
    for before, after in ((c["k_raw"], kr), (c["v_raw"], vr), (c["k_cache"], kc), (c["v_cache"], vc)):
        assert np.array_equal(before.float().numpy()[~mask], after[~mask])


def test_kv_write_one_step_equals_token_by_token():
    """The sconv cache carries the state: writing T tokens at once equals T
    one-token steps in order (each reading the raw vectors the previous ones
    wrote)."""
    lens, T = [11, 6], 4
    c = _case(lens, T=T, seed=8)
    all_at_once = oracle.kv_write_ref(**c)
    state = dict(c)
    for t in range(T):
        step = dict(state, k_new=c["k_new"][:, t:t + 1], v_new=c["v_new"][:, t:t + 1],
                    seq_lens=torch.tensor([L - T + t + 1 for L in lens], dtype=torch.int32))
        kr, vr, kc, vc = oracle.kv_write_ref(**step)
        state.update(k_raw=torch.from_numpy(kr).to(torch.bfloat16),
                     v_raw=torch.from_numpy(vr).to(torch.bfloat16),
                     k_cache=torch.from_numpy(kc).to(torch.bfloat16),
                     v_cache=torch.from_numpy(vc).to(torch.bfloat16))
    for a, b in zip(all_at_once, (state["k_raw"], state["v_raw"], state["k_cache"], state["v_cache"])):
        assert np.array_equal(a, b.float().numpy())


def test_kv_write_e4m3_codes():
    """E4M3 codes: the fp32 sum divided by the scale, rounded (nearest even,
    saturating); decoding them returns the bf16-path value within half an
    E4M3 step (times the scale)."""
    c = _case([10, 3], T=3, seed=9)
    ks = torch.tensor([0.01, 0.02], dtype=torch.float32)
    vs = torch.tensor([0.015, 0.005], dtype=torch.float32)
    codes = dict(c, k_cache=torch.zeros(c["k_cache"].shape, dtype=torch.uint8),
                 v_cache=torch.zeros(c["v_cache"].shape, dtype=torch.uint8), k_scale=ks, v_scale=vs)
    _, _, kc8, vc8 = oracle.kv_write_ref(**codes)
    _, _, kc16, vc16 = oracle.kv_write_ref(**c)
    P = c["k_raw"].shape[2]
    for cache8, cache16, sc in ((kc8, kc16, ks), (vc8, vc16, vs)):
        for b, L in enumerate(c["seq_lens"].tolist()):
            for p in range(L - 3, L):
                pg = int(c["block_table"][b, p // P])
                for h in range(2):
                    dec = oracle.e4m3_to_float(cache8[pg, h, p % P]) * float(sc[h])
                    ref = cache16[pg, h, p % P]
                    step = np.maximum(np.abs(ref), 2.0 ** -6 * float(sc[h])) * 2.0 ** -3
                    assert np.all(np.abs(dec - np.clip(ref, -448 * float(sc[h]), 448 * float(sc[h])))
                                  <= step / 2 + 1e-2 * step)
