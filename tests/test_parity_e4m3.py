"""GPU parity of the E4M3 (FP8) KV-cache path against the fp64 oracle.

The oracle dequantises the codes exactly (code value x per-KV-head scale) and
applies the definition.  Up to three query tokens: the FP8 kernel runs the
codes through E4M3 tensor-core MMAs, with the query split into two E4M3
terms and P into three (several tokens as one-token chunks of one launch).
Four and more: the multi-token kernel widens the codes to bf16 in shared
memory (exactly) and folds the scales into the logit multiplier and the
final normalisation.  Same tolerances as the bf16 path: max |out_fp32 -
oracle| <= 2e-3, max |lse - oracle| <= 1e-3.
"""

import numpy as np
import pytest
import torch

import oracle
from relative_bias_gqa_b200 import workloads as W

pytestmark = pytest.mark.gpu

OUT_TOL = 2e-3
LSE_TOL = 1e-3


@pytest.fixture(scope="module")
def ra():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from relative_bias_gqa_b200 import rel_attn
    return rel_attn


def e4m3(case):
    kc, vc, ks, vs = W.to_e4m3(case)
    return kc, vc, ks, vs


def run_gpu(ra, case, codes, num_splits=0, out_fp32=True):
    kc, vc, ks, vs = codes
    out, lse = ra.rel_attn_decode_e4m3(case.q, kc, vc, ks, vs, case.block_table, case.seq_lens,
                                       case.rel_table, case.window, num_splits,
                                       max_seq_len=case.max_seq_len, out_fp32=out_fp32,
                                       exact_buckets=case.exact_buckets,
                                       max_distance=case.max_distance)
    torch.cuda.synchronize()
    return out, lse


def run_oracle(case, codes):
    kc, vc, ks, vs = codes
    return oracle.rel_attn_decode_fp8kv_ref(case.q, kc, vc, ks, vs, case.block_table,
                                            case.seq_lens, case.rel_table, case.window,
                                            exact_buckets=case.exact_buckets,
                                            max_distance=case.max_distance)


def check(out, lse, ref_out, ref_lse):
    o = out.float().cpu().numpy().astype(np.float64)
    l = lse.cpu().numpy().astype(np.float64)
    assert np.isfinite(o).all() and np.isfinite(l).all()
    eo = np.abs(o - ref_out).max()
    el = np.abs(l - ref_lse).max()
    assert eo <= OUT_TOL and el <= LSE_TOL, (eo, el)


def small(L, window=0, NB=1280, seed=0, Hkv=2, lens=None, G=6, T=1, **kw):
    lens = lens if lens is not None else [L]
    return W.make_case(seq_lens=lens, q_tokens=T, num_q_heads=G * Hkv, num_kv_heads=Hkv,
                       window=window, num_buckets=NB, seed=seed, extra_pages=2, **kw).to("cuda")


SMALL = [
    dict(L=1), dict(L=63), dict(L=64), dict(L=65), dict(L=127), dict(L=128), dict(L=129),
    dict(L=300), dict(L=1000), dict(L=3001), dict(L=5000, seed=3),
    dict(L=1500, window=1), dict(L=1500, window=64), dict(L=2500, window=1024),
    dict(L=900, NB=8), dict(L=2000, NB=1030), dict(L=200, window=1024, NB=1024),
    dict(L=6000, NB=364, exact_buckets=64, max_distance=5000),
    # the previous Inkling's group sizes
    dict(L=1, G=4), dict(L=129, G=4), dict(L=3001, G=4), dict(L=2500, G=4, window=512, NB=1024),
    dict(L=1, G=8), dict(L=129, G=8), dict(L=3001, G=8), dict(L=5000, G=8, seed=5),
]


@pytest.mark.parametrize("kw", SMALL, ids=[str(k) for k in SMALL])
@pytest.mark.parametrize("splits", [1, 3, 0])
def test_small_cases(ra, kw, splits):
    case = small(**kw)
    codes = e4m3(case)
    check(*run_gpu(ra, case, codes, splits), *run_oracle(case, codes))


def test_batched_mixed_lengths(ra):
    case = small(0, Hkv=3, lens=[5, 64, 65, 300, 1111, 2049, 129, 2])
    codes = e4m3(case)
    ref = run_oracle(case, codes)
    for splits in (1, 2, 5, 0):
        check(*run_gpu(ra, case, codes, splits), *ref)


def test_split_count_invariance(ra):
    case = small(20000)
    codes = e4m3(case)
    ref = run_oracle(case, codes)
    for s in (1, 2, 3, 5, 8, 13, 18, 37, 64, 157):
        check(*run_gpu(ra, case, codes, s), *ref)


@pytest.mark.parametrize("T", [1, 8])
def test_bf16_output_is_rounded_fp32(ra, T):
    """bf16 output is the fp32 output rounded (one token: the FP8 kernel;
    eight: the widened multi-token kernel)."""
    case = small(2600, T=T)
    codes = e4m3(case)
    for splits in (1, 4):
        o32, l32 = run_gpu(ra, case, codes, splits, out_fp32=True)
        o16, l16 = run_gpu(ra, case, codes, splits, out_fp32=False)
        assert torch.equal(o32.to(torch.bfloat16), o16)
        assert torch.equal(l32, l16)


def test_nan_codes_in_unseen_slots_do_not_matter(ra):
    """E4M3 NaN codes (0x7F) in every cache slot no query can see."""
    for kw in (dict(L=3001), dict(L=2500, window=1024, NB=1024), dict(L=1500, window=100)):
        case = small(**kw)
        kc, vc, ks, vs = e4m3(case)
        ref = run_oracle(case, (kc, vc, ks, vs))
        L = int(case.seq_lens[0])
        lo = max(0, L - 1 - case.window + 1) if case.window > 0 else 0
        seen = torch.zeros(kc.shape[0], kc.shape[2], dtype=torch.bool)
        bt = case.block_table[0].cpu()
        for j in range(lo, L):
            seen[int(bt[j // 64]), j % 64] = True
        mask = (~seen).to(kc.device)[:, None, :, None].expand_as(kc)
        kp, vp = kc.clone(), vc.clone()
        kp[mask] = 0x7F
        vp[mask] = 0x7F
        for splits in (1, 4):
            clean = run_gpu(ra, case, (kc, vc, ks, vs), splits)
            bad = run_gpu(ra, case, (kp, vp, ks, vs), splits)
            assert torch.equal(clean[0], bad[0]) and torch.equal(clean[1], bad[1])
            check(*bad, *ref)


@pytest.mark.parametrize("T", [1, 8])
def test_scales_are_per_kv_head(ra, T):
    """Distinct scales per head: doubling head 1's V scale doubles only its rows
    (one token, and eight through the widened multi-token kernel)."""
    case = small(3000, T=T)
    kc, vc, ks, vs = e4m3(case)
    o1, l1 = run_gpu(ra, case, (kc, vc, ks, vs), 3)
    vs2 = vs.clone()
    vs2[1] *= 2
    o2, l2 = run_gpu(ra, case, (kc, vc, ks, vs2), 3)
    assert torch.equal(o1[:, :, :6], o2[:, :, :6])
    assert torch.allclose(o2[:, :, 6:], 2 * o1[:, :, 6:], rtol=1e-6, atol=0)
    check(o2, l2, *run_oracle(case, (kc, vc, ks, vs2)))
    assert torch.equal(l1, l2)


def test_full_100k(ra):
    case = W.make_workload("full_100k", seed=0, device="cuda")
    codes = e4m3(case)
    ref = run_oracle(case, codes)
    for s in (1, 7, 18, 37, 148, 0):
        check(*run_gpu(ra, case, codes, s), *ref)


def test_sliding_100k(ra):
    case = W.make_workload("sliding_100k", seed=1, device="cuda")
    codes = e4m3(case)
    ref = run_oracle(case, codes)
    for s in (1, 4, 0):
        check(*run_gpu(ra, case, codes, s), *ref)


def test_one_hot_key_probe(ra):
    """One key dominates its row (P = 1 there, tiny elsewhere): the hardest
    case for the three-term split of P, whose largest term then carries
    almost all of the output."""
    for j_star in (0, 64, 500, 999):
        case = small(1000, Hkv=1)
        case.rel_table.zero_()
        q = case.q[0, 0, 0].float()
        pg = int(case.block_table[0, j_star // 64])
        case.k_cache[pg, 0, j_star % 64] = (q * (40.0 / q.norm())).to(torch.bfloat16)
        codes = e4m3(case)
        check(*run_gpu(ra, case, codes, 0), *run_oracle(case, codes))


def test_query_magnitudes(ra):
    """Query rows of very different scales (1e-3 .. 30) and a row with tiny
    elements among large ones: the per-row power of two and the two-term
    E4M3 split of the query keep q . k exact."""
    case = small(2000, Hkv=2)
    g = torch.Generator(device="cuda").manual_seed(7)
    scale = torch.tensor([1e-3, 0.05, 1.0, 3.0, 30.0, 0.3] * 2, device="cuda")
    case.q.copy_((case.q.float() * scale[None, None, :, None]).to(torch.bfloat16))
    case.q[0, 0, 3, ::2] = (torch.randn(64, generator=g, device="cuda") * 1e-4).to(torch.bfloat16)
    codes = e4m3(case)
    check(*run_gpu(ra, case, codes, 3), *run_oracle(case, codes))


@pytest.mark.parametrize("name", ["v1_full_100k"])
def test_previous_model_full_layer(ra, name):
    case = W.make_workload(name, seed=0, device="cuda")
    codes = e4m3(case)
    ref = run_oracle(case, codes)
    for s in (1, 18, 0):
        check(*run_gpu(ra, case, codes, s), *ref)


@pytest.mark.parametrize("T", [1, 8])
def test_injected_wait_limit_times_out_cleanly(ra, T):
    """As for the bf16 kernel: a 1 ns wait bound makes the E4M3 kernels abort
    promptly with TIMEOUT and NaN rows (one token: the FP8 kernel; eight: the
    widened multi-token kernel, whose softmax warps also wait for K copies);
    the default bound then works again."""
    import time
    case = W.make_workload("full_100k", seed=4, device="cuda", num_q_heads=12, num_kv_heads=2,
                           q_tokens=T)
    codes = e4m3(case)
    shape = ra.shape_of(case.q, codes[0], case.block_table, case.rel_table,
                        max_seq_len=case.max_seq_len, out_fp32=True)
    ws = ra.Workspace.for_shape(shape, 0, "cuda")
    kc, vc, ks, vs = codes
    call = lambda: ra.rel_attn_decode_e4m3(case.q, kc, vc, ks, vs, case.block_table, case.seq_lens,
                                           case.rel_table, 0, 0, workspace=ws,
                                           max_seq_len=case.max_seq_len, out_fp32=True)
    call()
    torch.cuda.synchronize()
    assert ws.read_status() == ra.REL_ATTN_OK
    try:
        ra.rel_attn_set_wait_limit(1)
        t0 = time.perf_counter()
        out, lse = call()
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
    finally:
        ra.rel_attn_set_wait_limit(0)
    assert elapsed < 1.0
    assert ws.read_status() == ra.REL_ATTN_ERR_TIMEOUT
    assert torch.isnan(out).any()
    out, lse = call()
    torch.cuda.synchronize()
    check(out, lse, *run_oracle(case, codes))
    assert ws.read_status() == ra.REL_ATTN_OK


MULTI = [
    dict(T=2, L=2), dict(T=2, L=129), dict(T=2, L=3001),
    dict(T=5, L=5), dict(T=5, L=700, window=64),
    dict(T=8, L=8), dict(T=8, L=130), dict(T=8, L=4000, seed=2), dict(T=8, L=2500, window=1024),
    dict(T=9, L=9), dict(T=9, L=3001),
    dict(T=9, L=1700, G=4, window=512, NB=1024), dict(T=6, L=2100, G=4),
    dict(T=8, L=3001, G=8), dict(T=3, L=129, G=8),
    dict(T=4, L=6000, NB=364, exact_buckets=64, max_distance=5000),
]


@pytest.mark.parametrize("kw", MULTI, ids=[str(k) for k in MULTI])
@pytest.mark.parametrize("splits", [1, 3, 0])
def test_several_query_tokens(ra, kw, splits):
    """A verify step over the E4M3 cache: token t of T sees the keys up to
    position L - T + t."""
    case = small(**kw)
    codes = e4m3(case)
    out, lse = run_gpu(ra, case, codes, splits)
    ref_out, ref_lse = run_oracle(case, codes)
    check(out, lse, ref_out, ref_lse)


@pytest.mark.parametrize("T", [3, 6])
def test_several_query_tokens_batched(ra, T):
    """Mixed lengths in one batch: three tokens (one-token chunks) and six
    (codes widened in shared memory)."""
    case = small(0, lens=[9, 130, 2049, 700], T=T, seed=4)
    codes = e4m3(case)
    out, lse = run_gpu(ra, case, codes, 0)
    ref_out, ref_lse = run_oracle(case, codes)
    check(out, lse, ref_out, ref_lse)


def test_verify_256k_eight_tokens_one_kv_head(ra):
    """The verify shape at full length (262,144 keys, 8 tokens) on one KV
    head: the oracle computes all 6 x 8 rows."""
    case = small(262_144, T=8, Hkv=1, seed=7)
    codes = e4m3(case)
    out, lse = run_gpu(ra, case, codes, 0)
    ref_out, ref_lse = run_oracle(case, codes)
    check(out, lse, ref_out, ref_lse)


def test_previous_model_full_layer_eight_tokens_one_kv_head(ra):
    """The 64/8 full-attention layer (G = 8) at 100K keys with an 8-token
    verify over E4M3, one KV head: the widened 64-wide four-group instance
    at full size against the oracle's 8 x 8 rows."""
    case = small(100_000, T=8, G=8, Hkv=1, seed=11)
    codes = e4m3(case)
    out, lse = run_gpu(ra, case, codes, 0)
    ref_out, ref_lse = run_oracle(case, codes)
    check(out, lse, ref_out, ref_lse)


def _all_finite_codes(shape, gen):
    """Uniform E4M3 codes over the 254 finite ones (0x7f and 0xff are NaN):
    subnormal codes (exponent field 0) and both zeros included."""
    c = torch.randint(0, 254, shape, generator=gen, dtype=torch.int16)
    c = c + (c >= 0x7F).to(torch.int16)
    return c.to(torch.uint8)


@pytest.mark.parametrize("kw", [dict(T=6, L=3001), dict(T=5, L=700, window=64, G=8),
                                dict(T=8, L=4000, seed=2), dict(T=9, L=1700, G=4, window=512, NB=1024),
                                dict(T=6, L=2500, G=8), dict(T=8, L=130, G=8)],
                         ids=lambda k: str(k))
def test_several_query_tokens_equal_bf16_on_the_decoded_codes(ra, kw):
    """With unit scales a multi-token E4M3 call equals, bit for bit, the bf16
    call on the codes' values (every E4M3 value is a bf16 value) wherever
    both use the same softmax-group layout (six tokens and more, five at
    G = 8): the kernel widens the codes to bf16 in shared memory and then
    runs the bf16 arithmetic.  (At four tokens, and five for G <= 6, the E4M3
    instances split the rows over four groups instead of two; the lazy
    reference max is then moved per group of rows, so results agree to
    rounding: the oracle tests cover them.)  Every finite code occurs, subnormal ones included; one
    split, so that both calls walk the same pages."""
    case = small(**kw)
    gen = torch.Generator().manual_seed(11)
    kc = _all_finite_codes(case.k_cache.shape, gen).to("cuda")
    vc = _all_finite_codes(case.v_cache.shape, gen).to("cuda")
    ones = torch.ones(case.k_cache.shape[1], dtype=torch.float32, device="cuda")
    out8, lse8 = run_gpu(ra, case, (kc, vc, ones, ones), 1)
    kb = kc.view(torch.float8_e4m3fn).to(torch.bfloat16)
    vb = vc.view(torch.float8_e4m3fn).to(torch.bfloat16)
    out16, lse16 = ra.rel_attn_decode(case.q, kb, vb, case.block_table, case.seq_lens,
                                      case.rel_table, case.window, 1, max_seq_len=case.max_seq_len,
                                      out_fp32=True, exact_buckets=case.exact_buckets,
                                      max_distance=case.max_distance)
    torch.cuda.synchronize()
    assert torch.isfinite(out8).all()
    assert torch.equal(out8, out16) and torch.equal(lse8, lse16)


def test_several_query_tokens_nan_codes_in_unseen_slots_do_not_matter(ra):
    """Several tokens over E4M3 NaN codes in every slot no query sees (the
    widened path and the one-token chunks)."""
    for kw in (dict(L=3001, T=8), dict(L=2500, T=4, window=1024, NB=1024), dict(L=3001, T=3)):
        case = small(**kw)
        kc, vc, ks, vs = e4m3(case)
        ref = run_oracle(case, (kc, vc, ks, vs))
        L, T = int(case.seq_lens[0]), kw["T"]
        lo = max(0, L - T - case.window + 1) if case.window > 0 else 0
        seen = torch.zeros(kc.shape[0], kc.shape[2], dtype=torch.bool)
        bt = case.block_table[0].cpu()
        for j in range(lo, L):
            seen[int(bt[j // 64]), j % 64] = True
        mask = (~seen).to(kc.device)[:, None, :, None].expand_as(kc)
        kp, vp = kc.clone(), vc.clone()
        kp[mask] = 0x7F
        vp[mask] = 0xFF
        for splits in (1, 4):
            clean = run_gpu(ra, case, (kc, vc, ks, vs), splits)
            bad = run_gpu(ra, case, (kp, vp, ks, vs), splits)
            assert torch.equal(clean[0], bad[0]) and torch.equal(clean[1], bad[1])
            check(*bad, *ref)


def test_up_to_three_tokens_match_one_token_calls(ra):
    """Up to three tokens run as one-token chunks of one launch: token t of
    a T-token call equals a one-token call whose sequence ends at that token
    (same splits: the same chunks, bit for bit)."""
    T, L = 3, 3001
    case = small(L, T=T, seed=9)
    codes = e4m3(case)
    out, lse = run_gpu(ra, case, codes, 3)
    for t in range(T):
        one = W.make_case(seq_lens=[L - T + t + 1], q_tokens=1, num_q_heads=12, num_kv_heads=2,
                          num_buckets=1280, seed=9, extra_pages=2).to("cuda")
        one.q.copy_(case.q[:, t:t + 1])
        one.block_table.copy_(case.block_table[:, :one.block_table.shape[1]])
        kc, vc, ks, vs = codes
        o1, l1 = ra.rel_attn_decode_e4m3(one.q, kc, vc, ks, vs, one.block_table, one.seq_lens,
                                         case.rel_table, 0, 3, max_seq_len=L, out_fp32=True)
        torch.cuda.synchronize()
        assert torch.equal(o1[:, 0], out[:, t]) and torch.equal(l1[:, 0], lse[:, t]), t


def test_rejects_missing_scales(ra):
    import ctypes
    one = small(300)
    kc, vc, ks, vs = e4m3(one)
    shape = ra.shape_of(one.q, kc, one.block_table, one.rel_table, max_seq_len=300)
    ws = ra.Workspace.for_shape(shape, 1, one.q.device)
    out = torch.empty_like(one.q)
    rc = ra.lib.rel_attn_decode_e4m3(ctypes.byref(shape), one.q.data_ptr(), kc.data_ptr(),
                                     vc.data_ptr(), None, vs.data_ptr(), one.block_table.data_ptr(),
                                     one.seq_lens.data_ptr(), one.rel_table.data_ptr(), 0, 1,
                                     out.data_ptr(), None, ws.buf.data_ptr(), ws.nbytes, None)
    assert rc == ra.REL_ATTN_ERR_INVALID_ARG
