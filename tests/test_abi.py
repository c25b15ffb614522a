"""C-ABI checks that need no GPU: the library loads, exports every entry point
the header declares, validates arguments before touching CUDA, and its host
copy of the bucket table (the one handed to the kernels) equals the oracle's
bucket function bit for bit."""

import ctypes
import os
import re

import numpy as np
import pytest
import torch

from relative_bias_gqa_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def ra():
    build_mod.build()
    from relative_bias_gqa_b200 import rel_attn
    return rel_attn


def header_functions():
    txt = open(os.path.join(ROOT, "include", "rel_attn.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(rel_attn_\w+)\s*\(", txt)))


def test_exports_every_declared_symbol(ra):
    names = header_functions()
    assert set(names) == set(ra.EXPORTED)
    lib = ctypes.CDLL(build_mod.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert "sm_100a" in ra.version()


def shape(ra, **kw):
    base = dict(batch=1, q_tokens=1, num_q_heads=48, num_kv_heads=8, num_pages=1563,
                max_pages_per_seq=1563, num_buckets=1280, max_seq_len=100_000)
    base.update(kw)
    return ra.make_shape(**base)


@pytest.mark.parametrize("nb", [1280, 1024, 1030, 8, 1])
def test_host_bucket_table_matches_oracle(ra, nb):
    import oracle
    s = shape(ra, num_buckets=nb)
    d = np.concatenate([np.arange(0, 70_000), np.arange(70_000, 1 << 21, 7),
                        [(1 << 20) - 1, 1 << 20, (1 << 20) + 1, 5 << 20]])
    want = oracle.bucket_of_distance(d, nb)
    f = ra.lib.rel_attn_bucket
    got = np.array([f(ctypes.byref(s), int(x)) for x in d])
    assert np.array_equal(got, want)
    assert f(ctypes.byref(s), -1) == -1


def test_host_bucket_every_distance_nb1280(ra):
    import oracle
    s = shape(ra)
    e = oracle.log_bucket_edges(1280)
    # every edge and its neighbours
    d = np.unique(np.concatenate([e - 1, e, e + 1]))
    d = d[d >= 0]
    got = np.array([ra.rel_attn_bucket(s, int(x)) for x in d])
    assert np.array_equal(got, oracle.bucket_of_distance(d, 1280))


# (NB, E, Dmax) triples: the standard tables, the geometries the GPU parity
# tests run, dense tables where consecutive edges repeat, and extremes of the
# integer ranges.  Exact powers (E * (Dmax/E)^(k/NL) an integer) must not
# round up: 1024 * 2^(10k/256) is an integer at k = 0, 128, 256.
EDGE_TRIPLES = [
    (1280, 1024, 1 << 20), (1030, 1024, 1 << 20), (1536, 1024, 1 << 20),
    (364, 64, 5000), (200, 16, 100000), (600, 100, 1500), (1024 + 512, 1024, (1 << 31) - 1),
    (513, 1, (1 << 31) - 1), (1100, 1000, 1000 * 3 ** 4), (1088, 1024, 1 << 30),
]


@pytest.mark.parametrize("nb,e,dmax", EDGE_TRIPLES, ids=[str(t) for t in EDGE_TRIPLES])
def test_host_edges_exact_for_other_geometries(ra, nb, e, dmax):
    """The library's edge table (long double, settled by exact integer
    comparison near integers) equals the oracle's exact-integer edges: each
    edge, and the distances one either side, get the same bucket."""
    import oracle
    s = shape(ra, num_buckets=nb, exact_buckets=e, max_distance=dmax)
    edges = oracle.log_bucket_edges(nb, e, dmax)
    d = np.unique(np.concatenate([edges - 1, edges, edges + 1, np.arange(0, min(e + 10, 4000)),
                                  [dmax - 1, dmax, dmax + 1]]))
    d = d[(d >= 0) & (d < (1 << 31) - 1)]
    want = oracle.bucket_of_distance(d, nb, e, dmax)
    got = np.array([ra.rel_attn_bucket(s, int(x)) for x in d])
    assert np.array_equal(got, want)


BAD = [
    dict(q_tokens=0), dict(q_tokens=10), dict(head_dim=64), dict(page_size=16),
    dict(num_q_heads=47), dict(num_q_heads=24), dict(num_q_heads=40), dict(num_q_heads=56),
    dict(num_q_heads=80), dict(num_q_heads=64, q_tokens=9),
    dict(num_kv_heads=0), dict(batch=0),
    dict(num_buckets=0), dict(num_buckets=1024 + 513), dict(num_pages=0),
    dict(max_pages_per_seq=0), dict(out_fp32=2), dict(max_seq_len=-1),
    dict(num_pages=1 << 23),
]


@pytest.mark.parametrize("kw", BAD)
def test_invalid_shape_rejected_before_any_cuda_call(ra, kw):
    s = shape(ra, **kw)
    fake = ctypes.c_void_p(1 << 20)       # never dereferenced: validation fails first
    rc = ra.lib.rel_attn_decode(ctypes.byref(s), fake, fake, fake, fake, fake, fake, 0, 0,
                                fake, None, fake, 1 << 30, None)
    assert rc == ra.REL_ATTN_ERR_INVALID_ARG
    assert ra.rel_attn_workspace_bytes(s, 4) == 0


# Group sizes with instances: 48/8 (G = 6), the previous Inkling's 64/8 full
# (G = 8, up to 8 tokens: 8 x 8 rows fill the 64 query slots) and 64/16
# sliding (G = 4) layers; nine tokens for G = 4 and 6.
GOOD = [dict(num_q_heads=48, num_kv_heads=8, q_tokens=t) for t in range(1, 10)] + \
       [dict(num_q_heads=64, num_kv_heads=8, q_tokens=t) for t in range(1, 9)] + \
       [dict(num_q_heads=64, num_kv_heads=16, q_tokens=t) for t in range(1, 10)]


@pytest.mark.parametrize("kw", GOOD, ids=[f"{k['num_q_heads']}/{k['num_kv_heads']}-T{k['q_tokens']}" for k in GOOD])
def test_supported_group_shapes(ra, kw):
    s = shape(ra, **kw)
    rows = kw["q_tokens"] * kw["num_q_heads"]
    assert ra.rel_attn_workspace_bytes(s, 3) == 256 + (3 * rows * 4 + 255) // 256 * 256 + 3 * rows * 128 * 4


@pytest.mark.parametrize("kw", [dict(num_q_heads=40, num_kv_heads=8, q_tokens=1),   # G = 5
                                dict(num_q_heads=64, num_kv_heads=8, q_tokens=9),   # 72 rows
                                dict(num_q_heads=48, num_kv_heads=8, q_tokens=10)])
def test_e4m3_rejects_unsupported_shapes(ra, kw):
    s = shape(ra, **kw)
    fake = ctypes.c_void_p(1 << 20)       # never dereferenced: validation fails first
    rc = ra.lib.rel_attn_decode_e4m3(ctypes.byref(s), fake, fake, fake, fake, fake, fake, fake,
                                     fake, 0, 1, fake, None, fake, 1 << 30, None)
    assert rc == ra.REL_ATTN_ERR_INVALID_ARG


def test_e4m3_needs_both_scales(ra):
    s = shape(ra, num_q_heads=48, num_kv_heads=8, q_tokens=8)
    fake = ctypes.c_void_p(1 << 20)       # never dereferenced: validation fails first
    for ks, vs in ((None, fake), (fake, None)):
        rc = ra.lib.rel_attn_decode_e4m3(ctypes.byref(s), fake, fake, fake, ks, vs, fake, fake,
                                         fake, 0, 1, fake, None, fake, 1 << 30, None)
        assert rc == ra.REL_ATTN_ERR_INVALID_ARG


def test_invalid_pointers_and_splits(ra):
    s = shape(ra)
    f = ctypes.c_void_p(1 << 20)
    call = ra.lib.rel_attn_decode
    assert call(ctypes.byref(s), None, f, f, f, f, f, 0, 0, f, None, f, 1 << 30, None) == ra.REL_ATTN_ERR_INVALID_ARG
    assert call(ctypes.byref(s), f, f, f, f, f, f, 0, 257, f, None, f, 1 << 30, None) == ra.REL_ATTN_ERR_INVALID_ARG
    odd = ctypes.c_void_p((1 << 20) + 8)
    assert call(ctypes.byref(s), odd, f, f, f, f, f, 0, 0, f, None, f, 1 << 30, None) == ra.REL_ATTN_ERR_INVALID_ARG
    assert call(ctypes.byref(s), f, f, f, f, f, f, 0, 0, f, None, odd, 1 << 30, None) == ra.REL_ATTN_ERR_INVALID_ARG
    assert call(ctypes.byref(s), f, f, f, f, f, f, 0, 0, f, None, f, 16, None) == ra.REL_ATTN_ERR_WORKSPACE_TOO_SMALL
    assert call(None, f, f, f, f, f, f, 0, 0, f, None, f, 1 << 30, None) == ra.REL_ATTN_ERR_INVALID_ARG


def test_split_heuristic_values(ra):
    # 148 SMs: batch-1 48/8 fills one wave with 18 splits per KV head
    assert ra.rel_attn_choose_splits(shape(ra), 0, 148) == 18
    # a sliding window of 1,024 has 9 tiles: never more splits than tiles
    assert ra.rel_attn_choose_splits(shape(ra), 1024, 148) == 9
    # small contexts: at most one split per 128-key tile
    assert ra.rel_attn_choose_splits(shape(ra, max_seq_len=300), 0, 148) == 3
    # 32 sequences x 8 heads > 148 SMs: about twelve CTAs per SM in all
    s = shape(ra, batch=32, max_seq_len=131_072, max_pages_per_seq=2048, num_pages=40000)
    assert ra.rel_attn_choose_splits(s, 0, 148) == 7         # ceil(12 * 148 / 256)
    # many units: one split each
    s = shape(ra, batch=2048, max_seq_len=131_072, max_pages_per_seq=2048, num_pages=40000)
    assert ra.rel_attn_choose_splits(s, 0, 148) == 1
    for sm in (1, 7, 148, 1000):
        assert 1 <= ra.rel_attn_choose_splits(shape(ra), 0, sm) <= 256
    # the previous Inkling's layers: 64/8 full behaves like 48/8 (8 KV heads);
    # 64/16 sliding has 16 units per split and a 512-key window (5 tiles)
    assert ra.rel_attn_choose_splits(shape(ra, num_q_heads=64), 0, 148) == 18
    assert ra.rel_attn_choose_splits(shape(ra, num_q_heads=64, num_kv_heads=16), 0, 148) == 9
    assert ra.rel_attn_choose_splits(shape(ra, num_q_heads=64, num_kv_heads=16), 512, 148) == 5


def test_workspace_bytes(ra):
    s = shape(ra)
    assert ra.rel_attn_workspace_bytes(s, 1) == 256
    rows = 48
    want = 256 + ((18 * rows * 4 + 255) // 256) * 256 + 18 * rows * 128 * 4
    assert ra.rel_attn_workspace_bytes(s, 18) == want
    assert ra.rel_attn_workspace_bytes(s, 256) > ra.rel_attn_workspace_bytes(s, 18)


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU error path")
def test_no_device_reported_without_gpu(ra):
    s = shape(ra)
    f = ctypes.c_void_p(1 << 20)
    rc = ra.lib.rel_attn_decode(ctypes.byref(s), f, f, f, f, f, f, 0, 4, f, None, f, 1 << 30, None)
    assert rc == ra.REL_ATTN_ERR_NO_DEVICE


def test_error_strings(ra):
    for code in range(-6, 1):
        assert ra.error_string(code) and ra.error_string(code) != "unknown error"


@pytest.mark.parametrize("L,T,window,nb", [(100_000, 1, 0, 1280), (262_144, 8, 0, 1280),
                                            (100_000, 1, 1024, 1024), (20_000, 3, 0, 1280),
                                            (5, 1, 0, 1280), (2048, 2, 100, 364)])
@pytest.mark.parametrize("e4m3", [False, True])
def test_split_pages_partition(ra, L, T, window, nb, e4m3):
    """Every split count gives contiguous, ordered page ranges that cover
    exactly the pages some query can see, tiles stay two pages long inside,
    and near-query splits are no longer than far ones."""
    pages = (L + 63) // 64 + 1
    s = shape(ra, q_tokens=T, num_buckets=nb, max_pages_per_seq=pages, num_pages=pages,
              max_seq_len=L, exact_buckets=min(1024, nb) if nb <= 1024 else 1024)
    lo = max(0, L - T - window + 1) if window > 0 else 0
    first, last = lo // 64, (L - 1) // 64
    for S in (1, 2, 3, 7, 18, 37, 64, 148, 256):
        prev = first
        sizes = []
        for sp in range(S):
            a, b = ra.rel_attn_split_pages(s, L, window, S, sp, e4m3=e4m3)
            assert a == prev and b >= a
            assert (a - first) % 2 == 0 or a == last + 1      # inner boundaries keep 2-page tiles
            sizes.append(b - a)
            prev = b
        assert prev == last + 1
        big = [x for x in sizes if x > 0]
        if len(big) > 2:
            assert big[-1] <= max(big[:-1])


@pytest.mark.parametrize("name", ["rel_attn_split_pages", "rel_attn_split_pages_e4m3"])
def test_split_pages_rejects_bad_arguments(ra, name):
    s = shape(ra)
    import ctypes
    a, b = ctypes.c_int(), ctypes.c_int()
    f = getattr(ra.lib, name)
    assert f(ctypes.byref(s), 100, 0, 4, 4, ctypes.byref(a), ctypes.byref(b)) == ra.REL_ATTN_ERR_INVALID_ARG
    assert f(ctypes.byref(s), 100, 0, 0, 0, ctypes.byref(a), ctypes.byref(b)) == ra.REL_ATTN_ERR_INVALID_ARG
    assert f(ctypes.byref(s), 0, 0, 4, 0, ctypes.byref(a), ctypes.byref(b)) == ra.REL_ATTN_ERR_INVALID_ARG
    assert f(ctypes.byref(s), 1 << 30, 0, 4, 0, ctypes.byref(a), ctypes.byref(b)) == ra.REL_ATTN_ERR_INVALID_ARG
    assert f(ctypes.byref(s), 100, 0, 4, 0, None, ctypes.byref(b)) == ra.REL_ATTN_ERR_INVALID_ARG


def test_e4m3_partition_gives_the_exact_range_fewer_pages(ra):
    """The E4M3 weights put fewer pages in the split nearest the queries
    (its tiles carry a relative-row chunk twice their K/V bytes)."""
    L = 100_000
    pages = (L + 63) // 64 + 1
    s = shape(ra, q_tokens=1, num_buckets=1280, max_pages_per_seq=pages, num_pages=pages,
              max_seq_len=L, exact_buckets=1024)
    a16, b16 = ra.rel_attn_split_pages(s, L, 0, 18, 17)
    a8, b8 = ra.rel_attn_split_pages(s, L, 0, 18, 17, e4m3=True)
    assert b16 == b8 == (L - 1) // 64 + 1
    assert b8 - a8 < b16 - a16


def _span_oracle(nb, e, dmax, T):
    """Largest number of bucket indices that 127 + T consecutive distances
    span, from the oracle's bucket function (bucket() is non-decreasing, so
    windows starting where a bucket starts suffice)."""
    import oracle
    edges = oracle.log_bucket_edges(nb, e, dmax) if nb > e else np.array([], dtype=np.int64)
    starts = np.unique(np.concatenate([np.arange(0, e + 1), edges])).astype(np.int64)
    starts = starts[starts < (1 << 31) - 200]
    b0 = oracle.bucket_of_distance(starts, nb, e, dmax)
    b1 = oracle.bucket_of_distance(starts + 126 + T, nb, e, dmax)
    return int((b1 - b0 + 1).max())


@pytest.mark.parametrize("nb,e,dmax", EDGE_TRIPLES + [(600, 100, 8000), (350, 100, 1500)],
                         ids=[str(t) for t in EDGE_TRIPLES + [(600, 100, 8000), (350, 100, 1500)]])
@pytest.mark.parametrize("T", [1, 2, 8])
def test_bucket_tables_too_dense_for_a_chunk_are_rejected(ra, nb, e, dmax, T):
    """A tile's 127 + T distances must span at most 128 bucket indices for
    one token (136 for several): one relative-row chunk then holds every
    bucket the tile needs.  Denser tables are refused before any CUDA call;
    the others pass validation (and fail later only for the fake pointers,
    with NO_DEVICE on a machine without a GPU)."""
    s = shape(ra, num_buckets=nb, exact_buckets=e, max_distance=dmax, q_tokens=T,
              num_q_heads=48, num_kv_heads=8)
    fake = ctypes.c_void_p(1 << 20)
    rc = ra.lib.rel_attn_decode(ctypes.byref(s), fake, fake, fake, fake, fake, fake, 0, 1, fake,
                                None, fake, 1 << 30, None)
    too_dense = _span_oracle(nb, e, dmax, T) > (128 if T == 1 else 136)
    if too_dense:
        assert rc == ra.REL_ATTN_ERR_INVALID_ARG
    elif not torch.cuda.is_available():
        assert rc == ra.REL_ATTN_ERR_NO_DEVICE


@pytest.mark.parametrize("nb,e,dmax", EDGE_TRIPLES + [(600, 100, 8000), (350, 100, 1500)],
                         ids=[str(t) for t in EDGE_TRIPLES + [(600, 100, 8000), (350, 100, 1500)]])
@pytest.mark.parametrize("T", [2, 3, 4, 8])
def test_e4m3_span_rule_follows_the_path(ra, nb, e, dmax, T):
    """Over an E4M3 cache up to three tokens run as one-token chunks (the
    one-token span rule applies), four and more through the multi-token
    kernel (the T-token rule)."""
    s = shape(ra, num_buckets=nb, exact_buckets=e, max_distance=dmax, q_tokens=T,
              num_q_heads=48, num_kv_heads=8)
    fake = ctypes.c_void_p(1 << 20)
    rc = ra.lib.rel_attn_decode_e4m3(ctypes.byref(s), fake, fake, fake, fake, fake, fake, fake,
                                     fake, 0, 1, fake, None, fake, 1 << 30, None)
    tt = 1 if T <= 3 else T
    too_dense = _span_oracle(nb, e, dmax, tt) > (128 if tt == 1 else 136)
    if too_dense:
        assert rc == ra.REL_ATTN_ERR_INVALID_ARG
    elif not torch.cuda.is_available():
        assert rc == ra.REL_ATTN_ERR_NO_DEVICE


def test_dense_table_in_the_edge_tests_is_too_dense(ra):
    assert _span_oracle(600, 100, 1500, 1) > 128 and _span_oracle(600, 100, 1500, 2) > 136
    assert _span_oracle(1280, 1024, 1 << 20, 1) == 128 and _span_oracle(1280, 1024, 1 << 20, 8) == 135
