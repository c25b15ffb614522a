"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Tolerances: max |out_fp32 - oracle| <= 2e-3, max |lse - oracle| <= 1e-3;
key selection (paging and masking) bit-exact.  bf16 outputs must equal the
round-to-nearest-even of the fp32 outputs.
"""

import math

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


def run_gpu(ra, case, num_splits=0, out_fp32=True, workspace=None):
    out, lse = ra.rel_attn_decode(case.q, case.k_cache, case.v_cache, case.block_table,
                                  case.seq_lens, case.rel_table, case.window, num_splits,
                                  workspace=workspace, max_seq_len=case.max_seq_len,
                                  out_fp32=out_fp32, exact_buckets=case.exact_buckets,
                                  max_distance=case.max_distance)
    torch.cuda.synchronize()
    return out, lse


def run_oracle(case, batch_indices=None):
    return oracle.rel_attn_decode_ref(case.q, case.k_cache, case.v_cache, case.block_table,
                                      case.seq_lens, case.rel_table, case.window,
                                      exact_buckets=case.exact_buckets,
                                      max_distance=case.max_distance,
                                      batch_indices=batch_indices)


def check(out, lse, ref_out, ref_lse, rows=None):
    o = out.float().cpu().numpy().astype(np.float64)
    l = lse.cpu().numpy().astype(np.float64)
    if rows is not None:
        o, l, ref_out, ref_lse = o[rows], l[rows], ref_out[rows], ref_lse[rows]
    assert np.isfinite(o).all() and np.isfinite(l).all()
    eo = np.abs(o - ref_out).max()
    el = np.abs(l - ref_lse).max()
    assert eo <= OUT_TOL and el <= LSE_TOL, (eo, el)
    return eo, el


def small(L, T=1, window=0, NB=1280, seed=0, Hkv=2, lens=None, **kw):
    lens = lens if lens is not None else [L]
    return W.make_case(seq_lens=lens, q_tokens=T, num_q_heads=6 * Hkv, num_kv_heads=Hkv,
                       window=window, num_buckets=NB, seed=seed, extra_pages=2, **kw).to("cuda")


# -------------------------------------------------------------- small shapes
SMALL = [
    dict(L=1), dict(L=63), dict(L=64), dict(L=65), dict(L=127), dict(L=128),
    dict(L=129), dict(L=300), dict(L=1000), dict(L=3001),
    dict(L=8, T=8), dict(L=9, T=8), dict(L=700, T=2), dict(L=1500, T=3),
    dict(L=2100, T=5), dict(L=4000, T=8), dict(L=777, T=7), dict(L=5000, T=6),
    dict(L=1500, window=1), dict(L=1500, window=64), dict(L=2500, window=1024),
    dict(L=2500, T=8, window=1024, NB=1024), dict(L=3000, T=4, window=100),
    dict(L=900, NB=8), dict(L=2000, NB=1030), dict(L=200, window=1024, NB=1024),
    # other bucket geometries: a short exact range with dense (repeated) tail
    # edges, and distances past max_distance clamped into the last bucket
    dict(L=6000, NB=364, exact_buckets=64, max_distance=5000),
    dict(L=3000, T=8, NB=200, exact_buckets=16, max_distance=100000),
    dict(L=2200, T=2, NB=600, exact_buckets=100, max_distance=1500),
]


@pytest.mark.parametrize("kw", SMALL, ids=[str(k) for k in SMALL])
@pytest.mark.parametrize("splits", [1, 3, 0])
def test_small_cases(ra, kw, splits):
    case = small(**kw)
    out, lse = run_gpu(ra, case, splits)
    check(out, lse, *run_oracle(case))


def test_batched_small_mixed_lengths(ra):
    case = small(0, T=2, Hkv=3, lens=[5, 64, 65, 300, 1111, 2049, 129, 2])
    for splits in (1, 2, 5, 0):
        out, lse = run_gpu(ra, case, splits)
        check(out, lse, *run_oracle(case))


def test_bf16_output_is_rounded_fp32(ra):
    case = small(2600, T=3)
    for splits in (1, 4):
        o32, l32 = run_gpu(ra, case, splits, out_fp32=True)
        o16, l16 = run_gpu(ra, case, splits, out_fp32=False)
        assert torch.equal(o32.to(torch.bfloat16), o16)
        assert torch.equal(l32, l16)


def test_split_count_invariance_long(ra):
    """Splits are cost-weighted toward the query end: with 313 pages every
    segment of the weighting (exact range, narrow tail buckets, far pages)
    falls inside some split for these counts."""
    case = small(20000, T=1)
    ref = run_oracle(case)
    for s in (2, 3, 5, 8, 13, 18, 37, 64, 150, 157):
        out, lse = run_gpu(ra, case, s)
        check(out, lse, *ref)


def test_split_count_invariance_small(ra):
    case = small(5000, T=1)
    ref = run_oracle(case)
    for s in list(range(1, 41)) + [64, 100, 255, 256]:
        out, lse = run_gpu(ra, case, s)
        check(out, lse, *ref)


# --------------------------------------------------- exact key-set identity
@pytest.mark.parametrize("T,window,L", [(1, 0, 1000), (3, 77, 1000), (8, 0, 333), (8, 1024, 3000),
                                         (1, 1024, 2500), (2, 5, 129)])
def test_key_set_identity_bit_exact(ra, T, window, L):
    """Q = 0 and R = 0 give uniform weights: exp(lse) is the number of keys a
    row selects and out * |J| counts, per bit c < 18, the selected positions
    with bit c set -- both integers that must match exactly."""
    case = small(L, T=T, window=window)
    case.q.zero_()
    case.rel_table.zero_()
    P = case.page_size
    pos = torch.arange(L, device="cuda")
    bits = ((pos[:, None] >> torch.arange(18, device="cuda")[None]) & 1).to(torch.bfloat16)
    vals = torch.zeros(L, 128, dtype=torch.bfloat16, device="cuda")
    vals[:, :18] = bits
    pages = case.block_table[0].long()[pos // P]
    for h in range(case.num_kv_heads):
        case.v_cache[pages, h, pos % P] = vals
    out, lse = run_gpu(ra, case, 0)
    for t in range(T):
        p = L - T + t
        J = [j for j in range(p + 1) if window <= 0 or p - j <= window - 1]
        cnt = torch.round(torch.exp(lse[0, t].double())).cpu()
        assert torch.all(cnt == len(J)), (t, cnt, len(J))
        want = torch.tensor([sum((j >> c) & 1 for j in J) for c in range(18)], dtype=torch.float64)
        got = torch.round(out[0, t, :, :18].double().cpu() * len(J))
        assert torch.all(got == want[None]), t


def test_poisoned_slots_do_not_matter(ra):
    for kw in (dict(L=3001, T=1, window=0), dict(L=2500, T=8, window=1024, NB=1024),
               dict(L=1500, T=3, window=100)):
        case = small(**kw)
        ref = run_oracle(case)
        for splits in (1, 4):
            clean = run_gpu(ra, case, splits)
            bad = run_gpu(ra, W.poison_unused(case), splits)
            assert torch.equal(clean[0], bad[0]) and torch.equal(clean[1], bad[1])
            check(*bad, *ref)


def test_one_hot_key_probe(ra):
    """A key aligned with a large multiple of q dominates its row: out ~= v_{j*}."""
    L = 1000
    for j_star in (0, 63, 64, 127, 128, 500, 998, 999):
        case = small(L, T=1, Hkv=1)
        case.rel_table.zero_()
        q = case.q[0, 0, 0].float()
        P = case.page_size
        pg = int(case.block_table[0, j_star // P])
        case.k_cache[pg, 0, j_star % P] = (q * (40.0 / q.norm())).to(torch.bfloat16)
        out, lse = run_gpu(ra, case, 0)
        ref_o, ref_l = run_oracle(case)
        check(out, lse, ref_o, ref_l)
        v = case.v_cache[pg, 0, j_star % P].float().cpu().numpy()
        assert np.abs(out[0, 0, 0].cpu().numpy() - v).max() < 5e-2


@pytest.mark.parametrize("target", [0, 7, 130, 1023, 1024, 1025, 1049, 1100, 1193, 1228])
def test_bucket_probe_counts(ra, target):
    """R row `target` holds a large value on one coordinate, q is one-hot there
    and K = 0: each row's mass sits on the keys whose distance falls in bucket
    `target`, so exp(lse - big) counts them exactly."""
    L = 262_144 if target >= 1193 else 20_000
    case = W.make_case(seq_lens=[L], q_tokens=1, num_q_heads=6, num_kv_heads=1,
                       window=0, num_buckets=1280, seed=1, device="cuda")
    case.k_cache.zero_()
    case.q.zero_()
    case.q[..., 0] = 8.0
    case.rel_table.zero_()
    case.rel_table[0, target, 0] = 16.0
    out, lse = run_gpu(ra, case, 0)
    check(out, lse, *run_oracle(case))
    big = 8.0 * 16.0 / math.sqrt(128)
    d = np.arange(L)
    n_target = int((oracle.bucket_of_distance(d, 1280) == target).sum())
    n_other = L - n_target
    want = big + math.log(n_target + n_other * math.exp(-big))
    assert abs(float(lse[0, 0, 0]) - want) < 2e-4, (target, float(lse[0, 0, 0]), want)


# ------------------------------------------------------ named workloads
def test_tiny_2k(ra):
    case = W.make_workload("tiny_2k", seed=0).to("cuda")
    ref = run_oracle(case)
    for splits in (1, 2, 7, 16, 0):
        check(*run_gpu(ra, case, splits), *ref)


def test_sliding_100k(ra):
    for seed in (0, 1):
        case = W.make_workload("sliding_100k", seed=seed, device="cuda")
        ref = run_oracle(case)
        for splits in (1, 4, 0):
            check(*run_gpu(ra, case, splits), *ref)


def test_full_100k_with_split_sweep(ra):
    case = W.make_workload("full_100k", seed=0, device="cuda")
    ref = run_oracle(case)
    for s in list(range(1, 65)) + [72, 96, 128, 148, 200, 255, 256, 0]:
        check(*run_gpu(ra, case, s), *ref)


def test_verify_t8_256k(ra):
    case = W.make_workload("verify_t8_256k", seed=0, device="cuda")
    ref = run_oracle(case)
    for splits in (1, 8, 0):
        check(*run_gpu(ra, case, splits), *ref)


def _sub_case(case, idx):
    """Compact copy holding only sequences `idx` (their pages, remapped)."""
    P = case.page_size
    rows, tables = [], []
    nxt = 0
    for b in idx:
        n = math.ceil(int(case.seq_lens[b]) / P)
        rows.append(case.block_table[b, :n].long())
        tables.append(torch.arange(nxt, nxt + n, dtype=torch.int32))
        nxt += n
    pages = torch.cat(rows)
    bt = torch.full((len(idx), case.block_table.shape[1]), -1, dtype=torch.int32)
    for i, t in enumerate(tables):
        bt[i, :len(t)] = t
    import dataclasses
    return dataclasses.replace(
        case, q=case.q[idx].cpu(), k_cache=case.k_cache[pages].cpu(),
        v_cache=case.v_cache[pages].cpu(), block_table=bt,
        seq_lens=case.seq_lens[idx].cpu(), rel_table=case.rel_table.cpu())


def test_batched_32_sampled(ra):
    case = W.make_workload("batched_32", seed=0, device="cuda")
    idx = [0, 5, 17, 31]
    sub = _sub_case(case, idx)
    ref_o, ref_l = run_oracle(sub)
    for splits in (1, 3, 0):
        out, lse = run_gpu(ra, case, splits)
        check(out[idx], lse[idx], ref_o, ref_l)


# ------------------------------------------------------------- error paths
def test_bad_sequence_length_reports_and_writes_nan(ra):
    case = small(500, T=1)
    case.seq_lens.fill_(10_000)                      # beyond the block table's capacity
    from relative_bias_gqa_b200.rel_attn import Workspace
    shape = ra.shape_of(case.q, case.k_cache, case.block_table, case.rel_table, out_fp32=True)
    for splits in (1, 3):
        ws = Workspace.for_shape(shape, splits, "cuda")
        out, lse = run_gpu(ra, case, splits, workspace=ws)
        assert torch.isnan(out).all() and torch.isnan(lse).all()
        assert ws.read_status() == ra.REL_ATTN_ERR_BAD_SEQ
        assert ws.read_status() == ra.REL_ATTN_OK    # reading clears it


def test_status_clean_after_normal_call(ra):
    case = small(3000, T=2)
    from relative_bias_gqa_b200.rel_attn import Workspace
    shape = ra.shape_of(case.q, case.k_cache, case.block_table, case.rel_table, out_fp32=True)
    ws = Workspace.for_shape(shape, 0, "cuda")
    run_gpu(ra, case, 0, workspace=ws)
    assert ws.read_status() == ra.REL_ATTN_OK


# ------------------------------------------- other GQA group sizes (G = 4, 8)
# The previous Inkling's layers: 64 query / 8 KV heads on full attention
# (G = 8, up to 6 tokens) and 64 / 16 on sliding-window layers (G = 4, window
# 512).  Each (G, T) pair has its own kernel instance.
def small_g(L, G, T=1, window=0, NB=1280, seed=0, Hkv=2, lens=None, **kw):
    lens = lens if lens is not None else [L]
    return W.make_case(seq_lens=lens, q_tokens=T, num_q_heads=G * Hkv, num_kv_heads=Hkv,
                       window=window, num_buckets=NB, seed=seed, extra_pages=2, **kw).to("cuda")


GROUP_CASES = (
    [dict(G=8, T=t, L=L) for t in range(1, 7) for L in (t, 129, 2100)] +
    [dict(G=4, T=t, L=L) for t in range(1, 9) for L in (t, 129, 2100)] +
    [dict(G=8, T=1, L=3001, window=1024, NB=1024), dict(G=8, T=6, L=3000, window=100),
     dict(G=4, T=1, L=3001, window=512, NB=1024), dict(G=4, T=8, L=2500, window=512, NB=1024),
     dict(G=4, T=5, L=1500, window=64), dict(G=8, T=3, L=5000, seed=3),
     dict(G=8, T=5, L=3000, NB=200, exact_buckets=16, max_distance=100000),
     dict(G=4, T=7, L=6000, NB=364, exact_buckets=64, max_distance=5000)]
)


@pytest.mark.parametrize("kw", GROUP_CASES, ids=[str(k) for k in GROUP_CASES])
def test_other_group_sizes(ra, kw):
    case = small_g(**kw)
    ref = run_oracle(case)
    for splits in (1, 3, 0):
        check(*run_gpu(ra, case, splits), *ref)


@pytest.mark.parametrize("G,T", [(8, 2), (8, 6), (4, 3), (4, 8)])
def test_other_group_sizes_batched(ra, G, T):
    case = small_g(0, G, T=T, Hkv=3, lens=[T, 64, 65 + T, 300, 1111, 2049, 129, T + 1])
    ref = run_oracle(case)
    for splits in (1, 2, 5, 0):
        check(*run_gpu(ra, case, splits), *ref)


@pytest.mark.parametrize("name", ["v1_full_100k", "v1_sliding_100k"])
def test_previous_model_layers_100k(ra, name):
    case = W.make_workload(name, seed=0, device="cuda")
    ref = run_oracle(case)
    for splits in (1, 7, 0):
        check(*run_gpu(ra, case, splits), *ref)


@pytest.mark.parametrize("G,T", [(8, 6), (4, 8)])
def test_other_group_sizes_verify_256k(ra, G, T):
    """Full-size verify with the G = 8 / G = 4 instances (one KV head keeps the
    oracle fast; the sequence still spans every split)."""
    case = W.make_case(seq_lens=[262_144], q_tokens=T, num_q_heads=G, num_kv_heads=1,
                       window=0, num_buckets=1280, seed=0).to("cuda")
    ref = run_oracle(case)
    for splits in (1, 18, 0):
        check(*run_gpu(ra, case, splits), *ref)
