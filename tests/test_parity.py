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
    # dense tail buckets (nearly one per distance past the exact range): the
    # densest tables one relative-row chunk still covers
    dict(L=2200, T=2, NB=600, exact_buckets=100, max_distance=8000),
    dict(L=3000, T=8, NB=350, exact_buckets=100, max_distance=1500),
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
                                         (1, 1024, 2500), (2, 5, 129), (9, 0, 700), (9, 100, 2000)])
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
               dict(L=1500, T=3, window=100), dict(L=2222, T=9, window=0)):
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


def test_full_100k_every_split_count(ra):
    """The 100K full-attention decode with every split count 1..256 (and the
    heuristic's) against one oracle result."""
    case = W.make_workload("full_100k", seed=0, device="cuda")
    ref = run_oracle(case)
    shape = ra.shape_of(case.q, case.k_cache, case.block_table, case.rel_table, out_fp32=True)
    from relative_bias_gqa_b200.rel_attn import Workspace
    ws = Workspace.for_shape(shape, 256, "cuda")
    worst = (0.0, 0.0)
    for s in list(range(1, 257)) + [0]:
        eo, el = check(*run_gpu(ra, case, s, workspace=ws), *ref)
        worst = (max(worst[0], eo), max(worst[1], el))
    assert ws.read_status() == ra.REL_ATTN_OK


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


def test_batched_32_every_sequence(ra):
    """All 32 sequences of the mixed-length batch against the oracle, one
    sequence at a time on the host (a compact copy of its pages keeps the
    fp64 working set small)."""
    case = W.make_workload("batched_32", seed=0, device="cuda")
    runs = [run_gpu(ra, case, splits) for splits in (1, 3, 0)]
    for b in range(case.batch):
        ref_o, ref_l = run_oracle(_sub_case(case, [b]))
        for out, lse in runs:
            check(out[b:b + 1], lse[b:b + 1], ref_o, ref_l)


# ------------------------------------------- full-size key sets and poison
def _zero_q_r_bits_v(case):
    """Q = 0 and R = 0 (uniform weights over the selected keys) and V row of
    position j holding the bits of j in its first 18 dims (0/1, exact in
    bf16), on every KV head, through the case's shuffled block table."""
    case.q.zero_()
    case.rel_table.zero_()
    P = case.page_size
    for b in range(case.batch):
        L = int(case.seq_lens[b])
        pos = torch.arange(L, device="cuda")
        bits = ((pos[:, None] >> torch.arange(18, device="cuda")[None]) & 1).to(torch.bfloat16)
        pages = case.block_table[b].long()[pos // P]
        vals = torch.zeros(L, 128, dtype=torch.bfloat16, device="cuda")
        vals[:, :18] = bits
        for h in range(case.num_kv_heads):
            case.v_cache[pages, h, pos % P] = vals


def _check_key_sets(case, out, lse, one_split):
    """Each row must select exactly its key set J (a contiguous position
    range).  One split: exp(lse) = |J| (to the nearest integer up to 16,384
    keys, else to 4e-6 relative: fp32 log2 / exp rounding) and out[c] =
    #{j in J : bit c of j} / |J| to a quarter of 1/|J| -- the partial
    kernel's sums of 0/1 values are exact and out is one rounded division,
    so a key missing, added or swapped moves some out[c] by about 1/(2|J|).
    Several splits: the merge's fp32 weights carry ~1e-6 relative error, so
    the check resolves whole pages (64 keys: >= 1e-5 relative at 262,144
    keys), which is what a split boundary can get wrong."""
    T, W = case.q_tokens, case.window
    o = out.double().cpu().numpy()
    l = lse.double().cpu().numpy()
    for b in range(case.batch):
        L = int(case.seq_lens[b])
        for t in range(T):
            p = L - T + t
            lo = 0 if W <= 0 else max(0, p - W + 1)
            n = p - lo + 1
            cnt = np.array([_bit_count_range(lo, p, c) for c in range(18)], dtype=np.float64)
            est = np.exp(l[b, t])
            strict = one_split or n <= 16384      # merge error ~1e-6 << 1/(4|J|)
            if strict and n <= 16384:
                assert np.all(np.round(est) == n), (b, t, est, n)
            else:
                rel = 4e-6 if strict else 1e-5
                assert np.all(np.abs(est / n - 1.0) <= rel), (b, t, est, n)
            err = np.abs(o[b, t, :, :18] - cnt[None] / n).max()
            tol = 0.25 / n if strict else max(0.25 / n, 4e-6)
            assert err <= tol, (b, t, err, tol)


def _bit_count_range(lo, hi, c):
    """#{j in [lo, hi] : bit c of j is set}, in closed form."""
    def upto(x):                                   # over [0, x)
        period = 1 << (c + 1)
        return (x // period) * (1 << c) + max(0, x % period - (1 << c))
    return upto(hi + 1) - upto(lo)


@pytest.mark.parametrize("name", ["full_100k", "sliding_100k", "verify_t8_256k"])
def test_key_set_identity_full_size(ra, name):
    case = W.make_workload(name, seed=2, device="cuda")
    _zero_q_r_bits_v(case)
    for splits in (1, 5, 0):
        out, lse = run_gpu(ra, case, splits)
        _check_key_sets(case, out, lse, one_split=splits == 1)


@pytest.mark.parametrize("name", ["full_100k", "sliding_100k", "verify_t8_256k"])
def test_poisoned_slots_full_size(ra, name):
    """NaN in every pool page no sequence owns (64 of them, shuffled in among
    the owned ones), in the slots past L and before the window: the outputs
    are bit-identical to the clean run and match the oracle."""
    case = W.make_workload(name, seed=3, device="cuda", extra_pages=64)
    ref = run_oracle(case)
    bad = W.poison_unused(case)
    for splits in (1, 7, 0):
        clean = run_gpu(ra, case, splits)
        dirty = run_gpu(ra, bad, splits)
        assert torch.equal(clean[0], dirty[0]) and torch.equal(clean[1], dirty[1])
        check(*dirty, *ref)


@pytest.mark.parametrize("T", [2, 3, 4, 5, 6, 7])
def test_verify_256k_every_token_count(ra, T):
    """Full-size speculative verify for every token count below 8 (G = 6; one
    KV head keeps the oracle fast, the sequence still spans every split)."""
    case = W.make_case(seq_lens=[262_144], q_tokens=T, num_q_heads=6, num_kv_heads=1,
                       window=0, num_buckets=1280, seed=T).to("cuda")
    ref = run_oracle(case)
    for splits in (1, 18, 0):
        check(*run_gpu(ra, case, splits), *ref)


# ------------------------------------------------------- merge entry points
def test_split_phase_partial_then_combine(ra):
    """rel_attn_partial + rel_attn_combine (the split-phase entry points)
    give exactly what rel_attn_decode gives, and match the oracle."""
    case = small(0, T=3, Hkv=2, lens=[5000, 700, 129])
    ref = run_oracle(case)
    for splits in (2, 7, 40):
        prep = ra.Prepared(case.q, case.k_cache, case.v_cache, case.block_table, case.seq_lens,
                           case.rel_table, case.window, splits, max_seq_len=case.max_seq_len,
                           out_fp32=True)
        prep.partial()
        prep.combine()
        torch.cuda.synchronize()
        a = (prep.out.clone(), prep.lse.clone())
        check(*a, *ref)
        prep.decode()
        torch.cuda.synchronize()
        assert torch.equal(prep.out, a[0]) and torch.equal(prep.lse, a[1])
        assert prep.workspace.read_status() == ra.REL_ATTN_OK


def test_many_sequences_and_heads(ra):
    """968 (sequence, KV head) pairs in one call: 121 sequences x 8 KV heads,
    lengths 2..901, checked on four sequences."""
    lens = [(37 * i) % 900 + 2 for i in range(121)]
    case = W.make_case(seq_lens=lens, q_tokens=1, num_q_heads=48, num_kv_heads=8, window=0,
                       num_buckets=1280, seed=12).to("cuda")
    idx = [0, 1, 60, 120]
    ref_o, ref_l = run_oracle(case, batch_indices=idx)
    for splits in (3, 0):
        out, lse = run_gpu(ra, case, splits)
        check(out[idx], lse[idx], ref_o[idx], ref_l[idx])


def test_one_workspace_across_shapes(ra):
    """One workspace serves calls of different shapes and split counts in
    turn (it holds only the status word and each call's own partials)."""
    from relative_bias_gqa_b200.rel_attn import Workspace
    big = small(0, T=2, Hkv=3, lens=[3000, 100, 2500])
    shape = ra.shape_of(big.q, big.k_cache, big.block_table, big.rel_table, out_fp32=True)
    ws = Workspace.for_shape(shape, 64, "cuda")
    cases = [big, small(2000, T=1, Hkv=2), small(0, T=5, Hkv=1, lens=[900, 4000])]
    refs = [run_oracle(c) for c in cases]
    for _ in range(2):
        for c, ref, splits in zip(cases, refs, (64, 5, 17)):
            check(*run_gpu(ra, c, splits, workspace=ws), *ref)
    assert ws.read_status() == ra.REL_ATTN_OK


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


@pytest.mark.parametrize("splits", [1, 3])
def test_block_table_entry_outside_pool_writes_nan(ra, splits):
    """One block-table entry of sequence 0 points outside the pool: every row
    of sequence 0 comes back NaN (all its KV heads walk that page) and the
    status says BAD_SEQ; sequence 1 is untouched and still matches the
    oracle.  Both through the workspace entry and the allocation-free one."""
    import ctypes
    from relative_bias_gqa_b200.rel_attn import Workspace
    case = small(0, T=2, Hkv=2, lens=[2000, 1500])
    ref_o, ref_l = run_oracle(case, batch_indices=[1])
    for bad_entry in (case.k_cache.shape[0] + 7, -3):
        case.block_table[0, 5] = bad_entry
        shape = ra.shape_of(case.q, case.k_cache, case.block_table, case.rel_table,
                            max_seq_len=case.max_seq_len, out_fp32=True)
        ws = Workspace.for_shape(shape, splits, "cuda")
        out, lse = run_gpu(ra, case, splits, workspace=ws)
        assert torch.isnan(out[0]).all() and torch.isnan(lse[0]).all()
        check(out[1:], lse[1:], ref_o[1:], ref_l[1:])
        assert ws.read_status() == ra.REL_ATTN_ERR_BAD_SEQ
        out2 = torch.zeros_like(out)
        lse2 = torch.zeros_like(lse)
        rc = ra.lib.rel_attn_decode_static(
            ctypes.byref(shape), case.q.data_ptr(), case.k_cache.data_ptr(),
            case.v_cache.data_ptr(), case.block_table.data_ptr(), case.seq_lens.data_ptr(),
            case.rel_table.data_ptr(), case.window, splits, out2.data_ptr(), lse2.data_ptr(),
            torch.cuda.current_stream().cuda_stream)
        torch.cuda.synchronize()
        assert rc == ra.REL_ATTN_OK
        assert torch.isnan(out2[0]).all() and torch.isnan(lse2[0]).all()
        assert torch.equal(out2[1:], out[1:]) and torch.equal(lse2[1:], lse[1:])


@pytest.mark.parametrize("workload,T", [("full_100k", 1), ("verify_t8_256k", 8)])
def test_injected_wait_limit_times_out_cleanly(ra, workload, T):
    """A 1 ns bound on every device wait (it runs out at the device timer's
    next tick) makes the waits for TMA copies run out: the call must come back promptly with REL_ATTN_ERR_TIMEOUT in the
    status word and NaN rows (never a hang), and the next call with the
    default bound must be correct again on the same workspace."""
    import time
    from relative_bias_gqa_b200.rel_attn import Workspace
    case = W.make_workload(workload, seed=4, device="cuda", num_q_heads=6 * 2, num_kv_heads=2)
    assert case.q_tokens == T
    shape = ra.shape_of(case.q, case.k_cache, case.block_table, case.rel_table,
                        max_seq_len=case.max_seq_len, out_fp32=True)
    ws = Workspace.for_shape(shape, 0, "cuda")
    run_gpu(ra, case, 0, workspace=ws)                   # warm: attributes, tensor maps
    assert ws.read_status() == ra.REL_ATTN_OK
    try:
        ra.rel_attn_set_wait_limit(1)
        t0 = time.perf_counter()
        out, lse = run_gpu(ra, case, 0, workspace=ws)
        elapsed = time.perf_counter() - t0
    finally:
        ra.rel_attn_set_wait_limit(0)
    assert elapsed < 1.0, elapsed                        # far below the 2 s default bound
    assert ws.read_status() == ra.REL_ATTN_ERR_TIMEOUT
    assert torch.isnan(out).any() and torch.isnan(lse).any()
    assert ws.read_status() == ra.REL_ATTN_OK            # reading cleared it
    check(*run_gpu(ra, case, 0, workspace=ws), *run_oracle(case))
    assert ws.read_status() == ra.REL_ATTN_OK


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
    [dict(G=8, T=t, L=L) for t in range(1, 9) for L in (t, 129, 2100)] +
    [dict(G=4, T=t, L=L) for t in range(1, 10) for L in (t, 129, 2100)] +
    [dict(G=6, T=9, L=L) for L in (9, 10, 129, 2100, 5000)] +
    [dict(G=8, T=8, L=3000, window=1024, NB=1024), dict(G=8, T=7, L=2500, window=100),
     dict(G=6, T=9, L=3000, window=1024, NB=1024), dict(G=4, T=9, L=1700, window=512, NB=1024),
     dict(G=6, T=9, L=3000, NB=200, exact_buckets=16, max_distance=100000)] +
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


@pytest.mark.parametrize("G,T", [(8, 2), (8, 6), (8, 8), (4, 3), (4, 8), (6, 9), (4, 9)])
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


@pytest.mark.parametrize("G,T", [(8, 6), (4, 8), (8, 7), (8, 8), (6, 9), (4, 9)])
def test_other_group_sizes_verify_256k(ra, G, T):
    """Full-size verify with the G = 8 / G = 4 instances (one KV head keeps the
    oracle fast; the sequence still spans every split)."""
    case = W.make_case(seq_lens=[262_144], q_tokens=T, num_q_heads=G, num_kv_heads=1,
                       window=0, num_buckets=1280, seed=0).to("cuda")
    ref = run_oracle(case)
    for splits in (1, 18, 0):
        check(*run_gpu(ra, case, splits), *ref)


def test_result_written_into_mapped_host_memory(ra):
    """out and lse may be mapped pinned host memory (the header allows it):
    the call then stores the result straight to the host, bit for bit what
    the same call writes into device memory."""
    try:
        from cuda.bindings import runtime as cudart
    except ImportError:
        from cuda import cudart
    case = small(3001, T=2, seed=6)
    for S in (1, 3):
        out_d, lse_d = run_gpu(ra, case, S, out_fp32=False)
        out_h = torch.empty(out_d.shape, dtype=out_d.dtype).pin_memory()
        lse_h = torch.empty(lse_d.shape, dtype=lse_d.dtype).pin_memory()
        for t in (out_h, lse_h):
            err, dptr = cudart.cudaHostGetDevicePointer(t.data_ptr(), 0)
            if int(err) != 0 or int(dptr) != t.data_ptr():
                pytest.skip("pinned memory is not mapped at its host address")
        ra.rel_attn_decode(case.q, case.k_cache, case.v_cache, case.block_table, case.seq_lens,
                           case.rel_table, case.window, S, out=out_h, lse=lse_h,
                           max_seq_len=case.max_seq_len, out_fp32=False)
        torch.cuda.synchronize()
        assert torch.equal(out_h, out_d.cpu()) and torch.equal(lse_h, lse_d.cpu())
