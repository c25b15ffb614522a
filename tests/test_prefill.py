"""GPU parity of the chunked prefill (rel_attn_prefill, through the C ABI)
against the fp64 oracle: C query tokens per sequence at positions
L - C .. L - 1, each attending causally (and within the window) to the keys
up to it -- the oracle's definition for a step of C tokens.  Tolerances as
for the decode: 2e-3 on the fp32 output, 1e-3 on the lse.
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


def run(ra, case, splits=0, out_fp32=True):
    out, lse = ra.rel_attn_prefill(case.q, case.k_cache, case.v_cache, case.block_table,
                                   case.seq_lens, case.rel_table, case.window, splits,
                                   max_seq_len=case.max_seq_len, out_fp32=out_fp32,
                                   exact_buckets=case.exact_buckets, max_distance=case.max_distance)
    torch.cuda.synchronize()
    return out, lse


def check(out, lse, case):
    ref_o, ref_l = oracle.rel_attn_decode_ref(case.q, case.k_cache, case.v_cache, case.block_table,
                                              case.seq_lens, case.rel_table, case.window,
                                              exact_buckets=case.exact_buckets,
                                              max_distance=case.max_distance)
    o = out.double().cpu().numpy()
    l = lse.double().cpu().numpy()
    assert np.isfinite(o).all() and np.isfinite(l).all()
    eo, el = np.abs(o - ref_o).max(), np.abs(l - ref_l).max()
    assert eo <= OUT_TOL and el <= LSE_TOL, (eo, el)


CASES = [
    dict(C=1, lens=[1]), dict(C=7, lens=[7]), dict(C=8, lens=[8]), dict(C=9, lens=[9]),
    dict(C=17, lens=[1000]), dict(C=100, lens=[100]), dict(C=129, lens=[2100]),
    dict(C=513, lens=[513]), dict(C=300, lens=[300], window=64),
    dict(C=200, lens=[3000], window=1024, NB=1024), dict(C=64, lens=[64, 200, 1111]),
    dict(C=33, lens=[40, 5000], G=8), dict(C=45, lens=[45, 777], G=4),
    # nine tokens at G = 8 (72 query rows, the MTP verify the decode instances
    # do not cover): an 8-token and a 1-token chunk
    dict(C=9, lens=[9, 2100, 20000], G=8),
    dict(C=24, lens=[1500], NB=364, exact_buckets=64, max_distance=5000),
]


@pytest.mark.parametrize("kw", CASES, ids=[str(k) for k in CASES])
@pytest.mark.parametrize("splits", [1, 3, 0])
def test_prefill_matches_oracle(ra, kw, splits):
    kw = dict(kw)
    C, G = kw.pop("C"), kw.pop("G", 6)
    lens = kw.pop("lens")
    case = W.make_case(seq_lens=lens, q_tokens=C, num_q_heads=2 * G, num_kv_heads=2,
                       num_buckets=kw.pop("NB", 1280), seed=C + len(lens), extra_pages=2,
                       **kw).to("cuda")
    check(*run(ra, case, splits), case)


def test_prefill_equals_decode_for_one_chunk(ra):
    """Up to 9 tokens the prefill is one decode step: identical results."""
    for C in (1, 5, 8):
        case = W.make_case(seq_lens=[3000], q_tokens=C, num_q_heads=12, num_kv_heads=2,
                           seed=C).to("cuda")
        a = run(ra, case, 3)
        b = ra.rel_attn_decode(case.q, case.k_cache, case.v_cache, case.block_table,
                               case.seq_lens, case.rel_table, 0, 3, max_seq_len=3000,
                               out_fp32=True)
        torch.cuda.synchronize()
        assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_prefill_8k_one_kv_head(ra):
    """An 8,192-token prefill over an 8,192-token context (one KV head keeps
    the oracle to seconds)."""
    case = W.make_case(seq_lens=[8192], q_tokens=8192, num_q_heads=6, num_kv_heads=1,
                       seed=9).to("cuda")
    check(*run(ra, case, 0), case)


def test_prefill_bf16_output_is_rounded_fp32(ra):
    case = W.make_case(seq_lens=[700], q_tokens=77, num_q_heads=12, num_kv_heads=2,
                       seed=3).to("cuda")
    o32, l32 = run(ra, case, 1, out_fp32=True)
    o16, l16 = run(ra, case, 1, out_fp32=False)
    assert torch.equal(o32.to(torch.bfloat16), o16) and torch.equal(l32, l16)


def test_prefill_rejects_short_sequence(ra):
    """seq_len below the token count: the sequence's rows come back NaN and
    the status word says BAD_SEQ."""
    case = W.make_case(seq_lens=[100], q_tokens=20, num_q_heads=12, num_kv_heads=2,
                       seed=4).to("cuda")
    case.seq_lens.fill_(10)
    shape = ra.shape_of(case.q, case.k_cache, case.block_table, case.rel_table, out_fp32=True)
    ws = ra.Workspace(ra.prefill_workspace_bytes(shape, 1), "cuda")
    out, lse = ra.rel_attn_prefill(case.q, case.k_cache, case.v_cache, case.block_table,
                                   case.seq_lens, case.rel_table, 0, 1, workspace=ws,
                                   out_fp32=True)
    torch.cuda.synchronize()
    assert torch.isnan(out).all()
    assert ws.read_status() == ra.REL_ATTN_ERR_BAD_SEQ
