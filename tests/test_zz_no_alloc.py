"""The allocation-free entry point, rel_attn_decode_static.

It serves callers that cannot allocate device memory (a plugin that is given
only its input and output buffers, or an engine that has reserved all of HBM
for its KV cache): the scratch space comes from a fixed 4 MiB array inside
the library.  Its results must match rel_attn_decode's on the same inputs,
call after call, even though the array keeps the previous call's contents.
This file is collected last so that a run stopping at the first failure has
already run every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

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


def _static_call(ra, case, num_splits, out_fp32=True):
    shape = ra.shape_of(case.q, case.k_cache, case.block_table, case.rel_table,
                        max_seq_len=case.max_seq_len, out_fp32=out_fp32)
    out = torch.full(case.q.shape, float("nan"), device="cuda",
                     dtype=torch.float32 if out_fp32 else torch.bfloat16)
    lse = torch.full(case.q.shape[:3], float("nan"), device="cuda", dtype=torch.float32)
    rc = ra.lib.rel_attn_decode_static(
        ctypes.byref(shape), case.q.data_ptr(), case.k_cache.data_ptr(), case.v_cache.data_ptr(),
        case.block_table.data_ptr(), case.seq_lens.data_ptr(), case.rel_table.data_ptr(),
        case.window, num_splits, out.data_ptr(), lse.data_ptr(),
        torch.cuda.current_stream().cuda_stream)
    return rc, out, lse


def _reference_call(ra, case, num_splits):
    out, lse = ra.rel_attn_decode(case.q, case.k_cache, case.v_cache, case.block_table,
                                  case.seq_lens, case.rel_table, case.window, num_splits,
                                  max_seq_len=case.max_seq_len, out_fp32=True)
    return out, lse


def test_static_entry_matches_workspace_entry_two_calls_in_a_row(ra):
    """Both entry points launch the same kernels with the same split count,
    so their results must be bit-identical; the first case also runs more
    splits than the second, so the second call finds the first one's
    partials still in the shared array."""
    cases = [
        (W.make_case(seq_lens=[5000], q_tokens=1, num_q_heads=48, num_kv_heads=8,
                     window=0, num_buckets=1280, seed=3).to("cuda"), 37),
        (W.make_case(seq_lens=[2500, 900], q_tokens=3, num_q_heads=12, num_kv_heads=2,
                     window=1024, num_buckets=1024, seed=4).to("cuda"), 0),
    ]
    for case, splits in cases:            # two calls in a row on the shared array
        rc, out, lse = _static_call(ra, case, splits)
        assert rc == ra.REL_ATTN_OK, ra.error_string(rc)
        torch.cuda.synchronize()
        ref_out, ref_lse = _reference_call(ra, case, splits)
        torch.cuda.synchronize()
        assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)


def test_static_entry_against_the_oracle(ra):
    """The allocation-free call checked directly against the fp64 oracle, with
    one split (no partials: the kernel writes the output itself), then with
    several splits after a call that used more of the array."""
    import oracle
    case = W.make_case(seq_lens=[3001, 64, 129], q_tokens=2, num_q_heads=18, num_kv_heads=3,
                       window=0, num_buckets=1280, seed=6).to("cuda")
    ref_o, ref_l = oracle.rel_attn_decode_ref(case.q, case.k_cache, case.v_cache,
                                              case.block_table, case.seq_lens,
                                              case.rel_table, case.window)
    for splits in (1, 40, 5, 1):
        rc, out, lse = _static_call(ra, case, splits)
        assert rc == ra.REL_ATTN_OK, ra.error_string(rc)
        torch.cuda.synchronize()
        eo = np.abs(out.double().cpu().numpy() - ref_o).max()
        el = np.abs(lse.double().cpu().numpy() - ref_l).max()
        assert np.isfinite(eo) and eo <= OUT_TOL, (splits, eo)
        assert np.isfinite(el) and el <= LSE_TOL, (splits, el)


def test_static_entry_rejects_shapes_beyond_its_scratch(ra):
    case = W.make_case(seq_lens=[300] * 16, q_tokens=8, num_q_heads=48, num_kv_heads=8,
                       window=0, num_buckets=1280, seed=5).to("cuda")
    shape = ra.shape_of(case.q, case.k_cache, case.block_table, case.rel_table)
    assert ra.rel_attn_workspace_bytes(shape, 64) > (4 << 20)
    rc, out, _ = _static_call(ra, case, 64)
    torch.cuda.synchronize()
    assert rc == ra.REL_ATTN_ERR_WORKSPACE_TOO_SMALL
    assert torch.isnan(out).all()          # nothing was launched
