"""Row-block geometry of the partial kernel's instances, read from the kernel
header itself: a host program compiled against rel_attn_kernels.cuh prints,
for every G (heads per KV head) and T (query tokens), the group width N, the
softmax group count and each group's tokens and query slots; the checks below
are the layout rules the kernel relies on (no GPU needed).
"""

import os
import subprocess

import pytest

from relative_bias_gqa_b200 import build as B

PROGRAM = r"""
#include <cstdio>
#include "rel_attn_kernels.cuh"
using namespace relattn;
int main() {
  for (int f8 = 0; f8 <= 1; ++f8)
  for (int G = 1; G <= 8; ++G) {
    for (int T = 1; T <= 9; ++T) {
      const int N = group_width_for(G, T, f8 != 0), NG = softmax_groups(G, T, f8 != 0);
      const int A = (T == 1) ? 8 : (cs_end(T, G, NG, 8) <= N ? 8 : 4);
      std::printf("%d %d %d %d %d %d", f8, G, T, N, NG, A);
      for (int q = 0; q < NG; ++q)
        std::printf(" %d:%d:%d", cs_tok_begin(T, NG, q), cs_slot(T, G, NG, q, A), cs_rows(T, G, NG, q));
      std::printf("\n");
    }
  }
  return 0;
}
"""


@pytest.fixture(scope="module")
def table(tmp_path_factory):
    d = tmp_path_factory.mktemp("geom")
    src = d / "geom.cu"
    src.write_text(PROGRAM)
    exe = d / "geom"
    cmd = [B.find_nvcc(), "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
           "-I", B.INCLUDE, "-I", B.CSRC, "-o", str(exe), str(src)]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout
    rows = {}
    for line in out.splitlines():
        f = line.split()
        F8, G, T, N, NG, A = map(int, f[:6])
        groups = [tuple(map(int, g.split(":"))) for g in f[6:]]
        rows[(G, T) if not F8 else (G, T, "e4m3")] = (N, NG, A, groups)
    return rows


SUPPORTED = [(6, t) for t in range(1, 10)] + [(8, t) for t in range(1, 9)] + [(4, t) for t in range(1, 10)]


def test_supported_shapes_have_instances(table):
    for G, T in SUPPORTED:
        assert table[(G, T)][0] in (16, 32, 48, 64), (G, T)
    assert table[(8, 9)][0] == 0                                  # 72 rows > 64 slots


def test_inkling2_instances(table):
    # 48/8 heads: N and group counts of the measured instances; nine tokens
    # (an 8-head MTP chain's verify step) need the 64-wide instance
    assert [table[(6, t)][0] for t in range(1, 10)] == [16, 32, 32, 32, 48, 48, 64, 64, 64]
    assert [table[(6, t)][1] for t in range(1, 10)] == [2, 2, 2, 2, 2, 3, 4, 4, 3]
    # 7 and 8 tokens: 8-aligned blocks in the 64-wide tile; 9 tokens 4-aligned
    assert [table[(6, t)][2] for t in range(6, 10)] == [8, 8, 8, 4]


def test_wide_instances(table):
    # 64/8 heads with 7 and 8 tokens: four groups of up to 16 rows, 8-aligned
    assert [table[(8, t)][:3] for t in (7, 8)] == [(64, 4, 8), (64, 4, 8)]
    # nine tokens at G = 6: three groups of three tokens, 18 rows each at
    # 4-aligned query slots 0 / 20 / 40
    assert [g[2] for g in table[(6, 9)][3]] == [18, 18, 18]
    assert [g[1] for g in table[(6, 9)][3]] == [0, 20, 40]
    # nine tokens at G = 4: three groups of 12 rows, 8-aligned in 48 columns
    assert table[(4, 9)][:3] == (48, 3, 8)
    # six tokens: three groups of two tokens for every G
    assert [table[(g, 6)][1] for g in (4, 6, 8)] == [3, 3, 3]


@pytest.mark.parametrize("G,T", [k for k in SUPPORTED if k[1] >= 2])
def test_column_split_layout(table, G, T):
    N, NG, A, groups = table[(G, T)]
    assert len(groups) == NG
    # tokens: a partition of [0, T) in order, every group non-empty
    starts = [g[0] for g in groups] + [T]
    assert starts[0] == 0 and all(starts[q] < starts[q + 1] for q in range(NG))
    for q, (tb, slot, rows) in enumerate(groups):
        assert rows == (starts[q + 1] - tb) * G
        assert slot % A == 0
        # the group's P units (A rows each) end before the next group's slots
        end = slot + -(-rows // A) * A
        nxt = groups[q + 1][1] if q + 1 < NG else N
        assert end <= nxt <= N
        # at most the per-group row capacity of the instance (N / NG, or
        # ceil(T / NG) * G when the tokens do not split evenly)
        assert rows <= max(N // NG, -(-T // NG) * G)
        # tensor-memory loads: RG = the instance's row capacity per group,
        # read as 8-column loads from the slot (A = 8) or from the 8-aligned
        # column below it, RG + 4 columns (A = 4); they must end inside the
        # group's N-column buffer (S, each O half, X0 and X1 are N wide, and
        # X1 is the last block of the allocation)
        RG = -(-T // NG) * G
        base, cols = (slot, -(-RG // 8) * 8) if A == 8 else (slot & ~7, -(-(RG + 4) // 8) * 8)
        assert base + cols <= N, (q, base, cols)


@pytest.mark.parametrize("G", [4, 6, 8])
def test_one_token_instance(table, G):
    N, NG, A, groups = table[(G, 1)]
    assert N == 16 and NG == 2 and G <= N


def test_e4m3_widened_instances(table):
    """Over an E4M3 cache the softmax warps also widen the codes: four groups
    at four tokens (and five for G <= 6), 8-aligned; otherwise the bf16
    instances' layout."""
    assert [table[(G, 4, "e4m3")][:3] for G in (4, 6, 8)] == [(32, 4, 8)] * 3
    assert [table[(G, 5, "e4m3")][:3] for G in (4, 6)] == [(32, 4, 8), (48, 4, 8)]
    assert table[(8, 5, "e4m3")] == table[(8, 5)]
    for G in (4, 6, 8):
        for T in (6, 7, 8, 9):
            assert table[(G, T, "e4m3")] == table[(G, T)]
    # column-split instances (several tokens): every group has tokens, slots
    # do not overlap, and the block fits N
    for (key, (N, NG, A, groups)) in table.items():
        if len(key) == 3 and N and key[1] >= 2:
            ends = [slot + rows for (_, slot, rows) in groups]
            assert all(rows > 0 for (_, _, rows) in groups) and max(ends) <= N, key
            assert all(groups[i][1] + groups[i][2] <= groups[i + 1][1] for i in range(NG - 1)), key

