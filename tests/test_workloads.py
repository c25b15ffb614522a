"""Seeded input generator: named workload shapes, block-table structure and
determinism (CPU only; the generator holds none of the attention arithmetic)."""

import math

import pytest
import torch

from relative_bias_gqa_b200 import workloads as W

SHAPES = {
    # name: (Hq, Hkv, T, window, NB, seq_lens)
    "sliding_100k": (48, 8, 1, 1024, 1024, [100_000]),
    "full_100k": (48, 8, 1, 0, 1280, [100_000]),
    "v1_full_100k": (64, 8, 1, 0, 1280, [100_000]),
    "v1_sliding_100k": (64, 16, 1, 512, 1024, [100_000]),
    "tiny_2k": (6, 1, 1, 0, 1280, [2048]),
}


@pytest.mark.parametrize("name", sorted(SHAPES))
def test_named_workload_shapes(name):
    Hq, Hkv, T, window, NB, lens = SHAPES[name]
    c = W.make_workload(name, seed=0)
    assert tuple(c.q.shape) == (len(lens), T, Hq, 128)
    assert c.k_cache.shape[1:] == (Hkv, 64, 128) and c.v_cache.shape == c.k_cache.shape
    assert tuple(c.rel_table.shape) == (Hkv, NB, 128)
    assert c.window == window and c.seq_lens.tolist() == lens
    assert c.q.dtype == c.k_cache.dtype == c.rel_table.dtype == torch.bfloat16
    # each sequence's pages are distinct pool pages; the rest of its row is -1
    bt = c.block_table
    for b, L in enumerate(lens):
        n = math.ceil(L / 64)
        row = bt[b].tolist()
        assert len(set(row[:n])) == n and min(row[:n]) >= 0 and max(row[:n]) < c.k_cache.shape[0]
        assert all(x == -1 for x in row[n:])


def test_batched_lengths_and_shared_pool():
    c = W.make_workload("batched_32", seed=0)
    lens = c.seq_lens.tolist()
    assert len(lens) == 32 and min(lens) >= 16384 and max(lens) <= 131072
    used = [p for b, L in enumerate(lens) for p in c.block_table[b, :math.ceil(L / 64)].tolist()]
    assert len(used) == len(set(used))                  # no page shared by two sequences


def test_seeded_and_reproducible():
    a = W.make_case(seq_lens=[300, 77], q_tokens=3, num_q_heads=16, num_kv_heads=2, seed=5)
    b = W.make_case(seq_lens=[300, 77], q_tokens=3, num_q_heads=16, num_kv_heads=2, seed=5)
    c = W.make_case(seq_lens=[300, 77], q_tokens=3, num_q_heads=16, num_kv_heads=2, seed=6)
    for x, y in ((a.q, b.q), (a.k_cache, b.k_cache), (a.v_cache, b.v_cache),
                 (a.rel_table, b.rel_table), (a.block_table, b.block_table)):
        assert torch.equal(x, y)
    assert not torch.equal(a.q, c.q)
