"""Seeded synthetic inputs for relative-bias GQA decode attention.

This module only draws and lays out inputs; it holds none of the attention
arithmetic, so both the CUDA path and the CPU oracle may be fed from it.

Shapes follow the Inkling model descriptions:
  * "vLLM、Inkling 2 Smallを初日サポート GB200で630 tok/s", section
    "モデルの構成" (table rows "Heads" and "Sliding window"): 48 query / 8 KV
    heads on every layer, sliding window 1,024; the previous Inkling's
    full-attention layers 64 query / 8 KV heads, its sliding layers 64 / 16
    with window 512.
  * "vLLM TML Inkling 지원", section "TML Inkling 모델 아키텍처": GQA with head
    size 128, context up to 1M tokens, up to 9 tokens per speculative step.
  * same page, section "Sconv 캐시 및 TP 샤딩": the KV cache is held by a
    unified (paged) KV-cache manager; the page size (64) is this library's.

Recipe (fixed draw order, all values drawn in fp32 then rounded to bf16 by
round-to-nearest-even):
  1. sequence lengths (CPU generator seeded with ``seed``) when they are random;
  2. q ~ N(0, 1)            [B, T, Hq, D]
  3. k pool ~ N(0, 1)       [num_pages, Hkv, P, D]
  4. v pool ~ N(0, 1)       [num_pages, Hkv, P, D]
  5. rel table ~ N(0, 0.02) [Hkv, NB, D]
     (2-5 from a generator on ``device`` seeded with ``seed``)
  6. page order: a random permutation of the pool (CPU generator seeded with
     ``seed + 1``) unless the case asks for a contiguous cache.
The block table is int32 [B, max_pages_per_seq], padded with -1.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import torch

PAGE_SIZE = 64
EXACT_BUCKETS = 1024
MAX_DISTANCE = 1 << 20


@dataclasses.dataclass
class DecodeCase:
    name: str
    q: torch.Tensor            # [B, T, Hq, D] bf16
    k_cache: torch.Tensor      # [num_pages, Hkv, P, D] bf16
    v_cache: torch.Tensor      # [num_pages, Hkv, P, D] bf16
    block_table: torch.Tensor  # [B, max_pages_per_seq] int32, -1 padded
    seq_lens: torch.Tensor     # [B] int32
    rel_table: torch.Tensor    # [Hkv, NB, D] bf16
    window: int                # <= 0: full attention
    num_buckets: int
    exact_buckets: int = EXACT_BUCKETS
    max_distance: int = MAX_DISTANCE

    @property
    def batch(self) -> int:
        return self.q.shape[0]

    @property
    def q_tokens(self) -> int:
        return self.q.shape[1]

    @property
    def num_q_heads(self) -> int:
        return self.q.shape[2]

    @property
    def num_kv_heads(self) -> int:
        return self.k_cache.shape[1]

    @property
    def head_dim(self) -> int:
        return self.q.shape[3]

    @property
    def page_size(self) -> int:
        return self.k_cache.shape[2]

    @property
    def max_seq_len(self) -> int:
        return int(self.seq_lens.max().item())

    def to(self, device) -> "DecodeCase":
        return dataclasses.replace(
            self,
            q=self.q.to(device), k_cache=self.k_cache.to(device),
            v_cache=self.v_cache.to(device),
            block_table=self.block_table.to(device),
            seq_lens=self.seq_lens.to(device),
            rel_table=self.rel_table.to(device))


def _randn_bf16(shape, gen, device, std=1.0):
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def make_case(*, seq_lens: Sequence[int], q_tokens: int = 1,
              num_q_heads: int = 48, num_kv_heads: int = 8,
              head_dim: int = 128, page_size: int = PAGE_SIZE,
              window: int = 0, num_buckets: int = 1280,
              exact_buckets: int = EXACT_BUCKETS,
              max_distance: int = MAX_DISTANCE,
              seed: int = 0, device="cpu", contiguous: bool = False,
              extra_pages: int = 0, max_pages_per_seq: Optional[int] = None,
              rel_std: float = 0.02, name: str = "case") -> DecodeCase:
    """Draw one decode problem; see the module docstring for the recipe."""
    seq_lens = [int(x) for x in seq_lens]
    B = len(seq_lens)
    pages_needed = [math.ceil(L / page_size) for L in seq_lens]
    num_pages = sum(pages_needed) + extra_pages
    if max_pages_per_seq is None:
        max_pages_per_seq = max(pages_needed)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    q = _randn_bf16((B, q_tokens, num_q_heads, head_dim), gen, device)
    k = _randn_bf16((num_pages, num_kv_heads, page_size, head_dim), gen, device)
    v = _randn_bf16((num_pages, num_kv_heads, page_size, head_dim), gen, device)
    rel = _randn_bf16((num_kv_heads, num_buckets, head_dim), gen, device,
                      std=rel_std)
    if contiguous:
        order = torch.arange(num_pages, dtype=torch.int64)
    else:
        cgen = torch.Generator()
        cgen.manual_seed(seed + 1)
        order = torch.randperm(num_pages, generator=cgen)
    bt = torch.full((B, max_pages_per_seq), -1, dtype=torch.int32)
    pos = 0
    for b, n in enumerate(pages_needed):
        bt[b, :n] = order[pos:pos + n].to(torch.int32)
        pos += n
    return DecodeCase(
        name=name, q=q, k_cache=k, v_cache=v, block_table=bt.to(device),
        seq_lens=torch.tensor(seq_lens, dtype=torch.int32, device=device),
        rel_table=rel, window=window, num_buckets=num_buckets,
        exact_buckets=exact_buckets, max_distance=max_distance)


def batched_lengths(batch: int = 32, lo: int = 16384, hi: int = 131072,
                    seed: int = 0) -> list:
    """Context lengths drawn uniformly from [lo, hi] (CPU generator)."""
    g = torch.Generator()
    g.manual_seed(seed)
    return torch.randint(lo, hi + 1, (batch,), generator=g).tolist()


# The named workloads (shapes from the Inkling model descriptions).
WORKLOADS = {
    # tiny oracle-scale case: 6 query heads / 1 KV head, 2,048 keys, contiguous cache
    "tiny_2k": dict(seq_lens=[2048], num_q_heads=6, num_kv_heads=1, window=0,
                    num_buckets=1280, contiguous=True),
    # sliding window of 1,024 over a 100,000-token context
    "sliding_100k": dict(seq_lens=[100_000], window=1024, num_buckets=1024),
    # full attention over a 100,000-token context
    "full_100k": dict(seq_lens=[100_000], window=0, num_buckets=1280),
    # speculative verify: 8 causal query tokens at the end of 262,144 keys
    "verify_t8_256k": dict(seq_lens=[262_144], q_tokens=8, window=0,
                           num_buckets=1280),
    # 32 sequences with lengths uniform in [16,384, 131,072], one shared pool
    "batched_32": dict(seq_lens=None, window=0, num_buckets=1280),
    # the previous Inkling's layers over a 100,000-token context: full
    # attention with 64 query / 8 KV heads, sliding window 512 with 64 / 16
    "v1_full_100k": dict(seq_lens=[100_000], window=0, num_buckets=1280,
                         num_q_heads=64, num_kv_heads=8),
    "v1_sliding_100k": dict(seq_lens=[100_000], window=512, num_buckets=1024,
                            num_q_heads=64, num_kv_heads=16),
}


def make_workload(name: str, seed: int = 0, device="cpu", **overrides) -> DecodeCase:
    spec = dict(WORKLOADS[name])
    if spec.get("seq_lens") is None:
        spec["seq_lens"] = batched_lengths(seed=seed)
    spec.update(overrides)
    return make_case(seed=seed, device=device, name=name, **spec)


def visible_page_range(seq_len: int, q_tokens: int, window: int,
                       page_size: int = PAGE_SIZE):
    """Logical pages [first, last] that hold keys some query token can see.

    Pure index bookkeeping used by input poisoning: keys j with
    p_0 - W + 1 <= j <= L - 1 (p_0 = L - T), or 0 <= j <= L - 1 when W <= 0.
    """
    lo = 0 if window <= 0 else max(0, seq_len - q_tokens - window + 1)
    return lo // page_size, (seq_len - 1) // page_size


def poison_unused(case: DecodeCase, value: float = float("nan")) -> DecodeCase:
    """Return a copy whose never-visible cache slots hold ``value``.

    Poisoned: every page no sequence can see, the slots past seq_len in each
    sequence's last page, and the slots before the window start in its first
    visible page.  A correct kernel's output does not depend on them.
    """
    k = case.k_cache.clone()
    v = case.v_cache.clone()
    P = case.page_size
    used = torch.zeros(k.shape[0], dtype=torch.bool)
    bt = case.block_table.cpu()
    lens = case.seq_lens.cpu().tolist()
    T = case.q_tokens
    for b, L in enumerate(lens):
        first, last = visible_page_range(L, T, case.window, P)
        for lp in range(first, last + 1):
            used[int(bt[b, lp])] = True
    unused = (~used).nonzero().flatten().to(k.device)
    k[unused] = value
    v[unused] = value
    for b, L in enumerate(lens):
        first, last = visible_page_range(L, T, case.window, P)
        tail = L - last * P
        if tail < P:
            pg = int(bt[b, last])
            k[pg, :, tail:] = value
            v[pg, :, tail:] = value
        lo = 0 if case.window <= 0 else max(0, L - T - case.window + 1)
        head = lo - first * P
        if head > 0:
            pg = int(bt[b, first])
            k[pg, :, :head] = value
            v[pg, :, :head] = value
    return dataclasses.replace(case, k_cache=k, v_cache=v)


def to_e4m3(case: DecodeCase):
    """An E4M3 copy of the case's KV cache: one scale per KV head (the head's
    largest |value| over the pool / 448, the largest finite E4M3 value) and
    the codes of value / scale, rounded to nearest even by torch's float8
    conversion.  Returns (k_codes uint8, v_codes uint8, k_scale fp32 [Hkv],
    v_scale fp32 [Hkv]) on the case's device."""
    out = []
    for pool in (case.k_cache, case.v_cache):
        x = pool.float()
        amax = x.abs().amax(dim=(0, 2, 3)).clamp_min(1e-30)
        scale = (amax / 448.0).to(torch.float32)
        codes = (x / scale.view(1, -1, 1, 1)).to(torch.float8_e4m3fn).view(torch.uint8)
        out.append((codes.contiguous(), scale.contiguous()))
    (kc, ks), (vc, vs) = out
    return kc, vc, ks, vs
