"""fp64 CPU oracle for relative-bias GQA decode attention and the KV-cache
producer step that feeds it.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py`` (its ``cpu_baseline`` leg and its ``--impl reference`` arm) may
import this package.  The product package ``relative_bias_gqa_b200`` never
imports it, and the two share no code: the oracle is written from the
definition of the operation, independently of the CUDA path.

Every function here is pinned by ``tests/test_oracle.py`` against brute
force, closed forms, invariants and a textbook library special case.
"""

from .rel_attn_ref import (  # noqa: F401
    EXACT_BUCKETS,
    MAX_DISTANCE,
    log_bucket_edges,
    bucket_of_distance,
    attend_at_positions,
    rel_attn_decode_ref,
    rel_attn_decode_split_ref,
    rel_attn_decode_bruteforce,
    e4m3_to_float,
    dequant_kv,
    rel_attn_decode_fp8kv_ref,
)
from .kv_write_ref import (  # noqa: F401
    short_conv_ref,
    short_conv_fp32,
    bf16_rne,
    e4m3_rne_satfinite,
    kv_write_ref,
)
