"""B200-native relative-bias GQA decode attention.

The compute path is a CUDA library (``librel_attn.so``, built for sm_100a from
``csrc/``) behind a C ABI (``include/rel_attn.h``); ``rel_attn`` is the thin
ctypes binding over it.  Importing the package does not load the library;
``from relative_bias_gqa_b200 import rel_attn`` does, and fails loudly when it
has not been built.
"""

__all__ = ["rel_attn", "workloads"]
