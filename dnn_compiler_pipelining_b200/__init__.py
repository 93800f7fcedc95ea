"""B200-native fused attention forward (causal / non-causal, grouped-query heads).

The compute path is the C-ABI library ``libattn_b200.so`` (hand-written sm_100a
kernels); ``dnn_compiler_pipelining_b200.attn`` is its thin ctypes binding.
Importing this package does not load the library; the first call does, and
fails loudly if it has not been built.
"""
__all__ = ["attn", "inputs"]
