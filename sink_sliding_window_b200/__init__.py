"""B200-native sink attention: causal grouped-query attention with a learned
per-head attention sink, sliding windows and packed documents.

The compute path is the C-ABI library ``libsinkattn.so`` (hand-written CUDA
for sm_100a) declared in ``include/sink_attn.h``; ``sink_sliding_window_b200.ops``
is a thin ctypes binding over it.  Loading fails loudly if the library has
not been built: there is no CPU fallback.
"""
