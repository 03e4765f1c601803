"""Lightning Attention-2 causal linear attention for B200 (sm_100a).

The compute lives in ``libla2.so`` (hand-written CUDA behind a C ABI declared in
``include/la2.h``); ``linear_attention_la2_b200.la2`` is the thin ctypes binding.
Importing this package does not load the library; ``la2`` does, and fails loudly
when it is missing.
"""

__all__ = ["inputs"]
