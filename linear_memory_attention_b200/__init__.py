"""B200-native linear-memory relation-KL kernel (LinearARD's Phase 1 / Phase 2).

The compute path is the C-ABI library ``liblard.so`` (hand-written CUDA for
sm_100a); ``linear_memory_attention_b200.lard`` is its thin ctypes binding.
Importing the package itself loads nothing, so that the synthetic input
generator (``synth``) is usable without a GPU; the binding raises if the
library is missing.
"""
__all__ = ["lard", "synth"]
