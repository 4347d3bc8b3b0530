"""B200-native Infini-attention layer forward (compressive memory, segment recurrence).

The compute path is the CUDA library ``libinfini_attn.so`` (hand-written
sm_100a kernels behind a C ABI, declared in ``include/infini_attn.h``).
``api`` is its thin Python binding; ``synth`` and ``configs`` describe the
seeded synthetic workloads.
"""

__all__ = ["api", "configs", "synth"]
