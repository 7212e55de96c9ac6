"""B200-native Lizard hybrid attention (gated linear + sliding window + meta tokens).

The compute path is the CUDA library ``liblizard.so`` (built from ``csrc/``),
reached through :mod:`gated_linear_sliding_chunkwise_b200.lizard`.  Importing
this package does not load the library; importing ``.lizard`` does, and fails
loudly when it is missing.
"""

__all__ = ["lizard", "synth"]
