"""paired_heads_b200 -- B200-native forward pass of causal, rotary-embedded, varlen multi-head
attention, including the paired-head variant of the modded-nanogpt "Paired Head Attention" record.

The compute lives in the C-ABI library ``libpha.so`` (hand-written sm_100a CUDA, declared in
``include/pha.h``). ``paired_heads_b200.pha`` is the thin ctypes binding over it; importing it
fails loudly if the library is missing. ``paired_heads_b200.synth`` draws the seeded synthetic
workloads. Importing this package itself loads nothing.
"""
__all__ = ["pha", "synth"]
