"""B200-native (sm_100a) Kimi-K3 MoE feed-forward layer.

The compute runs in the C-ABI library ``libmoe_sm100.so`` built from ``csrc/``;
``api`` is a thin ctypes binding to it (argument marshalling only).  ``synth``
draws the seeded synthetic workloads.
"""
__all__ = ["api", "synth"]
