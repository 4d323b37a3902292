"""W4A8 MoE expert FFN for NVIDIA B200 (sm_100a).

The compute runs in the CUDA library ``libw4a8.so`` built from ``csrc/``; the
Python layer in :mod:`.binding` only marshals torch tensors into its C ABI.
"""

from . import synth  # noqa: F401  (seeded input generators)

__all__ = ["synth"]
