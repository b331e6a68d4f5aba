"""B200-native FP8 block-scaled GEMMs (dense NT, contiguous and masked M-grouped).

The compute path is the C-ABI library ``libdg.so`` built from ``csrc/``; the
Python layer in :mod:`moe_grouped_gemm_05_b200.binding` only marshals
arguments.  Importing this package does not load the library; the first call
does, and raises if it is missing.
"""
__all__ = ["binding", "synth"]
