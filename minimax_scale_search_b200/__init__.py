"""B200-native exact minimax FP16 group-scale selection (W4, group size 128).

The CUDA library (``libcq.so``, C ABI in ``include/cq.h``) is loaded by
``minimax_scale_search_b200.cq``; ``synth`` holds the seeded input generators.
"""

__all__ = ["cq", "synth"]
