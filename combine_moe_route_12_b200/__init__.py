"""B200-native (sm_100a) hot path of an expert-parallel MoE layer.

Router top-k -> per-expert capacity clip -> expert-contiguous, EP-rank-grouped
dispatch layout -> row permute -> grouped SwiGLU FFN (tcgen05/TMEM) -> weighted
combine, plus a two-stream chunked entry point.  The kernels live in the C-ABI
library ``libmoe_b200.so`` (``include/moe_b200.h``); ``combine_moe_route_12_b200.moe``
is the thin ctypes binding over it.  ``workload`` holds the seeded input
generators and nothing of the layer's arithmetic.
"""
__all__ = ["workload"]
