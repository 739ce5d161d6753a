"""B200-native forward pass of a capacity-limited Mixture-of-Experts layer.

The layer's four stages (router softmax/top-k, capacity-limited dispatch with token dropping,
per-expert FFN, router-weighted combine onto the residual) run in hand-written sm_100a CUDA
kernels behind the C-ABI library ``libmoe_b200.so``.  :mod:`.moe` is its thin ctypes binding;
it raises if the library is missing or no GPU is present.  There is no CPU fallback.
"""

__all__ = ["moe", "inputs"]
