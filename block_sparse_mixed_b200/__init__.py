"""Block-sparse mixed-precision causal attention (TriAttention-style) for B200.

The compute path is a C-ABI CUDA library (``libtria.so``, sm_100a) with three
calls -- ``tria_quantize_kv``, ``tria_prefill`` and ``tria_decode`` -- and a thin
ctypes binding in :mod:`block_sparse_mixed_b200.tria`. Importing this package
loads nothing; the binding loads the library on first use and raises if it is
missing. There is no CPU fallback.
"""
__all__ = ["tria", "workloads"]
