"""Packed ternary weight matmul for NVIDIA B200 (sm_100a).

The CUDA library and its thin ctypes binding live in
`packed_weight_matmul_b200.tq`; importing this package alone loads nothing.
"""
__all__ = ["tq", "inputs"]
