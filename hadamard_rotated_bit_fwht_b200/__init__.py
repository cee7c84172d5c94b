"""Hadamard-rotated low-bit KV cache for NVIDIA B200 (sm_100a).

The compute lives in libkvq.so (C ABI: include/kvq.h), built from csrc/ by
``python -m hadamard_rotated_bit_fwht_b200.build``; ``kvq`` is its Python
binding and ``synth`` the seeded synthetic-input generator.
"""
__all__ = ["kvq", "synth", "build"]
