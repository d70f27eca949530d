"""Seeded synthetic KV-cache inputs shared by the tests, the oracle checks and bench.py.

This package only draws input tensors. It holds none of the codec's arithmetic
(no factorisation, rotation, quantiser or allocator), so both the CUDA path and
the CPU oracle may be fed from it without sharing method code.
"""
from .kv import CONFIGS, config, gen_layer_tensor, gen_cache_numpy, gen_cache_torch, bf16_bytes  # noqa: F401
