"""Quantized-KV scaled-dot-product attention for NVIDIA B200 (sm_100a).

The compute path lives in the C-ABI library ``libqkv.so`` (CUDA kernels under
``csrc/``); :mod:`quantized_kv_attention_split_b200.qkv` is the Python binding.
Importing this package loads nothing; the binding loads the library on first
use and raises if it is missing.
"""
__all__ = ["qkv", "synthetic"]
