"""Routed MoE layer with a GPU-resident (layer, expert) LRU slot cache for NVIDIA B200.

The layer runs in libmoe.so (CUDA for sm_100a, C ABI in include/moe.h);
``api`` is its argument-marshalling Python face, ``workloads`` draws seeded
synthetic inputs, ``build`` compiles the library in-tree.
"""
__all__ = ["api", "workloads", "build"]
