"""Causal packed-document flash attention for NVIDIA B200 (sm_100a).

The product is ``libfapk.so`` (C ABI: ``include/fapk.h``) built from
``csrc/``; ``fapk`` is its thin Python binding and ``workloads`` the seeded
synthetic input generator.  Importing the package does not load the CUDA
library; the first call through ``fapk`` does, and fails loudly if it is
missing.
"""
__all__ = ["fapk", "workloads", "build"]
