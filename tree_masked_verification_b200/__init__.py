"""Hybrid Tree Attention (LongSpec verification attention) on B200.

Importing the package loads nothing: ``inputs`` holds the seeded workload
generator and ``hta`` the ctypes binding to ``liblongspec_hta.so``, which is
loaded on first use and fails loudly if it is missing.
"""
__all__ = ["inputs", "hta"]
