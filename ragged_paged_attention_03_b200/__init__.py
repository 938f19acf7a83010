"""Ragged paged attention on NVIDIA B200 (sm_100a).

The compute lives in ``librpa_b200.so`` (CUDA kernels plus a C ABI declared in
``include/rpa.h``); ``binding`` marshals torch tensors into that ABI and
nothing else.  ``inputs`` draws the seeded synthetic workloads.
"""
__all__ = ["binding", "inputs"]
