"""Exact IO-aware attention for B200 (sm_100a).

The compute lives in ``libfa.so`` (CUDA, built from ``csrc/``); ``binding`` marshals
torch tensors into its C ABI.  ``inputs`` and ``traffic`` are host-side helpers.
"""
