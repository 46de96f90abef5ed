"""B200 (sm_100a) rotated W4G128 linear layer (ParoQuant inference hot path).

The compute lives in libparo.so (C ABI, include/paro.h); `binding` marshals
torch tensors into it. Importing this package does not load the library;
the first binding call does, and fails loudly if it is missing.
"""
__all__ = ["binding", "build"]
