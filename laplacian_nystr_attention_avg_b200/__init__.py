"""Laplacian-kernel Nystrom attention (LaplacianFormer) on B200 (sm_100a).

The compute path is the C-ABI library ``liblfa.so`` built from ``csrc/``;
``lfa`` is its thin ctypes binding. Importing this package loads nothing: the
library is opened on first use and a missing library is an error, never a
fallback.
"""
__all__ = ["inputs", "lfa"]
