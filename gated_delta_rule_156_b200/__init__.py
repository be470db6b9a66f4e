"""Kimi Delta Attention (KDA) forward for B200 (sm_100a).

The kernels live in the in-tree ``libkda.so`` (sources under ``csrc/``, public
C ABI in ``include/kda.h``); this package only marshals torch tensors into
that ABI.
"""
from .kda import (KdaError, KdaShape, chunk_fwd, library, library_path,  # noqa: F401
                  recurrent_step)

__all__ = ["chunk_fwd", "recurrent_step", "library", "library_path",
           "KdaError", "KdaShape"]
