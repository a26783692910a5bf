"""B200-native (sm_100a) compressed-sparse-attention layer of DeepSeek-V4-Pro.

libcsa.so holds every kernel (C4A/C128A compressor, lightning indexer on tcgen05, radix-select
top-k, sparse MQA with sink on tcgen05, HCA attention, fused decode) behind the C ABI in
include/csa.h. This package is its thin Python binding: `ops` marshals torch tensors into the
ABI, `build` compiles the library in-tree.
"""

from ._lib import CsaError, load  # noqa: F401
from . import ops  # noqa: F401

__all__ = ["CsaError", "load", "ops"]
