"""ctypes loader and prototypes for libcsa.so (the C ABI in include/csa.h).

The library is built in-tree by ``long_context_decode_c4a_b200.build``. Loading fails loudly if
it is missing: there is no fallback implementation.
"""

from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_float, c_int, c_int64, c_size_t, c_void_p

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libcsa.so")

CSA_OK = 0
CSA_ERR_INVALID_ARG = 1
CSA_ERR_UNSUPPORTED = 2
CSA_ERR_CUDA = 3
CSA_ERR_TIMEOUT = 4
CSA_ERR_WORKSPACE = 5
CSA_ERR_BOUNDS = 6

CSA_WS_INDEXER_TOPK = 1
CSA_WS_SPARSE_ATTN = 2
CSA_WS_HCA_ATTN = 3
CSA_WS_DECODE_FUSED = 4
CSA_WS_HCA_DECODE_FUSED = 5
CSA_WS_OUTPUT_PROJ = 6
CSA_WS_Q_PROJ = 7


class CompressorCfg(ctypes.Structure):
    _fields_ = [("ratio", c_int), ("overlap", c_int), ("d", c_int), ("rope_dim", c_int),
                ("rope_base", c_float), ("eps", c_float)]


class DecodeArgs(ctypes.Structure):
    """Mirror of csa_decode_args."""
    _fields_ = [
        ("B", c_int), ("H", c_int), ("d", c_int), ("rope_dim", c_int), ("H_I", c_int), ("d_I", c_int),
        ("ratio", c_int), ("window", c_int), ("topk", c_int),
        ("rope_base", c_float), ("eps", c_float), ("scale", c_float),
        ("pos", c_void_p), ("kv", c_void_p), ("score", c_void_p), ("idx_kv", c_void_p), ("idx_score", c_void_p),
        ("win_kv", c_void_p), ("q", c_void_p), ("q_idx", c_void_p), ("w", c_void_p), ("sink", c_void_p),
        ("gamma", c_void_p), ("idx_gamma", c_void_p),
        ("state_kv", c_void_p), ("state_score", c_void_p), ("idx_state_kv", c_void_p), ("idx_state_score", c_void_p),
        ("cache", c_void_p), ("cache_bstride", c_int64), ("idx_cache", c_void_p), ("idx_bstride", c_int64),
        ("max_entries", c_int), ("ring", c_void_p), ("ring_bstride", c_int64), ("ring_cap", c_int),
        ("topk_idx", c_void_p), ("cache_f32", c_void_p), ("out", c_void_p), ("out_is_f32", c_int),
        ("ws", c_void_p), ("ws_bytes", c_size_t), ("stage_events", c_void_p),
    ]


class HcaDecodeArgs(ctypes.Structure):
    """Mirror of hca_decode_args."""
    _fields_ = [
        ("B", c_int), ("H", c_int), ("d", c_int), ("rope_dim", c_int), ("ratio", c_int), ("window", c_int),
        ("rope_base", c_float), ("eps", c_float), ("scale", c_float),
        ("pos", c_void_p), ("kv", c_void_p), ("score", c_void_p), ("win_kv", c_void_p), ("q", c_void_p),
        ("sink", c_void_p), ("gamma", c_void_p), ("state_kv", c_void_p), ("state_score", c_void_p),
        ("cache", c_void_p), ("cache_bstride", c_int64), ("max_entries", c_int),
        ("ring", c_void_p), ("ring_bstride", c_int64), ("ring_cap", c_int),
        ("cache_f32", c_void_p), ("out", c_void_p), ("out_is_f32", c_int), ("ws", c_void_p), ("ws_bytes", c_size_t),
        ("stage_events", c_void_p),
    ]


# name -> (restype, argtypes)
PROTOTYPES = {
    "csa_status_string": (c_char_p, [c_int]),
    "csa_last_error": (c_char_p, []),
    "csa_version": (c_int, []),
    "csa_workspace_size": (c_int, [c_int, c_int, c_int, c_int, c_int, POINTER(c_size_t)]),
    "csa_state_reset": (c_int, [POINTER(CompressorCfg), c_int, c_void_p, c_void_p, c_void_p]),
    "csa_compress": (c_int, [POINTER(CompressorCfg), c_int, c_int, c_void_p, c_void_p, c_void_p, c_void_p,
                             c_void_p, c_void_p, c_void_p, c_int64, c_int, c_void_p, c_void_p]),
    "csa_indexer_topk": (c_int, [c_int, c_int, c_int, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p,
                                 c_void_p, c_int64, c_int, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "csa_sparse_attn": (c_int, [c_int, c_int, c_int, c_int, c_int, c_float, c_float, c_void_p, c_void_p,
                                c_void_p, c_int64, c_int, c_int, c_void_p, c_int64, c_int, c_void_p, c_int,
                                c_void_p, c_void_p, c_int, c_void_p, c_size_t, c_void_p]),
    "hca_attn": (c_int, [c_int, c_int, c_int, c_int, c_int, c_float, c_float, c_int, c_void_p, c_void_p,
                         c_void_p, c_int64, c_int, c_int, c_void_p, c_int64, c_int, c_void_p, c_void_p, c_int,
                         c_void_p, c_size_t, c_void_p]),
    "csa_decode_fused": (c_int, [POINTER(DecodeArgs), c_void_p]),
    "hca_decode_fused": (c_int, [POINTER(HcaDecodeArgs), c_void_p]),
    "csa_get_device_status": (c_int, [c_void_p, c_void_p, POINTER(c_int)]),
    "csa_watchdog_selftest": (c_int, [c_void_p, c_size_t, ctypes.c_longlong, c_void_p]),
    "csa_indexer_topk_noalloc": (c_int, [c_int, c_int, c_int, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p,
                                         c_void_p, c_int64, c_int, c_void_p, c_void_p]),
    "csa_output_projection": (c_int, [c_int, c_int, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p, c_void_p,
                                      c_void_p, c_void_p, c_size_t, c_void_p]),
    "csa_indexer_scores": (c_int, [c_int, c_int, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p, c_void_p,
                                   c_int64, c_int, c_void_p, c_void_p, c_size_t, c_void_p]),
    "csa_topk": (c_int, [c_int, c_int, c_int, c_int, c_void_p, c_void_p, c_int, c_void_p, c_void_p, c_size_t,
                         c_void_p]),
    "csa_linear": (c_int, [c_int, c_int, c_int, c_void_p, c_void_p, c_void_p, c_int, c_void_p, c_size_t, c_void_p]),
    "csa_q_projection": (c_int, [c_int, c_int, c_int, c_int, c_int, c_int, c_float, c_float, c_void_p, c_void_p,
                                 c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                                 c_void_p]),
    "csa_window_projection": (c_int, [c_int, c_int, c_int, c_int, c_float, c_void_p, c_void_p, c_void_p, c_void_p,
                                      c_void_p, c_size_t, c_void_p]),
}

_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libcsa.so once and attach the prototypes. Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with `python -m long_context_decode_c4a_b200.build` "
            "(the CSA kernels have no non-CUDA implementation)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in PROTOTYPES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


class CsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        lib = load()
        msg = lib.csa_status_string(status).decode()
        detail = lib.csa_last_error().decode()
        super().__init__(f"{where}: {msg} ({status}){': ' + detail if detail else ''}")
        self.status = status


def check(status: int, where: str) -> None:
    if status != CSA_OK:
        raise CsaError(status, where)
