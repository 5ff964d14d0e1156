"""ctypes loader for libspkv.so (the C ABI declared in include/spkv.h).

Argument marshalling only: every step of the decode path runs in the CUDA
kernels of libspkv.so.  There is no fallback: if the library is missing this
module raises at import time.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libspkv.so")

SPKV_OK = 0
STATUS_NAMES = {0: "SPKV_OK", 1: "SPKV_ERR_INVALID_ARG", 2: "SPKV_ERR_UNSUPPORTED", 3: "SPKV_ERR_WORKSPACE",
                4: "SPKV_ERR_CUDA"}
DEVERR_PAGE_ID, DEVERR_BITS, DEVERR_RECORD, DEVERR_CTX, DEVERR_TIMEOUT, DEVERR_RADIUS = 1, 2, 4, 8, 16, 32

# Exported entry points (must match include/spkv.h).
EXPORTS = (
    "spkv_status_string",
    "spkv_encode_keys",
    "spkv_decode_default_splits",
    "spkv_decode_workspace_bytes",
    "spkv_decode_attention",
    "spkv_dense_decode",
    "spkv_decompress_then_dot",
    "spkv_debug_logits",
    "spkv_decode_attention_static_ws",
    "spkv_decode_attention_ex",
    "spkv_debug_logits_ex",
    "spkv_decode_attention_append",
    "spkv_decode_attention_partial",
    "spkv_merge_partials",
    "spkv_debug_wait_timeout",
    "spkv_rdr_workspace_bytes",
    "spkv_rdr_plan",
    "spkv_encode_keys_packed",
    "spkv_nonuniform_tables",
    "spkv_encode_keys_nonuniform",
    "spkv_decode_nonuniform_workspace_bytes",
    "spkv_decode_attention_nonuniform",
)
PARTIAL_FLOATS = 132  # floats per (sequence, query head) shard record
DECODE_EXACT_Q = 1  # SPKV_DECODE_EXACT_Q
STATIC_WS_BYTES = 16 * 1024 * 1024  # SPKV_STATIC_WS_BYTES
RDR_INFEASIBLE, RDR_PAGES, RDR_BAD_RANGE = 1, 2, 4  # SPKV_RDR_* status bits


class SpkvError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what} failed: {STATUS_NAMES.get(status, status)}")
        self.status = status


class SpkvCacheC(ctypes.Structure):
    """Mirror of `spkv_cache` (host struct of device pointers)."""

    _fields_ = [
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("page_size", ctypes.c_int32),
        ("num_pages", ctypes.c_int32),
        ("code_arena", ctypes.c_void_p),
        ("code_arena_bytes", ctypes.c_uint64),
        ("hdr", ctypes.c_void_p),
        ("rad_lo_log2", ctypes.c_void_p),
        ("rad_step_log2", ctypes.c_void_p),
        ("v_pages", ctypes.c_void_p),
        ("keep_mask", ctypes.c_void_p),
        ("err_flags", ctypes.c_void_p),
        ("tiers", ctypes.c_uint32),
    ]


_P = ctypes.c_void_p
_I = ctypes.c_int32


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python compressed_kv_decode_ada_b200/build.py` "
            "(the CUDA library is required; there is no CPU fallback)")
    L = ctypes.CDLL(LIB_PATH)
    L.spkv_status_string.restype = ctypes.c_char_p
    L.spkv_status_string.argtypes = [ctypes.c_int]
    L.spkv_encode_keys.restype = ctypes.c_int
    L.spkv_encode_keys.argtypes = [ctypes.POINTER(SpkvCacheC), _P, _P, _P, _I, _I, _P, _I, _P]
    L.spkv_decode_default_splits.restype = ctypes.c_int32
    L.spkv_decode_default_splits.argtypes = [_I, _I, _I]
    L.spkv_decode_workspace_bytes.restype = ctypes.c_size_t
    L.spkv_decode_workspace_bytes.argtypes = [_I, _I, _I, _I, _I]
    L.spkv_decode_attention.restype = ctypes.c_int
    L.spkv_decode_attention.argtypes = [ctypes.POINTER(SpkvCacheC), _P, _I, _I, _P, _I, _P, _I, _P, _I, _P,
                                        ctypes.c_size_t, _I, _P]
    L.spkv_dense_decode.restype = ctypes.c_int
    L.spkv_dense_decode.argtypes = [_P, _P, _I, _I, _P, _P, _P, _I, _I, _P, _I, _P, _I, _P, _I, _P,
                                    ctypes.c_size_t, _I, _P]
    L.spkv_decompress_then_dot.restype = ctypes.c_int
    L.spkv_decompress_then_dot.argtypes = [ctypes.POINTER(SpkvCacheC), _P, _P, _I, _I, _P, _I, _P, _I, _P, _I,
                                           _P, ctypes.c_size_t, _I, _P]
    L.spkv_decode_attention_static_ws.restype = ctypes.c_int
    L.spkv_decode_attention_static_ws.argtypes = [ctypes.POINTER(SpkvCacheC), _P, _I, _I, _P, _I, _P, _I, _P, _I,
                                                  _I, _P]
    L.spkv_debug_logits.restype = ctypes.c_int
    L.spkv_debug_logits.argtypes = [ctypes.POINTER(SpkvCacheC), _P, _I, _I, _P, _I, _P, _I, _P, _P]
    L.spkv_decode_attention_ex.restype = ctypes.c_int
    L.spkv_decode_attention_ex.argtypes = [ctypes.POINTER(SpkvCacheC), _P, _I, _I, _P, _I, _P, _I, _P, _I, _P,
                                           ctypes.c_size_t, _I, ctypes.c_uint32, _P]
    L.spkv_decode_attention_append.restype = ctypes.c_int
    L.spkv_decode_attention_append.argtypes = [ctypes.POINTER(SpkvCacheC), _P, _P, _P, _I, _I, _P, _I, _P, _I, _P,
                                               _I, _P, ctypes.c_size_t, _I, ctypes.c_uint32, _P]
    L.spkv_decode_attention_partial.restype = ctypes.c_int
    L.spkv_decode_attention_partial.argtypes = [ctypes.POINTER(SpkvCacheC), _P, _I, _I, _P, _I, _P, _I, _P, _P,
                                                ctypes.c_size_t, _I, ctypes.c_uint32, _P]
    L.spkv_merge_partials.restype = ctypes.c_int
    L.spkv_merge_partials.argtypes = [_P, _I, _I, _I, _P, _I, _P]
    L.spkv_debug_wait_timeout.restype = ctypes.c_int
    L.spkv_debug_wait_timeout.argtypes = [_P, _P, ctypes.c_uint64, _P]
    L.spkv_debug_logits_ex.restype = ctypes.c_int
    L.spkv_debug_logits_ex.argtypes = [ctypes.POINTER(SpkvCacheC), _P, _I, _I, _P, _I, _P, _I, _P, ctypes.c_uint32,
                                       _P]
    L.spkv_rdr_workspace_bytes.restype = ctypes.c_size_t
    L.spkv_rdr_workspace_bytes.argtypes = [ctypes.c_int64]
    L.spkv_rdr_plan.restype = ctypes.c_int
    L.spkv_rdr_plan.argtypes = [_P, _P, _I, ctypes.c_int64, _I, _P, _P, _P, ctypes.c_uint32, _I, _P, _P, _P, _P,
                                _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
    L.spkv_encode_keys_packed.restype = ctypes.c_int
    L.spkv_encode_keys_packed.argtypes = [ctypes.POINTER(SpkvCacheC), _P, _P, _P, _I, ctypes.c_int64, _P, _P, _I,
                                          _P]
    L.spkv_nonuniform_tables.restype = ctypes.c_int
    L.spkv_nonuniform_tables.argtypes = [_I, _I, _P, _P, _P]
    L.spkv_encode_keys_nonuniform.restype = ctypes.c_int
    L.spkv_encode_keys_nonuniform.argtypes = [ctypes.POINTER(SpkvCacheC), _P, _P, _P, _I, _I, _P, _I, _I, _P, _P]
    L.spkv_decode_nonuniform_workspace_bytes.restype = ctypes.c_size_t
    L.spkv_decode_nonuniform_workspace_bytes.argtypes = [_I, _I, _I, _I, _I, _I]
    L.spkv_decode_attention_nonuniform.restype = ctypes.c_int
    L.spkv_decode_attention_nonuniform.argtypes = [ctypes.POINTER(SpkvCacheC), _P, _I, _I, _P, _I, _P, _I, _I, _P, _P,
                                                   _P, _P, _I, _P, _P, ctypes.c_size_t, _I, _P]
    return L


lib = _load()


def check(status: int, what: str) -> None:
    if status != SPKV_OK:
        raise SpkvError(status, what)
