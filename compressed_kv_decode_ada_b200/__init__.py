"""compressed_kv_decode_ada_b200: Spherical KV angle-domain attention (ADA)
paged decode on NVIDIA B200 (sm_100a).

The compute lives in libspkv.so (C ABI, include/spkv.h); this package is its
thin Python binding plus seeded synthetic workloads.  Importing it fails
loudly when the CUDA library has not been built.
"""
from ._lib import LIB_PATH, SpkvError, lib  # noqa: F401
from .cache import SpkvCache  # noqa: F401
from .ops import (alloc_workspace, debug_logits, decode_attention, decode_attention_append,  # noqa: F401
                  decode_attention_nonuniform, decode_attention_partial, decode_attention_static_ws,
                  decompress_then_dot, default_splits, dense_decode, encode_keys, encode_keys_nonuniform,
                  encode_keys_packed, merge_partials, nonuniform_tables, rdr_plan, rdr_workspace_bytes,
                  workspace_bytes)
from .rdr import allocate_packed, build_packed_cache  # noqa: F401
