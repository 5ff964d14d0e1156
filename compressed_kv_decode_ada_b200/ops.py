"""Python entry points with the C ABI's names; argument marshalling only.

Each function checks shapes/dtypes/devices of torch tensors, then calls the
entry point of libspkv.so of the same name on the current CUDA stream.  All
arithmetic of the decode path happens in the CUDA kernels.
"""
from __future__ import annotations

import ctypes

import torch

from ._lib import DECODE_EXACT_Q, PARTIAL_FLOATS, check, lib
from .cache import HEAD_DIM, SpkvCache


def _stream(stream=None) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t, dtype, name, dims=None):
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dims is not None and t.dim() != dims:
        raise ValueError(f"{name} must have {dims} dims, got {tuple(t.shape)}")


def default_splits(B: int, num_kv_heads: int, max_ctx: int) -> int:
    return int(lib.spkv_decode_default_splits(B, num_kv_heads, max_ctx))


def workspace_bytes(B: int, num_q_heads: int, num_kv_heads: int, max_ctx: int, num_splits: int = 0) -> int:
    return int(lib.spkv_decode_workspace_bytes(B, num_q_heads, num_kv_heads, max_ctx, num_splits))


def alloc_workspace(B, num_q_heads, num_kv_heads, max_ctx, num_splits=0, device="cuda") -> torch.Tensor:
    n = workspace_bytes(B, num_q_heads, num_kv_heads, max_ctx, num_splits)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device)


def encode_keys(cache: SpkvCache, keys: torch.Tensor, start_pos: torch.Tensor, block_table: torch.Tensor,
                values: torch.Tensor | None = None, stream=None) -> None:
    """spkv_encode_keys: keys/values [B, n_new, H_kv, 128] bf16 -> page slots."""
    _need(keys, torch.bfloat16, "keys", 4)
    B, n_new, hkv, d = keys.shape
    if hkv != cache.num_kv_heads or d != HEAD_DIM:
        raise ValueError("keys must be [B, n_new, H_kv, 128]")
    if values is not None:
        _need(values, torch.bfloat16, "values", 4)
        if values.shape != keys.shape:
            raise ValueError("values must match keys")
    _need(start_pos, torch.int32, "start_pos", 1)
    _need(block_table, torch.int32, "block_table", 2)
    if start_pos.shape[0] != B or block_table.shape[0] != B:
        raise ValueError("start_pos / block_table batch mismatch")
    c = cache.c_struct()
    check(lib.spkv_encode_keys(ctypes.byref(c), _ptr(keys), _ptr(values), _ptr(start_pos), B, n_new,
                               _ptr(block_table), block_table.shape[1], _stream(stream)), "spkv_encode_keys")


def encode_keys_nonuniform(cache: SpkvCache, keys: torch.Tensor, start_pos: torch.Tensor, block_table: torch.Tensor,
                           bits: int, edge_cos: torch.Tensor, values: torch.Tensor | None = None,
                           stream=None) -> None:
    """spkv_encode_keys_nonuniform: as encode_keys, with the non-uniform angle
    quantiser at b = bits (every page must have that width); edge_cos: the
    [126, 2^b - 1] fp64 polar edge cosines (nonuniform_tables(128, bits)[0])
    on the device."""
    _need(keys, torch.bfloat16, "keys", 4)
    B, n_new, hkv, d = keys.shape
    if hkv != cache.num_kv_heads or d != HEAD_DIM:
        raise ValueError("keys must be [B, n_new, H_kv, 128]")
    if values is not None:
        _need(values, torch.bfloat16, "values", 4)
        if values.shape != keys.shape:
            raise ValueError("values must match keys")
    _need(start_pos, torch.int32, "start_pos", 1)
    _need(block_table, torch.int32, "block_table", 2)
    _need(edge_cos, torch.float64, "edge_cos", 2)
    if start_pos.shape[0] != B or block_table.shape[0] != B:
        raise ValueError("start_pos / block_table batch mismatch")
    if tuple(edge_cos.shape) != (HEAD_DIM - 2, (1 << bits) - 1):
        raise ValueError("edge_cos must be [126, 2^b - 1]")
    c = cache.c_struct()
    check(lib.spkv_encode_keys_nonuniform(ctypes.byref(c), _ptr(keys), _ptr(values), _ptr(start_pos), B, n_new,
                                          _ptr(block_table), block_table.shape[1], int(bits), _ptr(edge_cos),
                                          _stream(stream)), "spkv_encode_keys_nonuniform")


def decode_attention_nonuniform(cache: SpkvCache, q: torch.Tensor, block_table: torch.Tensor,
                                ctx_lens: torch.Tensor, max_ctx: int, bits: int, edge_cos: torch.Tensor,
                                mid_cos: torch.Tensor, mid_sin: torch.Tensor, out=None, out_dtype=torch.float32,
                                logits: torch.Tensor | None = None, ws=None, num_splits: int = 0,
                                stream=None) -> torch.Tensor:
    """spkv_decode_attention_nonuniform: ADA decode of a cache written by
    encode_keys_nonuniform at b = bits; the three tables are
    nonuniform_tables(128, bits) as fp64 device tensors.  logits (optional):
    [B, Hq, max_ctx] fp32, filled for t < ctx_lens."""
    _batch_checks(q, block_table, ctx_lens)
    for t, name, shape in ((edge_cos, "edge_cos", (HEAD_DIM - 2, (1 << bits) - 1)),
                           (mid_cos, "mid_cos", (HEAD_DIM - 2, 1 << bits)),
                           (mid_sin, "mid_sin", (HEAD_DIM - 2, 1 << bits))):
        _need(t, torch.float64, name, 2)
        if tuple(t.shape) != shape:
            raise ValueError(f"{name} must be {shape}")
    B, Hq, _ = q.shape
    out = _out_buffer(out, B, Hq, out_dtype, q.device)
    if logits is not None:
        _need(logits, torch.float32, "logits", 3)
    need = int(lib.spkv_decode_nonuniform_workspace_bytes(B, Hq, cache.num_kv_heads, int(max_ctx), int(num_splits),
                                                          int(bits)))
    if need == 0:
        raise ValueError("invalid shape for spkv_decode_nonuniform_workspace_bytes")
    if ws is None:
        ws = torch.empty(need + 256, dtype=torch.uint8, device=q.device)
    base = ws.data_ptr()
    off = (-base) % 256  # the entry point wants a 256-byte aligned workspace
    c = cache.c_struct()
    check(lib.spkv_decode_attention_nonuniform(
        ctypes.byref(c), _ptr(q), B, Hq, _ptr(block_table), block_table.shape[1], _ptr(ctx_lens), int(max_ctx),
        int(bits), _ptr(edge_cos), _ptr(mid_cos), _ptr(mid_sin), _ptr(out), 1 if out.dtype == torch.bfloat16 else 0,
        _ptr(logits), ctypes.c_void_p(base + off), ws.numel() - off, int(num_splits), _stream(stream)),
        "spkv_decode_attention_nonuniform")
    return out


def _out_buffer(out, B, Hq, out_dtype, device):
    if out is None:
        out = torch.empty((B, Hq, HEAD_DIM), dtype=out_dtype, device=device)
    if out.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("out must be float32 or bfloat16")
    _need(out, out.dtype, "out", 3)
    return out


def _batch_checks(q, block_table, ctx_lens):
    _need(q, torch.bfloat16, "q", 3)
    _need(block_table, torch.int32, "block_table", 2)
    _need(ctx_lens, torch.int32, "ctx_lens", 1)
    B = q.shape[0]
    if block_table.shape[0] != B or ctx_lens.shape[0] != B:
        raise ValueError("batch mismatch between q, block_table and ctx_lens")
    if q.shape[2] != HEAD_DIM:
        raise ValueError("q must be [B, Hq, 128]")


def _ws(ws, B, Hq, Hkv, max_ctx, num_splits, device):
    # a caller's workspace is passed as is: the library checks its size
    if ws is None:
        need = workspace_bytes(B, Hq, Hkv, max_ctx, num_splits)
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=device)
    return ws, ws.numel() * ws.element_size()


def decode_attention(cache: SpkvCache, q: torch.Tensor, block_table: torch.Tensor, ctx_lens: torch.Tensor,
                     max_ctx: int, out=None, out_dtype=torch.float32, ws=None, num_splits: int = 0,
                     stream=None, exact_q: bool = False) -> torch.Tensor:
    """spkv_decode_attention: ADA decode straight from the codes; returns out [B, Hq, 128].

    exact_q=True calls spkv_decode_attention_ex with SPKV_DECODE_EXACT_Q (the
    unquantised unit query in f_b)."""
    _batch_checks(q, block_table, ctx_lens)
    B, Hq, _ = q.shape
    out = _out_buffer(out, B, Hq, out_dtype, q.device)
    ws, wsb = _ws(ws, B, Hq, cache.num_kv_heads, max_ctx, num_splits, q.device)
    c = cache.c_struct()
    args = (ctypes.byref(c), _ptr(q), B, Hq, _ptr(block_table), block_table.shape[1], _ptr(ctx_lens), int(max_ctx),
            _ptr(out), int(out.dtype == torch.bfloat16), _ptr(ws), wsb, int(num_splits))
    if exact_q:
        check(lib.spkv_decode_attention_ex(*args, DECODE_EXACT_Q, _stream(stream)), "spkv_decode_attention_ex")
    else:
        check(lib.spkv_decode_attention(*args, _stream(stream)), "spkv_decode_attention")
    return out


def decode_attention_append(cache: SpkvCache, new_keys: torch.Tensor, new_values: torch.Tensor, q: torch.Tensor,
                            block_table: torch.Tensor, ctx_lens: torch.Tensor, max_ctx: int, out=None,
                            out_dtype=torch.float32, ws=None, num_splits: int = 0, stream=None,
                            exact_q: bool = False) -> torch.Tensor:
    """spkv_decode_attention_append: write token ctx_lens[b] - 1 of every sequence
    (new_keys / new_values [B, H_kv, 128] bf16) into its page, then decode over
    ctx_lens[b] tokens, in the decode's own launches."""
    _batch_checks(q, block_table, ctx_lens)
    B, Hq, _ = q.shape
    for t, name in ((new_keys, "new_keys"), (new_values, "new_values")):
        _need(t, torch.bfloat16, name, 3)
        if tuple(t.shape) != (B, cache.num_kv_heads, HEAD_DIM):
            raise ValueError(f"{name} must be [B, H_kv, 128]")
    out = _out_buffer(out, B, Hq, out_dtype, q.device)
    ws, wsb = _ws(ws, B, Hq, cache.num_kv_heads, max_ctx, num_splits, q.device)
    c = cache.c_struct()
    check(lib.spkv_decode_attention_append(ctypes.byref(c), _ptr(new_keys), _ptr(new_values), _ptr(q), B, Hq,
                                           _ptr(block_table), block_table.shape[1], _ptr(ctx_lens), int(max_ctx),
                                           _ptr(out), int(out.dtype == torch.bfloat16), _ptr(ws), wsb,
                                           int(num_splits), DECODE_EXACT_Q if exact_q else 0, _stream(stream)),
          "spkv_decode_attention_append")
    return out


def decode_attention_partial(cache: SpkvCache, q: torch.Tensor, block_table: torch.Tensor, ctx_lens: torch.Tensor,
                             max_ctx: int, partial=None, ws=None, num_splits: int = 0, stream=None,
                             exact_q: bool = False) -> torch.Tensor:
    """spkv_decode_attention_partial: this shard's records [B, Hq, 132] (M, L, 0, 0, o[128])."""
    _batch_checks(q, block_table, ctx_lens)
    B, Hq, _ = q.shape
    if partial is None:
        partial = torch.empty((B, Hq, PARTIAL_FLOATS), dtype=torch.float32, device=q.device)
    _need(partial, torch.float32, "partial", 3)
    if tuple(partial.shape) != (B, Hq, PARTIAL_FLOATS):
        raise ValueError("partial must be [B, Hq, 132]")
    ws, wsb = _ws(ws, B, Hq, cache.num_kv_heads, max_ctx, num_splits, q.device)
    c = cache.c_struct()
    check(lib.spkv_decode_attention_partial(ctypes.byref(c), _ptr(q), B, Hq, _ptr(block_table), block_table.shape[1],
                                            _ptr(ctx_lens), int(max_ctx), _ptr(partial), _ptr(ws), wsb,
                                            int(num_splits), DECODE_EXACT_Q if exact_q else 0, _stream(stream)),
          "spkv_decode_attention_partial")
    return partial


def merge_partials(partials: torch.Tensor, out=None, out_dtype=torch.float32, stream=None) -> torch.Tensor:
    """spkv_merge_partials: combine shard records [R, B, Hq, 132] into out [B, Hq, 128]."""
    _need(partials, torch.float32, "partials", 4)
    R, B, Hq, n = partials.shape
    if n != PARTIAL_FLOATS:
        raise ValueError("partials must be [R, B, Hq, 132]")
    out = _out_buffer(out, B, Hq, out_dtype, partials.device)
    check(lib.spkv_merge_partials(_ptr(partials), R, B, Hq, _ptr(out), int(out.dtype == torch.bfloat16),
                                  _stream(stream)), "spkv_merge_partials")
    return out


def decode_attention_static_ws(cache: SpkvCache, q: torch.Tensor, block_table: torch.Tensor,
                               ctx_lens: torch.Tensor, max_ctx: int, out=None, out_dtype=torch.float32,
                               num_splits: int = 0, stream=None) -> torch.Tensor:
    """spkv_decode_attention_static_ws: ADA decode for callers that cannot allocate
    device memory while decoding -- the workspace is the library's own fixed
    device array (SPKV_STATIC_WS_BYTES), shared by every call on the device, so
    calls must not overlap on the GPU.  `out` may be preallocated to make the
    call allocation-free on the Python side too."""
    _batch_checks(q, block_table, ctx_lens)
    B, Hq, _ = q.shape
    out = _out_buffer(out, B, Hq, out_dtype, q.device)
    c = cache.c_struct()
    check(lib.spkv_decode_attention_static_ws(ctypes.byref(c), _ptr(q), B, Hq, _ptr(block_table),
                                              block_table.shape[1], _ptr(ctx_lens), int(max_ctx), _ptr(out),
                                              int(out.dtype == torch.bfloat16), int(num_splits), _stream(stream)),
          "spkv_decode_attention_static_ws")
    return out


def dense_decode(k_pages: torch.Tensor, v_pages: torch.Tensor, q: torch.Tensor, block_table: torch.Tensor,
                 ctx_lens: torch.Tensor, max_ctx: int, keep_mask=None, err=None, out=None,
                 out_dtype=torch.float32, ws=None, num_splits: int = 0, stream=None) -> torch.Tensor:
    """spkv_dense_decode: the uncompressed bf16 paged decode (comparison path)."""
    _need(k_pages, torch.bfloat16, "k_pages", 4)
    _need(v_pages, torch.bfloat16, "v_pages", 4)
    _batch_checks(q, block_table, ctx_lens)
    num_pages, hkv = k_pages.shape[0], k_pages.shape[1]
    B, Hq, _ = q.shape
    out = _out_buffer(out, B, Hq, out_dtype, q.device)
    ws, wsb = _ws(ws, B, Hq, hkv, max_ctx, num_splits, q.device)
    check(lib.spkv_dense_decode(_ptr(k_pages), _ptr(v_pages), num_pages, hkv, _ptr(keep_mask), _ptr(err), _ptr(q),
                                B, Hq, _ptr(block_table), block_table.shape[1], _ptr(ctx_lens), int(max_ctx),
                                _ptr(out), int(out.dtype == torch.bfloat16), _ptr(ws), wsb, int(num_splits),
                                _stream(stream)), "spkv_dense_decode")
    return out


def decompress_then_dot(cache: SpkvCache, k_scratch: torch.Tensor, q: torch.Tensor, block_table: torch.Tensor,
                        ctx_lens: torch.Tensor, max_ctx: int, out=None, out_dtype=torch.float32, ws=None,
                        num_splits: int = 0, stream=None) -> torch.Tensor:
    """spkv_decompress_then_dot: materialise k~ into k_scratch, then dense decode."""
    _need(k_scratch, torch.bfloat16, "k_scratch", 4)
    _batch_checks(q, block_table, ctx_lens)
    B, Hq, _ = q.shape
    out = _out_buffer(out, B, Hq, out_dtype, q.device)
    ws, wsb = _ws(ws, B, Hq, cache.num_kv_heads, max_ctx, num_splits, q.device)
    c = cache.c_struct()
    check(lib.spkv_decompress_then_dot(ctypes.byref(c), _ptr(k_scratch), _ptr(q), B, Hq, _ptr(block_table),
                                       block_table.shape[1], _ptr(ctx_lens), int(max_ctx), _ptr(out),
                                       int(out.dtype == torch.bfloat16), _ptr(ws), wsb, int(num_splits),
                                       _stream(stream)), "spkv_decompress_then_dot")
    return out


def debug_logits(cache: SpkvCache, q: torch.Tensor, block_table: torch.Tensor, ctx_lens: torch.Tensor,
                 max_ctx: int, stream=None, exact_q: bool = False) -> torch.Tensor:
    """spkv_debug_logits(_ex): ADA logits [B, Hq, max_ctx] fp32 (NaN where not written)."""
    _batch_checks(q, block_table, ctx_lens)
    B, Hq, _ = q.shape
    logits = torch.full((B, Hq, max(max_ctx, 1)), float("nan"), dtype=torch.float32, device=q.device)
    c = cache.c_struct()
    check(lib.spkv_debug_logits_ex(ctypes.byref(c), _ptr(q), B, Hq, _ptr(block_table), block_table.shape[1],
                                   _ptr(ctx_lens), int(max_ctx), _ptr(logits), DECODE_EXACT_Q if exact_q else 0,
                                   _stream(stream)), "spkv_debug_logits_ex")
    return logits


def encode_keys_packed(cache: SpkvCache, keys: torch.Tensor, seq_start: torch.Tensor, dst_pos: torch.Tensor,
                       block_table: torch.Tensor, values: torch.Tensor | None = None, stream=None) -> None:
    """spkv_encode_keys_packed: keys/values [total_tokens, H_kv, 128] bf16, token t of sequence s
    to position dst_pos[t] of s (negative: skipped)."""
    _need(keys, torch.bfloat16, "keys", 3)
    total, hkv, d = keys.shape
    if hkv != cache.num_kv_heads or d != HEAD_DIM:
        raise ValueError("keys must be [total_tokens, H_kv, 128]")
    if values is not None:
        _need(values, torch.bfloat16, "values", 3)
        if values.shape != keys.shape:
            raise ValueError("values must match keys")
    _need(seq_start, torch.int32, "seq_start", 1)
    _need(dst_pos, torch.int32, "dst_pos", 1)
    _need(block_table, torch.int32, "block_table", 2)
    B = seq_start.shape[0] - 1
    if dst_pos.shape[0] != total or block_table.shape[0] != B:
        raise ValueError("dst_pos / block_table shape mismatch")
    c = cache.c_struct()
    check(lib.spkv_encode_keys_packed(ctypes.byref(c), _ptr(keys), _ptr(values), _ptr(seq_start), B, total,
                                      _ptr(dst_pos), _ptr(block_table), block_table.shape[1], _stream(stream)),
          "spkv_encode_keys_packed")


def rdr_workspace_bytes(total_tokens: int) -> int:
    return int(lib.spkv_rdr_workspace_bytes(int(total_tokens)))


def rdr_plan(keys: torch.Tensor, seq_start: torch.Tensor, q_norms: torch.Tensor, budget_bytes: torch.Tensor,
             protect: torch.Tensor | None = None, tier_mask: int = 0xF, max_pages_out: int | None = None,
             ws: torch.Tensor | None = None, stream=None) -> dict:
    """spkv_rdr_plan over sequences concatenated in keys [total_tokens, H_kv, 128] bf16.

    Returns a dict of device tensors: tier [T] uint8 (b, 0 = evicted),
    dst_pos [T] int32 (-1 = evicted), page_bits [B, max_pages_out] uint8,
    page_keep [B, max_pages_out] int16 (the uint16 slot masks' bits),
    n_pages [B] int32, lambda, rate, dist [B] float64, status [B] int32
    (SPKV_RDR_* bits).  max_pages_out defaults to ceil(T / 16) + 3, enough
    for any sequence of the batch."""
    _need(keys, torch.bfloat16, "keys", 3)
    total, hkv, d = keys.shape
    if d != HEAD_DIM:
        raise ValueError("keys must be [total_tokens, H_kv, 128]")
    _need(seq_start, torch.int32, "seq_start", 1)
    B = seq_start.shape[0] - 1
    _need(q_norms, torch.float32, "q_norms", 2)
    _need(budget_bytes, torch.float64, "budget_bytes", 1)
    if tuple(q_norms.shape) != (B, hkv) or budget_bytes.shape[0] != B:
        raise ValueError("q_norms must be [B, H_kv] and budget_bytes [B]")
    if protect is not None:
        _need(protect, torch.uint8, "protect", 1)
        if protect.shape[0] != total:
            raise ValueError("protect must be [total_tokens]")
    dev = keys.device
    if max_pages_out is None:
        max_pages_out = (total + 15) // 16 + 3
    if ws is None:
        ws = torch.empty(rdr_workspace_bytes(total), dtype=torch.uint8, device=dev)
    out = dict(tier=torch.empty(total, dtype=torch.uint8, device=dev),
               dst_pos=torch.empty(total, dtype=torch.int32, device=dev),
               page_bits=torch.zeros((B, max(max_pages_out, 1)), dtype=torch.uint8, device=dev),
               page_keep=torch.zeros((B, max(max_pages_out, 1)), dtype=torch.int16, device=dev),
               n_pages=torch.empty(B, dtype=torch.int32, device=dev),
               **{k: torch.empty(B, dtype=torch.float64, device=dev) for k in ("lambda", "rate", "dist")},
               status=torch.empty(B, dtype=torch.int32, device=dev))
    check(lib.spkv_rdr_plan(_ptr(keys), _ptr(seq_start), B, total, hkv, _ptr(q_norms), _ptr(protect),
                            _ptr(budget_bytes), int(tier_mask), int(max_pages_out), _ptr(out["tier"]),
                            _ptr(out["dst_pos"]), _ptr(out["page_bits"]), _ptr(out["page_keep"]),
                            _ptr(out["n_pages"]), _ptr(out["lambda"]), _ptr(out["rate"]), _ptr(out["dist"]),
                            _ptr(out["status"]), _ptr(ws), ws.numel(), _stream(stream)), "spkv_rdr_plan")
    return out


def nonuniform_tables(d: int, b: int):
    """spkv_nonuniform_tables: (edge_cos [d-2, 2^b-1], mid_cos [d-2, 2^b],
    mid_sin [d-2, 2^b]) as fp64 numpy arrays (host computation)."""
    import numpy as np

    n = 1 << b
    ec = np.empty((max(d - 2, 1), n - 1), np.float64)
    mc = np.empty((max(d - 2, 1), n), np.float64)
    ms = np.empty((max(d - 2, 1), n), np.float64)
    check(lib.spkv_nonuniform_tables(d, b, ec.ctypes.data, mc.ctypes.data, ms.ctypes.data), "spkv_nonuniform_tables")
    return ec[:d - 2], mc[:d - 2], ms[:d - 2]
