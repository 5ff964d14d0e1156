"""CPU checks of the C ABI: the library loads, exports every entry point that
include/spkv.h declares, and rejects bad arguments on the host before any
launch (no GPU is touched by these calls)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "spkv.h")).read()
    return sorted(set(re.findall(r"SPKV_API\s+[\w\s\*]+?\b(spkv_\w+)\(", src)))


@pytest.fixture(scope="module")
def lib():
    import compressed_kv_decode_ada_b200 as m

    return m


def test_header_declares_the_entry_points(lib):
    names = _declared()
    assert set(names) == set(lib._lib.EXPORTS), names


def test_library_exports_every_declared_symbol(lib):
    raw = ctypes.CDLL(lib.LIB_PATH)
    for name in _declared():
        assert hasattr(raw, name), name


def test_status_strings(lib):
    assert lib.lib.spkv_status_string(0) == b"SPKV_OK"
    assert lib.lib.spkv_status_string(3) == b"SPKV_ERR_WORKSPACE"
    assert lib.lib.spkv_status_string(99) == b"SPKV_ERR_UNKNOWN"


def _fake_cache(m, **over):
    c = m._lib.SpkvCacheC()
    c.num_kv_heads, c.head_dim, c.page_size, c.num_pages = 2, 128, 16, 10
    c.code_arena, c.code_arena_bytes, c.hdr = 0x10000, 1 << 20, 0x20000
    c.rad_lo_log2, c.rad_step_log2, c.v_pages = 0x30000, 0x40000, 0x50000
    c.keep_mask, c.err_flags = None, None
    for k, v in over.items():
        setattr(c, k, v)
    return c


def _decode(m, c, B=1, Hq=4, ws_bytes=1 << 20, splits=4, q=0x60000):
    L = m.lib
    return L.spkv_decode_attention(ctypes.byref(c), q, B, Hq, 0x70000, 8, 0x80000, 128, 0x90000, 0, 0xA0000,
                                   ws_bytes, splits, None)


def test_host_argument_checks(lib):
    m = lib
    L = m.lib
    assert L.spkv_decode_attention(None, 0, 0, 1, 0, 0, 0, 0, 0, 0, 0, 0, 0, None) == 1
    assert _decode(m, _fake_cache(m, head_dim=64)) == 2
    assert _decode(m, _fake_cache(m, page_size=32)) == 2
    assert _decode(m, _fake_cache(m), Hq=6) == 2           # G = 3
    assert _decode(m, _fake_cache(m), Hq=3) == 1           # Hq not a multiple of H_kv
    assert _decode(m, _fake_cache(m, code_arena=0x10001)) == 1  # misaligned arena
    assert _decode(m, _fake_cache(m), q=0x60002) == 1      # misaligned q
    assert _decode(m, _fake_cache(m), ws_bytes=16) == 3    # workspace too small
    assert _decode(m, _fake_cache(m), B=5000) == 2         # batch beyond the supported maximum
    assert _decode(m, _fake_cache(m), B=0) == 0            # empty batch: nothing to do
    # flags: unknown bits are rejected before anything else; known bits pass the checks
    c = _fake_cache(m)
    assert L.spkv_decode_attention_ex(ctypes.byref(c), 0x1000, 0, 8, 0x2000, 4, 0x3000, 64, 0x4000, 0, 0x5000,
                                      1 << 20, 0, 2, None) == 1
    assert L.spkv_decode_attention_ex(ctypes.byref(c), 0x1000, 0, 8, 0x2000, 4, 0x3000, 64, 0x4000, 0, 0x5000,
                                      1 << 20, 1, 1, None) == 0  # empty batch, one split: no device query
    assert L.spkv_debug_logits_ex(ctypes.byref(c), 0x1000, 1, 8, 0x2000, 4, 0x3000, 64, 0x4000, 4, None) == 1
    # encode: negative sizes / misaligned keys
    c = _fake_cache(m)
    assert L.spkv_encode_keys(ctypes.byref(c), 0x1000, None, 0x2000, -1, 1, 0x3000, 4, None) == 1
    assert L.spkv_encode_keys(ctypes.byref(c), 0x1004, None, 0x2000, 1, 1, 0x3000, 4, None) == 1
    assert L.spkv_encode_keys(ctypes.byref(c), 0x1000, None, 0x2000, 0, 1, 0x3000, 4, None) == 0


def _static(m, c, B=1, Hq=4, splits=4, q=0x60000, max_ctx=128):
    cp = ctypes.byref(c) if c is not None else None
    return m.lib.spkv_decode_attention_static_ws(cp, q, B, Hq, 0x70000, 8, 0x80000, max_ctx, 0x90000, 0, splits, None)


def test_static_ws_argument_checks_match_decode(lib):
    """spkv_decode_attention_static_ws runs spkv_decode_attention's argument checks
    before its own capacity check: a bad argument gets the same status from both
    entry points, also when its workspace would exceed the fixed array."""
    m = lib
    L = m.lib

    def dec(c, B=1, Hq=4, splits=4, q=0x60000, max_ctx=128):
        cp = ctypes.byref(c) if c is not None else None
        return L.spkv_decode_attention(cp, q, B, Hq, 0x70000, 8, 0x80000, max_ctx, 0x90000, 0, 0xA0000, 1 << 20,
                                       splits, None)

    cases = [
        (None, {}),                                   # no cache
        (_fake_cache(m, head_dim=64), {}),             # unsupported head dim
        (_fake_cache(m), dict(Hq=6)),                  # G = 3
        (_fake_cache(m), dict(Hq=3)),                  # Hq not a multiple of H_kv
        (_fake_cache(m), dict(q=0x60002)),             # misaligned q
        (_fake_cache(m), dict(B=5000, splits=4096)),   # batch beyond the maximum, workspace far beyond 16 MiB
        (_fake_cache(m), dict(B=1024, max_ctx=1 << 24, splits=4096)),  # too many pages, huge workspace
        (_fake_cache(m), dict(B=0)),                   # empty batch
        (_fake_cache(m), dict(B=1024, splits=4096)),   # valid, but 39 MB of workspace: both too small
    ]
    want = [1, 2, 2, 1, 1, 2, 2, 0, 3]
    for (c, kw), w in zip(cases, want):
        assert dec(c, **kw) == w, kw
        assert _static(m, c, **kw) == w, kw
    need = m.workspace_bytes(1024, 4, 2, 128, 4096)
    assert need > m._lib.STATIC_WS_BYTES


def test_nonuniform_host_argument_checks(lib):
    """The non-uniform encode / decode reject bad arguments before any launch."""
    m = lib
    L = m.lib
    c = _fake_cache(m)
    enc = lambda bits, ec: L.spkv_encode_keys_nonuniform(ctypes.byref(c), 0x1000, None, 0x2000, 1, 1, 0x3000, 4,  # noqa: E731
                                                          bits, ec, None)
    assert enc(5, 0x4000) == 2           # b outside {3, 4, 6, 8}
    assert enc(4, None) == 1             # no edge table
    assert enc(4, 0x4004) == 1           # misaligned edge table

    def dec(Hq=4, bits=4, ec=0x4000, ws=0x100000, ws_bytes=1 << 24, splits=2, B=1):
        return L.spkv_decode_attention_nonuniform(ctypes.byref(c), 0x60000, B, Hq, 0x70000, 8, 0x80000, 128, bits,
                                                  ec, 0x5000, 0x6000, 0x90000, 0, None, ws, ws_bytes, splits, None)
    assert dec(Hq=6) == 2                # G = 3
    assert dec(bits=7) == 2
    assert dec(ec=None) == 1
    assert dec(ws=0x100010) == 3         # workspace not 256-byte aligned
    assert dec(ws_bytes=16) == 3         # workspace too small
    assert dec(B=0) == 0                 # empty batch
    # explicit split count: no device query
    want = ((2 * 1 * 4 * 132 * 4 + 255) // 256) * 256 + 127 * 16 * 8
    assert L.spkv_decode_nonuniform_workspace_bytes(1, 4, 2, 128, 2, 4) == want
    assert L.spkv_decode_nonuniform_workspace_bytes(1, 4, 2, 128, 2, 5) == 0


def test_workspace_formula(lib):
    # (C + B H_kv) segments x 6 consumer-warp slots x G partials of 132 floats
    # (rounded to 16 bytes), then one 4-byte row counter per kv row (rounded)
    def want(B, Hq, Hkv, C):
        part = (C + B * Hkv) * 6 * (Hq // Hkv) * 132 * 4
        return (part + 15) // 16 * 16 + (B * Hkv * 4 + 15) // 16 * 16
    assert lib.workspace_bytes(8, 32, 8, 32768, 296) == want(8, 32, 8, 296)
    assert lib.workspace_bytes(2, 8, 8, 100, 5) == want(2, 8, 8, 5)
    assert lib.workspace_bytes(3, 8, 1, 100, 5) == want(3, 8, 1, 5)
    assert lib.workspace_bytes(2, 7, 2, 100, 5) == 0  # Hq not a multiple of H_kv


def test_rdr_host_argument_checks(lib):
    """spkv_rdr_plan / spkv_encode_keys_packed reject bad arguments before any
    CUDA call; an empty batch is a no-op."""
    L = lib.lib
    P = 0x10000  # an aligned stand-in pointer, never dereferenced

    def plan(B=2, total=10, Hkv=8, mask=0xF, maxp=8, keys=P, ws=P, ws_bytes=1 << 20, page=P):
        return L.spkv_rdr_plan(keys, P, B, total, Hkv, P, None, P, mask, maxp, P, P, page, page, P, P, P, P, P,
                               ws, ws_bytes, None)

    assert plan(Hkv=0) == 1 and plan(Hkv=33) == 1
    assert plan(mask=0) == 1 and plan(mask=0x10) == 1
    assert plan(B=-1) == 1 and plan(total=-1) == 1 and plan(maxp=-1) == 1
    assert plan(keys=P + 8) == 1          # keys must be 16-byte aligned
    assert plan(page=None) == 1           # page outputs needed when max_pages_out > 0
    assert plan(ws_bytes=16) == 3         # workspace: 8 bytes per token
    assert plan(B=0) == 0                 # empty batch
    assert L.spkv_rdr_workspace_bytes(0) == 16
    assert L.spkv_rdr_workspace_bytes(1000) == 8000
    assert L.spkv_rdr_workspace_bytes(1001) == 8016
    c = _fake_cache(lib)
    assert L.spkv_encode_keys_packed(ctypes.byref(c), P, None, P, -1, 4, P, P, 4, None) == 1
    assert L.spkv_encode_keys_packed(ctypes.byref(c), P + 4, None, P, 1, 4, P, P, 4, None) == 1
    assert L.spkv_encode_keys_packed(ctypes.byref(c), P, None, P, 1, 0, P, P, 4, None) == 0
