"""spkv_decode_attention_static_ws: the decode entry point for callers that
cannot allocate device memory while they decode (its workspace is the
library's own fixed device array).  Checked through the C ABI against
spkv_decode_attention with a caller-allocated workspace, on two calls in a
row (the second reuses what the first left in the shared array), and for the
size limit.  This file is collected last on purpose."""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu



@pytest.fixture(scope="module")
def spkv():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import compressed_kv_decode_ada_b200 as m
    from compressed_kv_decode_ada_b200 import synthetic, workload

    return m, synthetic, workload


def _static_ws_call(m, cache, q, block_table, ctx, max_ctx, out, num_splits=0):
    c = cache.c_struct()
    return m.lib.spkv_decode_attention_static_ws(
        ctypes.byref(c), ctypes.c_void_p(q.data_ptr()), q.shape[0], q.shape[1],
        ctypes.c_void_p(block_table.data_ptr()), block_table.shape[1], ctypes.c_void_p(ctx.data_ptr()), max_ctx,
        ctypes.c_void_p(out.data_ptr()), 0, num_splits, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_static_workspace_matches_allocated_workspace(spkv):
    m, synthetic, workload = spkv
    results = []
    for cfg, kw in (("llama3_8b_b8_h32x8_t32768_b4", dict(B=3, ctx=[2000, 513, 4100])), ("ragged_rdr_b32_h32x8_t1k-64k_mixed_b_mask25", dict(B=4, ctx=("loguniform", 40, 3000)))):
        wl = synthetic.make_workload(cfg, device="cuda", **kw)
        cache = workload.build_cache(wl)
        ctx = wl.ctx_tensor()
        ref = m.decode_attention(cache, wl.q, wl.block_table, ctx, wl.max_ctx)
        results.append((wl, cache, ctx, ref))
    # two calls in a row on each workload: the second starts from what the
    # previous call left in the shared array
    for wl, cache, ctx, ref in results + results:
        out = torch.empty_like(ref)
        st = _static_ws_call(m, cache, wl.q, wl.block_table, ctx, wl.max_ctx, out)
        torch.cuda.synchronize()
        assert st == 0, m.lib.spkv_status_string(st)
        assert cache.error_flags() == 0
        # the same kernels at the same split count: bit-identical output
        assert torch.equal(out, ref)


def test_static_workspace_rejects_sizes_beyond_its_capacity(spkv):
    m, synthetic, workload = spkv
    wl = synthetic.make_workload("llama3_8b_b8_h32x8_t32768_b4", device="cuda", B=2, ctx=[64, 64])
    cache = workload.build_cache(wl)
    # 1024 sequences of up to 2^20 tokens with 4096 splits need far more than 16 MiB
    need = m.workspace_bytes(1024, 32, 8, 1 << 20, 4096)
    assert need > m._lib.STATIC_WS_BYTES
    q = torch.zeros((1024, 32, 128), dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros((1024, 1), dtype=torch.int32, device="cuda")
    ctx = torch.zeros(1024, dtype=torch.int32, device="cuda")
    out = torch.empty((1024, 32, 128), dtype=torch.float32, device="cuda")
    st = _static_ws_call(m, cache, q, bt, ctx, 1 << 20, out, num_splits=4096)
    assert st == 3  # SPKV_ERR_WORKSPACE


def test_static_workspace_capacity_boundary(spkv):
    """An explicit split count whose workspace just fits the fixed array runs and
    equals the caller-workspace call bit for bit; one more split is rejected."""
    m, synthetic, workload = spkv
    wl = synthetic.make_workload("llama3_8b_b8_h32x8_t32768_b4", device="cuda", B=8,
                                 ctx=[64, 300, 17, 1000, 16, 512, 129, 2048])
    cache = workload.build_cache(wl)
    ctx = wl.ctx_tensor()
    cap = m._lib.STATIC_WS_BYTES
    lo, hi = 1, 1 << 16  # largest C whose workspace fits
    while lo < hi:
        mid = (lo + hi + 1) // 2
        if m.workspace_bytes(wl.B, wl.Hq, wl.Hkv, wl.max_ctx, mid) <= cap:
            lo = mid
        else:
            hi = mid - 1
    c_max = lo
    assert m.workspace_bytes(wl.B, wl.Hq, wl.Hkv, wl.max_ctx, c_max + 1) > cap
    ref = m.decode_attention(cache, wl.q, wl.block_table, ctx, wl.max_ctx, num_splits=c_max)
    out = torch.empty_like(ref)
    st = _static_ws_call(m, cache, wl.q, wl.block_table, ctx, wl.max_ctx, out, num_splits=c_max)
    torch.cuda.synchronize()
    assert st == 0, m.lib.spkv_status_string(st)
    assert cache.error_flags() == 0
    assert torch.equal(out, ref)
    st = _static_ws_call(m, cache, wl.q, wl.block_table, ctx, wl.max_ctx, out, num_splits=c_max + 1)
    assert st == 3  # SPKV_ERR_WORKSPACE
