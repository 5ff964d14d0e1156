"""Failure detection without a GPU fault: the decode kernels' bounded waits.

Every mbarrier wait in the kernels gives up after a limit, sets
SPKV_DEVERR_TIMEOUT and lets the kernel return; spkv_debug_wait_timeout runs
that routine on a barrier that nothing completes (no fault, no trap, no
endless loop), and the context must stay usable afterwards."""
import pytest
import torch


def test_wait_timeout_hook_rejects_bad_arguments():
    from compressed_kv_decode_ada_b200._lib import lib

    assert lib.spkv_debug_wait_timeout(None, None, 1000, None) == 1
    assert lib.spkv_debug_wait_timeout(0x1000, 0x2000, 0, None) == 1
    assert lib.spkv_debug_wait_timeout(0x1000, 0x2000, 2_000_000_000, None) == 1


@pytest.mark.gpu
def test_bounded_wait_gives_up_sets_the_flag_and_the_context_survives():
    import ctypes

    import compressed_kv_decode_ada_b200 as m
    from compressed_kv_decode_ada_b200 import synthetic, workload
    from compressed_kv_decode_ada_b200._lib import DEVERR_TIMEOUT, check, lib

    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    status = torch.zeros(3, dtype=torch.int32, device="cuda")
    limit_ns = 20_000_000  # 20 ms
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    check(lib.spkv_debug_wait_timeout(ctypes.c_void_p(err.data_ptr()), ctypes.c_void_p(status.data_ptr()), limit_ns,
                                      stream), "spkv_debug_wait_timeout")
    torch.cuda.synchronize()
    st = status.cpu().tolist()
    assert st[0] == 1 and st[2] == 1                 # the wait gave up and raised the abort flag
    assert 20_000 <= st[1] < 1_000_000               # after the limit, not forever
    assert int(err.item()) & DEVERR_TIMEOUT
    # the context is still usable: a small decode right after is correct
    wl = synthetic.make_workload("tiny_b1_h1_t4096_b4", device="cuda", ctx=[100])
    cache = workload.build_cache(wl)
    out = m.decode_attention(cache, wl.q, wl.block_table, wl.ctx_tensor(), wl.max_ctx)
    torch.cuda.synchronize()
    assert cache.error_flags() == 0
    from tests import helpers
    err2 = helpers.max_abs_diff_groups(out.cpu().numpy(), wl, helpers.all_groups(wl), helpers.oracle_seq)
    assert err2 <= 2e-3
