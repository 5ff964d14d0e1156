"""Parity at the full workload sizes, in the launch configuration the bench
times (default split count), on (sequence, kv head) groups the oracle can
compute one by one, plus properties that hold at any size."""
import numpy as np
import pytest
import torch

from tests import helpers

pytestmark = pytest.mark.gpu

OUT_TOL = 2e-3


@pytest.fixture(scope="module")
def spkv():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import compressed_kv_decode_ada_b200 as m
    from compressed_kv_decode_ada_b200 import synthetic, workload

    return m, synthetic, workload


@pytest.mark.parametrize("cfg,groups", [
    ("llama3_8b_b8_h32x8_t32768_b4", [(0, 0), (7, 7), (3, 5)]),
    ("long_b1_h32x8_t131072_b4", [(0, 0), (0, 6)]),
    ("ragged_rdr_b32_h32x8_t1k-64k_mixed_b_mask25", [(0, 0), (31, 7), (17, 3)]),
    ("70b_b16_h64x8_t16384_b4_encode", [(0, 0), (15, 7)]),
])
def test_full_size_sampled_parity(spkv, cfg, groups):
    m, synthetic, workload = spkv
    wl = synthetic.make_workload(cfg, device="cuda")
    cache = workload.build_cache(wl)
    wl.extras["code_offset"] = cache.page_code_offset
    out = m.decode_attention(cache, wl.q, wl.block_table, wl.ctx_tensor(), wl.max_ctx)
    torch.cuda.synchronize()
    assert cache.error_flags() == 0
    assert torch.isfinite(out).all()
    outn = out.cpu().numpy()
    err = helpers.max_abs_diff_groups(outn, wl, groups, helpers.oracle_seq)
    assert err <= OUT_TOL, err
    # the encoded bytes of every sampled group are the oracle's codes (off the
    # cell edges; edge-adjacent differences within the 1e-6 budget)
    helpers.check_codes(wl, cache, groups)
    # property at any size: every output row is a convex combination of value rows
    vmax = wl.values.float().abs().amax().item()
    assert outn.max() <= vmax + 1e-3 and outn.min() >= -vmax - 1e-3
