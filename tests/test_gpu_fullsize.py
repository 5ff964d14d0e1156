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


def test_full_size_exact_query_sampled_parity(spkv):
    """The exact-query variant (the unquantised unit query in f_b) at the full
    Llama shape, default split count, on sampled groups against the oracle."""
    m, synthetic, workload = spkv
    wl = synthetic.make_workload("llama3_8b_b8_h32x8_t32768_b4", device="cuda")
    cache = workload.build_cache(wl)
    out = m.decode_attention(cache, wl.q, wl.block_table, wl.ctx_tensor(), wl.max_ctx, exact_q=True)
    torch.cuda.synchronize()
    assert cache.error_flags() == 0
    err = helpers.max_abs_diff_groups(out.cpu().numpy(), wl, [(0, 0), (7, 7), (3, 5)], helpers.oracle_seq_exact_q)
    assert err <= OUT_TOL, err


def test_full_size_sharded_form_equals_one_shot(spkv):
    """The page-sharded form at the full Llama shape on one GPU: two shards'
    partial decodes merged by spkv_merge_partials against the one-shot decode
    (same arithmetic up to the split of the softmax sums: 2^-14 max|v|)."""
    m, synthetic, workload = spkv
    from compressed_kv_decode_ada_b200 import sharded

    wl = synthetic.make_workload("llama3_8b_b8_h32x8_t32768_b4", device="cuda")
    cache = workload.build_cache(wl)
    one = m.decode_attention(cache, wl.q, wl.block_table, wl.ctx_tensor(), wl.max_ctx)
    parts = []
    for r in range(2):
        bt, lc = sharded.shard_batch(wl.block_table_np, wl.ctx, 2, r)
        parts.append(m.decode_attention_partial(cache, wl.q, torch.as_tensor(bt, device="cuda"),
                                                torch.as_tensor(lc, device="cuda"), int(lc.max())))
    merged = m.merge_partials(torch.stack(parts))
    torch.cuda.synchronize()
    assert cache.error_flags() == 0
    vmax = wl.values.float().abs().amax().item()
    assert (merged - one).abs().max().item() <= 2.0 ** -14 * vmax
