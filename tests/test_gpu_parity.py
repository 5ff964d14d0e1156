"""GPU <-> oracle parity of the ADA decode path through the C ABI.

Tolerances (stated in the design notes, from the target of the method's
evaluation): angle and radius codes bit-exact except codes on a cell edge
(|t - k| <= 1e-12 max(1,|t|) for the oracle's scaled position t), which are
counted and must be < 1e-6 of all codes; logits |d logit| <= 1e-4 ||q|| r~ /
sqrt(d) (i.e. |d f_b| <= 1e-4); outputs <= 2e-3 absolute (fp32 output,
unit-variance values).  The oracle encodes the keys itself: no oracle input
comes from the CUDA path.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tests import helpers

pytestmark = pytest.mark.gpu

OUT_TOL = 2e-3
FB_TOL = 1e-4
# workload shapes (compressed_kv_decode_ada_b200.synthetic.WORKLOADS), shrunk per test
TINY = "tiny_b1_h1_t4096_b4"
LLAMA = "llama3_8b_b8_h32x8_t32768_b4"
RAGGED = "ragged_rdr_b32_h32x8_t1k-64k_mixed_b_mask25"


@pytest.fixture(scope="module")
def spkv():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import compressed_kv_decode_ada_b200 as m
    from compressed_kv_decode_ada_b200 import synthetic, workload

    return m, synthetic, workload


def _build(spkv, cfg, **kw):
    m, synthetic, workload = spkv
    wl = synthetic.make_workload(cfg, device="cuda", **kw)
    cache = workload.build_cache(wl)
    wl.extras["code_offset"] = cache.page_code_offset
    torch.cuda.synchronize()
    assert cache.error_flags() == 0
    return wl, cache


def _decode(spkv, wl, cache, **kw):
    m = spkv[0]
    out = m.decode_attention(cache, wl.q, wl.block_table, wl.ctx_tensor(), wl.max_ctx, **kw)
    torch.cuda.synchronize()
    assert cache.error_flags() == 0
    return out


# ------------------------------------------------------------------ encode

def _check_codes(wl, cache, groups):
    return helpers.check_codes(wl, cache, groups)


def test_encode_codes_bit_exact_tiny(spkv):
    wl, cache = _build(spkv, TINY)
    _check_codes(wl, cache, helpers.all_groups(wl))


def test_encode_codes_bit_exact_mixed_tiers(spkv):
    wl, cache = _build(spkv, RAGGED, B=6, ctx=("loguniform", 17, 1500))
    assert set(np.unique(wl.page_bits)) == {3, 4, 6, 8}
    _check_codes(wl, cache, helpers.all_groups(wl))


def test_encode_append_in_steps_matches_one_shot(spkv):
    """Appending a sequence one token (then 5 tokens) at a time gives the same bytes."""
    m, synthetic, workload = spkv
    wl, cache = _build(spkv, RAGGED, B=2, ctx=[37, 50], mask=False)
    ref = cache.arena.clone()
    cache2 = m.SpkvCache(wl.num_pages, wl.Hkv, wl.page_bits, wl.rad_lo, wl.rad_step)
    for b in range(wl.B):
        s, n = int(wl.seq_off[b]), int(wl.ctx[b])
        pos = 0
        step = 1 if b == 0 else 5
        while pos < n:
            k = min(step, n - pos)
            m.encode_keys(cache2, wl.keys[s + pos:s + pos + k].unsqueeze(0),
                          torch.tensor([pos], dtype=torch.int32, device="cuda"),
                          wl.block_table[b:b + 1].contiguous(), values=wl.values[s + pos:s + pos + k].unsqueeze(0))
            pos += k
    torch.cuda.synchronize()
    assert torch.equal(cache2.arena, ref)
    assert torch.equal(cache2.v_pages, cache.v_pages)


def test_encode_thread_and_warp_forms_write_the_same_bytes(spkv):
    """Bulk encode runs one thread per key for large calls and one warp per key
    for a few keys (decode-step appends); the two forms must write the same
    bytes: one call of 2,800 keys vs the same keys 8 tokens (64 keys) at a time."""
    m, synthetic, workload = spkv
    wl = synthetic.make_workload(RAGGED, device="cuda", B=1, ctx=[350], mask=False)
    one = m.SpkvCache(wl.num_pages, wl.Hkv, wl.page_bits, wl.rad_lo, wl.rad_step)
    steps = m.SpkvCache(wl.num_pages, wl.Hkv, wl.page_bits, wl.rad_lo, wl.rad_step)
    n = int(wl.ctx[0])
    bt = wl.block_table[0:1].contiguous()
    m.encode_keys(one, wl.keys[:n].unsqueeze(0), torch.zeros(1, dtype=torch.int32, device="cuda"), bt,
                  values=wl.values[:n].unsqueeze(0))
    for pos in range(0, n, 8):
        k = min(8, n - pos)
        m.encode_keys(steps, wl.keys[pos:pos + k].unsqueeze(0), torch.tensor([pos], dtype=torch.int32, device="cuda"),
                      bt, values=wl.values[pos:pos + k].unsqueeze(0))
    torch.cuda.synchronize()
    assert one.error_flags() == 0 and steps.error_flags() == 0
    assert len(set(int(b) for b in wl.page_bits)) > 1  # several tiers
    assert torch.equal(one.arena, steps.arena)
    assert torch.equal(one.v_pages, steps.v_pages)


def test_packed_and_per_sequence_prefill_write_the_same_bytes(spkv):
    """A ragged batch prefilled by one spkv_encode_keys_packed call (the
    default) and by one spkv_encode_keys call per sequence: identical pages."""
    m, synthetic, workload = spkv
    wl = synthetic.make_workload(RAGGED, device="cuda", B=5, ctx=[700, 1, 33, 2049, 160])
    packed = m.SpkvCache(wl.num_pages, wl.Hkv, wl.page_bits, wl.rad_lo, wl.rad_step, keep_mask=wl.keep_mask)
    perseq = m.SpkvCache(wl.num_pages, wl.Hkv, wl.page_bits, wl.rad_lo, wl.rad_step, keep_mask=wl.keep_mask)
    workload.prefill(packed, wl)
    workload.prefill(perseq, wl, packed=False)
    torch.cuda.synchronize()
    assert packed.error_flags() == 0 and perseq.error_flags() == 0
    assert torch.equal(packed.arena, perseq.arena)
    assert torch.equal(packed.v_pages, perseq.v_pages)


def _last_tokens(wl):
    idx = torch.tensor([int(wl.seq_off[b]) + int(wl.ctx[b]) - 1 for b in range(wl.B)], device=wl.keys.device)
    return wl.keys[idx].contiguous(), wl.values[idx].contiguous()


@pytest.mark.parametrize("cfg,kw", [
    (RAGGED, dict(B=4, ctx=[37, 1, 2049, 700])),        # mixed tiers, mask, a one-token sequence (wide ring)
    (LLAMA, dict(B=3, ctx=[16, 1000, 4097])),           # b = 4 only (narrow ring), page-aligned and ragged ends
])
def test_fused_append_equals_encode_then_decode(spkv, cfg, kw):
    """spkv_decode_attention_append writes token ctx - 1 exactly as spkv_encode_keys
    does (over junk left in the slot) and returns the same output as the two-call path."""
    m = spkv[0]
    wl, cache = _build(spkv, cfg, **kw)
    ref_out = _decode(spkv, wl, cache)
    ref_arena, ref_v = cache.arena.clone(), cache.v_pages.clone()
    new_k, new_v = _last_tokens(wl)
    g = torch.Generator(device="cuda").manual_seed(5)
    junk_k = torch.randn(new_k.shape, generator=g, device="cuda").to(torch.bfloat16)
    junk_v = torch.randn(new_v.shape, generator=g, device="cuda").to(torch.bfloat16)
    last = (wl.ctx_tensor() - 1).to(torch.int32)
    m.encode_keys(cache, junk_k.unsqueeze(1).contiguous(), last, wl.block_table, values=junk_v.unsqueeze(1).contiguous())
    torch.cuda.synchronize()
    assert not torch.equal(cache.arena, ref_arena)
    out = m.decode_attention_append(cache, new_k, new_v, wl.q, wl.block_table, wl.ctx_tensor(), wl.max_ctx)
    torch.cuda.synchronize()
    assert cache.error_flags() == 0
    assert torch.equal(cache.arena, ref_arena)
    assert torch.equal(cache.v_pages, ref_v)
    assert torch.equal(out, ref_out)


def test_fused_append_oracle_parity_exact_query(spkv):
    """The fused append with the exact-query flag against the oracle, from a cache
    whose last tokens were never encoded."""
    m, synthetic, workload = spkv
    wl = synthetic.make_workload(RAGGED, device="cuda", B=3, ctx=[300, 17, 1500], Hq=8, Hkv=2)
    cache = m.SpkvCache(wl.num_pages, wl.Hkv, wl.page_bits, wl.rad_lo, wl.rad_step, keep_mask=wl.keep_mask)
    for b in range(wl.B):  # prefill all but the last token of every sequence
        s, n = int(wl.seq_off[b]), int(wl.ctx[b])
        if n > 1:
            m.encode_keys(cache, wl.keys[s:s + n - 1].unsqueeze(0).contiguous(),
                          torch.zeros(1, dtype=torch.int32, device="cuda"), wl.block_table[b:b + 1].contiguous(),
                          values=wl.values[s:s + n - 1].unsqueeze(0).contiguous())
    new_k, new_v = _last_tokens(wl)
    out = m.decode_attention_append(cache, new_k, new_v, wl.q, wl.block_table, wl.ctx_tensor(), wl.max_ctx,
                                    exact_q=True)
    torch.cuda.synchronize()
    assert cache.error_flags() == 0
    err = helpers.max_abs_diff_groups(out.cpu().numpy(), wl, helpers.all_groups(wl), helpers.oracle_seq_exact_q)
    assert err <= OUT_TOL, err


# ------------------------------------------------------------------ decode

def test_decode_parity_tiny(spkv):
    wl, cache = _build(spkv, TINY)
    out = _decode(spkv, wl, cache).cpu().numpy()
    err = helpers.max_abs_diff_groups(out, wl, helpers.all_groups(wl), helpers.oracle_seq)
    assert err <= OUT_TOL, err


@pytest.mark.parametrize("kw", [
    dict(B=2, ctx=[1000, 4099]),                       # G = 4, ragged tails, RoPE keys
    dict(B=3, ctx=[16, 1, 2500], Hq=16, Hkv=2),       # G = 8, one-token and one-page contexts
    dict(B=2, ctx=[777, 3001], Hq=4, Hkv=2),           # G = 2
])
def test_decode_parity_small_shapes(spkv, kw):
    wl, cache = _build(spkv, LLAMA, **kw)
    out = _decode(spkv, wl, cache).cpu().numpy()
    err = helpers.max_abs_diff_groups(out, wl, helpers.all_groups(wl), helpers.oracle_seq)
    assert err <= OUT_TOL, err


def test_decode_parity_mixed_tiers_and_mask(spkv):
    wl, cache = _build(spkv, RAGGED, B=5, ctx=("loguniform", 20, 5000))
    out = _decode(spkv, wl, cache).cpu().numpy()
    err = helpers.max_abs_diff_groups(out, wl, helpers.all_groups(wl), helpers.oracle_seq)
    assert err <= OUT_TOL, err


def test_debug_logits_parity(spkv):
    """|d f_b| <= 1e-4: logits within 1e-4 ||q|| r~ / sqrt(d) of the oracle's."""
    m = spkv[0]
    wl, cache = _build(spkv, RAGGED, B=3, ctx=[300, 1200, 64], Hq=8, Hkv=2)
    lg = m.debug_logits(cache, wl.q, wl.block_table, wl.ctx_tensor(), wl.max_ctx).cpu().numpy()
    for b, h in helpers.all_groups(wl):
        n = int(wl.ctx[b])
        _, ref = helpers.oracle_seq(wl, b, h, want_logits=True)
        keys, bits = wl.keys_bits(b, h), wl.token_bits(b)
        _, rc = oracle.encode(keys, bits, float(wl.rad_lo[h]), float(wl.rad_step[h]))
        scale = helpers.logit_scale(wl, b, h, rc)
        got = lg[b, h * wl.G:(h + 1) * wl.G, :n].astype(np.float64)
        ev = np.isinf(ref)
        assert np.array_equal(np.isinf(got), ev)
        d = np.abs(got[~ev] - ref[~ev]) / scale[~ev]
        assert d.max() <= FB_TOL, d.max()


def test_exact_query_decode_parity(spkv):
    """The exact-query variant (SPKV_DECODE_EXACT_Q) against the oracle's,
    mixed tiers, mask and ragged lengths; and its logits to |d f_b| <= 1e-4."""
    m = spkv[0]
    wl, cache = _build(spkv, RAGGED, B=4, ctx=[2000, 333, 17, 4100], Hq=8, Hkv=2)
    out = _decode(spkv, wl, cache, exact_q=True).cpu().numpy()
    err = helpers.max_abs_diff_groups(out, wl, helpers.all_groups(wl), helpers.oracle_seq_exact_q)
    assert err <= OUT_TOL, err
    lg = m.debug_logits(cache, wl.q, wl.block_table, wl.ctx_tensor(), wl.max_ctx, exact_q=True).cpu().numpy()
    for b, h in helpers.all_groups(wl):
        n = int(wl.ctx[b])
        _, ref = helpers.oracle_seq(wl, b, h, want_logits=True, exact_q=True)
        keys, bits = wl.keys_bits(b, h), wl.token_bits(b)
        _, rc = oracle.encode(keys, bits, float(wl.rad_lo[h]), float(wl.rad_step[h]))
        scale = helpers.logit_scale(wl, b, h, rc)
        got = lg[b, h * wl.G:(h + 1) * wl.G, :n].astype(np.float64)
        ev = np.isinf(ref)
        assert np.array_equal(np.isinf(got), ev)
        d = np.abs(got[~ev] - ref[~ev]) / scale[~ev]
        assert d.max() <= FB_TOL, d.max()


def test_exact_query_decode_parity_b4_pairs(spkv):
    """Exact query on an all-b=4 cache (the narrow ring and the paired b = 4 loop), G = 4."""
    wl, cache = _build(spkv, LLAMA, B=2, ctx=[1000, 2049])
    out = _decode(spkv, wl, cache, exact_q=True).cpu().numpy()
    err = helpers.max_abs_diff_groups(out, wl, helpers.all_groups(wl), helpers.oracle_seq_exact_q)
    assert err <= OUT_TOL, err


def _reorder_tol(wl):
    # A different split count changes only the fp32 summation order and the
    # running maxima at which p is split into bf16 hi + lo parts for the
    # tensor-core P.V (residual below 2^-16 of p): bound 2^-14 max|v|.
    return 2.0 ** -14 * float(wl.values.float().abs().max())


def test_split_count_invariance(spkv):
    wl, cache = _build(spkv, RAGGED, B=4, ctx=("loguniform", 100, 4000))
    ref = _decode(spkv, wl, cache, num_splits=1)
    for s in (2, 7, 33, 0):
        out = _decode(spkv, wl, cache, num_splits=s)
        assert torch.max(torch.abs(out - ref)).item() <= _reorder_tol(wl)


def test_block_table_permutation_invariance(spkv):
    wl1, c1 = _build(spkv, RAGGED, B=3, ctx=[500, 1700, 33], extra_pages=7, perm_seed=11)
    wl2, c2 = _build(spkv, RAGGED, B=3, ctx=[500, 1700, 33], extra_pages=7, perm_seed=12)
    assert not np.array_equal(wl1.block_table_np, wl2.block_table_np)
    o1, o2 = _decode(spkv, wl1, c1), _decode(spkv, wl2, c2)
    assert torch.max(torch.abs(o1 - o2)).item() <= _reorder_tol(wl1)


def test_bf16_output_matches_fp32(spkv):
    wl, cache = _build(spkv, LLAMA, B=2, ctx=[2000, 900])
    o32 = _decode(spkv, wl, cache)
    o16 = _decode(spkv, wl, cache, out_dtype=torch.bfloat16)
    # round-to-nearest bf16: at most half a unit in the last place (2^-8 relative)
    assert torch.all(torch.abs(o16.float() - o32) <= torch.abs(o32) * 2.0 ** -8 + 1e-30)


# ------------------------------------------------------------ edge cases

def test_empty_and_fully_evicted_sequences_give_zero(spkv):
    m = spkv[0]
    wl, cache = _build(spkv, LLAMA, B=3, ctx=[0, 40, 300], Hq=4, Hkv=1)
    # evict every slot of sequence 1
    km = cache.keep_mask if cache.keep_mask is not None else torch.full(
        (wl.num_pages, wl.Hkv), -1, dtype=torch.int16, device="cuda")
    pages = wl.block_table_np[1, :3]
    km[torch.as_tensor(pages, device="cuda").long()] = 0
    cache.keep_mask = km
    out = _decode(spkv, wl, cache).cpu().numpy()
    assert np.all(out[0] == 0) and np.all(out[1] == 0)
    ref = helpers.oracle_seq(wl, 2, 0)
    assert np.max(np.abs(out[2] - ref)) <= OUT_TOL
    # B = 0 is a no-op
    m.decode_attention(cache, wl.q[:0], wl.block_table[:0], wl.ctx_tensor()[:0], 0)


def test_context_beyond_max_ctx_sets_flag_and_zero(spkv):
    m = spkv[0]
    wl, cache = _build(spkv, LLAMA, B=2, ctx=[64, 64], Hq=4, Hkv=1)
    ctx = torch.tensor([64, 64], dtype=torch.int32, device="cuda")
    out = m.decode_attention(cache, wl.q, wl.block_table, ctx, 32)  # max_ctx too small
    torch.cuda.synchronize()
    assert cache.error_flags() & 8
    assert torch.all(out == 0)


def test_bad_page_id_and_bad_header_are_flagged_not_fatal(spkv):
    m = spkv[0]
    wl, cache = _build(spkv, LLAMA, B=2, ctx=[100, 100], Hq=4, Hkv=1)
    bt = wl.block_table.clone()
    bt[0, 2] = wl.num_pages + 5
    cache.clear_errors()
    out = m.decode_attention(cache, wl.q, bt, wl.ctx_tensor(), wl.max_ctx)
    torch.cuda.synchronize()
    assert cache.error_flags() & 1
    assert torch.isfinite(out).all()
    hdr = cache.hdr.clone()
    cache.hdr[int(wl.block_table_np[1, 0]), 4] = 5  # b = 5 is not a tier
    cache.clear_errors()
    out = m.decode_attention(cache, wl.q, wl.block_table, wl.ctx_tensor(), wl.max_ctx)
    torch.cuda.synchronize()
    assert cache.error_flags() & 2
    assert torch.isfinite(out).all()
    cache.hdr.copy_(hdr)
    # sequence 0 is untouched by the bad header of sequence 1's first page
    ref = helpers.oracle_seq(wl, 0, 0)
    assert np.max(np.abs(out[0].cpu().numpy() - ref)) <= OUT_TOL


# ------------------------------------------------------ comparison paths

def test_dense_decode_parity(spkv):
    m, synthetic, workload = spkv
    wl = synthetic.make_workload(RAGGED, device="cuda", B=4, ctx=("loguniform", 30, 3000))
    kp, vp = workload.dense_pages(wl)
    km = torch.from_numpy(wl.keep_mask.view(np.int16)).cuda()
    out = m.dense_decode(kp, vp, wl.q, wl.block_table, wl.ctx_tensor(), wl.max_ctx, keep_mask=km).cpu().numpy()
    err = helpers.max_abs_diff_groups(out, wl, helpers.all_groups(wl), helpers.oracle_seq_dense)
    assert err <= OUT_TOL, err


def test_decompress_then_dot_parity(spkv):
    m = spkv[0]
    wl, cache = _build(spkv, RAGGED, B=3, ctx=("loguniform", 30, 2500))
    ks = torch.zeros_like(cache.v_pages)
    out = m.decompress_then_dot(cache, ks, wl.q, wl.block_table, wl.ctx_tensor(), wl.max_ctx).cpu().numpy()
    err = helpers.max_abs_diff_groups(out, wl, helpers.all_groups(wl), helpers.oracle_seq_decompress)
    assert err <= OUT_TOL, err
    # the materialised keys are bf16(r~ u~(c)) up to one bf16 ulp
    ksn = ks.view(torch.int16).cpu().numpy().view(np.uint16)
    for b, h in helpers.all_groups(wl)[:4]:
        keys, bits = wl.keys_bits(b, h), wl.token_bits(b)
        L, D = float(wl.rad_lo[h]), float(wl.rad_step[h])
        codes, rc = oracle.encode(keys, bits, L, D)
        want = oracle.bf16_to_f64(oracle.decompress(codes, bits, rc, L, D))
        n = int(wl.ctx[b])
        t = np.arange(n)
        got = oracle.bf16_to_f64(ksn[wl.block_table_np[b, t // 16], h, t % 16])
        assert np.all(np.abs(got - want) <= np.abs(want) * 2 ** -7 + 1e-30)
