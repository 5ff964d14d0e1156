"""GPU <-> oracle parity of the RDR controller (spkv_rdr_plan, technical
summary section 2.2) and of the cache it packs, through the C ABI.

The plan's decisions are integers decided in fp64 by the same operations on
both sides, so tiers, packed positions, pages, the multiplier lambda and the
rate are compared exactly; the distortion is a sum whose order differs
(sequential on the oracle, per CTA on the GPU) and is compared to 1e-11
relative (a recursive sum of n <= 2^16 positive terms is within (n - 1) u
< 7.3e-12 of the exact sum).  The decode of a packed cache is compared with the oracle's ADA
decode over the kept tokens in their original order, to the decode
tolerance 2e-3.
"""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

OUT_TOL = 2e-3
RAGGED = "ragged_rdr_b32_h32x8_t1k-64k_mixed_b_mask25"
LLAMA = "llama3_8b_b8_h32x8_t32768_b4"


@pytest.fixture(scope="module")
def spkv():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import compressed_kv_decode_ada_b200 as m
    from compressed_kv_decode_ada_b200 import synthetic

    return m, synthetic


def _keys_np(wl):
    return wl.keys.cpu().view(torch.int16).numpy().view(np.uint16)


def _plan(m, wl, ri, tier_mask=0xF, budget=None, protect=True, max_pages_out=None, seq_start=None):
    dev = wl.keys.device
    out = m.rdr_plan(wl.keys, torch.from_numpy(ri.seq_start if seq_start is None else seq_start).to(dev),
                     torch.from_numpy(ri.q_norms).to(dev),
                     torch.from_numpy(np.asarray(ri.budget if budget is None else budget, np.float64)).to(dev),
                     protect=torch.from_numpy(ri.protect).to(dev) if protect else None, tier_mask=tier_mask,
                     max_pages_out=max_pages_out)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in out.items()}


def _oracle_seq(keys, ri, b, tier_mask, budget, protect):
    s0, s1 = int(ri.seq_start[b]), int(ri.seq_start[b + 1])
    return oracle.rdr_plan(keys[s0:s1], ri.q_norms[b].astype(np.float64), float(budget[b]), tier_mask=tier_mask,
                           protect=ri.protect[s0:s1] if protect else None)


def _check(wl, ri, got, tier_mask=0xF, budget=None, protect=True):
    keys = _keys_np(wl)
    budget = ri.budget if budget is None else budget
    for b in range(wl.B):
        s0, s1 = int(ri.seq_start[b]), int(ri.seq_start[b + 1])
        tiers, lam, rate, dist, st = _oracle_seq(keys, ri, b, tier_mask, budget, protect)
        np.testing.assert_array_equal(got["tier"][s0:s1], tiers, err_msg=f"seq {b}")
        assert got["lambda"][b] == lam, (b, got["lambda"][b], lam)
        assert got["rate"][b] == rate, (b, got["rate"][b], rate)
        assert got["status"][b] == st, (b, got["status"][b], st)
        assert got["dist"][b] == pytest.approx(dist, rel=1e-11, abs=1e-300)
        dst, pb, pk = oracle.rdr_pack(tiers)
        np.testing.assert_array_equal(got["dst_pos"][s0:s1], dst, err_msg=f"seq {b}")
        assert got["n_pages"][b] == len(pb)
        np.testing.assert_array_equal(got["page_bits"][b, :len(pb)], pb)
        np.testing.assert_array_equal(got["page_keep"][b, :len(pb)].view(np.uint16), pk)


@pytest.mark.parametrize("Hkv,frac,mask", [(8, 0.35, 0xF), (8, 0.1, 0xF), (3, 0.3, 0x3), (1, 0.5, 0xA),
                                           (32, 0.2, 0x1), (5, 0.6, 0xE)])
def test_plan_matches_oracle_ragged(spkv, Hkv, frac, mask):
    """Ragged sequences (empty, one token, a partial page, several CTAs of
    the cluster) with sinks + recent window protected."""
    m, syn = spkv
    wl = syn.make_workload(RAGGED, B=6, ctx=[0, 1, 17, 700, 9000, 3001], Hq=Hkv, Hkv=Hkv, seed=11 + Hkv)
    ri = syn.make_rdr_inputs(wl, budget_frac=frac)
    _check(wl, ri, _plan(m, wl, ri, tier_mask=mask), tier_mask=mask)


def test_plan_without_protection(spkv):
    m, syn = spkv
    wl = syn.make_workload(RAGGED, B=3, ctx=[333, 4096, 50], Hq=8, Hkv=8, seed=21)
    ri = syn.make_rdr_inputs(wl, budget_frac=0.25)
    _check(wl, ri, _plan(m, wl, ri, protect=False), protect=False)


def test_plan_limits(spkv):
    """lambda = 0 (everything fits), budget 0 (everything evicted), a
    negative budget (infeasible: lambda = +inf), protected tokens alone over
    the budget."""
    m, syn = spkv
    wl = syn.make_workload(RAGGED, B=4, ctx=[200, 1000, 64, 2048], Hq=8, Hkv=8, seed=22)
    ri = syn.make_rdr_inputs(wl)
    full = wl.ctx.astype(np.float64) * 8 * (16 * 8 + 257)
    budget = np.array([full[0], 0.0, -1.0, 10.0 * 8 * 385])
    got = _plan(m, wl, ri, budget=budget, protect=False)
    _check(wl, ri, got, budget=budget, protect=False)
    assert got["lambda"][0] == 0.0 and np.all(got["tier"][:200] == 8)
    assert got["status"][2] == 1 and got["lambda"][2] == np.inf
    got = _plan(m, wl, ri, budget=budget, protect=True)
    _check(wl, ri, got, budget=budget, protect=True)
    assert got["status"][3] == 1  # all 64 tokens protected (sinks + window) > 10 tokens of bytes


def test_plan_page_capacity_and_bad_ranges(spkv):
    m, syn = spkv
    wl = syn.make_workload(RAGGED, B=2, ctx=[500, 300], Hq=8, Hkv=8, seed=23)
    ri = syn.make_rdr_inputs(wl, budget_frac=0.5)
    got = _plan(m, wl, ri, max_pages_out=4)
    ref = [_oracle_seq(_keys_np(wl), ri, b, 0xF, ri.budget, True) for b in range(2)]
    for b in range(2):
        s0, s1 = int(ri.seq_start[b]), int(ri.seq_start[b + 1])
        assert got["status"][b] & 2 and np.all(got["dst_pos"][s0:s1] == -1)
        np.testing.assert_array_equal(got["tier"][s0:s1], ref[b][0])
        assert got["n_pages"][b] == len(oracle.rdr_pack(ref[b][0])[1])
    bad = np.array([0, 600, 500], np.int32)  # second range runs backwards
    got = _plan(m, wl, ri, seq_start=bad)
    assert got["status"][1] == 4 and got["n_pages"][1] == 0


def test_plan_full_size_sequences_match_oracle(spkv):
    """Two sequences of 32768 tokens x 8 kv heads (the Llama-3-8B decode
    shape), budget 35% of b = 8."""
    m, syn = spkv
    wl = syn.make_workload(LLAMA, B=2)
    ri = syn.make_rdr_inputs(wl, budget_frac=0.35)
    _check(wl, ri, _plan(m, wl, ri))


def test_plan_ragged_workload_full_size(spkv):
    """The ragged 32-sequence workload (1K-64K tokens each) at full size:
    every sequence compared with the oracle."""
    m, syn = spkv
    wl = syn.make_workload(RAGGED)
    ri = syn.make_rdr_inputs(wl, budget_frac=0.35)
    _check(wl, ri, _plan(m, wl, ri))


def test_packed_cache_decode_matches_oracle(spkv):
    """plan -> packed tier-homogeneous pages -> spkv_encode_keys_packed ->
    ADA decode, against the oracle's ADA decode of the same tokens in their
    original order with the plan's tiers and evictions."""
    m, syn = spkv
    wl = syn.make_workload(RAGGED, B=3, ctx=[500, 2000, 70], Hq=8, Hkv=2, seed=24)
    ri = syn.make_rdr_inputs(wl, budget_frac=0.3)
    dev = wl.keys.device
    plan = m.rdr_plan(wl.keys, torch.from_numpy(ri.seq_start).to(dev), torch.from_numpy(ri.q_norms).to(dev),
                      torch.from_numpy(ri.budget).to(dev), protect=torch.from_numpy(ri.protect).to(dev))
    cache, bt, ctx = m.build_packed_cache(plan, wl.keys, wl.values, torch.from_numpy(ri.seq_start).to(dev),
                                          wl.rad_lo, wl.rad_step)
    max_ctx = int(ctx.max().item())
    out = m.decode_attention(cache, wl.q, bt, ctx, max_ctx)
    torch.cuda.synchronize()
    assert cache.error_flags() == 0
    out = out.cpu().numpy()
    tiers = plan["tier"].cpu().numpy()
    keys = _keys_np(wl)
    vals = wl.values.cpu().view(torch.int16).numpy().view(np.uint16)
    qb = wl.q.cpu().view(torch.int16).numpy().view(np.uint16)
    G = wl.Hq // wl.Hkv
    worst = 0.0
    for b in range(wl.B):
        s0, s1 = int(ri.seq_start[b]), int(ri.seq_start[b + 1])
        tb = tiers[s0:s1].astype(np.int32)
        keep = (tb > 0).astype(np.uint8)
        bits = np.where(tb > 0, tb, 8)
        for h in range(wl.Hkv):
            L, D = float(wl.rad_lo[h]), float(wl.rad_step[h])
            codes, rcode = oracle.encode(keys[s0:s1, h], bits, L, D)
            ref = oracle.ada_group(qb[b, h * G:(h + 1) * G], codes, bits, rcode, L, D, vals[s0:s1, h], keep=keep)
            worst = max(worst, float(np.max(np.abs(out[b, h * G:(h + 1) * G] - ref))))
    assert worst <= OUT_TOL, worst


def test_plan_extreme_weights(spkv):
    """Zero keys (w = 0: every cost ties at lambda = 0), huge keys (w above
    the fp32 filter's range) and tiny keys (below it) are decided exactly."""
    m, syn = spkv
    wl = syn.make_workload(RAGGED, B=3, ctx=[400, 1500, 900], Hq=8, Hkv=8, seed=25)
    k = wl.keys.float()
    k[0:30] = 0.0
    k[450:470] *= 1e35
    k[600:640] *= 1e-36
    k[1500:1520] = 0.0
    wl.keys = k.to(torch.bfloat16)
    for frac in (0.2, 0.5, 0.95):
        ri = syn.make_rdr_inputs(wl, budget_frac=frac)
        _check(wl, ri, _plan(m, wl, ri))
        _check(wl, ri, _plan(m, wl, ri, protect=False), protect=False)


def test_plan_sequence_longer_than_shared_memory(spkv):
    """One sequence of 140,000 tokens: each CTA's share (17,500) exceeds the
    16,384 weights it keeps in shared memory, so the rest is read from global
    memory on every pass."""
    m, syn = spkv
    wl = syn.make_workload(RAGGED, B=1, ctx=[140000], Hq=1, Hkv=1, seed=26)
    ri = syn.make_rdr_inputs(wl, budget_frac=0.4)
    _check(wl, ri, _plan(m, wl, ri))
