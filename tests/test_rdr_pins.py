"""Pins of the oracle's RDR controller (technical summary section 2.2,
readings R14-R17 in oracle/spkv_oracle.c).

The Lagrangian solve is pinned by brute force (no allocation with at most the
chosen rate has less surrogate distortion: Everett's theorem for the
multiplier found), the surrogate's eps_b by a Monte-Carlo RMS of the actual
angle quantiser, and the budget / protection rules by their definitions."""
import itertools
import math

import numpy as np
import pytest

import oracle

OPTIONS = (0, 3, 4, 6, 8)


def _keys(rng, T, H, d, scale=None):
    import torch

    x = rng.standard_normal((T, H, d)) * (scale if scale is not None else rng.lognormal(0, 0.7, (T, H, 1)))
    return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _w(keys, qn):
    kf = oracle.bf16_to_f64(keys)
    return (np.linalg.norm(kf, axis=2) * np.asarray(qn)[None, :]).sum(axis=1)


def _eps(b):
    return 1.0 if b == 0 else math.pi / (2 ** b * math.sqrt(12.0))


def _rate(b, H):
    return 0.0 if b == 0 else H * (16 * b + 1 + 256)


def test_eps_is_the_rms_error_of_the_angle_quantiser():
    rng = np.random.default_rng(1)
    phi = rng.uniform(0, math.pi, 200_000)
    for b in (3, 4, 6, 8):
        mids = np.array([oracle.angle_mid(oracle.angle_code(p, b, 0), b, 0) for p in phi[:20000]])
        rms = math.sqrt(np.mean((phi[:20000] - mids) ** 2))
        assert abs(rms / _eps(b) - 1.0) < 0.02, (b, rms, _eps(b))


@pytest.mark.parametrize("seed", [2, 3, 4])
def test_lagrangian_allocation_is_optimal_for_its_rate(seed):
    rng = np.random.default_rng(seed)
    T, H, d = 5, 2, 8
    keys = _keys(rng, T, H, d)
    qn = rng.uniform(0.5, 2.0, H)
    protect = np.zeros(T, np.uint8)
    protect[rng.integers(T)] = 1
    w = _w(keys, qn)
    full = T * _rate(8, H)
    for frac in (0.25, 0.4, 0.6, 0.85):  # (one protected token at b = 8 is 0.2 of full)
        tiers, lam, rate, dist, st = oracle.rdr_plan(keys, qn, frac * full, protect=protect)
        assert st == 0 and rate <= frac * full
        assert dist == pytest.approx(sum(w[t] * _eps(int(tiers[t])) for t in range(T)), rel=1e-12)
        assert rate == sum(_rate(int(b), H) for b in tiers)
        best = math.inf
        for choice in itertools.product(OPTIONS, repeat=T):
            if any(protect[t] and choice[t] != 8 for t in range(T)):
                continue
            r = sum(_rate(b, H) for b in choice)
            if r <= rate:
                best = min(best, sum(w[t] * _eps(choice[t]) for t in range(T)))
        assert dist <= best * (1 + 1e-12), (dist, best)


def test_budget_protection_and_limits():
    rng = np.random.default_rng(5)
    T, H, d = 64, 4, 32
    keys = _keys(rng, T, H, d)
    qn = np.ones(H)
    protect = np.zeros(T, np.uint8)
    protect[:4] = 1
    full = T * _rate(8, H)
    # everything fits: all at b_max, lambda = 0
    tiers, lam, rate, dist, st = oracle.rdr_plan(keys, qn, full, protect=protect)
    assert st == 0 and lam == 0.0 and np.all(tiers == 8)
    # tier mask {3, 4}: b_max = 4
    tiers, lam, rate, dist, st = oracle.rdr_plan(keys, qn, full, tier_mask=0x3, protect=protect)
    assert np.all(tiers == 4)
    # a tight budget: protected at b_max, the rest fits
    budget = 0.3 * full
    tiers, lam, rate, dist, st = oracle.rdr_plan(keys, qn, budget, protect=protect)
    assert st == 0 and rate <= budget and np.all(tiers[:4] == 8) and lam > 0
    # only the protected tokens fit: every other token evicted
    tiers, lam, rate, dist, st = oracle.rdr_plan(keys, qn, 4 * _rate(8, H), protect=protect)
    assert st == 0 and np.all(tiers[:4] == 8) and np.all(tiers[4:] == 0)
    # infeasible: the protected tokens alone exceed the budget
    tiers, lam, rate, dist, st = oracle.rdr_plan(keys, qn, 3 * _rate(8, H), protect=protect)
    assert st == 1 and np.all(tiers[:4] == 8) and np.all(tiers[4:] == 0)


def test_distortion_falls_as_the_budget_grows():
    rng = np.random.default_rng(6)
    keys = _keys(rng, 200, 4, 32)
    qn = rng.uniform(0.5, 2.0, 4)
    full = 200 * _rate(8, 4)
    prev_d, prev_r = math.inf, -1.0
    for frac in np.linspace(0.05, 1.0, 12):
        _, _, rate, dist, st = oracle.rdr_plan(keys, qn, frac * full)
        assert st == 0 and rate <= frac * full
        assert dist <= prev_d * (1 + 1e-12) and rate >= prev_r
        prev_d, prev_r = dist, rate


def test_high_weight_tokens_are_kept_first():
    """With equal rates per tier, the surrogate orders tokens by w_t: under a
    budget for half the tokens, every kept token weighs at least every evicted one."""
    rng = np.random.default_rng(7)
    T, H = 40, 2
    keys = _keys(rng, T, H, 16)
    qn = np.ones(H)
    tiers, _, _, _, st = oracle.rdr_plan(keys, qn, T / 2 * _rate(4, H), tier_mask=0x2)
    w = _w(keys, qn)
    kept, evicted = w[tiers > 0], w[tiers == 0]
    assert st == 0 and len(kept) and len(evicted)
    assert kept.min() >= evicted.max()


def test_infeasible_plan_reports_an_infinite_multiplier():
    rng = np.random.default_rng(8)
    keys = _keys(rng, 10, 2, 16)
    protect = np.ones(10, np.uint8)
    tiers, lam, rate, _, st = oracle.rdr_plan(keys, np.ones(2), 9 * _rate(8, 2), protect=protect)
    assert st == 1 and lam == math.inf and np.all(tiers == 8) and rate == 10 * _rate(8, 2)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_pack_makes_tier_homogeneous_pages(seed):
    """Every resident token lands in exactly one slot of a page of its own
    tier; pages are grouped by ascending tier; the keep bits are the occupied
    slots; a group of n tokens takes ceil(n / 16) pages."""
    rng = np.random.default_rng(seed)
    T = int(rng.integers(1, 300))
    tiers = rng.choice(OPTIONS, size=T, p=[0.2, 0.2, 0.3, 0.2, 0.1])
    dst, bits, keep = oracle.rdr_pack(tiers)
    assert np.all((dst < 0) == (tiers == 0))
    kept = dst[dst >= 0]
    assert len(np.unique(kept)) == len(kept)
    occupied = np.zeros((len(bits), 16), bool)
    occupied[kept // 16, kept % 16] = True
    for p in range(len(bits)):
        assert keep[p] == sum(1 << s for s in range(16) if occupied[p, s])
    assert np.all(bits[dst[tiers > 0] // 16] == tiers[tiers > 0])
    assert np.all(np.diff(bits.astype(int)) >= 0)
    assert len(bits) == sum(-(-int(np.sum(tiers == b)) // 16) for b in (3, 4, 6, 8))
    for b in (3, 4, 6, 8):  # ascending t within a tier
        assert np.all(np.diff(dst[tiers == b]) > 0)


@pytest.mark.parametrize("seed", [10, 11])
def test_packed_layout_gives_the_attention_of_the_kept_tokens(seed):
    """Attention over the packed pages (tokens moved to dst_pos, page bit
    widths, slot keep bits) equals attention over the kept tokens in their
    original order with the plan's tiers: the packing loses, duplicates and
    re-tiers nothing."""
    rng = np.random.default_rng(seed)
    T, H, d, G = 150, 2, 128, 2
    keys = _keys(rng, T, H, d)
    vals = _keys(rng, T, H, d, scale=1.0)
    qn = rng.uniform(0.5, 2.0, H)
    protect = np.zeros(T, np.uint8)
    protect[:4] = 1
    tiers, _, _, _, st = oracle.rdr_plan(keys, qn, 0.3 * T * _rate(8, H), protect=protect)
    assert st == 0 and np.any(tiers == 0) and len(set(tiers[tiers > 0].tolist())) > 1
    dst, pbits, pkeep = oracle.rdr_pack(tiers)
    n_slots = 16 * len(pbits)
    kept = np.nonzero(tiers > 0)[0]
    for h in range(H):
        q = _keys(rng, G, 1, d)[:, 0]
        L, D = -2.0, 0.05
        bits0 = np.where(tiers > 0, tiers, 8).astype(np.int32)
        c0, r0 = oracle.encode(keys[:, h], bits0, L, D)
        ref = oracle.ada_group(q, c0, bits0, r0, L, D, vals[:, h], keep=(tiers > 0).astype(np.uint8))
        # the packed sequence: slot s of page p holds the token with dst = 16 p + s
        pk = np.zeros((n_slots, d), np.uint16)
        pv = np.zeros((n_slots, d), np.uint16)
        pk[dst[kept]] = keys[kept, h]
        pv[dst[kept]] = vals[kept, h]
        sbits = np.repeat(pbits.astype(np.int32), 16)
        skeep = ((pkeep[:, None].astype(np.int64) >> np.arange(16)) & 1).reshape(-1).astype(np.uint8)
        c1, r1 = oracle.encode(pk, sbits, L, D)
        got = oracle.ada_group(q, c1, sbits, r1, L, D, pv, keep=skeep)
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("frac", [0.2, 0.45, 0.7])
def test_multiplier_is_the_smallest_that_fits(frac):
    """The solver's lambda fits the budget and the next smaller double does
    not (the bisection converges to adjacent doubles); its tiers are the
    per-token minimisers at lambda."""
    rng = np.random.default_rng(12)
    T, H, d = 300, 4, 64
    keys = _keys(rng, T, H, d)
    qn = rng.uniform(0.5, 2.0, H)
    budget = frac * T * _rate(8, H)
    tiers, lam, rate, _, st = oracle.rdr_plan(keys, qn, budget)
    assert st == 0 and 0.0 < lam < math.inf
    t_at, r_at = oracle.rdr_assign(keys, qn, lam)
    np.testing.assert_array_equal(t_at, tiers)
    assert r_at == rate <= budget
    _, r_below = oracle.rdr_assign(keys, qn, np.nextafter(lam, 0.0))
    assert r_below > budget
    # rate is non-increasing in lambda
    rates = [oracle.rdr_assign(keys, qn, x)[1] for x in np.geomspace(lam / 64, lam * 64, 25)]
    assert all(a >= b for a, b in zip(rates, rates[1:]))
