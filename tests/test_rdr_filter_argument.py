"""The RDR plan kernel's fp32 filter, restated in numpy, against the fp64
decision it must reproduce.

The kernel tries each token's tier in fp32 (cost = fma(wf, eps_b, lambda R(b))
per tier, the eviction cost wf) and keeps the fp32 winner only when it beats
every other fp32 cost by the factor 1 - 2^-16; otherwise it decides in fp64.
The argument: each fp32 cost is within 2^-22 of the real cost (for |w| and
lambda R(b) zero or in [2^-100, 1e30]) and the fp64 cost within 2^-51.9, so an
accepted fp32 winner is the strict fp64 winner.  This test checks the claim
on random weights and multipliers and on constructed near-ties, where the
filter must either abstain or agree.  (The kernel itself is compared with the
oracle bit for bit in tests/test_rdr_gpu.py.)"""
import math

import numpy as np

BITS = (3, 4, 6, 8)
MARGIN = np.float32(1.0) - np.float32(2.0 ** -16)


def _eps(b):
    return math.pi / (2.0 ** b * math.sqrt(12.0))


def _rate(b, H):
    return float(H * (16 * b + 1 + 256))


def _fp64_choice(w, lam, mask, H):
    """The oracle's per-token minimiser (ties: the larger b), operations as written."""
    best, bc = -1, w * 1.0 + lam * 0.0
    for i, b in enumerate(BITS):
        if mask >> i & 1:
            c = w * _eps(b) + lam * _rate(b, H)
            if c <= bc:
                best, bc = i, c
    return best


def _fmaf(a, b, c):
    """fp32 fused multiply-add: the product of two fp32 values is exact in
    fp64; the sum is rounded once to fp32 (through fp64, whose rounding is
    far below fp32's for these ranges)."""
    return np.float32(float(a) * float(b) + float(c))


def _fp32_filter(w, lam, mask, H):
    """(tier index or -1, accepted) as the kernel's rdr_choose_fp32."""
    if not (w == 0.0 or 2.0 ** -100 <= w <= 1e30):
        return None, False
    lr = [lam * _rate(b, H) for b in BITS]
    if not (math.isfinite(lam) and all((mask >> i & 1) == 0 or x == 0.0 or 2.0 ** -100 <= x <= 1e30
                                       for i, x in enumerate(lr))):
        return None, False
    wf = np.float32(w)
    best, second, bi = wf, np.float32(np.inf), -1
    for i, b in enumerate(BITS):
        rf = np.float32(lr[i]) if mask >> i & 1 else np.float32(np.inf)
        c = _fmaf(wf, np.float32(_eps(b)), rf)
        if c <= best:
            best, second, bi = c, best, i
        else:
            second = min(second, c)
    return bi, bool(best < second * MARGIN)


def test_accepted_fp32_decisions_equal_the_fp64_ones_random():
    rng = np.random.default_rng(0)
    accepted = 0
    for _ in range(20000):
        H = int(rng.choice([1, 2, 8, 32]))
        mask = int(rng.integers(1, 16))
        w = float(2.0 ** rng.uniform(-100, 99)) if rng.random() > 0.02 else 0.0
        lam = float(2.0 ** rng.uniform(-60, 60)) if rng.random() > 0.02 else 0.0
        bi, ok = _fp32_filter(w, lam, mask, H)
        if ok:
            accepted += 1
            assert bi == _fp64_choice(w, lam, mask, H), (w, lam, mask, H)
    assert accepted > 15000  # the filter decides the clear cases


def test_near_ties_are_never_decided_wrongly():
    """lambda at the crossing of two tiers' costs (or of a tier and
    eviction), nudged by relative 1e-12 .. 1e-3: an accepted decision is the
    fp64 one, and the filter abstains when the nudge is below its margin."""
    rng = np.random.default_rng(1)
    opts = [(-1, 1.0, 0.0)] + [(i, _eps(b), None) for i, b in enumerate(BITS)]
    abstained_close = 0
    for _ in range(20000):
        H = int(rng.choice([1, 8]))
        w = float(2.0 ** rng.uniform(-20, 40))
        (i, ei, _), (j, ej, _) = [opts[k] for k in rng.choice(5, 2, replace=False)]
        ri = 0.0 if i < 0 else _rate(BITS[i], H)
        rj = 0.0 if j < 0 else _rate(BITS[j], H)
        if ri == rj:
            continue
        lam_star = w * (ei - ej) / (rj - ri)
        if lam_star <= 0:
            continue
        rel = float(10.0 ** rng.uniform(-12, -3)) * (1 if rng.random() < 0.5 else -1)
        lam = lam_star * (1 + rel)
        mask = 0xF
        bi, ok = _fp32_filter(w, lam, mask, H)
        if ok:
            assert bi == _fp64_choice(w, lam, mask, H), (w, lam, i, j, rel)
        elif abs(rel) < 2.0 ** -20:
            abstained_close += 1
    assert abstained_close > 0
