"""Host pins of the bulk encoder's two reorganisations (spkv_encode.cuh), restated
in numpy and checked against the oracle, which decides each code from its plain
definition: the angle code is floor(phi 2^b / pi) (azimuth: floor(phi 2^b / 2 pi))
of the hyperspherical angles, with phi_i = atan2(sqrt(S_(i+1)), x_i) (technical
summary of "SPHERICAL KV: Angle-Domain Attention and Rate-Distortion Retention",
section 2.1).

1. The half-range search.  Rather than the full binary search over all 2^b - 1
   cell edges, the kernel lets the sign of x_i pick the half of [0, pi] the
   polar angle lies in and searches that half's 2^(b-1) edges in b - 1 steps
   (x > 0: the largest k with x^2 <= S c2[k]; x < 0: 2^(b-1) + the largest j
   with j = 0 or x^2 >= S c2[2^(b-1) + j], tested as -x^2 <= S (-c2[...]);
   x = 0: 2^(b-1), which the x < 0 branch gives; S = 0: 0), with
   c2[k] = cos^2(k pi / 2^b), adding the steps 2^(b-2), ..., 1 while the test
   holds; the bulk encoder keeps -c2 in the table's upper half, the decode's
   fused append puts the sign on S (both restated).  Restated here and compared, code by code, with the oracle's codes
   of random bf16 keys (equal off the cell edges) and with a brute-force scan
   of every edge (equal everywhere, ties included).
2. The slot words.  Codes are pushed four at a time (fields 4g .. 4g + 3,
   groups 31 down to 0) into a 64-bit accumulator (acc = acc << 4b | grp) and
   word w = stream bits [32 w, 32 w + 32) is taken once the lowest pushed code
   starts at or below bit 32 w; the four words of chunk w / 4 land at byte
   (16 (w / 4) + slot) 16 of the record.
   Restated here, and the record read back with the layout reader the GPU
   parity tests use (the chunk-major layout of the library header).

3. The non-uniform encoder's search: per-angle edges from the library's host
   tables, decided as x |x| <= S (c |c|) for either sign of c = cos theta by
   steps 2^(b-1) .. 1; restated and compared with a scan of every edge under
   the plain test and with the non-uniform oracle's codes off the cell edges.

These are restatements of the kernel's steps (the kernel itself needs a GPU);
what pins them is the oracle and the plain definitions, not the kernel.
"""
import math

import numpy as np
import pytest

import oracle
from tests import helpers

D = 128


def _cospi(t):
    """cos(pi t), exact at multiples of 1/2 (the edges a bf16 input can hit exactly)."""
    t = np.asarray(t, np.float64)
    r = np.cos(np.pi * t)
    half = np.isclose(t * 2, np.round(t * 2), rtol=0, atol=0)
    exact = np.array([1.0, 0.0, -1.0, 0.0])[np.mod(np.round(t * 2).astype(np.int64), 4)]
    return np.where(half, exact, r)


def _c2_polar(b):
    k = np.arange(1 << b)
    return 0.5 * (1.0 + _cospi(2.0 * k / (1 << b)))


def _suffix_sums(x):
    """S_i = sum_(j >= i) x_j^2 in the kernel's fixed order (groups of four,
    fma within a group, then the groups' sums from the top).  The square of a
    bf16 value is exact in fp64, so fma(x, x, s) rounds like x * x + s."""
    S = np.empty(D)
    T = 0.0
    for g in range(31, -1, -1):
        xs = x[4 * g:4 * g + 4]
        s3 = xs[3] * xs[3]
        s2 = xs[2] * xs[2] + s3
        s1 = xs[1] * xs[1] + s2
        s0 = xs[0] * xs[0] + s1
        S[4 * g:4 * g + 4] = (s0 + T, s1 + T, s2 + T, s3 + T)
        T = s0 + T
    return S


def _polar_half(x, S, c2, b, half_signed=True):
    """The kernel's half-range search (restated): the code starts at 0 (x > 0)
    or 2^(b-1) (x <= 0) and takes the steps 2^(b-2) .. 1 while
    x |x| <= S e[k]; e is the half-signed table (-c2 from 2^(b-1) on), or the
    plain one with the sign on S instead (the decode's fused append)."""
    H = 1 << (b - 1)
    pos = x > 0.0
    sx2 = x * abs(x)
    if half_signed:
        e = np.where(np.arange(1 << b) >= H, -c2, c2)
        sS = S
    else:
        e = c2
        sS = S if pos else -S
    k = 0 if pos else H
    step = H // 2
    while step >= 1:
        if sx2 <= sS * e[k + step]:
            k += step
        step //= 2
    return 0 if S == 0.0 else k


def _polar_scan(x, S, c2, b):
    """Brute force: the largest edge k the angle reaches, phi >= k pi / 2^b
    <=> x <= sqrt(S) cos(k pi / 2^b), decided on squares and signs."""
    if S == 0.0:
        return 0
    best = 0
    for k in range(1, 1 << b):
        cos_nonneg = 2 * k <= (1 << b)
        rhs = S * c2[k]
        reach = (x <= 0.0 or x * x <= rhs) if cos_nonneg else (x < 0.0 and x * x >= rhs)
        if reach:
            best = k
    return best


def _keys(n, seed):
    """bf16 keys N(0, 1) with log-normal channel scales and four x10 outlier channels."""
    rng = np.random.default_rng(seed)
    scale = np.exp(rng.normal(0.0, 0.5, D))
    scale[rng.choice(D, 4, replace=False)] *= 10.0
    x = (rng.standard_normal((n, D)) * scale).astype(np.float32)
    bits = (x.view(np.uint32) + 0x7FFF + ((x.view(np.uint32) >> 16) & 1)) >> 16  # round to nearest even
    return bits.astype(np.uint16)


@pytest.mark.parametrize("b", [3, 4, 6, 8])
def test_half_range_search_matches_the_oracle_codes(b):
    keys = _keys(48, seed=100 + b)
    # a few keys with exact ties and zeros: x_i = +-x_(i+1) pairs, zero tails
    keys[0, 64:] = 0
    keys[1, ::2] = keys[1, 1::2]
    keys[2, 100:] = 0x3F80  # 1.0: polar angles of pi/4-type ties
    keys[3, 126:] = 0x3F80
    c2 = _c2_polar(b)
    codes, _, apos, _ = oracle.encode(keys, b, 0.0, 0.05, positions=True)
    edge = helpers.near_integer(apos)
    n_checked = 0
    for t in range(keys.shape[0]):
        x = oracle.bf16_to_f64(keys[t])
        S = _suffix_sums(x)
        for i in range(126):
            got = _polar_half(x[i], S[i], c2, b)
            assert got == _polar_half(x[i], S[i], c2, b, half_signed=False)
            assert got == _polar_scan(x[i], S[i], c2, b), (t, i, x[i], S[i])
            if not edge[t, i]:
                assert got == codes[t, i], (t, i, got, codes[t, i], apos[t, i])
            n_checked += 1
    assert n_checked == 48 * 126


@pytest.mark.parametrize("b", [3, 4, 6, 8])
def test_half_range_search_on_exact_edges(b):
    """Inputs whose angle sits exactly on an edge that fp64 represents exactly
    (multiples of pi/4): decided to the upper cell, as the definition says."""
    c2 = _c2_polar(b)
    n = 1 << b
    # phi = pi/4 (x = 1, S = 2), pi/2 (x = 0), 3 pi/4 (x = -1, S = 2), 0, and a zero suffix
    assert _polar_half(1.0, 2.0, c2, b) == n // 4
    assert _polar_half(0.0, 5.0, c2, b) == n // 2
    assert _polar_half(-1.0, 2.0, c2, b) == 3 * n // 4
    assert _polar_half(3.0, 9.0, c2, b) == 0
    assert _polar_half(-3.0, 9.0, c2, b) == n - 1  # phi = pi: clamped to the last cell
    assert _polar_half(0.0, 0.0, c2, b) == 0
    for x, S in [(1.0, 2.0), (0.0, 5.0), (-0.0, 5.0), (-1.0, 2.0), (3.0, 9.0), (-3.0, 9.0)]:
        assert _polar_half(x, S, c2, b) == _polar_scan(x, S, c2, b)
        assert _polar_half(x, S, c2, b, half_signed=False) == _polar_scan(x, S, c2, b)
        phi = math.atan2(math.sqrt(max(S - x * x, 0.0)), x)
        assert _polar_half(x, S, c2, b) == oracle.angle_code(phi, b, False)


def _slot_words(codes, b, slot, rec):
    """The kernel's accumulator push (restated) into record bytes `rec`."""
    nwords = 4 * b
    acc, w = 0, nwords - 1
    stage = [0, 0, 0, 0]
    mask64 = (1 << 64) - 1
    for g in range(31, -1, -1):
        grp = 0
        for k in range(4):
            i = 4 * g + k
            grp |= (int(codes[i]) if i < 127 else 0) << (k * b)
        acc = ((acc << (4 * b)) | grp) & mask64
        i = 4 * g
        if i * b <= 32 * w:
            word = (acc >> (32 * w - i * b)) & 0xFFFFFFFF
            stage[w & 3] = word
            if (w & 3) == 0:
                off = ((w >> 2) * 16 + slot) * 16
                rec[off:off + 16] = np.array(stage, np.uint32).view(np.uint8)
            w -= 1
    assert w == -1


@pytest.mark.parametrize("b", [3, 4, 6, 8])
def test_slot_words_write_the_documented_layout(b):
    rng = np.random.default_rng(7 + b)
    rec = np.zeros(256 * b + 16, np.uint8)
    codes = rng.integers(0, 1 << b, size=(16, 127), dtype=np.int64)
    codes[0] = (1 << b) - 1  # all ones: every word boundary carries bits
    for s in range(16):
        _slot_words(codes[s], b, s, rec)
    got, _, pads = helpers.unpack_records(rec[None, :], b)
    assert np.array_equal(got[0], codes)
    assert np.all(pads == 0)


# ---------------------------------------------------------------- non-uniform

def _polar_nu(x, S, ec, b):
    """The non-uniform encoder's search (restated): the largest j with edge j
    reached, x |x| <= S (c |c|) for c = cos theta_j, by steps 2^(b-1) .. 1."""
    sx2 = x * abs(x)
    k = 0
    step = 1 << (b - 1)
    while step >= 1:
        c = ec[k + step - 1]
        if sx2 <= S * (c * abs(c)):
            k += step
        step //= 2
    return 0 if S == 0.0 else k


def _polar_nu_scan(x, S, ec):
    """Brute force with the plain test: phi >= theta <=> x <= sqrt(S) cos theta,
    i.e. x <= 0 or x^2 <= S c^2 for c >= 0, x < 0 and x^2 >= S c^2 for c < 0."""
    if S == 0.0:
        return 0
    best = 0
    for j, c in enumerate(ec, start=1):
        rhs = S * (c * c)
        reach = (x <= 0.0 or x * x <= rhs) if c >= 0.0 else (x < 0.0 and x * x >= rhs)
        if reach:
            best = j
    return best


@pytest.mark.parametrize("b", [3, 4, 6, 8])
def test_nonuniform_signed_square_search(b):
    """The signed-square search equals the plain edge scan everywhere (ties and
    zeros included) and the oracle's non-uniform codes off the cell edges."""
    from compressed_kv_decode_ada_b200 import ops
    from oracle import nonuniform as onu

    ec, _, _ = ops.nonuniform_tables(D, b)
    keys = _keys(12, seed=300 + b)
    keys[0, 64:] = 0
    keys[1, ::2] = keys[1, 1::2]
    n = 1 << b
    codes, _ = onu.encode(keys, b, 0.0, 0.05)
    n_checked = 0
    for t in range(keys.shape[0]):
        x = oracle.bf16_to_f64(keys[t])
        S = _suffix_sums(x)
        phi = oracle.angles(x)
        for i in range(126):
            got = _polar_nu(x[i], S[i], ec[i], b)
            assert got == _polar_nu_scan(x[i], S[i], ec[i]), (t, i)
            pos = n * float(onu.polar_cdf(phi[i], D, i + 1))
            if abs(pos - round(pos)) > 1e-9 * max(1.0, abs(pos)):
                assert got == codes[t, i], (t, i, got, codes[t, i], pos)
            n_checked += 1
        # a zero input is the middle code: phi = pi / 2 sits on the middle edge
        assert _polar_nu(0.0, 1.0, ec[0], b) == _polar_nu_scan(0.0, 1.0, ec[0])
    assert n_checked == 12 * 126
