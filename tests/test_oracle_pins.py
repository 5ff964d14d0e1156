"""Pins of the fp64 oracle against facts fixed outside the oracle itself.

Each test checks the oracle against something it does not compute itself: a
hand-derived closed form (tests/golden/closed_forms.txt), a textbook identity,
an error bound of the quantiser, brute force on tiny inputs, or a library
routine (numpy, torch).  Definitions: "SPHERICAL KV: Angle-Domain Attention and
Rate-Distortion Retention for Efficient Long-Context Inference", technical
summary section 2.1 (spherical parametrisation, logit from codes, f_b as a
cosine from angle codes), with the readings R1-R7 stated in oracle/spkv_oracle.c.
"""
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_forms.txt")
BITS = (3, 4, 6, 8)


def _bf16(x):
    """fp32 values -> bf16 bit patterns by truncation of exactly representable values."""
    a = np.asarray(x, np.float32)
    u = a.view(np.uint32)
    assert np.all((u & 0xFFFF) == 0), "test inputs must be exact bf16 values"
    return (u >> 16).astype(np.uint16)


def _rand_bf16(rng, shape, scale=1.0):
    import torch

    t = torch.from_numpy((rng.standard_normal(shape) * scale).astype(np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


# ------------------------------------------------------------------ golden

def _golden_lines(kind):
    out = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = [p.strip() for p in line.split("|")]
            if parts[0] == kind:
                out.append(parts[1:])
    return out


@pytest.mark.parametrize("case", _golden_lines("encode"))
def test_golden_encode(case):
    head, xs, codes, rcode = case
    d, b, L, delta = head.split()
    d, b, L, delta = int(d), int(b), float(L), float(delta)
    x = np.array([float(v) for v in xs.split()], np.float32)
    got_c, got_r = oracle.encode(_bf16(x)[None, :], b, L, delta)
    assert got_c[0].tolist() == [int(v) for v in codes.split()]
    assert int(got_r[0]) == int(rcode)


@pytest.mark.parametrize("case", _golden_lines("fb"))
def test_golden_fb(case):
    head, cq, ck, want = case
    d, b = (int(v) for v in head.split())
    cq = np.array([int(v) for v in cq.split()], np.int32)
    ck = np.array([int(v) for v in ck.split()], np.int32)
    assert len(cq) == d - 1
    assert oracle.fb(cq, ck, b) == pytest.approx(float(want), abs=1e-15)
    assert oracle.fb_nested(cq, ck, b) == pytest.approx(float(want), abs=1e-15)


# ------------------------------------------------------- chart invariants

@pytest.mark.parametrize("b", BITS + (12,))
def test_unit_norm_of_decoded_codes(b):
    """sin^2 + cos^2 telescopes: every decoded code vector has unit norm."""
    rng = np.random.default_rng(b)
    for d in (2, 3, 17, 128):
        for _ in range(20):
            c = rng.integers(0, 2 ** b, size=d - 1).astype(np.int32)
            u = oracle.unit_from_codes(c, b)
            assert abs(np.linalg.norm(u) - 1.0) <= 1e-13


def test_unquantised_round_trip():
    """Phi^-1(Phi(x)) = x/||x|| for the unquantised chart."""
    rng = np.random.default_rng(1)
    for d in (2, 3, 5, 128):
        for _ in range(50):
            x = rng.standard_normal(d)
            u = oracle.unit_from_angles(oracle.angles(x))
            assert np.max(np.abs(u - x / np.linalg.norm(x))) <= 1e-13


def test_angles_against_arccos_definition():
    """cos(phi_i) = x_i / ||x_{i:}|| (polar) and the azimuth's (cos, sin) = (x_{d-2}, x_{d-1}) / rho,
    computed here with numpy from cumulative sums, independently of the oracle."""
    rng = np.random.default_rng(2)
    d = 128
    for _ in range(50):
        x = rng.standard_normal(d)
        phi = oracle.angles(x)
        tail = np.sqrt(np.cumsum((x ** 2)[::-1])[::-1])
        assert np.all(phi[:-1] >= 0) and np.all(phi[:-1] <= math.pi)
        assert 0 <= phi[-1] < 2 * math.pi
        assert np.max(np.abs(np.cos(phi[:-1]) - x[:-2] / tail[:-2])) <= 1e-14
        rho = math.hypot(x[-2], x[-1])
        assert abs(math.cos(phi[-1]) - x[-2] / rho) <= 1e-14
        assert abs(math.sin(phi[-1]) - x[-1] / rho) <= 1e-14


def test_exact_dot_with_unquantised_angles():
    """||q|| ||k|| <Phi^-1 Phi(q^), Phi^-1 Phi(k^)> = q . k."""
    rng = np.random.default_rng(3)
    for _ in range(100):
        q, k = rng.standard_normal(128), rng.standard_normal(128)
        uq = oracle.unit_from_angles(oracle.angles(q))
        uk = oracle.unit_from_angles(oracle.angles(k))
        got = np.linalg.norm(q) * np.linalg.norm(k) * float(uq @ uk)
        assert abs(got - float(q @ k)) <= 1e-12 * np.linalg.norm(q) * np.linalg.norm(k)


def test_d2_closed_form():
    """d = 2: f_b is the cosine of the difference of the two azimuth midpoints."""
    for b in BITS:
        for cq in range(2 ** b):
            for ck in range(0, 2 ** b, max(1, 2 ** b // 8)):
                want = math.cos((cq - ck) * 2 * math.pi / 2 ** b)
                assert oracle.fb(np.array([cq]), np.array([ck]), b) == pytest.approx(want, abs=1e-15)


def test_d3_spherical_law_of_cosines():
    """d = 3: f_b = cos t1 cos t2 + sin t1 sin t2 cos(p1 - p2) on the cell midpoints."""
    rng = np.random.default_rng(4)
    for b in BITS:
        for _ in range(200):
            cq = np.array([rng.integers(2 ** b), rng.integers(2 ** b)], np.int32)
            ck = np.array([rng.integers(2 ** b), rng.integers(2 ** b)], np.int32)
            t1, t2 = (cq[0] + 0.5) * math.pi / 2 ** b, (ck[0] + 0.5) * math.pi / 2 ** b
            p1, p2 = (cq[1] + 0.5) * 2 * math.pi / 2 ** b, (ck[1] + 0.5) * 2 * math.pi / 2 ** b
            want = math.cos(t1) * math.cos(t2) + math.sin(t1) * math.sin(t2) * math.cos(p1 - p2)
            assert oracle.fb(cq, ck, b) == pytest.approx(want, abs=1e-15)


def test_prefix_form_equals_nested_form():
    rng = np.random.default_rng(5)
    for b in BITS:
        for _ in range(100):
            cq = rng.integers(0, 2 ** b, 127).astype(np.int32)
            ck = rng.integers(0, 2 ** b, 127).astype(np.int32)
            assert abs(oracle.fb(cq, ck, b) - oracle.fb_nested(cq, ck, b)) <= 1e-14


def test_fb_converges_to_cosine():
    """f_b -> cos(q, k) as b grows, about one halving of the error per bit."""
    rng = np.random.default_rng(6)
    pairs = [(rng.standard_normal(128), rng.standard_normal(128)) for _ in range(60)]
    errs = []
    for b in range(3, 17):
        e = []
        for q, k in pairs:
            cq = oracle.angle_codes(oracle.angles(q), b)
            ck = oracle.angle_codes(oracle.angles(k), b)
            cos = float(q @ k) / (np.linalg.norm(q) * np.linalg.norm(k))
            e.append(abs(oracle.fb(cq, ck, b) - cos))
        errs.append(np.mean(e))
    errs = np.array(errs)
    assert errs[-1] < 1e-3
    slope = np.polyfit(np.arange(3, 17), np.log2(errs), 1)[0]
    assert -1.3 < slope < -0.7, slope
    assert np.all(errs[2:] < errs[:-2])


# ------------------------------------------------------------ quantisers

@pytest.mark.parametrize("b", BITS)
def test_angle_code_is_the_cell_containing_phi(b):
    """Brute force: the code is the c with c w <= phi < (c+1) w, and the
    midpoint is within half a cell (w = pi/2^b polar, 2pi/2^b azimuth)."""
    rng = np.random.default_rng(7 + b)
    for az in (False, True):
        w = (2 * math.pi if az else math.pi) / 2 ** b
        for phi in rng.uniform(0, w * 2 ** b, 2000):
            c = oracle.angle_code(phi, b, az)
            assert 0 <= c < 2 ** b
            assert c * w <= phi * (1 + 1e-15) and phi < (c + 1) * w * (1 + 1e-15)
            assert abs(phi - oracle.angle_mid(c, b, az)) <= w / 2 * (1 + 1e-12)


def test_radius_code_is_nearest_log_grid_point():
    """Brute force over the 256 grid points 2^(L + c Delta): nearest in log2, ties up;
    |r~/r - 1| <= 2^(Delta/2) - 1 inside the range; r = 0 and out-of-range clamp."""
    rng = np.random.default_rng(8)
    L, delta = 2.5, 3.0 / 255
    grid = L + np.arange(256) * delta
    for r in 2 ** rng.uniform(L - 1, L + 4, 3000):
        c = oracle.radius_code(r, L, delta)
        lr = math.log2(r)
        if lr < L:
            assert c == 0
        elif lr > grid[-1]:
            assert c == 255
        else:
            dist = np.abs(grid - lr)
            best = np.flatnonzero(dist <= dist.min() + 1e-12)
            assert c in best
            assert abs(oracle.radius_value(c, L, delta) / r - 1) <= 2 ** (delta / 2) - 1 + 1e-12
    assert oracle.radius_code(0.0, L, delta) == 0


def test_bf16_rounding_matches_torch():
    """The oracle's fp64 -> bf16 rounding equals torch's round-to-nearest-even
    conversion for fp32-representable inputs."""
    import torch

    rng = np.random.default_rng(9)
    x = (rng.standard_normal(20000) * np.exp(rng.uniform(-20, 20, 20000))).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.f64_to_bf16(float(v)) for v in x], np.uint16)
    assert np.array_equal(got, want)


# ------------------------------------------------------------- attention

def _np_softmax_attention(qvec, kmat, v, keep=None):
    lg = kmat @ qvec / math.sqrt(qvec.shape[0])
    if keep is not None:
        lg = np.where(keep.astype(bool), lg, -np.inf)
    m = lg.max()
    if m == -np.inf:
        return np.zeros(v.shape[1])
    p = np.exp(lg - m)
    return (p @ v) / p.sum()


def test_ada_equals_dense_attention_on_decoded_vectors():
    """ADA(q, codes) = softmax((||q|| u~_q) . (r~ u~_k) / sqrt d) V with mixed bit widths and a mask."""
    rng = np.random.default_rng(10)
    d, T, G = 128, 96, 3
    q = _rand_bf16(rng, (G, d))
    keys = _rand_bf16(rng, (T, d), 2.0)
    v = _rand_bf16(rng, (T, d))
    bits = rng.choice(BITS, T).astype(np.int32)
    keep = (rng.random(T) > 0.3).astype(np.uint8)
    L, delta = 1.0, 6.0 / 255
    codes, rcode = oracle.encode(keys, bits, L, delta)
    out, lg = oracle.ada_group(q, codes, bits, rcode, L, delta, v, keep=keep, want_logits=True)
    vf = oracle.bf16_to_f64(v)
    for g in range(G):
        qf = oracle.bf16_to_f64(q[g])
        qphi = oracle.angles(qf)
        kmat = np.empty((T, d))
        qmat = np.empty((T, d))
        for t in range(T):
            b = int(bits[t])
            kmat[t] = oracle.radius_value(int(rcode[t]), L, delta) * oracle.unit_from_codes(codes[t], b)
            qmat[t] = np.linalg.norm(qf) * oracle.unit_from_codes(oracle.angle_codes(qphi, b), b)
        lgt = np.einsum("td,td->t", qmat, kmat) / math.sqrt(d)
        lgt = np.where(keep.astype(bool), lgt, -np.inf)
        p = np.exp(lgt - lgt.max())
        want = (p @ vf) / p.sum()
        assert np.max(np.abs(out[g] - want)) <= 1e-12
        assert np.array_equal(np.isinf(lg[g]), keep == 0)
        np.testing.assert_allclose(lg[g][keep == 1], lgt[keep == 1], rtol=0, atol=1e-12)


def test_query_is_coded_at_the_key_bit_width():
    """R3: the logit uses u~(c_q) with c_q found by the cell rule from
    independently computed query angles (numpy arccos/arctan2)."""
    rng = np.random.default_rng(11)
    d, T = 128, 8
    q = _rand_bf16(rng, (1, d))
    keys = _rand_bf16(rng, (T, d))
    v = _rand_bf16(rng, (T, d))
    b = 3
    codes, rcode = oracle.encode(keys, b, 0.0, 8.0 / 255)
    _, lg = oracle.ada_group(q, codes, b, rcode, 0.0, 8.0 / 255, v, want_logits=True)
    qf = oracle.bf16_to_f64(q[0])
    tail = np.sqrt(np.cumsum((qf ** 2)[::-1])[::-1])
    phi = np.arccos(np.clip(qf[:-2] / tail[:-2], -1, 1))
    az = math.atan2(qf[-1], qf[-2]) % (2 * math.pi)
    cq = np.concatenate([np.minimum(np.floor(phi * 2 ** b / math.pi), 2 ** b - 1),
                         [math.floor(az * 2 ** b / (2 * math.pi))]]).astype(np.int32)
    uq = oracle.unit_from_codes(cq, b)
    for t in range(T):
        uk = oracle.unit_from_codes(codes[t], b)
        want = np.linalg.norm(qf) * oracle.radius_value(int(rcode[t]), 0.0, 8.0 / 255) * float(uq @ uk) / math.sqrt(d)
        assert abs(lg[0, t] - want) <= 1e-12


def test_brute_force_attention_at_high_bit_width():
    """b = 30 with exact radii: ADA approaches plain softmax(q K^T / sqrt d) V."""
    rng = np.random.default_rng(12)
    d, T, G = 128, 64, 2
    q = _rand_bf16(rng, (G, d))
    keys = _rand_bf16(rng, (T, d))
    v = _rand_bf16(rng, (T, d))
    codes, _ = oracle.encode(keys, 30, 0.0, 1.0)
    kf = oracle.bf16_to_f64(keys)
    out = oracle.ada_group(q, codes, 30, np.zeros(T, np.uint8), 0.0, 1.0, v,
                           r_exact=np.linalg.norm(kf, axis=1))
    vf = oracle.bf16_to_f64(v)
    for g in range(G):
        want = _np_softmax_attention(oracle.bf16_to_f64(q[g]), kf, vf)
        assert np.max(np.abs(out[g] - want)) <= 1e-6


def _np_unit_from_codes(c, b):
    """Decoded unit vector, written out independently with numpy: cell
    midpoints, then cos of each angle times the running product of sines."""
    c = np.asarray(c, np.float64)
    d = c.shape[0] + 1
    phi = (c + 0.5) * math.pi / 2 ** b
    phi[-1] = (c[-1] + 0.5) * 2 * math.pi / 2 ** b
    u = np.empty(d)
    run = 1.0
    for j in range(d - 1):
        u[j] = run * math.cos(phi[j])
        run *= math.sin(phi[j])
    u[d - 1] = run
    return u


def test_exact_query_logit_is_cosine_with_the_decoded_key():
    """R13: with the exact query, logit = ||q|| r~ <q/||q||, u~(c_k)> / sqrt d, with
    the key decoded by an independent numpy routine; mixed widths and a mask."""
    rng = np.random.default_rng(13)
    d, T, G = 128, 40, 2
    q = _rand_bf16(rng, (G, d))
    keys = _rand_bf16(rng, (T, d), 1.5)
    v = _rand_bf16(rng, (T, d))
    bits = rng.choice(BITS, T).astype(np.int32)
    keep = (rng.random(T) > 0.25).astype(np.uint8)
    L, delta = -1.0, 7.0 / 255
    codes, rcode = oracle.encode(keys, bits, L, delta)
    out, lg = oracle.ada_group(q, codes, bits, rcode, L, delta, v, keep=keep, want_logits=True, exact_q=True)
    vf = oracle.bf16_to_f64(v)
    for g in range(G):
        qf = oracle.bf16_to_f64(q[g])
        want = np.array([float(qf @ _np_unit_from_codes(codes[t], int(bits[t])))
                         * 2.0 ** (L + int(rcode[t]) * delta) / math.sqrt(d) for t in range(T)])
        np.testing.assert_allclose(lg[g][keep == 1], want[keep == 1], rtol=0, atol=1e-12)
        assert np.all(np.isinf(lg[g][keep == 0]))
        x = np.where(keep.astype(bool), want, -np.inf)
        p = np.exp(x - x.max())
        assert np.max(np.abs(out[g] - (p @ vf) / p.sum())) <= 1e-12


def test_exact_query_high_bit_width_matches_dense_attention():
    """R13 with b = 30 keys and exact radii: only the key angles are quantised,
    so ADA reaches plain softmax(q K^T / sqrt d) V to about 2^-30."""
    rng = np.random.default_rng(14)
    d, T, G = 128, 64, 2
    q = _rand_bf16(rng, (G, d))
    keys = _rand_bf16(rng, (T, d))
    v = _rand_bf16(rng, (T, d))
    codes, _ = oracle.encode(keys, 30, 0.0, 1.0)
    kf = oracle.bf16_to_f64(keys)
    out = oracle.ada_group(q, codes, 30, np.zeros(T, np.uint8), 0.0, 1.0, v,
                           r_exact=np.linalg.norm(kf, axis=1), exact_q=True)
    vf = oracle.bf16_to_f64(v)
    for g in range(G):
        want = _np_softmax_attention(oracle.bf16_to_f64(q[g]), kf, vf)
        assert np.max(np.abs(out[g] - want)) <= 1e-7


def test_exact_query_zero_query_gives_uniform_attention():
    """R13: a zero query has f = 0, so every retained slot gets the same weight."""
    rng = np.random.default_rng(15)
    d, T = 128, 12
    q = np.zeros((1, d), np.uint16)
    keys = _rand_bf16(rng, (T, d))
    v = _rand_bf16(rng, (T, d))
    codes, rcode = oracle.encode(keys, 4, 0.0, 4.0 / 255)
    out, lg = oracle.ada_group(q, codes, 4, rcode, 0.0, 4.0 / 255, v, want_logits=True, exact_q=True)
    assert np.all(lg == 0.0)
    assert np.max(np.abs(out[0] - oracle.bf16_to_f64(v).mean(axis=0))) <= 1e-12


def test_dense_oracle_brute_force():
    rng = np.random.default_rng(13)
    d, T, G = 128, 50, 4
    q, k, v = _rand_bf16(rng, (G, d)), _rand_bf16(rng, (T, d)), _rand_bf16(rng, (T, d))
    keep = (rng.random(T) > 0.25).astype(np.uint8)
    out = oracle.dense_group(q, k, v, keep=keep)
    for g in range(G):
        want = _np_softmax_attention(oracle.bf16_to_f64(q[g]), oracle.bf16_to_f64(k), oracle.bf16_to_f64(v), keep)
        assert np.max(np.abs(out[g] - want)) <= 1e-12


def test_mask_equals_compaction():
    """Evicting slots gives the same output as attending over only the retained ones."""
    rng = np.random.default_rng(14)
    d, T = 128, 80
    q = _rand_bf16(rng, (2, d))
    keys, v = _rand_bf16(rng, (T, d)), _rand_bf16(rng, (T, d))
    bits = rng.choice(BITS, T).astype(np.int32)
    keep = (rng.random(T) > 0.4).astype(np.uint8)
    codes, rcode = oracle.encode(keys, bits, 0.5, 5.0 / 255)
    a = oracle.ada_group(q, codes, bits, rcode, 0.5, 5.0 / 255, v, keep=keep)
    idx = np.flatnonzero(keep)
    b_ = oracle.ada_group(q, codes[idx], bits[idx], rcode[idx], 0.5, 5.0 / 255, v[idx])
    assert np.max(np.abs(a - b_)) <= 1e-12


def test_empty_and_fully_evicted_give_zero():
    rng = np.random.default_rng(15)
    q = _rand_bf16(rng, (1, 128))
    keys, v = _rand_bf16(rng, (4, 128)), _rand_bf16(rng, (4, 128))
    codes, rcode = oracle.encode(keys, 4, 0.0, 0.05)
    out = oracle.ada_group(q, codes, 4, rcode, 0.0, 0.05, v, keep=np.zeros(4, np.uint8))
    assert np.all(out == 0)
    out = oracle.ada_group(q, codes[:0], 4, rcode[:0], 0.0, 0.05, v[:0])
    assert np.all(out == 0)


def test_decompress_is_radius_times_decoded_unit_vector():
    """k~ = bf16(r~ u~(c)); checked with torch's bf16 rounding of the fp64 product."""
    import torch

    rng = np.random.default_rng(16)
    keys = _rand_bf16(rng, (40, 128), 3.0)
    bits = rng.choice(BITS, 40).astype(np.int32)
    codes, rcode = oracle.encode(keys, bits, 2.0, 4.0 / 255)
    got = oracle.decompress(codes, bits, rcode, 2.0, 4.0 / 255)
    for t in range(40):
        kt = oracle.radius_value(int(rcode[t]), 2.0, 4.0 / 255) * oracle.unit_from_codes(codes[t], int(bits[t]))
        # torch rounds fp64 -> bf16 directly (round-to-nearest-even)
        want = torch.from_numpy(kt).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(got[t], want)


def test_encoded_radius_error_bound_on_random_keys():
    rng = np.random.default_rng(17)
    keys = _rand_bf16(rng, (500, 128), 1.5)
    kf = oracle.bf16_to_f64(keys)
    r = np.linalg.norm(kf, axis=1)
    L, delta = math.log2(r.min()), (math.log2(r.max()) - math.log2(r.min())) / 255
    _, rcode = oracle.encode(keys, 4, L, delta)
    rt = np.array([oracle.radius_value(int(c), L, delta) for c in rcode])
    assert np.max(np.abs(rt / r - 1)) <= 2 ** (delta / 2) - 1 + 1e-12
