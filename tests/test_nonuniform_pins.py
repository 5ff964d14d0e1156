"""Pins of the oracle's non-uniform angle quantiser (oracle/nonuniform.py,
reading R19: equal-mass polar cells under the angle law of a uniform
direction, median reconstruction, uniform azimuth).

The law is pinned by an independent numerical integral of sin^k and by the
d = 3 closed form; the quantiser by Monte-Carlo cell frequencies of uniform
directions, the median property and the edge count; the attention by its limit
(many bits, exact radii -> dense attention) and by its purpose (smaller f_b
error than the uniform quantiser on uniform directions)."""
import math

import numpy as np
import pytest
from scipy import integrate

import oracle
from oracle import nonuniform as nu


@pytest.mark.parametrize("d,i", [(3, 1), (8, 2), (128, 1), (128, 64), (128, 126)])
def test_cdf_is_the_integral_of_the_sine_power(d, i):
    k = d - 1 - i
    z = integrate.quad(lambda t: math.sin(t) ** k, 0.0, math.pi)[0]
    for theta in (0.3, 1.0, math.pi / 2, 2.0, 2.9):
        want = integrate.quad(lambda t: math.sin(t) ** k, 0.0, theta)[0] / z
        assert nu.polar_cdf(theta, d, i) == pytest.approx(want, abs=1e-10)


def test_d3_closed_form():
    """d = 3: phi_1 has density sin(phi)/2, F = (1 - cos phi)/2, so the edges
    are arccos(1 - 2 j / 2^b) and the medians arccos(1 - (2 j + 1) / 2^b)."""
    for b in (2, 3, 4):
        n = 1 << b
        np.testing.assert_allclose(nu.polar_edges(3, b)[0], np.arccos(1 - 2 * np.arange(1, n) / n), atol=1e-12)
        np.testing.assert_allclose(nu.polar_mids(3, b)[0], np.arccos(1 - (2 * np.arange(n) + 1) / n), atol=1e-12)


def test_cells_have_equal_mass_for_uniform_directions():
    rng = np.random.default_rng(0)
    d, b, N = 128, 3, 6000
    x = rng.standard_normal((N, d))
    n = 1 << b
    counts = np.zeros((d - 1, n))
    for t in range(N):
        c = nu.codes_from_angles(oracle.angles(x[t]), b)
        counts[np.arange(d - 1), c] += 1
    frac = counts / N
    sigma = math.sqrt((1 / n) * (1 - 1 / n) / N)
    assert np.max(np.abs(frac - 1 / n)) < 5.5 * sigma, np.max(np.abs(frac - 1 / n)) / sigma


def test_medians_split_their_cells_and_edges_are_quantiles():
    d, b = 128, 4
    n = 1 << b
    edges, mids = nu.polar_edges(d, b), nu.polar_mids(d, b)
    for i in (1, 40, 126):
        F_e = nu.polar_cdf(edges[i - 1], d, i)
        F_m = nu.polar_cdf(mids[i - 1], d, i)
        np.testing.assert_allclose(F_e, np.arange(1, n) / n, atol=1e-12)
        np.testing.assert_allclose(F_m, (np.arange(n) + 0.5) / n, atol=1e-12)
        lo = np.concatenate([[0.0], edges[i - 1]])
        hi = np.concatenate([edges[i - 1], [math.pi]])
        assert np.all((lo < mids[i - 1]) & (mids[i - 1] < hi))


def test_high_dimension_concentrates_near_half_pi():
    """phi_1 in d = 128 has standard deviation about 1/sqrt(126) around pi/2:
    every inner edge lies within 4 of them."""
    e = nu.polar_edges(128, 4)[0]
    assert np.all(np.abs(e - math.pi / 2) < 4 / math.sqrt(126))


def test_codes_count_the_edges_below_and_the_azimuth_is_r1():
    """The code of a polar angle is the number of edges at or below it (away
    from fp64 rounding of an edge); the azimuth code is R1's."""
    rng = np.random.default_rng(4)
    d, b = 16, 3
    e = nu.polar_edges(d, b)
    for _ in range(200):
        phi = np.concatenate([rng.uniform(0, math.pi, d - 2), [rng.uniform(0, 2 * math.pi)]])
        c = nu.codes_from_angles(phi, b)
        for i in range(d - 2):
            if np.min(np.abs(e[i] - phi[i])) > 1e-9:
                assert c[i] == np.searchsorted(e[i], phi[i], side="right")
        assert c[d - 2] == oracle.angle_code(phi[d - 2], b, True)
    # inside a cell, away from its edges: the cell's index
    mids = nu.polar_mids(d, b)
    assert np.all(nu.codes_from_angles(np.concatenate([mids[:, 5], [0.1]]), b)[:d - 2] == 5)


def test_unit_vectors_and_round_trip():
    rng = np.random.default_rng(1)
    for b in (3, 8):
        for _ in range(5):
            x = rng.standard_normal(128)
            u = nu.unit_from_codes(nu.codes_from_angles(oracle.angles(x), b), b)
            assert abs(np.linalg.norm(u) - 1) < 1e-12
            assert float(u @ (x / np.linalg.norm(x))) > (0.9 if b == 3 else 0.995)


def test_many_bits_with_exact_radii_is_dense_attention():
    rng = np.random.default_rng(2)
    import torch

    T, G, d = 40, 2, 128
    k = torch.randn(T, d).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    v = torch.randn(T, d).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    q = torch.randn(G, d).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    codes, rc = nu.encode(k, 20, -5.0, 0.05)
    r = np.linalg.norm(oracle.bf16_to_f64(k), axis=1)
    got = nu.ada_group(q, codes, 20, rc, -5.0, 0.05, v, r_exact=r)
    ref = oracle.dense_group(q, k, v)
    np.testing.assert_allclose(got, ref, atol=1e-4)
    assert rng is not None


def test_smaller_cosine_error_than_uniform_cells_on_uniform_directions():
    """The point of the variant: at b = 4, the fused cosine of uniformly
    random (q, k) directions is closer to the exact cosine than with the
    uniform quantiser (R1)."""
    rng = np.random.default_rng(3)
    b, d = 4, 128
    err_nu, err_u = [], []
    for _ in range(200):
        q, k = rng.standard_normal(d), rng.standard_normal(d)
        exact = float(q @ k / np.linalg.norm(q) / np.linalg.norm(k))
        pq, pk = oracle.angles(q), oracle.angles(k)
        f_nu = float(nu.unit_from_codes(nu.codes_from_angles(pq, b), b)
                     @ nu.unit_from_codes(nu.codes_from_angles(pk, b), b))
        f_u = oracle.fb(oracle.angle_codes(pq, b), oracle.angle_codes(pk, b), b)
        err_nu.append(abs(f_nu - exact))
        err_u.append(abs(f_u - exact))
    assert np.mean(err_nu) < 0.8 * np.mean(err_u), (np.mean(err_nu), np.mean(err_u))
