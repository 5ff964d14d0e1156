"""fp64 oracle of the non-uniform angle quantiser (an f_b variant).

Test infrastructure, like the rest of ``oracle/``: only tests/ may use it.

"SPHERICAL KV: Angle-Domain Attention and Rate-Distortion Retention for
Efficient Long-Context Inference", technical summary section 2.1, leaves the
angle quantiser open (it names b-bit angle codes and their fused cosine).
Reading R19 (this module): for a direction drawn uniformly on the unit
sphere of R^d, the polar angle phi_i (i = 1 .. d-2) has the density
sin^(d-1-i)(phi) / Z on [0, pi] (the factor of the d-dimensional volume
element), so in high d it concentrates near pi/2; the azimuth phi_(d-1) is
uniform on [0, 2 pi).  The non-uniform quantiser gives each polar angle
2^b cells of equal probability under that density -- edges at the j/2^b
quantiles, reconstruction at the cell's median, the (j + 1/2)/2^b quantile --
and keeps the uniform mid-rise azimuth of R1.  The cell is decided on the
probability scale, floor(2^b F(phi)); an input on an edge goes to the upper
cell, as in R1, up to the fp64 rounding of F (an input within that rounding
of an edge may land either side, as R10 allows for the uniform cells).

The CDF: with u = (1 - cos phi)/2, sin^k(phi) dphi is proportional to
(u (1 - u))^((k-1)/2) du, so u ~ Beta(a, a) with a = (k + 1)/2 and
F(phi) = I_u(a, a) (the regularised incomplete beta function).  Quantiles
come from its inverse (scipy.special.betaincinv, a library step).

Everything else is the oracle's: the angles and the unit-vector decode from
angles (R1, R2), the radius code (R4), the coded query (R3), logits divided
by sqrt(d) and softmax over retained tokens (R6, R7).
"""
from __future__ import annotations

import math

import numpy as np
from scipy import special

from . import angles, bf16_to_f64, radius_code, radius_value, unit_from_angles


def polar_shape(d: int, i: int) -> float:
    """a of the Beta(a, a) law of u = (1 - cos phi_i)/2, polar angle i (1-based)."""
    if not 1 <= i <= d - 2:
        raise ValueError("polar angles are 1 .. d-2")
    return (d - i) / 2.0


def polar_cdf(phi, d: int, i: int):
    """F(phi) for polar angle i of a uniform direction in R^d."""
    a = polar_shape(d, i)
    return special.betainc(a, a, (1.0 - np.cos(phi)) / 2.0)


def polar_quantile(p, d: int, i: int):
    a = polar_shape(d, i)
    u = special.betaincinv(a, a, np.asarray(p, np.float64))
    return np.arccos(np.clip(1.0 - 2.0 * u, -1.0, 1.0))


def polar_edges(d: int, b: int) -> np.ndarray:
    """[d-2, 2^b - 1] cell edges of the polar angles: F_i^-1(j / 2^b)."""
    n = 1 << b
    return np.stack([polar_quantile(np.arange(1, n) / n, d, i) for i in range(1, d - 1)])


def polar_mids(d: int, b: int) -> np.ndarray:
    """[d-2, 2^b] reconstruction angles (cell medians): F_i^-1((j + 1/2) / 2^b)."""
    n = 1 << b
    return np.stack([polar_quantile((np.arange(n) + 0.5) / n, d, i) for i in range(1, d - 1)])


def _shapes(d: int) -> np.ndarray:
    return (d - np.arange(1, d - 1)) / 2.0  # a of polar angles 1 .. d-2


def codes_from_angles(phi: np.ndarray, b: int) -> np.ndarray:
    """Codes [d-1] of the angles phi [d-1]: polar code = the cell of F_i(phi_i)
    on the probability scale, min(floor(2^b F_i(phi_i)), 2^b - 1) (an input on
    an edge lands in the upper cell, up to fp64 rounding of F); uniform
    azimuth (R1)."""
    phi = np.asarray(phi, np.float64)
    d = phi.shape[0] + 1
    n = 1 << b
    a = _shapes(d)
    F = special.betainc(a, a, (1.0 - np.cos(phi[:d - 2])) / 2.0)
    c = np.empty(d - 1, np.int32)
    c[:d - 2] = np.minimum(np.floor(F * n), n - 1).astype(np.int32)
    c[d - 2] = min(int(math.floor(phi[d - 2] * n / (2.0 * math.pi))), n - 1)  # R1 azimuth
    return c


def angles_from_codes(c: np.ndarray, b: int) -> np.ndarray:
    c = np.asarray(c, np.int64)
    d = c.shape[0] + 1
    n = 1 << b
    a = _shapes(d)
    phi = np.empty(d - 1, np.float64)
    u = special.betaincinv(a, a, (c[:d - 2] + 0.5) / n)
    phi[:d - 2] = np.arccos(np.clip(1.0 - 2.0 * u, -1.0, 1.0))
    phi[d - 2] = (c[d - 2] + 0.5) * 2.0 * math.pi / n
    return phi


def unit_from_codes(c: np.ndarray, b: int) -> np.ndarray:
    return unit_from_angles(angles_from_codes(c, b))


def encode(keys_bf16: np.ndarray, b: int, L: float, delta: float):
    """Keys [T, d] bf16 bits -> (codes [T, d-1], radius codes [T])."""
    x = bf16_to_f64(keys_bf16)
    T, d = x.shape
    codes = np.empty((T, d - 1), np.int32)
    rc = np.empty(T, np.int32)
    for t in range(T):
        codes[t] = codes_from_angles(angles(x[t]), b)
        rc[t] = radius_code(float(np.linalg.norm(x[t])), L, delta)
    return codes, rc


def ada_group(q_bf16: np.ndarray, codes: np.ndarray, b: int, rcode: np.ndarray, L: float, delta: float,
              v_bf16: np.ndarray, keep=None, r_exact=None) -> np.ndarray:
    """ADA attention of G queries [G, d] over T coded keys with this quantiser:
    logit = ||q|| r~ <u~(c_q), u~(c_k)> / sqrt(d), q coded at b (R3), softmax
    over retained tokens, P.V in fp64.  Returns out [G, d]."""
    q = bf16_to_f64(q_bf16)
    v = bf16_to_f64(v_bf16)
    G, d = q.shape
    T = codes.shape[0]
    uk = np.stack([unit_from_codes(codes[t], b) for t in range(T)]) if T else np.zeros((0, d))
    r = (np.asarray(r_exact, np.float64) if r_exact is not None
         else np.array([radius_value(int(c), L, delta) for c in rcode], np.float64))
    keep = np.ones(T, bool) if keep is None else np.asarray(keep).astype(bool)
    out = np.zeros((G, d), np.float64)
    for g in range(G):
        qn = float(np.linalg.norm(q[g]))
        if not np.any(keep):
            continue
        uq = unit_from_codes(codes_from_angles(angles(q[g]), b), b) if qn > 0 else np.zeros(d)
        lg = qn * r * (uk @ uq) / math.sqrt(d)
        lg = np.where(keep, lg, -np.inf)
        w = np.exp(lg - lg[keep].max())
        out[g] = (w[:, None] * v).sum(0) / w.sum()
    return out
