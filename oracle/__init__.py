"""fp64 CPU oracle for Spherical KV angle-domain attention (ADA) decode.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s cpu_baseline / reference arm may import this package.  The
product path (``compressed_kv_decode_ada_b200``) never imports it, and it never
imports the product path: the two share no code.

The arithmetic lives in ``spkv_oracle.c`` (plain C, IEEE fp64); this module
only builds it with gcc and marshals numpy arrays through ctypes.  Each wrapper
cites the definition it follows: "SPHERICAL KV: Angle-Domain Attention and
Rate-Distortion Retention for Efficient Long-Context Inference", technical
summary section 2.1 (Angle-Domain Attention) and section 2.2 (Rate-Distortion
Retention: ``rdr_plan``, ``rdr_assign``, ``rdr_pack``).  The readings where the
pages are silent are listed at the top of ``spkv_oracle.c`` (R1-R13) and at
the RDR controller in it (R14-R17); ``rdr_pack`` states R18 and
``nonuniform.py`` (the non-uniform angle quantiser) R19.

ctypes drops the GIL around each foreign call, so ``map_groups`` runs the
per-(sequence, kv head) oracle calls on a thread pool.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "spkv_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libspkv_oracle.so")
_lib = None

_d = ctypes.c_double
_i = ctypes.c_int
_p = ctypes.c_void_p


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, no fast-math, no FMA contraction) into oracle/libspkv_oracle.so."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        L.spkv_oracle_bf16_to_f64.restype = _d
        L.spkv_oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
        L.spkv_oracle_f64_to_bf16.restype = ctypes.c_uint16
        L.spkv_oracle_f64_to_bf16.argtypes = [_d]
        L.spkv_oracle_angles.argtypes = [_i, _p, _p]
        L.spkv_oracle_angle_pos.restype = _d
        L.spkv_oracle_angle_pos.argtypes = [_d, _i, _i]
        L.spkv_oracle_angle_code.restype = ctypes.c_int32
        L.spkv_oracle_angle_code.argtypes = [_d, _i, _i]
        L.spkv_oracle_angle_mid.restype = _d
        L.spkv_oracle_angle_mid.argtypes = [ctypes.c_int32, _i, _i]
        L.spkv_oracle_angle_codes.argtypes = [_i, _p, _i, _p]
        L.spkv_oracle_unit_from_angles.argtypes = [_i, _p, _p]
        L.spkv_oracle_unit_from_codes.argtypes = [_i, _p, _i, _p]
        L.spkv_oracle_fb.restype = _d
        L.spkv_oracle_fb.argtypes = [_i, _p, _p, _i]
        L.spkv_oracle_fb_nested.restype = _d
        L.spkv_oracle_fb_nested.argtypes = [_i, _p, _p, _i]
        L.spkv_oracle_radius_pos.restype = _d
        L.spkv_oracle_radius_pos.argtypes = [_d, _d, _d]
        L.spkv_oracle_radius_code.restype = ctypes.c_int32
        L.spkv_oracle_radius_code.argtypes = [_d, _d, _d]
        L.spkv_oracle_radius_value.restype = _d
        L.spkv_oracle_radius_value.argtypes = [ctypes.c_int32, _d, _d]
        L.spkv_oracle_encode.argtypes = [_i, _i, _p, _p, _d, _d, _p, _p, _p, _p]
        L.spkv_oracle_decompress.argtypes = [_i, _i, _p, _p, _p, _d, _d, _p]
        L.spkv_oracle_ada_group.argtypes = [_i, _i, _i, _p, _p, _p, _p, _p, _d, _d, _p, _p, _p, _p]
        L.spkv_oracle_ada_group_exact_q.argtypes = [_i, _i, _i, _p, _p, _p, _p, _p, _d, _d, _p, _p, _p, _p]
        L.spkv_oracle_rdr_plan.restype = _i
        L.spkv_oracle_rdr_plan.argtypes = [_i, _i, _i, _p, _p, _p, _d, ctypes.c_uint32, _p, _p, _p, _p]
        L.spkv_oracle_rdr_assign.restype = _d
        L.spkv_oracle_rdr_assign.argtypes = [_i, _i, _i, _p, _p, _p, ctypes.c_uint32, _d, _p]
        L.spkv_oracle_dense_group.argtypes = [_i, _i, _i, _p, _p, _p, _p, _p, _p]
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


# ----------------------------------------------------------- scalar pieces

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns; -0 becomes +0."""
    f = (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    f[f == 0.0] = 0.0
    return f


def f64_to_bf16(x: float) -> int:
    return int(lib().spkv_oracle_f64_to_bf16(float(x)))


def angles(x: np.ndarray) -> np.ndarray:
    """R1: hyperspherical angles phi[0..d-2] of x (fp64)."""
    x = _c(x, np.float64)
    d = x.shape[0]
    phi = np.empty(d - 1, np.float64)
    lib().spkv_oracle_angles(d, _ptr(x), _ptr(phi))
    return phi


def angle_pos(phi: float, b: int, azimuth: bool) -> float:
    return lib().spkv_oracle_angle_pos(float(phi), b, int(azimuth))


def angle_code(phi: float, b: int, azimuth: bool) -> int:
    return int(lib().spkv_oracle_angle_code(float(phi), b, int(azimuth)))


def angle_mid(c: int, b: int, azimuth: bool) -> float:
    return lib().spkv_oracle_angle_mid(int(c), b, int(azimuth))


def angle_codes(phi: np.ndarray, b: int) -> np.ndarray:
    phi = _c(phi, np.float64)
    d = phi.shape[0] + 1
    c = np.empty(d - 1, np.int32)
    lib().spkv_oracle_angle_codes(d, _ptr(phi), b, _ptr(c))
    return c


def unit_from_angles(phi: np.ndarray) -> np.ndarray:
    phi = _c(phi, np.float64)
    d = phi.shape[0] + 1
    u = np.empty(d, np.float64)
    lib().spkv_oracle_unit_from_angles(d, _ptr(phi), _ptr(u))
    return u


def unit_from_codes(codes: np.ndarray, b: int) -> np.ndarray:
    codes = _c(codes, np.int32)
    d = codes.shape[0] + 1
    u = np.empty(d, np.float64)
    lib().spkv_oracle_unit_from_codes(d, _ptr(codes), b, _ptr(u))
    return u


def fb(cq: np.ndarray, ck: np.ndarray, b: int) -> float:
    """R2 prefix form of f_b."""
    cq, ck = _c(cq, np.int32), _c(ck, np.int32)
    return lib().spkv_oracle_fb(cq.shape[0] + 1, _ptr(cq), _ptr(ck), b)


def fb_nested(cq: np.ndarray, ck: np.ndarray, b: int) -> float:
    """R2 nested form of f_b."""
    cq, ck = _c(cq, np.int32), _c(ck, np.int32)
    return lib().spkv_oracle_fb_nested(cq.shape[0] + 1, _ptr(cq), _ptr(ck), b)


def radius_pos(r: float, L: float, delta: float) -> float:
    return lib().spkv_oracle_radius_pos(float(r), float(L), float(delta))


def radius_code(r: float, L: float, delta: float) -> int:
    return int(lib().spkv_oracle_radius_code(float(r), float(L), float(delta)))


def radius_value(c: int, L: float, delta: float) -> float:
    return lib().spkv_oracle_radius_value(int(c), float(L), float(delta))


# ------------------------------------------------------------- batch pieces

def encode(keys_bf16: np.ndarray, bits: np.ndarray, L: float, delta: float, positions: bool = False):
    """Encode keys [n, d] (bf16 bit patterns) at per-key bit widths bits[n].

    Returns (codes [n, d-1] int32, rcode [n] uint8) and, with positions=True,
    also the scaled angle positions [n, d-1] and radius positions [n], whose
    distance to the nearest integer tells how close each code is to a cell edge.
    """
    keys = _c(keys_bf16, np.uint16)
    n, d = keys.shape
    bits = _c(np.broadcast_to(np.asarray(bits, np.int32), (n,)), np.int32)
    codes = np.empty((n, d - 1), np.int32)
    rcode = np.empty(n, np.uint8)
    apos = np.empty((n, d - 1), np.float64) if positions else None
    rpos = np.empty(n, np.float64) if positions else None
    lib().spkv_oracle_encode(d, n, _ptr(keys), _ptr(bits), float(L), float(delta), _ptr(codes),
                             _ptr(rcode), _ptr(apos), _ptr(rpos))
    if positions:
        return codes, rcode, apos, rpos
    return codes, rcode


def decompress(codes: np.ndarray, bits: np.ndarray, rcode: np.ndarray, L: float, delta: float) -> np.ndarray:
    """k~ = r~ u~(c) rounded to bf16 bit patterns, [n, d]."""
    codes = _c(codes, np.int32)
    n, dm1 = codes.shape
    bits = _c(np.broadcast_to(np.asarray(bits, np.int32), (n,)), np.int32)
    rcode = _c(rcode, np.uint8)
    out = np.empty((n, dm1 + 1), np.uint16)
    lib().spkv_oracle_decompress(dm1 + 1, n, _ptr(codes), _ptr(bits), _ptr(rcode), float(L), float(delta),
                                 _ptr(out))
    return out


def ada_group(q_bf16, kcodes, kbits, rcode, L, delta, v_bf16, keep=None, r_exact=None, want_logits=False,
              exact_q=False):
    """ADA attention of G query heads [G, d] against T coded keys of one kv head.

    logit = ||q|| r~ f_b(c_q, c_k) / sqrt(d); softmax over retained slots; P.V.
    exact_q: f = <q/||q||, u~(c_k)> (the unquantised unit query, reading R13).
    Returns out [G, d] (and logits [G, T] with -inf where evicted).
    """
    q = _c(q_bf16, np.uint16)
    G, d = q.shape
    kcodes = _c(kcodes, np.int32)
    T = kcodes.shape[0]
    kbits = _c(np.broadcast_to(np.asarray(kbits, np.int32), (T,)), np.int32)
    rcode = _c(rcode, np.uint8)
    r_exact = _c(r_exact, np.float64)
    keep = _c(keep, np.uint8)
    v = _c(v_bf16, np.uint16)
    out = np.empty((G, d), np.float64)
    lg = np.empty((G, T), np.float64) if want_logits else None
    fn = lib().spkv_oracle_ada_group_exact_q if exact_q else lib().spkv_oracle_ada_group
    fn(d, G, T, _ptr(q), _ptr(kcodes), _ptr(kbits), _ptr(rcode), _ptr(r_exact), float(L), float(delta), _ptr(keep),
       _ptr(v), _ptr(out), _ptr(lg))
    return (out, lg) if want_logits else out


def dense_group(q_bf16, k_bf16, v_bf16, keep=None, want_logits=False):
    """Dense attention: logit = q.k/sqrt(d), softmax over retained slots, P.V."""
    q = _c(q_bf16, np.uint16)
    G, d = q.shape
    k = _c(k_bf16, np.uint16)
    T = k.shape[0]
    keep = _c(keep, np.uint8)
    v = _c(v_bf16, np.uint16)
    out = np.empty((G, d), np.float64)
    lg = np.empty((G, T), np.float64) if want_logits else None
    lib().spkv_oracle_dense_group(d, G, T, _ptr(q), _ptr(k), _ptr(keep), _ptr(v), _ptr(out), _ptr(lg))
    return (out, lg) if want_logits else out


def map_groups(fn, items, threads: int | None = None):
    """Run fn over items on a thread pool (the C calls release the GIL)."""
    threads = threads or len(os.sched_getaffinity(0))
    with ThreadPoolExecutor(max_workers=threads) as ex:
        return list(ex.map(fn, items))


def rdr_plan(keys_bf16, q_norms, budget_bytes, tier_mask=0xF, protect=None):
    """RDR controller (readings R14-R17): tiers [T] (0 = evicted) for keys [T, H_kv, d].

    Returns (tiers, lambda, rate_bytes, distortion, status)."""
    k = _c(keys_bf16, np.uint16)
    T, Hkv, d = k.shape
    qn = _c(np.asarray(q_norms, np.float64).reshape(Hkv), np.float64)
    pr = _c(protect, np.uint8)
    tiers = np.empty(T, np.int32)
    lam, rate, dist = (ctypes.c_double() for _ in range(3))
    st = lib().spkv_oracle_rdr_plan(d, T, Hkv, _ptr(k), _ptr(qn), _ptr(pr), float(budget_bytes), int(tier_mask),
                                    _ptr(tiers), ctypes.byref(lam), ctypes.byref(rate), ctypes.byref(dist))
    return tiers, lam.value, rate.value, dist.value, int(st)



def rdr_assign(keys_bf16, q_norms, lam, tier_mask=0xF, protect=None):
    """Tiers [T] and total rate of the per-token minimisers at one multiplier lam."""
    k = _c(keys_bf16, np.uint16)
    T, Hkv, d = k.shape
    qn = _c(np.asarray(q_norms, np.float64).reshape(Hkv), np.float64)
    pr = _c(protect, np.uint8)
    tiers = np.empty(T, np.int32)
    rate = lib().spkv_oracle_rdr_assign(d, T, Hkv, _ptr(k), _ptr(qn), _ptr(pr), int(tier_mask), float(lam),
                                        _ptr(tiers))
    return tiers, rate


RDR_TIER_ORDER = (3, 4, 6, 8)


def rdr_pack(tiers, page=16):
    """Tier-homogeneous pages for a plan (section 2.2: every page holds one
    precision tier).  Reading: the resident tokens are grouped by tier in
    ascending b, ascending t within a tier, and each group fills whole pages
    of 16 slots (its last page partly); attention over the kept tokens does
    not depend on their order, since keys are stored after RoPE.

    Returns (dst_pos [T] int32: page * 16 + slot in the packed sequence, -1
    when evicted; page_bits [n_pages] uint8; page_keep [n_pages] uint16, bit s
    set when slot s holds a token)."""
    tiers = np.asarray(tiers).reshape(-1)
    dst = np.full(tiers.shape[0], -1, np.int32)
    bits, keep = [], []
    for b in RDR_TIER_ORDER:
        toks = [t for t in range(tiers.shape[0]) if int(tiers[t]) == b]
        for r, t in enumerate(toks):
            dst[t] = len(bits) * page + r
        for p0 in range(0, len(toks), page):
            n = min(page, len(toks) - p0)
            bits.append(b)
            keep.append((1 << n) - 1)
    return dst, np.array(bits, np.uint8), np.array(keep, np.uint16)
