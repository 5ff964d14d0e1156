"""Test-side helpers: read the documented page layout back, run the oracle on
(sequence, kv head) groups, and compare.  Layout parsing only (include/spkv.h);
the arithmetic being checked is the oracle's."""
from __future__ import annotations

import math

import numpy as np

import oracle

PAGE = 16


def unpack_records(rec_bytes: np.ndarray, bits: int):
    """rec_bytes: [n, 256 b + 16] uint8 records -> (codes [n, 16, 127], radius [n, 16], pad [n, 16])."""
    n = rec_bytes.shape[0]
    codes_region = rec_bytes[:, :256 * bits].reshape(n, bits, 16, 16)      # [rec, chunk, slot, byte]
    stream = codes_region.transpose(0, 2, 1, 3).reshape(n, 16, 16 * bits)  # [rec, slot, bytes]
    bitsarr = np.unpackbits(stream, axis=2, bitorder="little").reshape(n, 16, 128, bits)
    w = (1 << np.arange(bits)).astype(np.int64)
    fields = (bitsarr.astype(np.int64) * w).sum(axis=3)                    # [rec, slot, 128]
    return fields[:, :, :127].astype(np.int32), rec_bytes[:, 256 * bits:256 * bits + 16], fields[:, :, 127]


def gpu_codes_for_seq(arena: np.ndarray, wl, b: int, h: int):
    """Angle codes [ctx, 127] and radius codes [ctx] that the GPU stored for
    sequence b, kv head h (read through the block table and page headers)."""
    n = int(wl.ctx[b])
    npg = (n + PAGE - 1) // PAGE
    codes = np.zeros((npg * PAGE, 127), np.int32)
    rad = np.zeros(npg * PAGE, np.uint8)
    pads = np.zeros(npg * PAGE, np.int64)
    from compressed_kv_decode_ada_b200.cache import record_bytes

    for j in range(npg):
        pid = int(wl.block_table_np[b, j])
        bits = int(wl.page_bits[pid])
        rb = int(record_bytes(bits))
        off = int(wl.extras["code_offset"][pid]) + h * rb
        c, r, p = unpack_records(arena[off:off + rb][None, :], bits)
        codes[j * PAGE:(j + 1) * PAGE] = c[0]
        rad[j * PAGE:(j + 1) * PAGE] = r[0]
        pads[j * PAGE:(j + 1) * PAGE] = p[0]
    return codes[:n], rad[:n], pads[:n]


def near_integer(pos: np.ndarray, rel: float = 1e-12) -> np.ndarray:
    """Scaled positions within rel * max(1, |t|) of an integer: codes on a cell
    edge, where fp64 rounding may legitimately decide either way."""
    pos = np.asarray(pos, np.float64)
    fin = np.isfinite(pos)
    d = np.full(pos.shape, np.inf)
    d[fin] = np.abs(pos[fin] - np.round(pos[fin]))
    return d <= rel * np.maximum(1.0, np.abs(np.where(fin, pos, 0.0)))


def oracle_seq(wl, b: int, h: int, want_logits: bool = False, exact_q: bool = False):
    """Oracle ADA output for the G query heads of (b, h), encoding the keys itself."""
    keys = wl.keys_bits(b, h)
    bits = wl.token_bits(b)
    L, D = float(wl.rad_lo[h]), float(wl.rad_step[h])
    codes, rcode = oracle.encode(keys, bits, L, D)
    return oracle.ada_group(wl.q_bits(b, h), codes, bits, rcode, L, D, wl.values_bits(b, h), keep=wl.keep_of(b),
                            want_logits=want_logits, exact_q=exact_q)


def oracle_seq_exact_q(wl, b: int, h: int):
    return oracle_seq(wl, b, h, exact_q=True)


def oracle_seq_dense(wl, b: int, h: int):
    return oracle.dense_group(wl.q_bits(b, h), wl.keys_bits(b, h), wl.values_bits(b, h), keep=wl.keep_of(b))


def oracle_seq_decompress(wl, b: int, h: int):
    """Dense attention of the unquantised query over oracle-decompressed keys."""
    keys = wl.keys_bits(b, h)
    bits = wl.token_bits(b)
    L, D = float(wl.rad_lo[h]), float(wl.rad_step[h])
    codes, rcode = oracle.encode(keys, bits, L, D)
    kt = oracle.decompress(codes, bits, rcode, L, D)
    return oracle.dense_group(wl.q_bits(b, h), kt, wl.values_bits(b, h), keep=wl.keep_of(b))


def all_groups(wl):
    return [(b, h) for b in range(wl.B) for h in range(wl.Hkv)]


def max_abs_diff_groups(out_gpu: np.ndarray, wl, groups, fn, threads=None):
    """max |gpu - oracle| over the given (b, h) groups; out_gpu [B, Hq, 128]."""
    res = oracle.map_groups(lambda bh: fn(wl, *bh), groups, threads)
    worst = 0.0
    G = wl.G
    for (b, h), ref in zip(groups, res):
        got = out_gpu[b, h * G:(h + 1) * G].astype(np.float64)
        worst = max(worst, float(np.max(np.abs(got - ref))) if ref.size else 0.0)
    return worst


def logit_scale(wl, b, h, rcode_oracle):
    qn = np.linalg.norm(oracle.bf16_to_f64(wl.q_bits(b, h)), axis=1)  # [G]
    r = np.array([oracle.radius_value(int(c), float(wl.rad_lo[h]), float(wl.rad_step[h])) for c in rcode_oracle])
    return qn[:, None] * r[None, :] / math.sqrt(128.0)


def check_codes(wl, cache, groups):
    """The cache's codes for the (sequence, kv head) groups against oracle.encode:
    equal off the cell edges, and codes decided differently on an edge (fp64
    rounding either way) at most 1e-6 of all codes."""
    arena = cache.arena.cpu().numpy()
    n_codes = n_edge = n_mismatch_edge = 0
    for b, h in groups:
        gc, gr, pads = gpu_codes_for_seq(arena, wl, b, h)
        keys, bits = wl.keys_bits(b, h), wl.token_bits(b)
        oc, orc, apos, rpos = oracle.encode(keys, bits, float(wl.rad_lo[h]), float(wl.rad_step[h]), positions=True)
        edge_a, edge_r = near_integer(apos), near_integer(rpos)
        bad_a = (gc != oc) & ~edge_a
        bad_r = (gr != orc) & ~edge_r
        assert not bad_a.any(), f"angle code mismatch off a cell edge at (b={b}, h={h}): {np.argwhere(bad_a)[:5]}"
        assert not bad_r.any(), f"radius code mismatch off a cell edge at (b={b}, h={h})"
        assert np.all(pads == 0)
        n_codes += oc.size + orc.size
        n_edge += int(edge_a.sum() + edge_r.sum())
        n_mismatch_edge += int(((gc != oc) & edge_a).sum() + ((gr != orc) & edge_r).sum())
    # codes decided differently on a cell edge (fp64 rounding either way) must
    # stay below 1e-6 of all codes; exact ties (common with bf16 inputs, e.g.
    # |x_126| = |x_127|) are decided exactly by both sides and counted as matches
    assert n_mismatch_edge <= max(1, 1e-6 * n_codes), (n_mismatch_edge, n_edge, n_codes)
    return n_codes, n_edge, n_mismatch_edge
