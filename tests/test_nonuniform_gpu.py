"""GPU <-> oracle parity of the non-uniform angle quantiser (an f_b variant:
equal-probability cells of each polar angle's sin^(d-1-i) law, medians for
reconstruction, uniform azimuth; oracle/nonuniform.py).

Codes: the GPU decides phi_i >= theta_ij exactly against the host tables'
edges (accurate to 1e-12), the oracle decides floor(2^b F_i(phi_i)) on the
probability scale; codes must be equal except on a cell edge (the oracle's
scaled position within 1e-9 of an integer), and those must stay below 1e-6 of
all codes.  Logits: |d f_b| <= 1e-4 (tokens whose codes agree).  Outputs:
<= 2e-3 absolute.  The oracle encodes the keys itself."""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import nonuniform as onu
from tests import helpers

pytestmark = pytest.mark.gpu

OUT_TOL = 2e-3
FB_TOL = 1e-4
EDGE_REL = 1e-9
LLAMA = "llama3_8b_b8_h32x8_t32768_b4"


@pytest.fixture(scope="module")
def spkv():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import compressed_kv_decode_ada_b200 as m
    from compressed_kv_decode_ada_b200 import synthetic

    return m, synthetic


def _tables(m, bits):
    ec, mc, ms = m.ops.nonuniform_tables(128, bits)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    return dev(ec), dev(mc), dev(ms)


def _build(spkv, bits, **kw):
    """A workload whose every page has b = bits, encoded with the non-uniform quantiser."""
    m, synthetic = spkv
    wl = synthetic.make_workload(LLAMA, device="cuda", **kw)
    wl.page_bits = np.full(wl.num_pages, bits, np.int64)
    cache = m.SpkvCache(wl.num_pages, wl.Hkv, wl.page_bits, wl.rad_lo, wl.rad_step, keep_mask=wl.keep_mask)
    ec, mc, ms = _tables(m, bits)
    for b in range(wl.B):
        s, n = int(wl.seq_off[b]), int(wl.ctx[b])
        if n:
            m.encode_keys_nonuniform(cache, wl.keys[s:s + n].unsqueeze(0).contiguous(),
                                     torch.zeros(1, dtype=torch.int32, device="cuda"),
                                     wl.block_table[b:b + 1].contiguous(), bits, ec,
                                     values=wl.values[s:s + n].unsqueeze(0).contiguous())
    torch.cuda.synchronize()
    assert cache.error_flags() == 0
    wl.extras["code_offset"] = cache.page_code_offset
    return wl, cache, (ec, mc, ms)


def _positions(keys_bits, bits, L, D):
    """The oracle's scaled positions: 2^b F_i(phi_i) of the polar angles,
    phi 2^b / 2 pi of the azimuth, and the radius code's (floor = code)."""
    x = oracle.bf16_to_f64(keys_bits)
    T = x.shape[0]
    n = 1 << bits
    phi = np.stack([oracle.angles(x[t]) for t in range(T)]) if T else np.zeros((0, 127))
    apos = np.empty((T, 127))
    for j in range(126):
        apos[:, j] = n * onu.polar_cdf(phi[:, j], 128, j + 1)
    apos[:, 126] = phi[:, 126] * n / (2.0 * math.pi)
    r = np.linalg.norm(x, axis=1)
    with np.errstate(divide="ignore"):
        rpos = (np.log2(r) - L) / D + 0.5
    return apos, rpos


def _oracle_group(wl, b, h, bits):
    L, D = float(wl.rad_lo[h]), float(wl.rad_step[h])
    codes, rc = onu.encode(wl.keys_bits(b, h), bits, L, D)
    return codes, rc, L, D


@pytest.mark.parametrize("bits", [3, 4, 6, 8])
def test_nonuniform_encode_codes_match_the_oracle(spkv, bits):
    wl, cache, _ = _build(spkv, bits, B=2, ctx=[150, 37], Hq=8, Hkv=2)
    arena = cache.arena.cpu().numpy()
    n_codes = n_edge_mismatch = 0
    for b, h in helpers.all_groups(wl):
        gc, gr, pads = helpers.gpu_codes_for_seq(arena, wl, b, h)
        oc, orc, L, D = _oracle_group(wl, b, h, bits)
        apos, rpos = _positions(wl.keys_bits(b, h), bits, L, D)
        ea, er = helpers.near_integer(apos, EDGE_REL), helpers.near_integer(rpos, EDGE_REL)
        assert not ((gc != oc) & ~ea).any(), np.argwhere((gc != oc) & ~ea)[:5]
        assert not ((gr != orc) & ~er).any()
        assert np.all(pads == 0)
        n_codes += oc.size + orc.size
        n_edge_mismatch += int(((gc != oc) & ea).sum() + ((gr != orc) & er).sum())
    assert n_edge_mismatch <= max(1, 1e-6 * n_codes), (n_edge_mismatch, n_codes)


@pytest.mark.parametrize("bits,kw", [
    (4, dict(B=2, ctx=[300, 77], Hq=8, Hkv=2)),       # G = 4, ragged tails
    (3, dict(B=2, ctx=[129, 16], Hq=4, Hkv=2)),       # G = 2, a one-page context
    (6, dict(B=1, ctx=[200], Hq=16, Hkv=2)),          # G = 8
    (8, dict(B=2, ctx=[90, 33], Hq=2, Hkv=2)),        # G = 1
])
def test_nonuniform_decode_matches_the_oracle(spkv, bits, kw):
    m = spkv[0]
    wl, cache, (ec, mc, ms) = _build(spkv, bits, **kw)
    lg = torch.full((wl.B, wl.Hq, wl.max_ctx), float("nan"), device="cuda")
    out = m.decode_attention_nonuniform(cache, wl.q, wl.block_table, wl.ctx_tensor(), wl.max_ctx, bits, ec, mc, ms,
                                        logits=lg)
    torch.cuda.synchronize()
    assert cache.error_flags() == 0
    out, lg = out.cpu().numpy(), lg.cpu().numpy()
    arena = cache.arena.cpu().numpy()
    err = 0.0
    for b, h in helpers.all_groups(wl):
        n = int(wl.ctx[b])
        oc, rc, L, D = _oracle_group(wl, b, h, bits)
        keep = wl.keep_of(b)
        want = onu.ada_group(wl.q_bits(b, h), oc, bits, rc, L, D, wl.values_bits(b, h), keep=keep)
        err = max(err, float(np.abs(out[b, h * wl.G:(h + 1) * wl.G] - want).max()))
        # logits: ||q|| r~ f_b / sqrt(d) with the oracle's decoded vectors
        gc, _, _ = helpers.gpu_codes_for_seq(arena, wl, b, h)
        same = np.all(gc == oc, axis=1)
        uk = np.stack([onu.unit_from_codes(oc[t], bits) for t in range(n)])
        r = np.array([oracle.radius_value(int(c), L, D) for c in rc])
        q = oracle.bf16_to_f64(wl.q_bits(b, h))
        for g in range(wl.G):
            qn = float(np.linalg.norm(q[g]))
            uq = onu.unit_from_codes(onu.codes_from_angles(oracle.angles(q[g]), bits), bits)
            ref = qn * r * (uk @ uq) / math.sqrt(128.0)
            got = lg[b, h * wl.G + g, :n].astype(np.float64)
            live = np.asarray(keep, bool)[:n] if keep is not None else np.ones(n, bool)
            assert np.all(np.isinf(got[~live]))
            sel = live & same
            scale = qn * r[sel] / math.sqrt(128.0)
            d = np.abs(got[sel] - ref[sel]) / np.maximum(scale, 1e-30)
            assert d.max() <= FB_TOL, d.max()
    assert err <= OUT_TOL, err


@pytest.mark.parametrize("num_splits", [0, 3])
def test_nonuniform_decode_long_context_splits(spkv, num_splits):
    """A 5000-token context at b = 4 (G = 4): the default split count (about six
    CTAs per SM: one page per split here) and three splits (each warp walks
    many 32-token chunks, value rows batched eight at a time), against the
    oracle and against each other."""
    m = spkv[0]
    wl, cache, (ec, mc, ms) = _build(spkv, 4, B=1, ctx=[5000], Hq=8, Hkv=2)
    out = m.decode_attention_nonuniform(cache, wl.q, wl.block_table, wl.ctx_tensor(), wl.max_ctx, 4, ec, mc, ms,
                                        num_splits=num_splits)
    torch.cuda.synchronize()
    assert cache.error_flags() == 0
    out = out.cpu().numpy()
    err = 0.0
    for b, h in helpers.all_groups(wl):
        oc, rc, L, D = _oracle_group(wl, b, h, 4)
        want = onu.ada_group(wl.q_bits(b, h), oc, 4, rc, L, D, wl.values_bits(b, h), keep=wl.keep_of(b))
        err = max(err, float(np.abs(out[b, h * wl.G:(h + 1) * wl.G] - want).max()))
    assert err <= OUT_TOL, err


def test_nonuniform_full_size_sampled_parity(spkv):
    """The Llama-3-8B shape at full size (B = 8, 32768 tokens, 32 / 8 heads) with
    the non-uniform quantiser at b = 4, in the launch configuration the bench
    times (default split count): sampled (sequence, kv head) groups against the
    oracle (codes off the cell edges, outputs), and every output row a convex
    combination of value rows."""
    m = spkv[0]
    wl, cache, (ec, mc, ms) = _build(spkv, 4)
    out = m.decode_attention_nonuniform(cache, wl.q, wl.block_table, wl.ctx_tensor(), wl.max_ctx, 4, ec, mc, ms)
    torch.cuda.synchronize()
    assert cache.error_flags() == 0
    outn = out.cpu().numpy()
    arena = cache.arena.cpu().numpy()
    err = 0.0
    for b, h in [(0, 0), (7, 7), (3, 5)]:
        oc, rc, L, D = _oracle_group(wl, b, h, 4)
        gc, gr, _ = helpers.gpu_codes_for_seq(arena, wl, b, h)
        apos, rpos = _positions(wl.keys_bits(b, h), 4, L, D)
        assert not ((gc != oc) & ~helpers.near_integer(apos, EDGE_REL)).any()
        assert not ((gr != rc) & ~helpers.near_integer(rpos, EDGE_REL)).any()
        want = onu.ada_group(wl.q_bits(b, h), oc, 4, rc, L, D, wl.values_bits(b, h), keep=wl.keep_of(b))
        err = max(err, float(np.abs(outn[b, h * wl.G:(h + 1) * wl.G] - want).max()))
    assert err <= OUT_TOL, err
    vmax = wl.values.float().abs().amax().item()
    assert outn.max() <= vmax + 1e-3 and outn.min() >= -vmax - 1e-3


def test_nonuniform_edge_cases(spkv):
    """Empty and fully evicted sequences give 0, a bad page id and a page of
    another width set their device-error bits without a fault, and the
    untouched sequences keep their parity."""
    m = spkv[0]
    wl, cache, (ec, mc, ms) = _build(spkv, 4, B=3, ctx=[0, 40, 300], Hq=4, Hkv=1)
    km = cache.keep_mask if cache.keep_mask is not None else torch.full(
        (wl.num_pages, wl.Hkv), -1, dtype=torch.int16, device="cuda")
    km[torch.as_tensor(wl.block_table_np[1, :3], device="cuda").long()] = 0  # evict sequence 1
    cache.keep_mask = km

    def dec(bt):
        out = m.decode_attention_nonuniform(cache, wl.q, bt, wl.ctx_tensor(), wl.max_ctx, 4, ec, mc, ms)
        torch.cuda.synchronize()
        return out

    out = dec(wl.block_table).cpu().numpy()
    assert cache.error_flags() == 0
    assert np.all(out[0] == 0) and np.all(out[1] == 0)
    oc, rc, L, D = _oracle_group(wl, 2, 0, 4)
    want = onu.ada_group(wl.q_bits(2, 0), oc, 4, rc, L, D, wl.values_bits(2, 0), keep=wl.keep_of(2))
    assert np.abs(out[2] - want).max() <= OUT_TOL
    # a page id past the pool: flagged, skipped, no fault
    bt = wl.block_table.clone()
    bt[2, 3] = wl.num_pages + 7
    cache.clear_errors()
    out = dec(bt)
    assert cache.error_flags() & 1
    assert torch.isfinite(out).all()
    # a page written at another width: flagged
    hdr = cache.hdr.clone()
    cache.hdr[int(wl.block_table_np[2, 0]), 4] = 6
    cache.clear_errors()
    out = dec(wl.block_table)
    assert cache.error_flags() & 2
    assert torch.isfinite(out).all()
    cache.hdr.copy_(hdr)
    # B = 0 is a no-op
    m.decode_attention_nonuniform(cache, wl.q[:0], wl.block_table[:0], wl.ctx_tensor()[:0], wl.max_ctx, 4, ec, mc,
                                  ms)
    torch.cuda.synchronize()
