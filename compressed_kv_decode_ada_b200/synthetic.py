"""Seeded synthetic decode workloads (inputs only; none of the method's arithmetic).

Shapes follow the long-context decode workloads of the Spherical KV summary
(section 4: Llama-3.1-8B-class models, 8K-128K contexts, paged serving); the
datasets named there are not available, so seeded random tensors stand in:

  keys    per kv head, channel scale s_c ~ LogNormal(0, 0.5) with 4 outlier
          channels x10; k = N(0,1) * s_c, then (rope=True) a rotate-half RoPE
          rotation by token position with base 500000; stored bf16.
  values  N(0,1) bf16.  queries N(0,1) bf16.
  pages   16 tokens; the block table maps each sequence's pages to a seeded
          random permutation of the physical pages.
  tiers   one bit width per page: 4, or (mixed=True) b in {3,4,6,8} with
          probabilities {0.3,0.4,0.2,0.1} and the first page of every sequence
          at b = 8 (protected sink tokens).
  mask    (mask=True) each non-sink token is evicted with probability 0.25,
          the same decision for every kv head; the first 4 tokens are kept.
  radius  grid per kv head: L_h = min log2 ||k||, Delta_h = (max - min)/255
          over the keys of the cache, as fp32 (inputs of both the kernels and
          the oracle).

Every random draw comes from one torch.Generator seeded with the config seed,
on the device the tensors are made on (so a given seed gives the same data on
every run on the same device type).  This module imports neither the CUDA
library nor the oracle.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

HEAD_DIM = 128
PAGE = 16
ROPE_BASE = 500000.0

# The five workload shapes, by name.  'ctx' is a fixed length or
# ('loguniform', lo, hi).
TINY = "tiny_b1_h1_t4096_b4"
LLAMA3_8B = "llama3_8b_b8_h32x8_t32768_b4"
LONG_128K = "long_b1_h32x8_t131072_b4"
RAGGED_RDR = "ragged_rdr_b32_h32x8_t1k-64k_mixed_b_mask25"
SHAPE_70B = "70b_b16_h64x8_t16384_b4_encode"
WORKLOADS = {
    TINY: dict(B=1, Hq=1, Hkv=1, ctx=4096, rope=False, mixed=False, mask=False, seed=0),
    LLAMA3_8B: dict(B=8, Hq=32, Hkv=8, ctx=32768, rope=True, mixed=False, mask=False, seed=1),
    LONG_128K: dict(B=1, Hq=32, Hkv=8, ctx=131072, rope=True, mixed=False, mask=False, seed=2),
    RAGGED_RDR: dict(B=32, Hq=32, Hkv=8, ctx=("loguniform", 1024, 65536), rope=True, mixed=True, mask=True, seed=3),
    SHAPE_70B: dict(B=16, Hq=64, Hkv=8, ctx=16384, rope=True, mixed=False, mask=False, seed=4),
}
for _n, _c in WORKLOADS.items():
    _c["name"] = _n


@dataclass
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    ctx: np.ndarray              # [B] int32 context lengths
    seq_off: np.ndarray          # [B+1] token offsets into keys/values
    keys: torch.Tensor           # [Ntok, Hkv, 128] bf16
    values: torch.Tensor         # [Ntok, Hkv, 128] bf16
    q: torch.Tensor              # [B, Hq, 128] bf16
    block_table: torch.Tensor    # [B, max_pages] int32 (device); -1 past the end
    block_table_np: np.ndarray
    num_pages: int
    page_bits: np.ndarray        # [num_pages] int
    keep_mask: np.ndarray | None  # [num_pages, Hkv] uint16 or None
    token_keep: np.ndarray | None  # [Ntok] bool or None
    rad_lo: np.ndarray           # [Hkv] float32
    rad_step: np.ndarray         # [Hkv] float32
    seed: int
    extras: dict = field(default_factory=dict)

    @property
    def max_ctx(self) -> int:
        return int(self.ctx.max()) if self.B else 0

    @property
    def max_pages(self) -> int:
        return int(self.block_table_np.shape[1])

    @property
    def kv_tokens(self) -> int:
        return int(self.ctx.sum())

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def ctx_tensor(self, device=None) -> torch.Tensor:
        return torch.as_tensor(self.ctx.astype(np.int32), device=device or self.keys.device)

    # ---- per-(sequence, kv head) views for the oracle (host copies, bf16 bit patterns)
    def token_bits(self, b: int) -> np.ndarray:
        n = int(self.ctx[b])
        pages = self.block_table_np[b, (np.arange(n) // PAGE)]
        return self.page_bits[pages].astype(np.int32)

    def keys_bits(self, b: int, h: int) -> np.ndarray:
        s, e = int(self.seq_off[b]), int(self.seq_off[b + 1])
        return self.keys[s:e, h].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)

    def values_bits(self, b: int, h: int) -> np.ndarray:
        s, e = int(self.seq_off[b]), int(self.seq_off[b + 1])
        return self.values[s:e, h].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)

    def q_bits(self, b: int, h: int) -> np.ndarray:
        G = self.G
        return self.q[b, h * G:(h + 1) * G].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)

    def keep_of(self, b: int) -> np.ndarray | None:
        if self.token_keep is None:
            return None
        s, e = int(self.seq_off[b]), int(self.seq_off[b + 1])
        return self.token_keep[s:e].astype(np.uint8)


def _ctx_lengths(spec, B, gen, device):
    if isinstance(spec, tuple):
        _, lo, hi = spec
        u = torch.rand(B, generator=gen, device=device, dtype=torch.float64).cpu().numpy()
        return np.floor(np.exp(np.log(lo) + u * (np.log(hi) - np.log(lo)))).astype(np.int32)
    return np.full(B, int(spec), np.int32)


def _rope_(k: torch.Tensor, pos0: int) -> None:
    """In-place rotate-half RoPE on k [n, Hkv, 128] (fp32), positions pos0.."""
    n = k.shape[0]
    half = HEAD_DIM // 2
    inv = ROPE_BASE ** (-torch.arange(half, dtype=torch.float64, device=k.device) * 2.0 / HEAD_DIM)
    ang = (torch.arange(pos0, pos0 + n, dtype=torch.float64, device=k.device)[:, None] * inv[None, :])
    c, s = torch.cos(ang).float()[:, None, :], torch.sin(ang).float()[:, None, :]
    a, b = k[..., :half].clone(), k[..., half:].clone()
    k[..., :half] = a * c - b * s
    k[..., half:] = a * s + b * c


def make_workload(cfg: str | dict, device="cuda", *, B=None, ctx=None, Hq=None, Hkv=None, seed=None,
                  mixed=None, mask=None, rope=None, extra_pages: int = 0, perm_seed=None) -> Workload:
    """Build a seeded workload; keyword overrides shrink a config for parity tests.

    perm_seed (optional) draws the physical page permutation from its own
    generator, leaving every other draw unchanged."""
    c = dict(WORKLOADS[cfg]) if isinstance(cfg, str) else dict(cfg)
    for k_, v_ in dict(B=B, ctx=ctx, Hq=Hq, Hkv=Hkv, seed=seed, mixed=mixed, mask=mask, rope=rope).items():
        if v_ is not None:
            c[k_] = v_
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(int(c["seed"]))
    Bn, Hq_, Hkv_ = int(c["B"]), int(c["Hq"]), int(c["Hkv"])
    ctxs = np.asarray(c["ctx"], np.int32) if isinstance(c["ctx"], (list, np.ndarray)) else _ctx_lengths(
        c["ctx"], Bn, gen, device)
    seq_off = np.zeros(Bn + 1, np.int64)
    seq_off[1:] = np.cumsum(ctxs)
    ntok = int(seq_off[-1])

    # ---- pages and block table
    npg = (ctxs.astype(np.int64) + PAGE - 1) // PAGE
    num_pages = int(npg.sum()) + int(extra_pages)
    max_pages = max(int(npg.max()) if Bn else 1, 1)
    perm = torch.randperm(max(num_pages, 1), generator=gen, device=device).cpu().numpy()[:num_pages]
    if perm_seed is not None:
        g2 = torch.Generator(device="cpu")
        g2.manual_seed(int(perm_seed))
        perm = torch.randperm(max(num_pages, 1), generator=g2).numpy()[:num_pages]
    bt = np.full((Bn, max_pages), -1, np.int32)
    o = 0
    for b in range(Bn):
        bt[b, :npg[b]] = perm[o:o + npg[b]]
        o += int(npg[b])

    # ---- tiers (drawn per logical page, so that a different physical
    # permutation leaves every token's tier unchanged)
    page_bits = np.full(num_pages, 4, np.int64)
    if c.get("mixed"):
        nlog = int(npg.sum())
        r = torch.rand(max(nlog, 1), generator=gen, device=device, dtype=torch.float64).cpu().numpy()[:nlog]
        logical = np.select([r < 0.3, r < 0.7, r < 0.9], [3, 4, 6], 8).astype(np.int64)
        o = 0
        for b in range(Bn):
            if npg[b]:
                logical[o] = 8  # first page of every sequence: protected sinks at b_max
            page_bits[bt[b, :npg[b]]] = logical[o:o + npg[b]]
            o += int(npg[b])

    # ---- keys, values, queries
    scale = torch.exp(0.5 * torch.randn((Hkv_, HEAD_DIM), generator=gen, device=device))
    for h in range(Hkv_):
        idx = torch.randperm(HEAD_DIM, generator=gen, device=device)[:4]
        scale[h, idx] *= 10.0
    keys = torch.empty((ntok, Hkv_, HEAD_DIM), dtype=torch.bfloat16, device=device)
    values = torch.empty((ntok, Hkv_, HEAD_DIM), dtype=torch.bfloat16, device=device)
    chunk = 1 << 16
    for b in range(Bn):
        s0, n = int(seq_off[b]), int(ctxs[b])
        for p0 in range(0, n, chunk):
            m = min(chunk, n - p0)
            k = torch.randn((m, Hkv_, HEAD_DIM), generator=gen, device=device) * scale[None]
            if c.get("rope"):
                _rope_(k, p0)
            keys[s0 + p0:s0 + p0 + m] = k.to(torch.bfloat16)
            values[s0 + p0:s0 + p0 + m] = torch.randn((m, Hkv_, HEAD_DIM), generator=gen, device=device).to(
                torch.bfloat16)
    q = torch.randn((Bn, Hq_, HEAD_DIM), generator=gen, device=device).to(torch.bfloat16)

    # ---- retention mask
    keep_mask = token_keep = None
    if c.get("mask"):
        u = torch.rand(ntok, generator=gen, device=device).cpu().numpy()
        token_keep = u >= 0.25
        for b in range(Bn):
            token_keep[seq_off[b]:seq_off[b] + min(4, int(ctxs[b]))] = True
        keep_mask = np.full((num_pages, Hkv_), 0xFFFF, np.uint16)
        for b in range(Bn):
            tk = token_keep[seq_off[b]:seq_off[b + 1]]
            padded = np.ones(int(npg[b]) * PAGE, bool)
            padded[:len(tk)] = tk
            words = (padded.reshape(-1, PAGE).astype(np.uint32) << np.arange(PAGE, dtype=np.uint32)).sum(1)
            keep_mask[bt[b, :npg[b]], :] = words.astype(np.uint16)[:, None]

    # ---- radius grid per kv head (calibrated over this cache's keys)
    rad_lo = np.zeros(Hkv_, np.float32)
    rad_step = np.full(Hkv_, 1.0 / 255, np.float32)
    if ntok:
        r = torch.linalg.vector_norm(keys.double(), dim=2)  # [ntok, Hkv]
        lr = torch.log2(torch.clamp(r, min=1e-30))
        lo, hi = lr.min(0).values.cpu().numpy(), lr.max(0).values.cpu().numpy()
        rad_lo = lo.astype(np.float32)
        rad_step = np.maximum((hi - lo) / 255.0, 1e-6).astype(np.float32)

    return Workload(name=c["name"], B=Bn, Hq=Hq_, Hkv=Hkv_, ctx=ctxs, seq_off=seq_off, keys=keys, values=values,
                    q=q, block_table=torch.as_tensor(bt, device=device), block_table_np=bt, num_pages=num_pages,
                    page_bits=page_bits, keep_mask=keep_mask, token_keep=token_keep, rad_lo=rad_lo,
                    rad_step=rad_step, seed=int(c["seed"]))


def ada_step_bytes(wl: Workload) -> float:
    """Algorithmic HBM bytes of one ADA decode step over the whole batch.

    Per (token, kv head): 16 b bytes of angle codes, 1 radius byte, 256 bytes of
    bf16 values (and 1/8 byte of keep mask when a mask is used); per token:
    4/16 bytes of block table and 8/16 bytes of page header."""
    total = 0.0
    for b in range(wl.B):
        bits = wl.token_bits(b).astype(np.float64)
        per_head = 16.0 * bits + 1.0 + 256.0 + (0.125 if wl.keep_mask is not None else 0.0)
        total += float(per_head.sum()) * wl.Hkv + 0.75 * len(bits)
    return total


def dense_step_bytes(wl: Workload) -> float:
    """Algorithmic bytes of the bf16 dense decode: 512 B per (token, kv head)
    plus 4/16 bytes of block table per token."""
    n = float(wl.ctx.sum())
    return n * (512.0 * wl.Hkv + 0.25)


@dataclass
class RdrInputs:
    """Inputs of the RDR controller for the sequences of a workload."""
    seq_start: np.ndarray  # [B + 1] int32 (the workload's seq_off)
    q_norms: np.ndarray    # [B, H_kv] float32
    protect: np.ndarray    # [ntok] uint8
    budget: np.ndarray     # [B] float64 bytes


def make_rdr_inputs(wl: Workload, budget_frac: float = 0.35, sinks: int = 4, recent: int = 64,
                    seed: int | None = None) -> RdrInputs:
    """Seeded RDR inputs for a workload's keys (section 2.2's controller):

      q_norms  per (sequence, kv head) ~ sqrt(128) * LogNormal(0, 0.25), the
               magnitude of a 128-d standard normal query, as fp32;
      protect  the first `sinks` tokens (attention sinks) and the last
               `recent` tokens (the local window) of every sequence;
      budget   budget_frac x the bytes of the whole sequence at b = 8
               (T * H_kv * (16 * 8 + 1 + 256)).
    """
    gen = torch.Generator(device="cpu")
    gen.manual_seed(int(wl.seed if seed is None else seed) + 7919)
    qn = (math.sqrt(HEAD_DIM) * torch.exp(0.25 * torch.randn((wl.B, wl.Hkv), generator=gen,
                                                             dtype=torch.float64))).numpy().astype(np.float32)
    ntok = int(wl.seq_off[-1])
    protect = np.zeros(ntok, np.uint8)
    for b in range(wl.B):
        s0, s1 = int(wl.seq_off[b]), int(wl.seq_off[b + 1])
        protect[s0:min(s1, s0 + sinks)] = 1
        protect[max(s0, s1 - recent):s1] = 1
    full = wl.ctx.astype(np.float64) * wl.Hkv * (16 * 8 + 1 + 256)
    return RdrInputs(seq_start=wl.seq_off.astype(np.int32), q_norms=qn, protect=protect,
                     budget=np.floor(budget_frac * full))
