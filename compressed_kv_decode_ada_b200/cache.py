"""Device-memory owner for a compressed paged KV store (the spkv_cache struct).

PyTorch allocates every buffer; the layouts are those of include/spkv.h:
tier-homogeneous pages ("SPHERICAL KV ...", technical summary section 2.2),
each with a header {code_off16, bits} and one record of 256 b + 16 bytes per
kv head in a byte arena, plus bf16 value pages [num_pages, H_kv, 16, 128].
"""
from __future__ import annotations

import numpy as np
import torch

from ._lib import SpkvCacheC

HEAD_DIM = 128
PAGE = 16
BIT_WIDTHS = (3, 4, 6, 8)


def record_bytes(bits):
    """Bytes of one (page, kv head) record at bit width b: 16 slots x 16 b codes + 16 radius bytes."""
    return 256 * np.asarray(bits, np.int64) + 16


class SpkvCache:
    """Compressed key store + bf16 value pages on one CUDA device.

    page_bits: [num_pages] bit width of each physical page (b in {3,4,6,8}).
    rad_lo, rad_step: [H_kv] fp32 log2-radius grid (L_h, Delta_h).
    keep_mask: optional [num_pages, H_kv] uint16 retention bits (bit s = slot s).
    """

    def __init__(self, num_pages: int, num_kv_heads: int, page_bits, rad_lo, rad_step, device="cuda",
                 keep_mask=None):
        page_bits = np.asarray(page_bits, np.int64).reshape(-1)
        if page_bits.shape[0] != num_pages:
            raise ValueError("page_bits must have one entry per page")
        if not np.all(np.isin(page_bits, BIT_WIDTHS)):
            raise ValueError("page bit widths must be in {3, 4, 6, 8}")
        self.num_pages = int(num_pages)
        self.num_kv_heads = int(num_kv_heads)
        self.device = torch.device(device)
        block = record_bytes(page_bits) * num_kv_heads  # bytes of each page's records
        off = np.zeros(num_pages, np.int64)
        if num_pages > 1:
            off[1:] = np.cumsum(block[:-1])
        arena_bytes = int(block.sum()) if num_pages else 16
        hdr = np.zeros((num_pages, 8), np.uint8)
        hdr[:, 0:4] = (off // 16).astype("<u4").view(np.uint8).reshape(num_pages, 4)
        hdr[:, 4] = page_bits.astype(np.uint8)
        self.page_bits = page_bits
        # bit t set when some page uses tier t (b = 3, 4, 6, 8)
        self.tiers = int(sum(1 << t for t, b in enumerate(BIT_WIDTHS) if np.any(page_bits == b)))
        self.page_code_offset = off
        self.arena = torch.zeros(max(arena_bytes, 16), dtype=torch.uint8, device=self.device)
        self.arena_bytes = arena_bytes
        self.hdr = torch.from_numpy(hdr).to(self.device)
        self.v_pages = torch.zeros((num_pages, num_kv_heads, PAGE, HEAD_DIM), dtype=torch.bfloat16, device=self.device)
        self.rad_lo = torch.as_tensor(np.asarray(rad_lo, np.float32).reshape(num_kv_heads), device=self.device)
        self.rad_step = torch.as_tensor(np.asarray(rad_step, np.float32).reshape(num_kv_heads), device=self.device)
        self.keep_mask = None
        if keep_mask is not None:
            km = np.asarray(keep_mask).astype(np.uint16).reshape(num_pages, num_kv_heads)
            self.keep_mask = torch.from_numpy(km.view(np.int16)).to(self.device)
        self.err = torch.zeros(1, dtype=torch.int32, device=self.device)

    _DESCRIBED = frozenset(("num_pages", "num_kv_heads", "arena", "arena_bytes", "hdr", "v_pages", "rad_lo",
                            "rad_step", "keep_mask", "err", "tiers"))

    def __setattr__(self, name, value):
        if name in self._DESCRIBED:  # the cached descriptor no longer matches
            object.__setattr__(self, "_c", None)
        object.__setattr__(self, name, value)

    def c_struct(self) -> SpkvCacheC:
        """The spkv_cache descriptor of these buffers (rebuilt only after one
        of them is replaced)."""
        c = getattr(self, "_c", None)
        if c is not None:
            return c
        c = SpkvCacheC()
        c.num_kv_heads = self.num_kv_heads
        c.head_dim = HEAD_DIM
        c.page_size = PAGE
        c.num_pages = self.num_pages
        c.code_arena = self.arena.data_ptr()
        c.code_arena_bytes = self.arena_bytes
        c.hdr = self.hdr.data_ptr()
        c.rad_lo_log2 = self.rad_lo.data_ptr()
        c.rad_step_log2 = self.rad_step.data_ptr()
        c.v_pages = self.v_pages.data_ptr()
        c.keep_mask = self.keep_mask.data_ptr() if self.keep_mask is not None else None
        c.err_flags = self.err.data_ptr()
        c.tiers = self.tiers
        self._c = c
        return c

    def error_flags(self) -> int:
        """Device error bits (SPKV_DEVERR_*) accumulated so far (synchronises)."""
        return int(self.err.item()) & 0xFFFFFFFF

    def clear_errors(self) -> None:
        self.err.zero_()

    def resident_bytes(self) -> int:
        """Bytes of codes + radii + headers + values held for all pages."""
        return self.arena_bytes + self.hdr.numel() + self.v_pages.numel() * 2
