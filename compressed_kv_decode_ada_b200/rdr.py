"""Host side of a rate-distortion retention plan (technical summary section
2.2): turn the plan of spkv_rdr_plan into a compressed paged cache.

spkv_rdr_plan decides each token's tier (or eviction) and its position in
the sequence's packed, tier-homogeneous pages.  What is left is page
allocation, a host task: each sequence receives n_pages physical pages, the
headers get the pages' bit widths, the retention mask gets the occupied
slots (the same for every kv head, since the decision is per token), and
spkv_encode_keys_packed writes the codes and values to their slots.
"""
from __future__ import annotations

import numpy as np
import torch

from . import ops
from .cache import PAGE, SpkvCache


def allocate_packed(plan: dict, num_kv_heads: int, rad_lo, rad_step, device=None):
    """Physical pages for a plan: sequence s takes the next n_pages[s] pages.

    Returns (cache, block_table [B, max n_pages] int32 on the device,
    ctx_lens [B] int32 on the device: n_pages * 16)."""
    n_pages = plan["n_pages"].cpu().numpy().astype(np.int64)
    status = plan["status"].cpu().numpy()
    if np.any(status & 6):
        raise ValueError(f"plan status {status.tolist()}: pages exceed max_pages_out or bad ranges")
    bits = plan["page_bits"].cpu().numpy()
    keep = plan["page_keep"].cpu().numpy().view(np.uint16)
    B = n_pages.shape[0]
    total = int(n_pages.sum())
    base = np.concatenate([[0], np.cumsum(n_pages)[:-1]]).astype(np.int64)
    page_bits = np.concatenate([bits[s, :n_pages[s]] for s in range(B)]) if total else np.zeros(0, np.uint8)
    page_keep = np.concatenate([keep[s, :n_pages[s]] for s in range(B)]) if total else np.zeros(0, np.uint16)
    device = device if device is not None else plan["tier"].device
    cache = SpkvCache(max(total, 1), num_kv_heads, page_bits if total else np.array([8]), rad_lo, rad_step,
                      device=device,
                      keep_mask=np.repeat(page_keep if total else np.zeros(1, np.uint16), num_kv_heads))
    width = max(1, int(n_pages.max()) if B else 1)
    bt = np.zeros((B, width), np.int32)
    for s in range(B):
        bt[s, :n_pages[s]] = base[s] + np.arange(n_pages[s])
    ctx = (n_pages * PAGE).astype(np.int32)
    return cache, torch.from_numpy(bt).to(device), torch.from_numpy(ctx).to(device)


def build_packed_cache(plan: dict, keys: torch.Tensor, values: torch.Tensor, seq_start: torch.Tensor, rad_lo,
                       rad_step, stream=None):
    """allocate_packed, then spkv_encode_keys_packed of every resident token.

    keys, values: [total_tokens, H_kv, 128] bf16 on the device (the planned
    tokens).  Returns (cache, block_table, ctx_lens)."""
    cache, bt, ctx = allocate_packed(plan, keys.shape[1], rad_lo, rad_step, device=keys.device)
    ops.encode_keys_packed(cache, keys, seq_start, plan["dst_pos"], bt, values=values, stream=stream)
    return cache, bt, ctx
