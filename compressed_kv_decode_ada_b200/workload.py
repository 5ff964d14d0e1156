"""Prefill helper: build an SpkvCache for a synthetic workload and append all
of its keys and values through spkv_encode_keys (the CUDA encode kernel)."""
from __future__ import annotations

import torch

from .cache import SpkvCache
from .ops import encode_keys, encode_keys_packed
from .synthetic import Workload


def build_cache(wl: Workload, device=None, with_values: bool = True) -> SpkvCache:
    device = device or wl.keys.device
    cache = SpkvCache(wl.num_pages, wl.Hkv, wl.page_bits, wl.rad_lo, wl.rad_step, device=device,
                      keep_mask=wl.keep_mask)
    prefill(cache, wl, with_values=with_values)
    return cache


def prefill(cache: SpkvCache, wl: Workload, with_values: bool = True, packed: bool = True) -> None:
    """Encode every context token of every sequence into its page slot: one
    spkv_encode_keys call when every sequence has the same length, else one
    spkv_encode_keys_packed call over the concatenated tokens (packed=False:
    one spkv_encode_keys call per sequence instead)."""
    if wl.B == 0:
        return
    if len(set(int(n) for n in wl.ctx)) == 1:
        n = int(wl.ctx[0])
        if n == 0:
            return
        keys = wl.keys.view(wl.B, n, wl.Hkv, -1)
        vals = wl.values.view(wl.B, n, wl.Hkv, -1) if with_values else None
        start = torch.zeros(wl.B, dtype=torch.int32, device=cache.device)
        encode_keys(cache, keys, start, wl.block_table, values=vals)
        return
    if packed:
        key = ("packed_positions", str(cache.device))
        if key not in wl.extras:  # token t of sequence s goes to position t - seq_off[s]
            dev = cache.device
            seq_start = torch.as_tensor(wl.seq_off.astype("int32"), device=dev)
            dst = torch.cat([torch.arange(int(n), dtype=torch.int32, device=dev) for n in wl.ctx])
            wl.extras[key] = (seq_start, dst)
        seq_start, dst = wl.extras[key]
        encode_keys_packed(cache, wl.keys, seq_start, dst, wl.block_table, values=wl.values if with_values else None)
        return
    for b in range(wl.B):
        n = int(wl.ctx[b])
        if n == 0:
            continue
        s = int(wl.seq_off[b])
        keys = wl.keys[s:s + n].unsqueeze(0)
        vals = wl.values[s:s + n].unsqueeze(0) if with_values else None
        start = torch.zeros(1, dtype=torch.int32, device=cache.device)
        encode_keys(cache, keys, start, wl.block_table[b:b + 1].contiguous(), values=vals)


def dense_pages(wl: Workload, num_pages: int | None = None):
    """bf16 K and V pages [num_pages, H_kv, 16, 128] of the workload (layout copy
    through the block table; used by the dense comparison path)."""
    P = num_pages or wl.num_pages
    dev = wl.keys.device
    kp = torch.zeros((P, wl.Hkv, 16, 128), dtype=torch.bfloat16, device=dev)
    vp = torch.zeros_like(kp)
    for b in range(wl.B):
        n = int(wl.ctx[b])
        if n == 0:
            continue
        s = int(wl.seq_off[b])
        t = torch.arange(n, device=dev)
        pid = wl.block_table[b].long()[t // 16]
        kp[pid, :, t % 16] = wl.keys[s:s + n]
        vp[pid, :, t % 16] = wl.values[s:s + n]
    return kp, vp
