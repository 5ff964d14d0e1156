"""Page-sharded decode of long sequences across ranks (one process per GPU).

A sequence whose pages do not fit on one GPU, or that one GPU streams too
slowly (the 128K regime of the summary's section 4), is split by pages: rank
r of R holds a contiguous range of each sequence's pages, decodes it with
spkv_decode_attention_partial into per-(sequence, query head) records
(M, L, 0, 0, o[128]), the ranks all-gather the records (B * Hq * 528 bytes per
rank, the only exchange), and every rank combines them with
spkv_merge_partials into the attention over the whole sequence.  Attention
needs no token positions at decode time (keys are stored after RoPE), so a
shard is just a shorter page list.

The collective runs through torch.distributed (NCCL between GPUs); the local
and merge steps are passed in, so the host logic can be driven by any
process group.
"""
from __future__ import annotations

import numpy as np
import torch

from . import ops
from ._lib import PARTIAL_FLOATS

PAGE = 16


def shard_pages(n_pages: int, world: int, rank: int) -> tuple[int, int]:
    """Page range [p0, p1) of `rank`: equal contiguous shares, the first
    n_pages % world ranks one page more."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    base, extra = divmod(int(n_pages), world)
    p0 = rank * base + min(rank, extra)
    return p0, p0 + base + (1 if rank < extra else 0)


def shard_batch(block_table: np.ndarray, ctx: np.ndarray, world: int, rank: int):
    """This rank's block table [B, max_local_pages] (int32, -1 past the end) and
    context lengths [B]: the pages of shard_pages of every sequence, and the
    tokens in them (only the globally last page can be partial)."""
    block_table = np.asarray(block_table)
    ctx = np.asarray(ctx, np.int64)
    B = ctx.shape[0]
    ranges = [shard_pages((int(c) + PAGE - 1) // PAGE, world, rank) for c in ctx]
    width = max([1] + [p1 - p0 for p0, p1 in ranges])
    bt = np.full((B, width), -1, np.int32)
    lctx = np.zeros(B, np.int32)
    for b, (p0, p1) in enumerate(ranges):
        bt[b, :p1 - p0] = block_table[b, p0:p1]
        lctx[b] = max(0, min(int(ctx[b]), p1 * PAGE) - p0 * PAGE)
    return bt, lctx


def gather_partials(partial: torch.Tensor, group=None) -> torch.Tensor:
    """All ranks' records [R, B, Hq, 132] in rank order, on partial's device
    (all_gather_into_tensor; a gloo group exchanges host copies)."""
    import torch.distributed as dist

    world = dist.get_world_size(group)
    partial = partial.contiguous()
    if dist.get_backend(group) == "gloo":  # host-side process groups: stage through host memory
        host = partial.cpu()
        parts = [torch.empty_like(host) for _ in range(world)]
        dist.all_gather(parts, host, group=group)
        return torch.stack(parts).to(partial.device)
    out = torch.empty((world,) + tuple(partial.shape), dtype=partial.dtype, device=partial.device)
    dist.all_gather_into_tensor(out, partial, group=group)
    return out


def sharded_step(local_partial, merge, group=None):
    """One page-sharded decode step: local_partial() -> this rank's records
    [B, Hq, 132]; gather; merge(records [R, B, Hq, 132]) -> the output."""
    partial = local_partial()
    if partial.shape[-1] != PARTIAL_FLOATS:
        raise ValueError("records must have 132 floats")
    return merge(gather_partials(partial, group))


def sharded_decode(cache, q: torch.Tensor, block_table_local: torch.Tensor, ctx_local: torch.Tensor,
                   max_ctx_local: int, group=None, ws=None, num_splits: int = 0, out_dtype=torch.float32,
                   exact_q: bool = False, stream=None) -> torch.Tensor:
    """The page-sharded decode on this rank's GPU: spkv_decode_attention_partial
    over this rank's pages, all-gather, spkv_merge_partials.  Every rank returns
    the full output [B, Hq, 128]."""
    return sharded_step(
        lambda: ops.decode_attention_partial(cache, q, block_table_local, ctx_local, max_ctx_local, ws=ws,
                                             num_splits=num_splits, stream=stream, exact_q=exact_q),
        lambda recs: ops.merge_partials(recs, out_dtype=out_dtype, stream=stream),
        group)
