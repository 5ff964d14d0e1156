"""Page-sharded decode of long sequences (compressed_kv_decode_ada_b200.sharded).

CPU: the page partition, the per-rank block tables, and the whole N > 1 step
(records, all-gather in rank order, log-sum-exp merge) on two gloo ranks, with
each rank's records computed by the fp64 oracle over its own tokens and merged
by an independent numpy combine; the result must equal the oracle's attention
over the whole sequences.  GPU: two and three shards emulated on one GPU
(spkv_decode_attention_partial per shard, spkv_merge_partials) against the
one-shot decode and the oracle."""
import math
import os
import socket

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LOG2E = 1.0 / math.log(2.0)


def test_shard_pages_is_an_exact_partition():
    from compressed_kv_decode_ada_b200.sharded import shard_pages

    for n in (0, 1, 5, 16, 17, 1000):
        for world in (1, 2, 3, 8):
            ranges = [shard_pages(n, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == n
            assert all(ranges[i][1] == ranges[i + 1][0] for i in range(world - 1))
            sizes = [p1 - p0 for p0, p1 in ranges]
            assert max(sizes) - min(sizes) <= 1


def test_shard_batch_splits_tokens_and_pages():
    from compressed_kv_decode_ada_b200.sharded import shard_batch

    ctx = np.array([1, 16, 17, 100, 0], np.int32)
    bt = np.arange(5 * 7, dtype=np.int32).reshape(5, 7)
    for world in (1, 2, 3):
        tot = np.zeros(5, np.int64)
        pages = [[] for _ in range(5)]
        for r in range(world):
            lbt, lctx = shard_batch(bt, ctx, world, r)
            tot += lctx
            for b in range(5):
                n = (int(lctx[b]) + 15) // 16
                pages[b] += list(lbt[b, :n])
                assert np.all(lbt[b, n:] == -1)
        assert np.array_equal(tot, ctx)
        for b in range(5):
            assert pages[b] == list(bt[b, :(int(ctx[b]) + 15) // 16])


def _problem():
    """Three sequences of one kv head (G = 2 query heads), coded at b = 4 by the oracle."""
    import oracle

    rng = np.random.default_rng(7)
    ctx = np.array([1, 40, 75], np.int32)
    seqs = []
    for n in ctx:
        keys = (rng.standard_normal((n, 128)) * 1.3).astype(np.float32)
        vals = rng.standard_normal((n, 128)).astype(np.float32)
        kb = (torch.from_numpy(keys).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))
        vb = (torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))
        codes, rc = oracle.encode(kb, 4, 0.0, 5.0 / 255)
        seqs.append((codes, rc, vb))
    q = torch.from_numpy(rng.standard_normal((3, 2, 128)).astype(np.float32)).to(torch.bfloat16)
    q = q.view(torch.int16).numpy().view(np.uint16)
    return ctx, seqs, q


def _oracle_records(ctx, seqs, q, world, rank):
    """This rank's (M, L, 0, 0, o) records, from the oracle over its own tokens."""
    import oracle
    from compressed_kv_decode_ada_b200.sharded import shard_batch

    bt = np.tile(np.arange(8, dtype=np.int32), (3, 1))  # logical page j of every sequence
    lbt, lctx = shard_batch(bt, ctx, world, rank)
    rec = np.zeros((3, 2, 132), np.float64)
    for b, (codes, rc, vb) in enumerate(seqs):
        n = int(lctx[b])
        rec[b, :, 0] = -np.inf
        if n == 0:
            continue
        t0 = int(lbt[b, 0]) * 16
        sl = slice(t0, t0 + n)
        out, lg = oracle.ada_group(q[b], codes[sl], 4, rc[sl], 0.0, 5.0 / 255, vb[sl], want_logits=True)
        x = lg * LOG2E
        M = x.max(axis=1)
        rec[b, :, 0] = M
        rec[b, :, 1] = np.exp2(x - M[:, None]).sum(axis=1)
        rec[b, :, 4:] = out
    return torch.from_numpy(rec)


def _np_merge(recs):
    recs = recs.numpy()
    M = recs[..., 0].max(axis=0)
    w = np.where(np.isinf(recs[..., 0]), 0.0, np.exp2(recs[..., 0] - M) * recs[..., 1])
    num = (w[..., None] * recs[..., 4:]).sum(axis=0)
    den = w.sum(axis=0)
    return num / np.where(den > 0, den, 1.0)[..., None], recs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime
    import sys

    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    from compressed_kv_decode_ada_b200.sharded import sharded_step

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ctx, seqs, qq = _problem()
        got = {}

        def merge(recs):
            out, raw = _np_merge(recs)
            got["raw"] = raw
            return out

        out = sharded_step(lambda: _oracle_records(ctx, seqs, qq, world, rank), merge)
        order_ok = all(np.array_equal(got["raw"][r], _oracle_records(ctx, seqs, qq, world, r).numpy())
                       for r in range(world))
        q.put((rank, out, order_ok))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_page_sharded_step_equals_whole_sequence_attention(world):
    import oracle
    import torch.multiprocessing as mp

    port = _free_port()
    ctxm = mp.get_context("spawn")
    qu = ctxm.Queue()
    procs = [ctxm.Process(target=_rank_main, args=(r, world, port, qu)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((qu.get(timeout=120) for _ in range(world)), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    ctx, seqs, qq = _problem()
    for b, (codes, rc, vb) in enumerate(seqs):
        want = oracle.ada_group(qq[b], codes, 4, rc, 0.0, 5.0 / 255, vb)
        for rank, out, order_ok in res:
            assert order_ok
            assert np.max(np.abs(out[b] - want)) <= 1e-12


def _reorder_tol(wl):
    return 2.0 ** -14 * float(wl.values.float().abs().max())


@pytest.mark.gpu
@pytest.mark.parametrize("shards", [2, 3])
def test_gpu_page_shards_merge_to_the_one_shot_decode(shards):
    import compressed_kv_decode_ada_b200 as m
    from compressed_kv_decode_ada_b200 import synthetic, workload
    from compressed_kv_decode_ada_b200.sharded import shard_batch

    from tests import helpers

    wl = synthetic.make_workload("ragged_rdr_b32_h32x8_t1k-64k_mixed_b_mask25", device="cuda", B=3,
                                 ctx=[5000, 33, 2049], Hq=8, Hkv=2)
    cache = workload.build_cache(wl)
    full = m.decode_attention(cache, wl.q, wl.block_table, wl.ctx_tensor(), wl.max_ctx)
    bt = wl.block_table.cpu().numpy()
    recs = []
    for r in range(shards):
        lbt, lctx = shard_batch(bt, wl.ctx, shards, r)
        recs.append(m.decode_attention_partial(cache, wl.q, torch.from_numpy(lbt).cuda(),
                                               torch.from_numpy(lctx).cuda(), int(lctx.max())))
    out = m.merge_partials(torch.stack(recs))
    torch.cuda.synchronize()
    assert cache.error_flags() == 0
    assert torch.max(torch.abs(out - full)).item() <= _reorder_tol(wl)
    err = helpers.max_abs_diff_groups(out.cpu().numpy(), wl, helpers.all_groups(wl), helpers.oracle_seq)
    assert err <= 2e-3, err


def _gpu_rank_main(rank, world, port, q):
    """One rank of the composed sharded_decode on the one GPU: the CUDA partial
    over this rank's pages, the gloo all-gather (host-staged), the CUDA merge."""
    import datetime
    import sys

    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from compressed_kv_decode_ada_b200 import synthetic, workload
        from compressed_kv_decode_ada_b200.sharded import shard_batch, sharded_decode

        wl = synthetic.make_workload(*_SHARD_WL, device="cuda", **_SHARD_KW)
        cache = workload.build_cache(wl)
        lbt, lctx = shard_batch(wl.block_table.cpu().numpy(), wl.ctx, world, rank)
        out = sharded_decode(cache, wl.q, torch.from_numpy(lbt).cuda(), torch.from_numpy(lctx).cuda(),
                             int(lctx.max()))
        torch.cuda.synchronize()
        q.put((rank, out.cpu().numpy(), cache.error_flags()))
    finally:
        dist.destroy_process_group()


_SHARD_WL = ("ragged_rdr_b32_h32x8_t1k-64k_mixed_b_mask25",)
_SHARD_KW = dict(B=3, ctx=[5000, 33, 2049], Hq=8, Hkv=2)


@pytest.mark.gpu
@pytest.mark.parametrize("world", [2, 3])
def test_gpu_gloo_ranks_sharded_decode_end_to_end(world):
    """sharded_decode as one function on every rank (gloo ranks sharing the GPU;
    no kernel waits on another rank): every rank's output is the whole-sequence
    attention of the oracle and the one-shot decode."""
    import torch.multiprocessing as mp

    import compressed_kv_decode_ada_b200 as m
    from compressed_kv_decode_ada_b200 import synthetic, workload

    from tests import helpers

    port = _free_port()
    ctxm = mp.get_context("spawn")
    qu = ctxm.Queue()
    procs = [ctxm.Process(target=_gpu_rank_main, args=(r, world, port, qu)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((qu.get(timeout=300) for _ in range(world)), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    wl = synthetic.make_workload(*_SHARD_WL, device="cuda", **_SHARD_KW)
    cache = workload.build_cache(wl)
    full = m.decode_attention(cache, wl.q, wl.block_table, wl.ctx_tensor(), wl.max_ctx).cpu().numpy()
    for rank, out, err_flags in res:
        assert err_flags == 0
        assert np.max(np.abs(out - full)) <= _reorder_tol(wl)
        assert np.array_equal(out, res[0][1])  # every rank merged the same records
    err = helpers.max_abs_diff_groups(res[0][1], wl, helpers.all_groups(wl), helpers.oracle_seq)
    assert err <= 2e-3, err
