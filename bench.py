#!/usr/bin/env python
"""Benchmark: ADA paged decode KV tokens/s on B200 (one JSON line on rank 0).

One step = the whole decode hot path for one batch, in one library call
(spkv_decode_attention_append): append the step's new token (key and value)
of every sequence into its page, then decode over all ctx tokens of every
sequence (split kernel with the fused append + merge kernel).  Default workload: Llama-3-8B-shaped layer decode, B = 8,
32 query / 8 kv heads, d = 128, ctx = 32768, page 16, b = 4 (673 MB of codes,
radii and values per step: far larger than the 126 MB L2, so no flush is
needed between steps).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl spkv|reference]

N > 1 is launched by torchrun, one rank per GPU; every rank decodes its own
batch (independent sequences: weak scaling, no collective on the data path);
the step time is the max over ranks.  --impl reference times the fp64 CPU
oracle on the host cores instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def _dist():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def _synthetic_inputs():
    """The seeded input generators (compressed_kv_decode_ada_b200/synthetic.py),
    loaded from their file without importing the package: the package's
    __init__ maps libspkv.so, which the CPU oracle arm must not load."""
    import importlib.util

    name = "_spkv_synthetic_inputs"
    if name in sys.modules:
        return sys.modules[name]
    path = os.path.join(ROOT, "compressed_kv_decode_ada_b200", "synthetic.py")
    spec = importlib.util.spec_from_file_location(name, path)
    mod = importlib.util.module_from_spec(spec)
    sys.modules[name] = mod
    spec.loader.exec_module(mod)
    return mod


def _cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


# ------------------------------------------------------- rank helpers
def rank_workload(workload: str, rank: int) -> dict:
    """The batch a rank decodes: the named workload shape with its own seed
    (ranks decode independent sequences; there is no exchange between them)."""
    from compressed_kv_decode_ada_b200 import synthetic

    cfg = dict(synthetic.WORKLOADS[workload])
    cfg["seed"] = int(cfg["seed"]) + 1000 * rank
    return cfg


def max_over_ranks(values, device=None):
    """Element-wise max of per-rank timings (all ranks take this collective)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def whole_job_rate(units_per_rank: float, world: int, ms_per_step_max: float) -> float:
    """Units all ranks processed per second, timed by the slowest rank."""
    return units_per_rank * world / (ms_per_step_max * 1e-3)


# --------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during a region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path:
            return None
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------ GPU arm
def run_spkv(args, rank, world, local):
    import torch
    import torch.distributed as dist

    import compressed_kv_decode_ada_b200 as spkv
    from compressed_kv_decode_ada_b200 import synthetic, workload

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    cfg = rank_workload(args.workload, rank)
    if args.B:
        cfg["B"] = args.B  # smaller batch, for profiler captures only
    wl = synthetic.make_workload(cfg, device=dev)
    cache = workload.build_cache(wl)
    B, Hq, Hkv = wl.B, wl.Hq, wl.Hkv
    ctx = wl.ctx_tensor(dev)
    max_ctx = wl.max_ctx
    splits = spkv.default_splits(B, Hkv, max_ctx) if args.splits == 0 else args.splits
    ws = spkv.alloc_workspace(B, Hq, Hkv, max_ctx, splits, device=dev)
    out = torch.empty((B, Hq, 128), dtype=torch.float32, device=dev)
    # the step's new token: the last context position of every sequence
    last = torch.as_tensor((wl.ctx - 1).astype(np.int32), device=dev)
    new_idx = torch.as_tensor(wl.seq_off[1:] - 1, device=dev).long()
    new_k = wl.keys[new_idx].contiguous()     # [B, Hkv, 128]
    new_v = wl.values[new_idx].contiguous()
    stream = torch.cuda.current_stream(dev)

    def step(q, k, v, o):
        spkv.decode_attention_append(cache, k, v, q, wl.block_table, ctx, max_ctx, out=o, ws=ws,
                                     num_splits=splits, stream=stream)

    for _ in range(args.warmup):
        step(wl.q, new_k, new_v, out)
    torch.cuda.synchronize(dev)
    if cache.error_flags():
        raise RuntimeError(f"device error flags {cache.error_flags():#x}")

    # ---------------- timed region: K steps, per-step events around the decode call
    ev_dec = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        t_start.record(stream)
        for i in range(args.steps):
            ev_dec[i][0].record(stream)
            spkv.decode_attention_append(cache, new_k, new_v, wl.q, wl.block_table, ctx, max_ctx, out=out, ws=ws,
                                         num_splits=splits, stream=stream)
            ev_dec[i][1].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    total_ms = t_start.elapsed_time(t_end)
    dec_ms = sum(a.elapsed_time(b) for a, b in ev_dec) / args.steps
    ms_step = total_ms / args.steps
    ms_step, dec_ms = max_over_ranks([ms_step, dec_ms], device=dev)
    clocks = clk.summary()

    # ---------------- end to end through the public API with host buffers
    e2e_steps = max(3, min(args.steps, args.e2e_steps))
    # the step's inputs (q, new k, new v) travel in one pinned buffer and one copy
    nq, nk = wl.q.numel(), new_k.numel()
    in_h = torch.cat([wl.q.reshape(-1), new_k.reshape(-1), new_v.reshape(-1)]).cpu().pin_memory()
    in_d = torch.empty_like(in_h, device=dev)
    q_d = in_d[:nq].view(wl.q.shape)
    k_d = in_d[nq:nq + nk].view(new_k.shape)
    v_d = in_d[nq + nk:].view(new_v.shape)
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for i in range(e2e_steps + 2):
        if i == 2:
            e0.record(stream)
        in_d.copy_(in_h, non_blocking=True)
        step(q_d, k_d, v_d, out)
        out_h.copy_(out, non_blocking=True)
        stream.synchronize()  # the host reads the step's result
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    (e2e_ms,) = max_over_ranks([e2e_ms], device=dev)
    if cache.error_flags():
        raise RuntimeError(f"device error flags {cache.error_flags():#x}")

    extras = {}
    if rank == 0 and args.compare:
        extras = compare_paths(args, spkv, workload, wl, cache, ctx, max_ctx, splits, ws, stream, dev)
        if args.compare_workloads:
            extras["workloads"] = compare_workloads(args, spkv, workload, synthetic, stream, dev, _peaks()[0])

    tokens = wl.kv_tokens
    bytes_step = synthetic.ada_step_bytes(wl)
    result = None
    if rank == 0:
        peak, peak_kind = _peaks()
        achieved = bytes_step / (dec_ms * 1e-3) / 1e9
        traffic = _committed_traffic(args.workload)
        h2d = in_h.numel() * in_h.element_size()
        d2h = out_h.numel() * out_h.element_size()
        result = {
            "metric": "ADA decode KV tokens/s on 1 B200; achieved HBM GB/s as % of peak",
            "value": whole_job_rate(tokens, world, ms_step),
            "unit": "KV tokens/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms_step,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "f32",
            "data": "synthetic (seeded: N(0,1) bf16 keys x log-normal channel scales with 4 outliers, RoPE base "
                    "500000; N(0,1) bf16 values and queries)",
            "config": {"workload": wl.name, "B": B, "num_q_heads": Hq, "num_kv_heads": Hkv, "ctx": int(max_ctx),
                       "page": 16, "bits": sorted(set(int(b) for b in wl.page_bits)), "splits": splits,
                       "kv_tokens_per_step": tokens, "algorithmic_bytes_per_step": bytes_step,
                       "l2": "no flush: the step streams %.0f MB > 126 MB L2" % (bytes_step / 1e6),
                       "step": "spkv_decode_attention_append: append 1 token/sequence + decode, one call",
                       "parallelism": f"dp{world} (independent batches)"},
            "roofline": {"bound": "hbm", "kernel": "spkv_decode_attention_append (split kernel with the append + merge)",
                         "achieved": achieved, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                         "frac": achieved / peak, "frac_of_nominal_8TBs": achieved / NOMINAL_HBM_GBS,
                         "traffic": traffic, "decode_ms": dec_ms},
            "e2e": {"value": whole_job_rate(tokens, world, e2e_ms), "unit": "KV tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "gpu_launches": 2 * args.steps,
            "clocks": clocks,
        }
        if extras:
            result["comparison"] = extras
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return result


def compare_paths(args, spkv, workload, wl, cache, ctx, max_ctx, splits, ws, stream, dev):
    """Untimed-in-the-headline comparison: dense bf16 and decompress-then-dot
    decode of the same batch (same split count), and bulk encode throughput."""
    import torch

    from compressed_kv_decode_ada_b200 import synthetic

    n = max(5, args.compare_steps)
    res = {}

    def timeit(fn):
        for _ in range(3):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / n

    tokens = wl.kv_tokens
    ada_ms = timeit(lambda: spkv.decode_attention(cache, wl.q, wl.block_table, ctx, max_ctx, ws=ws,
                                                  num_splits=splits, stream=stream))
    res["ada_decode_ms"] = ada_ms
    # the step as two calls (spkv_encode_keys + spkv_decode_attention) vs the fused append
    last = (ctx - 1).to(torch.int32)
    idx = torch.as_tensor(wl.seq_off[1:] - 1, device=dev).long()
    nk, nv = wl.keys[idx].contiguous(), wl.values[idx].contiguous()

    def two_calls():
        spkv.encode_keys(cache, nk.unsqueeze(1), last, wl.block_table, values=nv.unsqueeze(1), stream=stream)
        spkv.decode_attention(cache, wl.q, wl.block_table, ctx, max_ctx, ws=ws, num_splits=splits, stream=stream)

    res["step_two_calls_ms"] = timeit(two_calls)
    res["step_fused_append_ms"] = timeit(lambda: spkv.decode_attention_append(
        cache, nk, nv, wl.q, wl.block_table, ctx, max_ctx, ws=ws, num_splits=splits, stream=stream))
    kp, vp = workload.dense_pages(wl)
    dense_ms = timeit(lambda: spkv.dense_decode(kp, vp, wl.q, wl.block_table, ctx, max_ctx, ws=ws,
                                                num_splits=splits, stream=stream))
    res["dense_decode_ms"] = dense_ms
    res["dense_tokens_per_s"] = tokens / (dense_ms * 1e-3)
    res["dense_achieved_gbs"] = synthetic.dense_step_bytes(wl) / (dense_ms * 1e-3) / 1e9
    del kp
    ks = torch.empty_like(cache.v_pages)
    dtd_ms = timeit(lambda: spkv.decompress_then_dot(cache, ks, wl.q, wl.block_table, ctx, max_ctx, ws=ws,
                                                     num_splits=splits, stream=stream))
    res["decompress_then_dot_ms"] = dtd_ms
    res["decompress_then_dot_tokens_per_s"] = tokens / (dtd_ms * 1e-3)
    res["ada_speedup_vs_dense"] = dense_ms / ada_ms
    res["ada_speedup_vs_decompress_then_dot"] = dtd_ms / ada_ms
    del ks, vp
    # bulk encode (prefill) of every context key and value
    enc_ms = timeit(lambda: workload.prefill(cache, wl))
    res["encode_ms"] = enc_ms
    res["encode_keys_per_s"] = tokens * wl.Hkv / (enc_ms * 1e-3)
    res["encode_unit"] = "(token, kv head) keys/s, with values"
    res["resident_bytes_per_token"] = {"ada": cache.resident_bytes() / tokens,
                                       "dense_bf16": 2 * wl.Hkv * 256.0}
    # f_b variants of the same batch: the exact (unquantised) unit query, and
    # the non-uniform angle quantiser at b = 4 (its own cache of the batch)
    exq_ms = timeit(lambda: spkv.decode_attention(cache, wl.q, wl.block_table, ctx, max_ctx, ws=ws,
                                                  num_splits=splits, stream=stream, exact_q=True))
    res["exact_q_decode_ms"] = exq_ms
    if len(set(int(c) for c in wl.ctx)) == 1:
        ec, mc, msn = (torch.from_numpy(np.ascontiguousarray(a)).to(dev) for a in spkv.nonuniform_tables(128, 4))
        nu = spkv.SpkvCache(wl.num_pages, wl.Hkv, np.full(wl.num_pages, 4, np.int64), wl.rad_lo, wl.rad_step,
                            device=dev, keep_mask=wl.keep_mask)
        n0 = int(wl.ctx[0])
        kv, vv = wl.keys.view(wl.B, n0, wl.Hkv, -1), wl.values.view(wl.B, n0, wl.Hkv, -1)
        zero = torch.zeros(wl.B, dtype=torch.int32, device=dev)
        nu_enc = timeit(lambda: spkv.encode_keys_nonuniform(nu, kv, zero, wl.block_table, 4, ec, values=vv,
                                                            stream=stream))
        nu_dec = timeit(lambda: spkv.decode_attention_nonuniform(nu, wl.q, wl.block_table, ctx, max_ctx, 4, ec, mc,
                                                                 msn, stream=stream))
        if nu.error_flags():
            raise RuntimeError(f"non-uniform cache: device error flags {nu.error_flags():#x}")
        res["nonuniform_b4"] = {"encode_ms": nu_enc, "encode_keys_per_s": tokens * wl.Hkv / (nu_enc * 1e-3),
                                "decode_ms": nu_dec, "decode_kv_tokens_per_s": tokens / (nu_dec * 1e-3)}
        del nu
    # the page-sharded form of the step on one GPU: two shards' partial
    # decodes (each a contiguous half of every sequence's pages) and the merge
    # of their records -- the kernels of a two-GPU step, run in sequence
    from compressed_kv_decode_ada_b200 import sharded

    shards = []
    for r in range(2):
        bt, lc = sharded.shard_batch(wl.block_table_np, wl.ctx, 2, r)
        shards.append((torch.as_tensor(bt, device=dev), torch.as_tensor(lc, device=dev), int(lc.max())))
    parts = torch.empty((2, wl.B, wl.Hq, 132), dtype=torch.float32, device=dev)

    def two_shards():
        for r, (bt, lc, mc_) in enumerate(shards):
            spkv.decode_attention_partial(cache, wl.q, bt, lc, mc_, partial=parts[r], ws=ws, stream=stream)
        spkv.merge_partials(parts, stream=stream)

    res["sharded_2_on_1gpu_ms"] = timeit(two_shards)
    # RDR controller (weights kernel + one cluster per sequence) over the
    # batch's context keys: 35% of the b = 8 bytes, sinks + last 64 protected
    ri = synthetic.make_rdr_inputs(wl, budget_frac=0.35)
    seq = torch.from_numpy(ri.seq_start).to(dev)
    qn = torch.from_numpy(ri.q_norms).to(dev)
    bud = torch.from_numpy(ri.budget).to(dev)
    prot = torch.from_numpy(ri.protect).to(dev)
    ntok = int(wl.keys.shape[0])
    rws = torch.empty(spkv.rdr_workspace_bytes(ntok), dtype=torch.uint8, device=dev)
    rdr_ms = timeit(lambda: spkv.rdr_plan(wl.keys, seq, qn, bud, protect=prot, ws=rws, stream=stream))
    res["rdr_plan_ms"] = rdr_ms
    res["rdr_plan_tokens_per_s"] = ntok / (rdr_ms * 1e-3)
    res["rdr_plan_key_bytes_gbs"] = wl.keys.numel() * 2 / (rdr_ms * 1e-3) / 1e9
    return res


def compare_workloads(args, spkv, workload, synthetic, stream, dev, peak):
    """The other full-size workloads of the method's evaluation (128K single
    sequence, the 70B shape with G = 8, the ragged mixed-tier batch with
    evictions), each in the bench's launch configuration: ADA decode and
    dense decode time, ADA achieved GB/s and its fraction of the peak, and the
    bulk encode of the workload's keys (with values)."""
    import torch

    n = max(5, args.compare_steps)

    def timeit(fn):
        for _ in range(3):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / n

    out = {}
    for name in (synthetic.LONG_128K, synthetic.SHAPE_70B, synthetic.RAGGED_RDR):
        if name == args.workload:
            continue
        wl = synthetic.make_workload(name, device=dev)
        cache = workload.build_cache(wl)
        ctx = wl.ctx_tensor()
        ws = spkv.alloc_workspace(wl.B, wl.Hq, wl.Hkv, wl.max_ctx, 0, device=dev)
        ada_ms = timeit(lambda: spkv.decode_attention(cache, wl.q, wl.block_table, ctx, wl.max_ctx, ws=ws,
                                                      stream=stream))
        gbs = synthetic.ada_step_bytes(wl) / (ada_ms * 1e-3) / 1e9
        kp, vp = workload.dense_pages(wl)
        dense_ms = timeit(lambda: spkv.dense_decode(kp, vp, wl.q, wl.block_table, ctx, wl.max_ctx, ws=ws,
                                                    stream=stream))
        del kp, vp
        enc_ms = timeit(lambda: workload.prefill(cache, wl))
        if cache.error_flags():
            raise RuntimeError(f"{name}: device error flags {cache.error_flags():#x}")
        out[name] = {"ada_decode_ms": ada_ms, "ada_achieved_gbs": gbs, "ada_frac_of_peak": gbs / peak,
                     "ada_kv_tokens_per_s": wl.kv_tokens / (ada_ms * 1e-3), "dense_decode_ms": dense_ms,
                     "ada_speedup_vs_dense": dense_ms / ada_ms, "encode_ms": enc_ms,
                     "encode_keys_per_s": wl.kv_tokens * wl.Hkv / (enc_ms * 1e-3)}
        del cache, ws, wl
        torch.cuda.empty_cache()
    return out


def decode_code_hash() -> str:
    """sha256[:16] of csrc/decode.cu with comments and blank lines removed:
    the key under which a DRAM-traffic capture stays valid (a comment edit
    does not change the kernel it describes)."""
    import re

    src = open(os.path.join(ROOT, "compressed_kv_decode_ada_b200", "csrc", "decode.cu")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    code = "\n".join(line.rstrip() for line in src.splitlines() if line.strip())
    return hashlib.sha256(code.encode()).hexdigest()[:16]


def _committed_traffic(workload):
    """ncu DRAM bytes per launch of the ADA split kernel, from the committed
    profile summary, if it was taken on the current kernel source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
    except Exception:
        return None
    ent = d.get(workload)
    if not ent or ent.get("decode_cu_code_sha256_16") != decode_code_hash():
        return None
    return ent.get("dram_bytes_per_launch")


# ------------------------------------------------------------ CPU oracle arm
def cpu_oracle(args, budget_s: float):
    """Time the fp64 oracle's decode (ADA attention from codes) on host cores
    over (sequence, kv head) groups of the same workload, one group per thread;
    the keys are encoded by the oracle beforehand (untimed).  Returns the line's
    cpu_baseline dict."""
    import torch

    import oracle

    synthetic = _synthetic_inputs()
    cfg = dict(synthetic.WORKLOADS[args.workload])
    wl = synthetic.make_workload(cfg, device="cpu", B=min(cfg["B"], 2))
    cores = _cores()
    groups = [(b, h) for b in range(wl.B) for h in range(wl.Hkv)]
    # tokens per group sized so the timed part stays within the budget
    per_tok_s = 6e-6 * wl.G / 4 + 4e-6
    T = int(min(wl.ctx.min(), max(256, budget_s * cores / max(1, len(groups)) / per_tok_s)))
    T = max(16, (T // 16) * 16)
    prepared = []
    for b, h in groups[:max(1, cores)]:
        keys = wl.keys_bits(b, h)[:T]
        bits = wl.token_bits(b)[:T]
        L, D = float(wl.rad_lo[h]), float(wl.rad_step[h])
        codes, rc = oracle.encode(keys, bits, L, D)
        prepared.append((wl.q_bits(b, h), codes, bits, rc, L, D, wl.values_bits(b, h)[:T]))
    # repeat whole passes over the sample until the budget is spent (at least one)
    passes = 0
    t0 = time.perf_counter()
    while True:
        oracle.map_groups(lambda a: oracle.ada_group(*a), prepared, threads=cores)
        passes += 1
        dt = time.perf_counter() - t0
        if dt >= budget_s:
            break
    token_heads = T * len(prepared) * passes
    value = token_heads / wl.Hkv / dt
    del torch
    return {"value": value, "unit": "KV tokens/s", "cores": min(cores, len(prepared)), "kind": "oracle",
            "sample": f"{passes} passes over {len(prepared)} (sequence, kv head) groups x {T} tokens of "
                      f"{wl.name} (G={wl.G}, b=4); KV tokens = token-heads / {wl.Hkv}; {dt:.1f} s"}


def run_rdr(args):
    """spkv_rdr_plan (weights kernel + plan kernel) over the workload's context
    keys: 35% of the b = 8 bytes, sinks + last 64 tokens protected; W warm-up
    and K timed calls, CUDA events on the launching stream."""
    import torch

    from compressed_kv_decode_ada_b200 import synthetic
    import compressed_kv_decode_ada_b200 as spkv

    dev = torch.device("cuda", 0)
    kw = {"B": args.B} if args.B else {}
    wl = synthetic.make_workload(args.workload, device=dev, **kw)
    ri = synthetic.make_rdr_inputs(wl, budget_frac=0.35)
    seq = torch.from_numpy(ri.seq_start).to(dev)
    qn = torch.from_numpy(ri.q_norms).to(dev)
    bud = torch.from_numpy(ri.budget).to(dev)
    prot = torch.from_numpy(ri.protect).to(dev)
    ntok = int(wl.keys.shape[0])
    ws = torch.empty(spkv.rdr_workspace_bytes(ntok), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        plan = spkv.rdr_plan(wl.keys, seq, qn, bud, protect=prot, ws=ws, stream=stream)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        plan = spkv.rdr_plan(wl.keys, seq, qn, bud, protect=prot, ws=ws, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / args.steps
    weights_bytes = ntok * (wl.Hkv * 256 + 1 + 8)
    return {"metric": "RDR plan: planned tokens/s", "value": ntok / (ms * 1e-3), "unit": "tokens/s",
            "ms_per_step": ms, "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
            "config": {"workload": wl.name, "B": wl.B, "num_kv_heads": wl.Hkv, "tokens": ntok, "budget_frac": 0.35,
                       "protected": "first 4 + last 64 tokens of each sequence",
                       "weights_kernel_algorithmic_bytes": weights_bytes},
            "status": plan["status"].cpu().tolist()[:8], "gpu_launches": 2 * args.steps}


def run_profile_only(args):
    """One path alone, for profiler captures: W warm-up and K calls of
    'ada' (spkv_decode_attention), 'dense' (spkv_dense_decode), 'dtd'
    (spkv_decompress_then_dot), 'encode' (spkv_encode_keys of every context
    key and value), or the non-uniform quantiser's 'nu_decode' / 'nu_encode'
    at b = 4 on the workload, so a capture can skip and count its
    launches exactly.  Prints one JSON line with the mean CUDA-event time."""
    import torch

    from compressed_kv_decode_ada_b200 import synthetic, workload
    import compressed_kv_decode_ada_b200 as spkv

    dev = torch.device("cuda", 0)
    kw = {"B": args.B} if args.B else {}
    wl = synthetic.make_workload(args.workload, device=dev, **kw)
    cache = workload.build_cache(wl)
    ctx = wl.ctx_tensor()
    max_ctx = wl.max_ctx
    stream = torch.cuda.current_stream(dev)
    ws = spkv.alloc_workspace(wl.B, wl.Hq, wl.Hkv, max_ctx, args.splits, device=dev)
    path = args.profile_only
    if path == "ada":
        fn = lambda: spkv.decode_attention(cache, wl.q, wl.block_table, ctx, max_ctx, ws=ws, num_splits=args.splits,
                                           stream=stream)
        per_call = ["split_kernel (ADA)", "merge_kernel"]
    elif path == "dense":
        kp, vp = workload.dense_pages(wl)
        fn = lambda: spkv.dense_decode(kp, vp, wl.q, wl.block_table, ctx, max_ctx, ws=ws, num_splits=args.splits,
                                       stream=stream)
        per_call = ["split_kernel (dense)", "merge_kernel"]
    elif path == "dtd":
        ks = torch.empty_like(cache.v_pages)
        fn = lambda: spkv.decompress_then_dot(cache, ks, wl.q, wl.block_table, ctx, max_ctx, ws=ws,
                                              num_splits=args.splits, stream=stream)
        per_call = ["decompress_kernel", "split_kernel (dense)", "merge_kernel"]
    elif path in ("nu_decode", "nu_encode"):
        # the non-uniform quantiser at b = 4: its own cache of the workload
        ec, mc, msn = (torch.from_numpy(np.ascontiguousarray(a)).to(dev) for a in spkv.nonuniform_tables(128, 4))
        cache = spkv.SpkvCache(wl.num_pages, wl.Hkv, np.full(wl.num_pages, 4, np.int64), wl.rad_lo, wl.rad_step,
                               device=dev, keep_mask=wl.keep_mask)
        n0 = int(wl.ctx[0])
        if len(set(int(c) for c in wl.ctx)) != 1:
            raise SystemExit("--profile-only nu_*: a workload with equal context lengths")
        kv, vv = wl.keys.view(wl.B, n0, wl.Hkv, -1), wl.values.view(wl.B, n0, wl.Hkv, -1)
        zero = torch.zeros(wl.B, dtype=torch.int32, device=dev)
        enc = lambda: spkv.encode_keys_nonuniform(cache, kv, zero, wl.block_table, 4, ec, values=vv, stream=stream)
        enc()
        if path == "nu_encode":
            fn = enc
            per_call = ["encode_kernel (non-uniform)"]
        else:
            fn = lambda: spkv.decode_attention_nonuniform(cache, wl.q, wl.block_table, ctx, max_ctx, 4, ec, mc, msn,
                                                          stream=stream)
            per_call = ["nu_table_kernel", "nu_decode_kernel", "merge_partials_kernel"]
    else:
        fn = lambda: workload.prefill(cache, wl)
        per_call = ["encode_kernel"]
    torch.cuda.synchronize(dev)
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / args.steps
    return {"profile_only": path, "workload": wl.name, "B": wl.B, "ms_per_call": ms, "calls": args.warmup + args.steps,
            "launches_per_call": per_call, "kv_tokens": wl.kv_tokens, "err_flags": cache.error_flags()}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="spkv", choices=["spkv", "reference"])
    ap.add_argument("--workload", default="llama3_8b_b8_h32x8_t32768_b4",
                    help="one of compressed_kv_decode_ada_b200.synthetic.WORKLOADS")
    ap.add_argument("--splits", type=int, default=0)
    ap.add_argument("--B", type=int, default=0, help="override the batch size (profiler captures)")
    ap.add_argument("--e2e-steps", type=int, default=500)
    ap.add_argument("--compare", type=int, default=1)
    ap.add_argument("--compare-steps", type=int, default=50)
    ap.add_argument("--compare-workloads", type=int, default=1,
                    help="also time the other full-size workloads (128K, 70B shape, ragged mixed tiers)")
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-only", choices=["ada", "dense", "dtd", "encode", "nu_decode", "nu_encode"],
                    default=None,
                    help="run one path alone, --warmup + --steps calls (one JSON line; profiler captures)")
    ap.add_argument("--rdr", action="store_true",
                    help="time only spkv_rdr_plan on the workload's keys (one JSON line; profiler captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank, world, local = _dist()

    if args.impl == "reference":
        if rank != 0:
            return 0
        cb = cpu_oracle(args, args.cpu_budget)
        line = {"metric": "ADA decode KV tokens/s on 1 B200; achieved HBM GB/s as % of peak", "impl": "reference",
                "value": cb["value"], "unit": "KV tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": args.workload}, "cpu_baseline": cb,
                "e2e": {"value": cb["value"], "unit": "KV tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0

    if args.rdr:
        if rank == 0:
            print(json.dumps(run_rdr(args)), flush=True)
        return 0

    if args.profile_only:
        if rank == 0:
            print(json.dumps(run_profile_only(args)), flush=True)
        return 0

    res = run_spkv(args, rank, world, local)
    if rank == 0:
        if not args.no_cpu_baseline and world == 1:
            res["cpu_baseline"] = cpu_oracle(args, args.cpu_budget)
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
