"""Multi-rank host logic of bench.py on CPU: two gloo ranks (127.0.0.1).

The decode shards by sequence: each rank decodes its own batch with no
exchange on the data path; the only collective is the max over ranks of the
step timings, and the reported value is all ranks' tokens over the slowest
rank's time."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import sys

    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        r, w, lr = bench._dist()
        ms = [1.0 + rank, 5.0 - rank]                # rank 0: [1, 5], rank 1: [2, 4]
        mx = bench.max_over_ranks(ms)
        cfg = bench.rank_workload("llama3_8b_b8_h32x8_t32768_b4", rank)
        q.put((r, w, lr, mx, cfg["seed"], bench.whole_job_rate(1000.0, w, mx[0])))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_decode_independent_batches():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, w0, l0, mx0, seed0, v0), (r1, w1, l1, mx1, seed1, v1) = res
    assert (r0, r1) == (0, 1) and w0 == w1 == 2 and (l0, l1) == (0, 1)
    assert mx0 == mx1 == [2.0, 5.0]          # element-wise max over ranks
    assert seed0 != seed1                     # independent batches per rank
    assert v0 == v1 == pytest.approx(1000.0 * 2 / 2e-3)


def test_single_process_needs_no_collective():
    import sys

    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks([3.0, 1.0]) == [3.0, 1.0]
    assert bench.whole_job_rate(10.0, 1, 1.0) == pytest.approx(1e4)


def test_reference_arm_maps_only_the_oracle_library():
    """bench.py --impl reference times the oracle alone: the process that runs
    it loads the input generators but neither the package nor libspkv.so."""
    import subprocess
    import sys

    code = (
        "import sys, types, bench\n"
        "args = types.SimpleNamespace(workload='llama3_8b_b8_h32x8_t32768_b4')\n"
        "cb = bench.cpu_oracle(args, 0.01)\n"
        "maps = open('/proc/self/maps').read()\n"
        "print(cb['kind'], cb['value'] > 0, 'compressed_kv_decode_ada_b200' in sys.modules,\n"
        "      'libspkv.so' in maps, 'libspkv_oracle.so' in maps)\n")
    out = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    assert out.stdout.split() == ["oracle", "True", "False", "False", "True"]
