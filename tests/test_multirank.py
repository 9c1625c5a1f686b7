"""The N > 1 path of bench.py on CPU: gloo ranks, max-over-ranks timing, weak-scaling workloads
and the reference arm under torchrun (rank 0 alone prints its line)."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    got = bench.max_over_ranks(10.0 + 5.0 * rank, torch.device("cpu"))
    w = bench.rank_workload("toy", rank, {})
    q.put((rank, got, w.seed, w.T, w.n_kv))
    dist.barrier()
    dist.destroy_process_group()


def _e2e_rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    dev = torch.device("cpu")
    ok = bench.e2e_over_ranks(100.0 + rank, None, dev)                       # both legs worked
    one_failed = bench.e2e_over_ranks(None if rank == 1 else 50.0,
                                      "out of pinned memory" if rank == 1 else None, dev)
    q.put((rank, ok, one_failed))
    dist.barrier()
    dist.destroy_process_group()


def test_e2e_leg_reduces_over_ranks_even_when_one_fails():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_e2e_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [(101.0, None), (101.0, None)]  # the slowest rank's time
    assert res[0][2] == (None, "the end-to-end leg failed on another rank")
    assert res[1][2] == (None, "out of pinned memory")


def test_max_over_ranks_and_weak_scaling_workloads():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [15.0, 15.0]        # both ranks see the slowest rank's time
    assert res[0][2] != res[1][2]                     # own sequences per rank
    assert res[0][3:] == res[1][3:]                   # same shape


def test_reference_arm_under_torchrun_prints_one_line():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0", "--workload", "toy",
           "--cpu-tokens", "64"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
