"""The multi-rank plumbing of bench.py on CPU: two gloo ranks reduce their timings to
the slowest rank's, the whole-job rate counts every rank's work, and the reference arm
launched with torchrun prints exactly one line from rank 0 while rank 1 exits at once.
(The GPU arm's collectives are the same calls on an NCCL group.)"""

import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r took (10 + r) ms per step and (3 - r) ms in the kernel
        got = bench.max_over_ranks([10.0 + rank, 3.0 - rank], world, "cpu", dist)
        dist.barrier()
        out_q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # element-wise max over ranks, identical on both ranks
    assert res[0] == res[1] == [11.0, 3.0]


def test_single_rank_is_identity():
    assert bench.max_over_ranks([1.5, 2.5], 1, "cpu") == [1.5, 2.5]


def test_whole_job_rate_counts_every_rank():
    # 4 ranks, each 2e12 FLOPs, slowest 10 ms -> 8e12 FLOP in 10 ms
    assert bench.whole_job_rate(4, 2e12, 10.0) == pytest.approx(8e14)
    assert bench.whole_job_rate(1, 2e12, 10.0) == pytest.approx(2e14)


def test_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--workload", "tiny", "--steps", "1", "--warmup", "3"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
