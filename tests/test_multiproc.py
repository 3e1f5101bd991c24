"""Host logic of the N-GPU benchmark on CPU: two `gloo` ranks.

The block shards as independent replicas (no data-path collective); the only
multi-rank steps are the barrier, the max-over-ranks time and the whole-job
throughput, and the reference arm printing from rank 0 alone.
"""

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
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(ws), LOCAL_RANK=str(rank))
    w, r, local = bench.dist_env()
    dist.init_process_group("gloo", rank=r, world_size=w,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        ms = 10.0 + 5.0 * r                      # rank 1 is the slow one
        m = bench.max_over_ranks(ms, torch.device("cpu"))
        dist.barrier()
        out.put((r, w, local, m, bench.job_tokens_per_s(8192, 4, w, 4 * m)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [x[:3] for x in res] == [(0, 2, 0), (1, 2, 1)]
    for _, _, _, m, tps in res:
        assert m == 15.0                         # every rank sees the max
        assert tps == pytest.approx(2 * 8192 * 4 / (4 * 15.0 / 1e3))


def test_single_rank_is_identity():
    assert bench.max_over_ranks(3.25, torch.device("cpu")) == 3.25
    assert bench.job_tokens_per_s(100, 10, 1, 1000.0) == pytest.approx(1000.0)


def test_reference_arm_prints_from_rank_zero_only():
    """torchrun with two CPU ranks: one JSON line, from rank 0."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "tiny",
           "--gpus", "2", "--steps", "1", "--warmup", "3", "--cpu-sample-tokens", "16"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT, env=env)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0
