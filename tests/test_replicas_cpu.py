"""The N > 1 host path on CPU: two gloo ranks (world size 2) through the same Replicas plumbing
that bench.py uses over NCCL, and the reference arm of bench.py under torchrun."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

from hybrid_softmax_linear_chunked_b200.replicas import Replicas, job_throughput

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    rep = Replicas.from_env("gloo", timeout_s=30)
    res = {"rank": rep.rank, "world": rep.world, "distributed": rep.distributed,
           "seed": rep.seed(7)}
    rep.barrier()
    # the slowest rank's time is the job's time
    res["max"] = rep.max(10.0 + 5.0 * rank)
    res["all"] = rep.all_values(100.0 + rank)
    res["value"] = job_throughput(32760, rep.world, res["max"])
    rep.close()
    out_q.put(res)


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted((q.get(timeout=5) for _ in procs), key=lambda r: r["rank"])
    assert [r["rank"] for r in res] == [0, 1]
    assert all(r["world"] == 2 and r["distributed"] for r in res)
    assert res[0]["seed"] != res[1]["seed"]          # each replica draws its own batch
    assert all(r["max"] == 15.0 for r in res)        # every rank sees the same max
    assert all(r["all"] == [100.0, 101.0] for r in res)
    # two replicas of 32760 tokens each, slowest rank 15 ms per step
    assert all(abs(r["value"] - 2 * 32760 / 0.015) < 1e-6 for r in res)


def test_single_process_needs_no_group(monkeypatch):
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    rep = Replicas.from_env("gloo")
    assert not rep.distributed and rep.world == 1
    assert rep.max(3.5) == 3.5 and rep.all_values(2.0) == [2.0]
    rep.close()


def test_reference_arm_under_torchrun():
    """Rank 0 alone runs and prints the reference line; the other rank exits 0 without work."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "2",
           "--warmup", "1"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["steps"] == 2
    assert line["value"] > 0 and line["higher_is_better"] is True
    assert line["e2e"]["value"] == line["value"]
    assert line["cpu_baseline"]["kind"] == "oracle"
