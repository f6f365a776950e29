"""Multi-process host logic on CPU: world size 2 over gloo.

The GPU path runs one replica per rank (sequences and kv groups share
nothing), so what needs covering without GPUs is the plumbing: joining the
group, the barrier, the max over ranks that times a step, the whole-job
rate, a rank that fails before a collective (the other gets an error within
the group's timeout instead of hanging), and the launcher path of bench.py's
reference arm (rank 0 alone prints; the other rank exits 0).
"""
import json
import os
import socket
import subprocess
import sys
import time

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank: int, world: int, port: int) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))


def _rank_collectives(rank, world, port, q):
    _env(rank, world, port)
    sys.path.insert(0, ROOT)
    from gated_block_sparse_b200 import dist as D
    w, r, _ = D.setup(backend="gloo", timeout_s=30)
    D.barrier(w)
    m = D.max_over_ranks(w, 1.5 + r)  # rank 1 is "slower"
    rate = D.whole_job_rate(1000.0, w, m)
    D.barrier(w)
    D.teardown(w)
    q.put((r, w, m, rate))


def test_two_rank_barrier_and_max_over_ranks():
    port, world = _free_port(), 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_collectives, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for r, (rr, w, m, rate) in enumerate(got):
        assert (rr, w) == (r, world)
        assert m == 2.5  # the max over ranks, seen by every rank
        assert abs(rate - 1000.0 * 2 / 2.5e-3) < 1e-6  # units of all ranks / slowest time


def _rank_fails_before_barrier(rank, world, port, q):
    _env(rank, world, port)
    sys.path.insert(0, ROOT)
    from gated_block_sparse_b200 import dist as D
    w, r, _ = D.setup(backend="gloo", timeout_s=5)
    D.barrier(w)  # both ranks are in
    if r == 1:
        os._exit(3)  # dies between steps, no collective in flight
    t0 = time.time()
    try:
        D.barrier(w)
        q.put(("no error", time.time() - t0))
    except Exception as e:  # noqa: BLE001 -- any collective error counts
        q.put((type(e).__name__, time.time() - t0))


def test_rank_that_dies_turns_the_next_collective_into_an_error():
    port, world = _free_port(), 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_fails_before_barrier, args=(r, world, port, q))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert procs[1].exitcode == 3
    kind, waited = q.get(timeout=10)
    assert kind != "no error"
    assert waited < 60  # bounded by the group's timeout, not a hang


def test_reference_arm_under_the_launcher_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--config", "c1", "--steps", "2", "--warmup", "3",
           "--cpu-seconds", "0.2"]
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0
