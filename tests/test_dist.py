"""Host-side multi-process logic of the bench (replicas only), on CPU with
the gloo backend at world size 2: the max-over-ranks step time, the
whole-job throughput, the barrier, and the reference arm running on rank 0
only."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r = bench.init_dist("gloo")
    assert (w, r) == (world, rank)
    bench.barrier()
    local_ms = 2.0 + rank              # rank 1 is the slow one
    ms, value = bench.job_rate(w, 100, local_ms)
    q.put((rank, ms, value))
    bench.barrier()
    dist.destroy_process_group()


def test_job_rate_is_max_over_ranks_and_counts_all_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    got = sorted(q.get(timeout=5) for _ in range(world))
    for _, ms, value in got:
        assert ms == 3.0                              # the slowest rank's time on every rank
        assert value == pytest.approx(2 * 100 / 3e-3)  # tokens of both ranks over it


def test_single_process_job_rate_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    ms, value = bench.job_rate(1, 256, 0.5)
    assert ms == 0.5 and value == pytest.approx(512000.0)


def _run_reference(env_extra):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config",
                           "tiny", "--steps", "2", "--warmup", "3"], capture_output=True, text=True, env=env,
                          timeout=300, cwd=ROOT)


def test_reference_arm_prints_one_line_on_rank0_and_nothing_elsewhere():
    r0 = _run_reference({"RANK": "0", "WORLD_SIZE": "1"})
    assert r0.returncode == 0, r0.stderr
    lines = [ln for ln in r0.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["value"] > 0 and rec["cpu_baseline"]["kind"] == "oracle"
    assert rec["e2e"]["h2d_bytes_per_step"] == 0
    r1 = _run_reference({"RANK": "1", "WORLD_SIZE": "2"})
    assert r1.returncode == 0, r1.stderr
    assert r1.stdout.strip() == ""
