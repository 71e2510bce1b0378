"""The N > 1 host path of bench.py on CPU: two gloo ranks (no GPU). Every
rank decodes its own replica, so the only cross-rank steps are the barrier
and the max-over-ranks time; the reference arm runs on rank 0 alone."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, port, q):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE="2", MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    world, r, local, pg = bench.init_ranks(None, backend="gloo")
    cpu = torch.device("cpu")
    ms = bench.max_over_ranks(pg, 1.5 + 2.0 * rank, cpu)      # rank 1 is the slow one
    pg.barrier()
    value = bench.job_tflops(world, 2e12, ms)
    pg.destroy_process_group()
    q.put((r, world, local, ms, value))


def test_two_gloo_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=180) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [g[0] for g in got] == [0, 1] and all(g[1] == 2 and g[2] == g[0] for g in got)
    assert all(g[3] == 3.5 for g in got)                                  # max over ranks
    assert all(abs(g[4] - 2 * 2e12 / 3.5e-3 / 1e12) < 1e-9 for g in got)  # whole-job throughput


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        os.environ.pop(k, None)
    world, rank, local, pg = bench.init_ranks(None, backend="gloo")
    assert (world, rank, local, pg) == (1, 0, 0, None)
    assert bench.max_over_ranks(None, 4.25, torch.device("cpu")) == 4.25


@pytest.mark.timeout(600)
def test_reference_arm_under_torchrun_prints_one_line_from_rank_0():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--workload", "tiny", "--steps", "2", "--warmup", "3"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["steps"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
