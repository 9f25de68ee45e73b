"""Host-side logic of the multi-process benchmark, on CPU with the gloo
backend and world size 2 (one process per GPU on a B200 machine, NCCL there):
the max-over-ranks timing, the per-rank inputs, the whole-job value, and the
reference arm's rank-0-only rule."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from vla_flow_matching_denoise_b200 import synth  # noqa: E402

torch = pytest.importorskip("torch")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, ws, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(ws), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    w, r, local, pg = bench.dist_setup(ws, backend="gloo")
    t = bench.max_over_ranks(10.0 + 5.0 * r, pg, "cpu")     # rank 1 is the slow one
    kp, vp, x0 = bench.rank_inputs(synth.WORKLOADS["tiny"], r)
    q.put((r, w, t, float(x0.sum()), int(kp[0].astype(np.int64).sum())))
    pg.barrier()
    pg.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_own_inputs():
    mp = torch.multiprocessing.get_context("spawn")
    q = mp.Queue()
    port = _free_port()
    ps = [mp.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, w0, t0, x0s, k0s), (r1, w1, t1, x1s, k1s) = res
    assert (r0, r1, w0, w1) == (0, 1, 2, 2)
    assert t0 == t1 == 15.0                     # both ranks see the slowest time
    assert x0s != x1s and k0s != k1s            # each rank has its own requests


def test_job_value_counts_every_rank():
    # 2 ranks x 64 requests x 10 Euler steps x 3 calls in 300 ms
    assert bench.job_value(2, 64, 10, 3, 300.0) == pytest.approx(2 * 64 * 10 * 3 / 0.3)
    assert bench.max_over_ranks(4.0, None, "cpu") == 4.0


def _run_bench(env_extra, *args):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], env=env, cwd=ROOT,
                          capture_output=True, text=True, timeout=600)


def test_reference_arm_other_ranks_exit_quietly():
    r = _run_bench({"RANK": "1", "WORLD_SIZE": "2"}, "--impl", "reference", "--workload", "tiny",
                   "--steps", "1", "--warmup", "0")
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_rank0_prints_one_line():
    r = _run_bench({"RANK": "0", "WORLD_SIZE": "1"}, "--impl", "reference", "--workload", "tiny",
                   "--steps", "1", "--warmup", "0")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0
