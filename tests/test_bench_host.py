"""Host-side logic of bench.py: the multi-rank timing reduction (gloo, two
processes on the CPU), the job-value arithmetic, rank gating of the CPU
reference arm, and the JSON line of the reference arm."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks(1.5 + rank)
        bench.barrier()
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    assert res == {0: 2.5, 1: 2.5}


def test_max_over_ranks_single_process():
    assert bench.max_over_ranks(3.25) == 3.25


def test_job_value():
    # 2 ranks x 10 steps x 1e12 flop in 4 s (slowest rank) -> 5 TFLOP/s
    assert bench.job_value(1e12, 2, 10, 4.0) == pytest.approx(5.0)


def test_reference_arm_other_ranks_do_no_work():
    class A:
        steps, warmup = 1, 0
    assert bench.run_reference(A(), bench.MlpWorkload(), rank=1, world=2) is None


def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    line = [ln for ln in r.stdout.splitlines() if ln.startswith("{")][-1]
    d = json.loads(line)
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["metric"] == bench.METRIC


def test_context_row_only_on_the_headline_pair():
    # The torch / cuBLAS context row is built from the MLP pair's weights: every
    # other workload (all subclasses of it) must skip it.
    import bench
    assert [k for k, W in bench.WORKLOADS.items() if bench.has_context_row(W())] == ["flux_mlp"]
