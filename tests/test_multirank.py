"""Multi-process host logic of the benchmark, on CPU with the gloo backend.

The GEMM shards into independent replicas, so the only cross-rank steps are
the barrier and the max-over-ranks of the step time; these run here with two
gloo ranks.  The reference arm must print exactly one line, from rank 0.
"""
import json
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, values, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dist.barrier()
        m = bench.max_over_ranks(values[rank], world, dist)
        out.put((rank, m, bench.job_value(10 ** 12, world, m)))
    finally:
        dist.destroy_process_group()


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_max_over_ranks_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    values = [1.25, 3.5]
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, values, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert [g[1] for g in got] == [3.5, 3.5]
    # two ranks of 1 TFLOP each in 3.5 ms -> 2 TFLOP / 3.5 ms
    assert got[0][2] == pytest.approx(2 / 3.5e-3, rel=1e-12)


def test_single_rank_max_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(2.5, 1) == 2.5
    assert bench.job_value(2 * 10 ** 12, 1, 1.0) == pytest.approx(2000.0)


def _run_bench(env_extra, args):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], env=env,
                          capture_output=True, text=True, timeout=600)


def test_reference_arm_prints_one_line_on_rank0_only():
    args = ["--impl", "reference", "--workload", "gemm_256", "--steps", "3", "--warmup", "3"]
    r1 = _run_bench({"RANK": "1", "WORLD_SIZE": "2"}, args + ["--gpus", "2"])
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    r0 = _run_bench({"RANK": "0", "WORLD_SIZE": "1"}, args)
    assert r0.returncode == 0
    lines = [l for l in r0.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e", "impl"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["config"]["workload"] == "gemm_256"
