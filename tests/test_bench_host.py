"""Host helpers of bench.py, checked without a GPU: the DRAM-traffic figure
is reported only for the kernel it was captured on (device code plus launch
configuration), the row samples of the CPU baseline are evenly spaced and
bounded, and the job value is whole-job throughput."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from tensor_core_gemm_fp16_b200 import binding  # noqa: E402


def test_traffic_is_keyed_to_the_captured_kernel():
    cfg = binding.tg_gemm_select_config(8192, 8192, 8192, 2)
    with open(os.path.join(ROOT, "profiles", "gemm_persistent_kernel_fused_8192.md")) as f:
        text = f.read()
    current = f"source_hash: {bench.kernel_source_hash(cfg)}" in text
    traffic = bench.profiled_traffic("fused_8192", cfg)
    if current:
        # one launch moves at least the algorithmic bytes
        assert traffic is not None and traffic >= 402_669_568
    else:
        assert traffic is None
    other = dict(cfg, id=cfg["id"] + 1)
    assert bench.profiled_traffic("fused_8192", other) is None
    assert bench.profiled_traffic("no_such_workload", cfg) is None
    assert bench.workload_kernel_hash("fused_8192") == bench.kernel_source_hash(cfg)


def test_evenly_spaced_rows():
    rows = bench.evenly_spaced(8192, 985)
    assert len(rows) == 985 and rows[0] == 0 and rows[-1] < 8192
    assert rows == sorted(set(rows))
    assert bench.evenly_spaced(10, 20) == list(range(10))


def test_job_value_is_whole_job_throughput():
    # 1e12 flop per rank-step, 2 ranks, 1 ms per step: 2000 TFLOP/s
    assert abs(bench.job_value(10 ** 12, 2, 1.0) - 2000.0) < 1e-9
