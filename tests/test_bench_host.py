"""Host-side measurement logic of bench.py, without a GPU: the choice of the tensor
peak from the recorded clocks, and the hash check that voids stale DRAM-traffic
entries."""

import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402

PEAKS = {"hbm_gbs": 6538.3, "bf16_tflops": 1662.5, "bf16_tflops_sustained": 1359.4}


def test_tensor_peak_follows_the_clocks():
    full = {"sm_mhz": 1965.0, "sm_max_mhz": 1965, "reasons": []}
    capped = {"sm_mhz": 1507.0, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"]}
    low = {"sm_mhz": 1700.0, "sm_max_mhz": 1965, "reasons": []}  # below 95 % of max, no reason given
    assert bench.tensor_peak(PEAKS, full) == (1662.5, "burst")
    assert bench.tensor_peak(PEAKS, capped) == (1359.4, "sustained")
    assert bench.tensor_peak(PEAKS, low) == (1359.4, "sustained")
    # no clock record: the larger (burst) figure, so a fraction is never inflated by it
    assert bench.tensor_peak(PEAKS, {"sm_mhz": None, "sm_max_mhz": None, "reasons": []}) == (1662.5, "burst")
    # a peaks file without a sustained figure
    assert bench.tensor_peak({"bf16_tflops": 1590.0}, capped) == (1590.0, "burst")


def test_traffic_entries_are_keyed_by_source_hash():
    with open(os.path.join(ROOT, "profiles", "gemm_traffic.json")) as f:
        table = json.load(f)
    for kernel, entry in table.items():
        assert kernel in bench.GEMM_SOURCES
        current = bench.gemm_kernel_hash(kernel) == entry["kernel_sha256_16"]
        for workload, nbytes in entry["bytes_per_launch_by_workload"].items():
            assert bench.gemm_traffic(kernel, workload) == (nbytes if current else None)
    # the dense default path's kernel has counters for the fused-QKV workload
    assert bench.gemm_traffic("gemm_bf16_pair_kernel", "c1") is not None


def test_reference_arm_reports_the_workloads_config(monkeypatch):
    """The reference arm times a bounded token sample of the workload, but its line
    carries the workload's own config, the one our arm reports (token counts included);
    the sample is described under cpu_baseline.  (The oracle step is replaced by a fixed
    time here: only the reporting is under test.)"""
    import argparse
    monkeypatch.setattr(bench, "oracle_linear_step", lambda case, tokens, backward: 100.0)
    args = argparse.Namespace(workload="c1", steps=1, warmup=3, moe="chunked", moe_backward=False,
                              moe_layer=False, weight_side=False)
    line = bench.run_reference(args, 0, 1)
    spec = bench.linear_spec("c1")
    assert line["impl"] == "reference"
    assert line["config"] == bench.workload_config("c1", spec.M, 1, spec.backward, args)
    assert line["config"]["tokens_per_gpu"] == spec.M
    assert str(spec.M) in line["cpu_baseline"]["sample"]
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
