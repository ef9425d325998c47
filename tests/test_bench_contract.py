"""bench.py's host-side contract, checked on CPU.

The JSON line's fixed parts (launch count, config keys, the reference arm's
line) and the DRAM-traffic figure that the roofline object takes from
profiles/traffic.json, which must belong to the kernel sources it was
measured on.
"""
import json
import os
import subprocess
import sys

import pytest

import bench
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_launch_count_per_step():
    # per k-means call: split + |x|^2 + 4 per round; per permute: hist, scan, scatter, gather;
    # select; two planning kernels + attention (un-permute fused)
    assert bench.kernel_launches_per_step(5) == 2 * (1 + 4 * 5) + 2 * 4 + 1 + 4 == 55
    assert bench.kernel_launches_per_step(2) == 2 * (1 + 4 * 2) + 13
    assert bench.kernel_launches_per_step(5, qk_fp8=True) == 55 - 1 + 4 == 58
    assert bench.kernel_launches_per_step(5, kv_gather=True) == 54
    assert bench.dynrad_launches_per_step("static") == 6 and bench.dynrad_launches_per_step("dynamic") == 7


def test_workload_config_keys():
    cfg = bench.workload_config(synth.WORKLOADS["480p-5s"], 1)
    for key in ("workload", "heads", "tokens", "head_dim", "cq", "ck", "kmeans_iters", "top_p", "l2"):
        assert key in cfg
    assert cfg["tokens"] == 32760 and cfg["heads"] == 40
    assert "warm_start" not in cfg
    warm = bench.workload_config(synth.WORKLOADS["480p-10s"], 1, iters=2)
    assert warm["kmeans_iters"] == 2 and "warm_start" in warm


@pytest.mark.parametrize("kernel,floor", [("kmeans_assign_tc_kernel", 335e6),   # one read of x (40 heads)
                                           ("sparse_attn_kernel", 1.0e9)])       # Q, K, V read + O written
def test_committed_traffic_belongs_to_the_kernel_sources(kernel, floor):
    """A committed DRAM figure is used only while the kernel's sources match the
    capture; then it must be at least the compulsory traffic.  A stale one reads as null."""
    got = bench.load_traffic(kernel, "480p-5s")
    assert got is None or (isinstance(got, int) and got > floor)
    assert bench.load_traffic(kernel, "no-such-workload") is None


def test_warmup_below_three_is_refused():
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "2"])


def test_reference_arm_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny", "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads([l for l in out.stdout.splitlines() if l.startswith("{")][-1])
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == bench.UNIT
    assert line["value"] > 0 and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
