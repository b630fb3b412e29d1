"""Host-side helpers of bench.py that need no GPU: the captured DRAM traffic
it reports beside the roofline is tied to the sources of the kernel it was
captured on."""
import copy
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_traffic_reported_for_the_captured_kernels_only():
    for config in bench.TRAFFIC:
        assert bench.measured_traffic(config, None) == bench.TRAFFIC[config]["bytes"], config
        # another token count is another workload: not the captured launch
        assert bench.measured_traffic(config, 4) is None
    assert bench.measured_traffic(2, None) is None  # never captured


def test_traffic_void_once_the_kernel_sources_change(monkeypatch):
    table = copy.deepcopy(bench.TRAFFIC)
    for t in table.values():
        t["sha"] = "0" * 16  # as if the sources had changed since the capture
    monkeypatch.setattr(bench, "TRAFFIC", table)
    for config in table:
        assert bench.measured_traffic(config, None) is None


def test_traffic_close_to_the_algorithmic_bytes():
    # the decode captures read each weight byte about once (a figure far above
    # the algorithmic bytes would mean re-reads the bench should not hide)
    qwen = [(1536, 1536), (1536, 256), (1536, 256), (1536, 1536), (1536, 8960), (1536, 8960), (8960, 1536)]
    weights = sum(di * do // 2 + 4 * do * di // 128 for di, do in qwen)
    for config in (1, 4):
        assert 0.95 < bench.TRAFFIC[config]["bytes"] / weights < 1.05, config
