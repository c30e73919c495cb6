"""bench.py's host-side legs on CPU: the oracle pool used for the
multi-core CPU baseline starts, runs the serving step's layers and cleans
up its shared memory."""
from __future__ import annotations

import bench
import workloads as W


def test_cpu_baseline_parallel_runs_and_reports_its_cores():
    c = bench.CFG
    idx_h = W.routed_indices("dsv3_prefill", device="cpu", T=256).numpy()
    hist_h = W.histogram_steps(15, c.L, c.E, 256 * c.K, c.stream).numpy()
    r = bench.cpu_baseline_parallel(idx_h, hist_h, 0.5)
    assert "unavailable" not in r, r
    assert r["value"] > 0 and 1 <= r["cores"] <= c.L and r["kind"] == "oracle"
