"""bench.py's output contract, checked on the CPU: the reference arm (the fp64 oracle timed on
the host) prints one JSON line with the keys the driver reads, and the GPU arm's helpers are
consistent. The GPU arm itself is run on the GPU machine."""
import json
import subprocess
import sys

import pytest

import bench


@pytest.mark.timeout(300)
def test_reference_arm_prints_one_contract_line():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "c1",
                          "--steps", "1", "--warmup", "3", "--cpu-threads", "2"],
                         capture_output=True, text=True, timeout=280, check=True)
    lines = [ln for ln in out.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["value"] > 0 and d["steps"] == 1 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["higher_is_better"] is True and d["vs_baseline"] is None
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] == 2
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert "workload" in d["config"]
    # the same config dict as the GPU arm on the same arguments
    from paged_kv_long_b200.inputs import WORKLOADS
    args = bench.main.__globals__["argparse"].Namespace(layout="paged", policy="makespan",
                                                          splits=None,
                                                          l2_flush_mb=bench.L2_FLUSH_BYTES >> 20)
    assert d["config"] == bench.bench_config(WORKLOADS["c1"], args, 1)
    # ms_per_step is the measured wall time of one sampled step, so the steps add up to the
    # timed seconds the line reports
    assert abs(d["ms_per_step"] * d["steps"] / 1e3 - d["timed_seconds"]) <= 0.5 * d["timed_seconds"]
    assert d["cpu_baseline"]["cpu_model"]


def test_warmup_below_three_is_refused():
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "2"])


def test_traffic_capture_is_keyed_to_the_kernel_sources():
    h = bench.kernel_sources_hash()
    assert len(h) == 16 and int(h, 16) >= 0
    cap = bench.TRAFFIC_CAPTURE
    assert cap is None or set(cap) == {"workload", "sources", "bytes_per_launch", "how"}


def test_roofline_peak_follows_the_timed_window_clocks():
    """Burst peak at full clock; sustained only when the timed steps ran power-capped (median SM
    clock below 95 % of max with sw_power_cap); burst when the clock record is missing."""
    peaks = {"bf16_tflops": 1642.9, "bf16_tflops_sustained": 1392.3}
    capped = {"sm_mhz": 1507, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    assert bench.roofline_peak(capped, peaks) == (1392.3, True)
    full = {"sm_mhz": 1965, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    assert bench.roofline_peak(full, peaks) == (1642.9, False)
    low_no_reason = {"sm_mhz": 1500, "sm_max_mhz": 1965.0, "reasons": []}
    assert bench.roofline_peak(low_no_reason, peaks) == (1642.9, False)
    missing = {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
    assert bench.roofline_peak(missing, peaks) == (1642.9, False)
