"""bench.py's reference arm (the float64 oracle on the host cores) prints one JSON line with
the keys of the benchmark contract, on the same metric, unit and workload as the GPU arm.
CPU only."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "2", "--warmup", "3"], capture_output=True, text=True,
                       timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    import bench
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["higher_is_better"] is True and d["steps"] == 2 and d["warmup"] == 3
    assert d["value"] > 0 and d["config"]["workload"] == bench.WORKLOAD
    # the very config dict the GPU arm reports (same keys, same values)
    import synth
    assert d["config"] == bench.decode_config(synth.WORKLOADS[bench.WORKLOAD], 1)
    # a short run decodes the whole batch every step
    assert d["sequences_per_step"] == synth.WORKLOADS[bench.WORKLOAD].batch
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
