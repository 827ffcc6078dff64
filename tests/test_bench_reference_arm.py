"""bench.py --impl reference (the oracle timed on host cores) prints one JSON
line with the contract's keys and the GPU arm's workload config; no GPU needed."""

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--cpu-seconds", "0.4"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads([l for l in r.stdout.splitlines() if l.startswith("{")][-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "GB/s"
    assert line["higher_is_better"] is True and line["metric"].startswith("quantized-KV decode attention")
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    cfg = line["config"]
    # the default workload is the largest: the long-context ragged stack (bf16 layers 0 and 31, K8V8 between)
    assert cfg["workload"] == "ragged_long" and cfg["batch"] == 4 and cfg["layers"] == 32
    assert cfg["layer_map_equiv_bits"] == 8.5 and 8192 <= cfg["context_min"] <= cfg["context"] <= 32768
    assert line["ms_per_step"] > 0
