"""Host-side parts of bench.py that need no GPU: the reference arm (the oracle
timed on the host cores) prints one JSON line with the contract's keys, and the
DRAM-traffic records are reported only for unchanged kernel sources."""
import json
import os
import subprocess
import sys

from conftest import ROOT


def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
                        "--warmup", "3"], cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["n_gpus"] == 1 and d["steps"] == 2 and d["warmup"] == 3
    assert d["value"] > 0 and d["higher_is_better"] is True and d["vs_baseline"] is None
    assert "workload" in d["config"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_traffic_records_follow_the_kernel_source():
    sys.path.insert(0, ROOT)
    import bench
    src = "ternary_neural_net_b200/csrc/binary_gemm_tc.cu"
    digest = bench.hashlib.sha256(open(os.path.join(ROOT, src), "rb").read()).hexdigest()[:16]
    recorded = {}
    for line in open(os.path.join(ROOT, "profiles", "traffic.txt")):
        f = line.split()
        if len(f) >= 3 and not line.startswith("#"):
            recorded[f[0]] = (float(f[1]), f[2])
    want = recorded["binary_gemm_tc_128x2"]
    got = bench.traffic_for("binary_gemm_tc_128x2", src)
    assert got == (want[0] if want[1] == digest else None)
    assert bench.traffic_for("no_such_kernel", src) is None
    # a record keyed to another file's digest is not reported for this one
    assert bench.traffic_for("binary_gemm_tc_128x2", "ternary_neural_net_b200/csrc/pack_signs.cu") is None
