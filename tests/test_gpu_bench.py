"""bench.py end to end on the GPU: one short run per option, and the JSON
line's contract keys and types (the keys the benchmark line promises)."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(*args):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--steps", "5",
                          "--warmup", "3", *args], capture_output=True, text=True, timeout=600,
                         cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    return json.loads(lines[0])


@pytest.mark.parametrize("extra", [
    ("--workload", "decode-M128-uniform"),
    ("--workload", "decode-M128-uniform", "--schedule", "separate", "--tiles", "64"),
    ("--workload", "M16384-hotpairs-dedup", "--combine", "two-level", "--no-cpu-baseline"),
])
def test_contract_line(extra):
    d = _bench(*extra)
    for key, typ in (("metric", str), ("value", float), ("unit", str), ("n_gpus", int),
                     ("steps", int), ("warmup", int), ("ms_per_step", float),
                     ("higher_is_better", bool), ("scaling", str), ("dtype", str),
                     ("data", str), ("config", dict), ("roofline", dict), ("e2e", dict),
                     ("gpu_launches", int), ("clocks", dict)):
        assert isinstance(d[key], typ), key
    assert d["n_gpus"] == 1 and d["steps"] == 5 and d["warmup"] == 3
    assert d["value"] > 0 and d["ms_per_step"] > 0 and d["vs_baseline"] is None
    assert "workload" in d["config"]
    r = d["roofline"]
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and 0 < r["frac"] < 2
    assert r["achieved"] == pytest.approx(r["frac"] * r["peak"], rel=1e-3)
    e = d["e2e"]
    assert e["value"] > 0 and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert d["gpu_launches"] >= 5 * 2                      # at least two kernels per step
    assert set(d["clocks"]) >= {"sm_mhz", "sm_max_mhz", "reasons"}
    if "--no-cpu-baseline" not in extra:
        c = d["cpu_baseline"]
        assert c["kind"] == "oracle" and c["cores"] == 1 and c["value"] > 0 and c["sample"]


def test_reference_arm_line():
    d = _bench("--impl", "reference", "--workload", "decode-M128-uniform")
    assert d["impl"] == "reference" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
