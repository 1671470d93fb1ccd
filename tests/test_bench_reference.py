"""The reference arm of bench.py (the fp64 oracle on the host) keeps the JSON
contract: one line with the same metric, unit and config as the CUDA arm,
impl = reference, a cpu_baseline record and a zero-copy e2e record."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "0", "--ref-rows", "8"],
                         cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    sys.path.insert(0, ROOT)
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["config"] == bench.workload_config(d["config"]["mask_adjusted_flops_per_step"], 1)
    assert d["config"]["mask_adjusted_flops_per_step"] == 4.0 * 128 * 32760 * 32760 * 12
    assert d["value"] > 0 and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["e2e"]["value"] == d["value"]


def test_cpu_baseline_config_timings(monkeypatch):
    # The oracle timings the bench adds to cpu_baseline, on shrunken copies of
    # the configurations (same code path as the benchmark, a few seconds).
    sys.path.insert(0, ROOT)
    import importlib.util
    import numpy as np
    import seeded_inputs as si
    spec = importlib.util.spec_from_file_location("bench_mod2", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    small = dict(si.CONFIGS)
    small["hybrid"] = dict(si.CONFIGS["hybrid"], T=4, H=2)
    small["stream"] = dict(si.CONFIGS["stream"], T=3, H=2)
    monkeypatch.setattr(si, "CONFIGS", small)
    monkeypatch.setattr(bench.si, "CONFIGS", small)
    w = dict(B=1, H=12, L=32760)
    res = bench.oracle_config_timings(w, wan_rows=100, wan_seconds=0.5, stream_rows=64)
    assert set(res) == {"wan13b", "tiny", "hybrid", "stream"}
    assert res["wan13b"]["projected"] and res["wan13b"]["projected_full_s"] == 32760 * 12 / 200.0
    assert not res["tiny"]["projected"] and res["tiny"]["rows"] == 48 * 2
    c = small["hybrid"]
    assert not res["hybrid"]["projected"] and res["hybrid"]["rows"] == 4 * c["Hg"] * c["Wg"] * 2
    st = res["stream"]
    assert st["projected"] and 0 < st["rows_sampled"] <= 64
    L = 3 * small["stream"]["Hg"] * small["stream"]["Wg"]
    assert np.isclose(st["projected_full_s"], L * 2 / st["rows_per_s"])
