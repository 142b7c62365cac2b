"""bench.py's reference arm (the oracle on the host cores) prints one JSON line with the
keys the bench contract names; runs on CPU in a few seconds."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_line_keys():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--config", "single_linear"], capture_output=True, text=True, timeout=300,
                       cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "higher_is_better", "scaling", "vs_baseline",
              "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["config"]["workload"] == "single_linear_step"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["higher_is_better"] is False and d["unit"] == "us"


def test_roofline_takes_the_binding_bound():
    """The Product class is reported against HBM when its bytes take longer than its
    multiply-adds (short contractions), else against the INT8 tensor peak; memory-bound
    classes always against HBM."""
    sys.path.insert(0, ROOT)
    import bench

    peaks = {"bf16": 1630.0, "hbm": 6544.7, "source": "measured"}
    M, D, H = 12608, 192, 768
    mlp = {"gemm": {"ms_per_step": 0.1, "launches_per_step": 6.0, "work_per_step": 22.31e9},
           "align": {"ms_per_step": 0.05, "launches_per_step": 6.0, "work_per_step": 5e7}}
    r = bench.roofline(mlp, peaks, "none", 6 * (M * D + D * H + M * H))
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["other_bound"]["bound"] == "tensor"
    assert abs(r["achieved"] - 6 * (M * D + D * H + M * H) / 1e-4 / 1e9) < 1.0
    trio = {"gemm": {"ms_per_step": 0.29, "launches_per_step": 6.0, "work_per_step": 356.95e9}}
    r = bench.roofline(trio, peaks, "none", 6 * (M * 768 + 768 * 3072 + M * 3072))
    assert r["bound"] == "tensor" and r["peak"] == 3260.0 and r["other_bound"]["bound"] == "hbm"
    sgd = {"sgd": {"ms_per_step": 0.05, "launches_per_step": 1.0, "work_per_step": 129.78e6}}
    r = bench.roofline(sgd, peaks, "none")
    assert r["bound"] == "hbm" and "other_bound" not in r and abs(r["frac"] - 129.78e6 / 5e-5 / 1e9 / 6544.7) < 1e-3
