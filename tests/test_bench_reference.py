"""The reference arm of bench.py (the CPU oracle, timed on the host cores) prints one JSON
line with the keys the measurement contract names; it runs without a GPU."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1", "--warmup", "3",
           "--cpu-sample-tokens", "32"]
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for k in ("metric", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["steps"] == 1 and d["warmup"] >= 3 and d["n_gpus"] == 1
    assert d["higher_is_better"] is True and d["vs_baseline"] is None
    assert "workload" in d["config"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["unit"] == d["unit"]
    assert cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_step_flops_counts_every_product():
    # the headline's work per fwd + bwd step, counted product by product: the two base GEMMs
    # (Y = X W^T, dX = dY W^) and the six rank-r products (X A, (s XA) B, dY B^T, (s G) A^T,
    # dA = X^T (s G), dB = (XA)^T dY), 2 m n k each
    sys.path.insert(0, ROOT)
    import bench
    M, d_in, d_out, r = 4096, 4096, 4096, 64
    products = [(M, d_out, d_in), (M, d_in, d_out),
                (M, r, d_in), (M, d_out, r), (M, r, d_out), (M, d_in, r), (d_in, r, M), (r, d_out, M)]
    assert bench.step_flops(M, d_in, d_out, r) == sum(2 * m * n * k for m, n, k in products) == 287762808832
    # a non-square layer as well
    M, d_in, d_out, r = 480, 1024, 16384, 16
    products = [(M, d_out, d_in), (M, d_in, d_out),
                (M, r, d_in), (M, d_out, r), (M, r, d_out), (M, d_in, r), (d_in, r, M), (r, d_out, M)]
    assert bench.step_flops(M, d_in, d_out, r) == sum(2 * m * n * k for m, n, k in products)
