"""The reference arm of bench.py (the oracle timed on host cores) runs without a
GPU and prints one JSON line with the fields the bench contract names."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "2", "--warmup", "3"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 3 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"] and d["cpu_baseline"]["sample"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["unit"] == d["unit"]
    assert "workload" in d["config"]


def test_rejects_short_warmup():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "1"],
                       cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0 and "warmup" in r.stderr


def test_failing_row_is_reported_not_fatal():
    """A row that raises is recorded as an error in the rows object; the
    other rows and the headline line still come out."""
    import types

    import torch

    import bench
    import workloads

    class Boom(RuntimeError):
        pass

    def fail(*a, **k):
        raise Boom("planted failure")

    fake = types.SimpleNamespace(empty_packed=fail, bnn_device_error=lambda: 0)
    args = types.SimpleNamespace(row_steps=3, warmup=3)
    pk = {"sm_max_mhz": 1965.0, "hbm_gbs": 6513.5}
    rows = bench.bench_rows(torch, fake, workloads, torch.device("cpu"), pk, args, lambda: None, lambda v: v, 1,
                            only=["pack_sign_weights"])
    assert list(rows) == ["pack_sign_weights"]
    assert rows["pack_sign_weights"]["error"].startswith("Boom: planted failure")
