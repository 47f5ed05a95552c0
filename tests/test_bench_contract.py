"""The reference leg of bench.py on CPU: its one JSON line carries the contract's keys,
the oracle's cpu_baseline (multi-thread figure, one-thread figure, CPU model) and an
e2e object with no host-device traffic."""
import contextlib
import io
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def test_reference_leg_prints_one_contract_line():
    import bench
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        rc = bench.main(["--impl", "reference", "--workload", "decode-tiny-f32", "--steps", "3", "--warmup", "3"])
    assert rc == 0
    lines = [ln for ln in buf.getvalue().splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 3 and d["warmup"] == 3
    assert d["value"] > 0 and d["unit"] == "GB/s" and d["dtype"] == "f64"
    assert d["config"]["workload"] == "decode-tiny-f32"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert cb["single_thread"]["value"] > 0 and "1 thread" in cb["single_thread"]["sample"]
    assert "cpu_model" in cb
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_bench_refuses_fewer_than_three_warmup_steps():
    import bench
    import pytest
    with pytest.raises(SystemExit):
        bench.main(["--impl", "reference", "--steps", "2", "--warmup", "1"])


def test_reference_leg_under_torchrun_prints_one_line_from_rank_zero():
    """Launched the way the N-GPU bench is (torchrun, two ranks), the reference leg runs on
    rank 0 only: one JSON line in all, and every rank exits 0."""
    import socket
    import subprocess
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--workload", "decode-tiny-f32", "--steps", "3", "--warmup", "3"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
