"""The benchmark's reference arm (the fp64 oracle timed on the host cores) and
its JSON line, run on the CPU: one process, and two ranks under torchrun where
only rank 0 may run and print."""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

REQUIRED = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
            "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"}


def _json_lines(out):
    return [json.loads(l) for l in out.splitlines() if l.startswith("{")]


def _check_line(d, n_gpus, steps, warmup):
    assert REQUIRED <= set(d), REQUIRED - set(d)
    assert d["impl"] == "reference" and d["n_gpus"] == n_gpus
    assert d["steps"] == steps and d["warmup"] == warmup
    assert d["value"] > 0 and d["ms_per_step"] > 0 and d["higher_is_better"] is True
    assert d["unit"] == "matrices/s" and d["dtype"] == "f64" and d["scaling"] == "weak"
    assert d["config"]["workload"] == "birkhoff_fwd_bwd_131072"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_reference_arm_single_process():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "2", "--warmup", "3"],
                       cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    _check_line(lines[0], 1, 2, 3)


def test_reference_arm_two_ranks_rank0_only():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           "bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    _check_line(lines[0], 2, 1, 3)


def test_product_arm_has_no_cpu_fallback():
    # without a GPU the CUDA arm must fail loudly rather than print a number
    import pytest
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    r = subprocess.run([sys.executable, "bench.py", "--steps", "1", "--warmup", "3", "--no-extras",
                        "--no-cpu-baseline"], cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0
    assert not _json_lines(r.stdout)


def test_measured_peaks_reader(tmp_path):
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import bench
    f = tmp_path / "peaks.json"
    f.write_text(json.dumps({"hbm_gbs": 6542.7, "bf16_tflops": 1590}))
    assert bench.measured_peaks(str(f)) == (6542.7, "measured")
    f.write_text(json.dumps({"hbm_gbs": {"value": 6500.0, "unit": "GB/s"}}))
    assert bench.measured_peaks(str(f)) == (6500.0, "measured")
    f.write_text(json.dumps({"bf16_tflops": 1590}))
    assert bench.measured_peaks(str(f)) == (bench.FALLBACK_HBM_GBS, "fallback")
    assert bench.measured_peaks(str(tmp_path / "absent.json")) == (bench.FALLBACK_HBM_GBS, "fallback")
