"""Tensor-core rate per MMA shape on this GPU (measurement support for the
attend's roofline, not a check of the method): builds and runs the probe
`tests/probes/mma_rate.cu` and prints cycles per tcgen05.mma for each form.
Passes when the probe completes on every SM; the rates are printed (-s)."""
import os
import shutil
import subprocess
import tempfile

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def test_mma_rate_probe_runs():
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    with tempfile.TemporaryDirectory() as td:
        exe = os.path.join(td, "mma_rate")
        subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                        "-I", os.path.join(HERE, "..", "include"), "-o", exe,
                        os.path.join(HERE, "probes", "mma_rate.cu")], check=True, timeout=300)
        out = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    print(out.stdout)
    assert out.returncode == 0, out.stdout + out.stderr
    lines = [ln for ln in out.stdout.splitlines() if "ok=" in ln]
    assert len(lines) == 8 and all("ok=148" in ln for ln in lines), out.stdout
