"""The decode's work division (slices, segments, partial slots) checked on
the host: tests/native/decode_slices_check.cu includes the same header the
decode kernels use and runs it over thousands of random batches."""
import os
import shutil
import subprocess

import pytest

from conftest import ROOT


def test_decode_slices_cover_every_token_once(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not found")
    exe = tmp_path / "decode_slices_check"
    src = os.path.join(ROOT, "tests", "native", "decode_slices_check.cu")
    inc = os.path.join(ROOT, "latent_attention_b200", "csrc")
    subprocess.run([nvcc, "-std=c++17", "-O2", "-Wno-deprecated-gpu-targets", "-o", str(exe), src, "-I", inc], check=True,
                   capture_output=True, text=True, timeout=300)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.startswith("ok ")
