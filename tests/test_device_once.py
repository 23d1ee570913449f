"""The launchers' per-device one-time set-up (enc::DeviceOnce in csrc/internal.h)
under concurrent first launches from many host threads: set-up runs exactly once
per device, every thread sees what it wrote, and a failed set-up is retried.
Host code only (nvcc compiles the CUDA C++ header); no GPU."""
import os
import shutil
import subprocess

import pytest

from audio_encoder_tower_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which(build.nvcc()) is None and not os.path.exists(build.nvcc()), reason="needs nvcc")
def test_device_once_under_racing_threads(tmp_path):
    exe = str(tmp_path / "device_once_host")
    cmd = [build.nvcc(), *build.ARCH, "-std=c++17", "-O2", "-I", os.path.join(ROOT, "audio_encoder_tower_b200", "csrc"),
           os.path.join(ROOT, "tests", "device_once_host.cu"), "-o", exe, "-Xcompiler", "-pthread"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip().splitlines()[-1] == "0 failures"
