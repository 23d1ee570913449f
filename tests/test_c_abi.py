"""The boundary as a C caller sees it: tests/c_abi_host.c includes every public
header under strict C99 (gcc -pedantic -Werror), links libenc_b200.so and runs
the calls that need no device. No GPU: nothing here reaches a CUDA call."""
import os
import shutil
import subprocess

import pytest

from audio_encoder_tower_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_program_links_and_runs(tmp_path):
    lib = build.build()
    exe = str(tmp_path / "c_abi_host")
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c_abi_host.c"), "-o", exe, "-L", os.path.dirname(lib), "-lenc_b200",
           "-Wl,-rpath," + os.path.dirname(lib)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    lines = r.stdout.strip().splitlines()
    assert r.returncode == 0, r.stdout + r.stderr
    assert lines[-1] == "0 failures"
    assert sum(1 for ln in lines if ln.startswith("ok ")) == 16
