"""The C ABI used from plain C: tests/c_consumer/consumer.c is compiled as C99 with gcc against
include/hq.h alone, linked to libhq.so and run (host-only calls; no GPU needed)."""
import os
import shutil
import subprocess

import pytest

from hadamard_rotated_precision_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_plain_c_consumer(tmp_path):
    lib = build.build()
    exe = tmp_path / "consumer"
    src = os.path.join(ROOT, "tests", "c_consumer", "consumer.c")
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), src, "-o",
                           str(exe), lib, "-Wl,-rpath," + os.path.dirname(lib)])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "c consumer: ok" in out.stdout
