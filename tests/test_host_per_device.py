"""Host-side unit test of the per-device launch set-up cache.

The head kernel's launch set-up (its shared-memory limit and the number of
CTA pairs that fit) belongs to the device it was done on, so the library
keeps it per device (``csrc/per_device.h``).  A machine with one GPU cannot
drive two devices from one process, so the cache itself is tested here on
the host: two fake devices used alternately get their own values, each set
up once; a failed set-up is retried; racing threads set up once.
"""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "block_canvas_denoising_b200", "csrc")


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_per_device_cache(tmp_path):
    exe = str(tmp_path / "per_device_test")
    subprocess.run(["g++", "-std=c++17", "-O1", "-pthread", "-I", CSRC,
                    os.path.join(HERE, "host", "per_device_test.cpp"), "-o", exe], check=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
