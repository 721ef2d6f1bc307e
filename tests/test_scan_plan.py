"""The chunk plan of the device offset scan (csrc/scan.cuh): every chunk a
positive multiple of 4 elements (the kernel moves int4), chunks covering the
array with none empty, no more blocks than 4 per SM, and the caller's
look-back words enough for one per chunk plus the chunk counter.  Built with
nvcc as a host program; nothing runs on a GPU."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def test_scan_plan(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("no nvcc")
    exe = str(tmp_path / "scan_plan_driver")
    subprocess.check_call([nvcc, "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-I",
                           os.path.join(ROOT, "include"), os.path.join(HERE, "scan_plan_driver.cu"), "-o", exe])
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
