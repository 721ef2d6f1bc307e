"""The device library's Hilbert keys are a state machine whose tables are
generated at compile time from Skilling's per-level steps
(csrc/hilbert_table.cuh).  These tests build the tables on the host with
g++ and check the keys they give against the oracle's transform
(Skilling, "Programming the Hilbert curve"): every grid point for 1..6 bits
per axis, random points for 7..10 bits."""
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def driver(tmp_path_factory):
    cxx = shutil.which("g++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    exe = str(tmp_path_factory.mktemp("ht") / "hilbert_table_driver")
    subprocess.check_call([cxx, "-O2", "-std=c++17", os.path.join(HERE, "hilbert_table_driver.cpp"), "-o", exe])
    return exe


def _keys(exe, q, bits):
    q = np.ascontiguousarray(q, dtype=np.uint32).reshape(-1, 3)
    inp = np.concatenate([np.array([bits, len(q)], np.uint32), q.ravel()]).tobytes()
    r = subprocess.run([exe], input=inp, capture_output=True, check=True)
    assert r.stderr.decode().strip() == "states 48"
    return np.frombuffer(r.stdout, dtype=np.uint32)


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5, 6])
def test_table_keys_every_point(driver, bits):
    g = np.arange(1 << bits, dtype=np.uint32)
    q = np.stack(np.meshgrid(g, g, g, indexing="ij"), -1).reshape(-1, 3)
    assert np.array_equal(_keys(driver, q, bits), oracle.hilbert_index_grid(q, bits))


@pytest.mark.parametrize("bits", [7, 8, 9, 10])
def test_table_keys_random_points(driver, bits):
    rng = np.random.default_rng(100 + bits)
    q = rng.integers(0, 1 << bits, size=(400_000, 3), dtype=np.uint32)
    assert np.array_equal(_keys(driver, q, bits), oracle.hilbert_index_grid(q, bits))
