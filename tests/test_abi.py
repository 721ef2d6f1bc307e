"""The C ABI library loads on a machine without a GPU and exports every
symbol that include/tess.h declares; host-side argument checks and
workspace queries work without touching a device."""
import ctypes
import os
import re

import pytest

import space_filling_curve_b200 as tess

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "tess.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tess_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from space_filling_curve_b200 import build
    build.build()
    return tess.lib()


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert len(names) >= 10
    for name in names:
        assert hasattr(lib, name), name
    # and the Python binding carries the same names
    for name in names:
        assert hasattr(tess, name), name


def test_status_strings_and_version(lib):
    assert tess.tess_status_string(0) == "ok"
    assert "workspace" in tess.tess_status_string(3)
    assert "sm_100a" in tess.tess_version()


def test_workspace_queries_are_host_only(lib):
    box = (467.84283, 467.84283, 467.84283)
    a = tess.tess_hilbert_sort_workspace(10_240_000)
    b = tess.tess_build_neighbors_workspace(10_240_000, box, 5.75, 0.5)
    assert a > 16 * 10_240_000 and b > 24 * 10_240_000
    assert tess.tess_hilbert_sort_workspace(0) == 0
    assert tess.tess_build_neighbors_workspace(10, box, -1.0, 0.5) == 0
    # sized for 10.24M atoms, the buffers fit comfortably in 180 GB
    assert a + b < 2 * 1024 ** 3


def test_argument_errors_are_reported_before_any_launch(lib):
    null = None
    box = (30.0, 30.0, 30.0)
    assert tess.tess_hilbert_sort(null, 10, box, 10, null, 0, null, null, null, null, null) == 1
    assert tess.tess_hilbert_sort(ctypes.c_void_p(256), 10, box, 11, ctypes.c_void_p(256), 1 << 20,
                                  ctypes.c_void_p(256), null, null, null, null) == 1
    # box below 2 (rc + skin): rejected on the host
    p = ctypes.c_void_p(256)
    assert tess.tess_build_neighbors(p, 10, (12.0, 30.0, 30.0), 6.0, 0.5, 16, 0, p, 1 << 30, p, p, p, null) == 2
    # workspace too small
    assert tess.tess_build_neighbors(p, 10, box, 6.0, 0.5, 16, 0, p, 16, p, p, p, null) == 3
    # unknown flag, or two search kinds at once
    for flags in (16, 64, 1 << 30, 2 | 4, 2 | 8, 4 | 8, 2 | 4 | 8):
        assert tess.tess_build_neighbors(p, 10, box, 6.0, 0.5, 16, flags, p, 1 << 30, p, p, p, null) == 1
    assert tess.tess_skin_check(p, p, 10, box, -0.5, p, null, null) == 1
    assert tess.tess_edge_aggregate(p, 10, box, 6.0, p, p, 16, p, 0, p, null, null, null, null) == 1
    # backward: F not a multiple of 4, cap above 512, box below 2 rc
    assert tess.tess_edge_aggregate_backward(p, 10, box, 6.0, p, p, 16, p, p, 6, p, p, null) == 1
    assert tess.tess_edge_aggregate_backward(p, 10, box, 6.0, p, p, 513, p, p, 64, p, p, null) == 1
    assert tess.tess_edge_aggregate_backward(p, 10, (10.0, 30.0, 30.0), 6.0, p, p, 16, p, p, 64, p, p, null) == 2
    # re-sort: no earlier order, workspace too small
    assert tess.tess_hilbert_resort(p, 10, box, 10, null, p, p, 1 << 20, p, p, null, null, null) == 1
    assert tess.tess_hilbert_resort(p, 10, box, 10, p, p, p, 16, p, p, null, null, null) == 3
    # closest pair: no workspace, workspace too small
    assert tess.tess_min_pair_distance(p, 10, box, p, p, 16, null, 0, p, p, null) == 1
    assert tess.tess_min_pair_distance(p, 10, box, p, p, 16, p, 16, p, p, null) == 3
    # step graph: missing buffers, small workspaces; nothing is created
    out = ctypes.c_void_p()
    assert tess.tess_step_graph_create(null, null, ctypes.byref(out)) == 1 and not out.value
    b = tess.StepBuffers()
    b.n, b.box, b.rc, b.skin, b.max_neighbors, b.bits, b.F = 10, tess._box(box), 6.0, 0.5, 16, 10, 8
    for name in ("pos", "feat", "ws_sort", "ws_list", "perm", "keys", "pos_sorted", "pos_cur", "nbr", "counts",
                 "overflow", "sort_status", "rebuild", "max_disp2", "control", "out"):
        setattr(b, name, 256)
    b.ws_sort_bytes, b.ws_list_bytes = 16, 16
    assert tess.tess_step_graph_create(ctypes.byref(b), null, ctypes.byref(out)) == 3 and not out.value
    b.control = None
    assert tess.tess_step_graph_create(ctypes.byref(b), null, ctypes.byref(out)) == 1 and not out.value


def test_static_sort_scratch_holds_the_largest_sort(lib):
    """The allocation-free sort's scratch array (its size in the header)
    holds the sort's workspace at the largest n it accepts."""
    src = open(os.path.join(ROOT, "include", "tess.h")).read()
    max_n = int(re.search(r"#define TESS_HILBERT_SORT_STATIC_MAX_N \(1 << (\d+)\)", src).group(1))
    nbytes = int(re.search(r"#define TESS_HILBERT_SORT_STATIC_BYTES \((\d+)u << 20\)", src).group(1)) << 20
    assert tess.HILBERT_SORT_STATIC_MAX_N == 1 << max_n
    assert tess.HILBERT_SORT_STATIC_BYTES == nbytes
    assert tess.tess_hilbert_sort_workspace(1 << max_n) <= nbytes

