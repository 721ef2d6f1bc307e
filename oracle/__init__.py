"""Plain CPU oracle for the neighbor-rebuild path -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline /
reference legs of ``bench.py`` may import this package.  The product library
(``space_filling_curve_b200``) never imports, loads or calls it, and the two
share no code: the C source here (``tess_oracle.c``) was written from the
definitions independently of the CUDA kernels.

Each function cites the passage it follows in its C counterpart.  The
source of the method is "Ab Initio Accuracy Beyond the Cutoff: Distributed
Message-Passing Equivariant Attention at Tens-of-Millions-of-Atom Scale"
(Tessera), abstract; the one-hop aggregation semantics is from the review of
arXiv 2505.06711 (ghost-atom message passing).  Open readings are marked
READING in the C source.

Arrays are numpy; positions are float32 ``[n, 3]`` or ``[n, 4]`` (the first
three columns are x, y, z), boxes are three float32 lengths.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tess_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

# Every operation one IEEE rounding in source order: no FMA contraction, no
# fast-math.  OpenMP only splits independent rows across threads.
CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared", "-std=c11"]


def build(force: bool = False) -> str:
    """Compile liboracle.so next to its source (gcc)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        path = build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64, i32, f32 = ctypes.c_int64, ctypes.c_int, ctypes.c_float
        L.oracle_set_threads.argtypes = [i32]
        L.oracle_get_threads.restype = i32
        L.oracle_quantize.argtypes = [f32, f32, i32]
        L.oracle_quantize.restype = ctypes.c_uint32
        L.oracle_hilbert_index.argtypes = [ctypes.c_uint32] * 3 + [i32]
        L.oracle_hilbert_index.restype = ctypes.c_uint32
        L.oracle_hilbert_index_many.argtypes = [P, i64, i32, P]
        L.oracle_morton_index.argtypes = [ctypes.c_uint32] * 3 + [i32]
        L.oracle_morton_index.restype = ctypes.c_uint32
        L.oracle_morton_index_many.argtypes = [P, i64, i32, P]
        L.oracle_morton_sort.argtypes = [P, i32, i64, P, i32, P, P]
        L.oracle_hilbert_keys.argtypes = [P, i32, i64, P, i32, P]
        L.oracle_hilbert_sort.argtypes = [P, i32, i64, P, i32, P, P]
        for name in ("oracle_neighbors_brute", "oracle_neighbors_cells"):
            fn = getattr(L, name)
            fn.argtypes = [P, i32, i64, P, f32, f32, i32, P, P]
            fn.restype = i32
        L.oracle_neighbors_of.argtypes = [P, i32, i64, P, f32, f32, i64, P, i64]
        L.oracle_neighbors_of.restype = i64
        L.oracle_pair_distances.argtypes = [P, i32, P, P, P, i64, P]
        L.oracle_neighbors_rows.argtypes = [P, i32, i64, P, f32, f32, P, i64, i32, P, P]
        L.oracle_edge_aggregate_rows.argtypes = [P, i32, i64, P, f32, P, P, i32, P, i32, P, i64, P, P]
        L.oracle_skin_check.argtypes = [P, P, i32, i64, P, f32, P]
        L.oracle_skin_check.restype = i32
        L.oracle_cutoff.argtypes = [ctypes.c_double, ctypes.c_double]
        L.oracle_cutoff.restype = ctypes.c_double
        L.oracle_edge_aggregate.argtypes = [P, i32, i64, P, f32, P, P, i32, P, i32, P, P, P, P, P]
        L.oracle_cutoff_deriv.argtypes = [ctypes.c_double, ctypes.c_double]
        L.oracle_cutoff_deriv.restype = ctypes.c_double
        L.oracle_edge_backward.argtypes = [P, i32, i64, P, f32, P, P, i32, P, P, i32, P, P]
        L.oracle_min_pair.argtypes = [P, i32, i64, P, P, P, i32, P, P, P]
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _pos(pos):
    pos = np.ascontiguousarray(pos, dtype=np.float32)
    if pos.ndim != 2 or pos.shape[1] < 3:
        raise ValueError("positions must be [n, 3] or [n, 4] float32")
    return pos, pos.shape[1]


def _box(box):
    b = np.ascontiguousarray(np.asarray(box, dtype=np.float32).reshape(3))
    return b


def set_threads(n: int) -> None:
    lib().oracle_set_threads(int(n))


def get_threads() -> int:
    return int(lib().oracle_get_threads())


def quantize(x: float, L: float, bits: int) -> int:
    """Grid cell of one coordinate, decided in fp32 (C1)."""
    return int(lib().oracle_quantize(float(np.float32(x)), float(np.float32(L)), int(bits)))


def hilbert_index(q0: int, q1: int, q2: int, bits: int) -> int:
    """Hilbert index of one grid point (Skilling's transform, C1)."""
    return int(lib().oracle_hilbert_index(int(q0), int(q1), int(q2), int(bits)))


def hilbert_index_grid(q: np.ndarray, bits: int) -> np.ndarray:
    """Hilbert indices of many integer grid points ``q[m, 3]`` (loops in C)."""
    q = np.ascontiguousarray(q, dtype=np.uint32).reshape(-1, 3)
    out = np.empty(len(q), dtype=np.uint32)
    lib().oracle_hilbert_index_many(_ptr(q), len(q), int(bits), _ptr(out))
    return out


def morton_index(q0: int, q1: int, q2: int, bits: int) -> int:
    """Morton (Z-order) index of one grid point."""
    return int(lib().oracle_morton_index(int(q0), int(q1), int(q2), int(bits)))


def morton_index_grid(q: np.ndarray, bits: int) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint32).reshape(-1, 3)
    out = np.empty(len(q), dtype=np.uint32)
    lib().oracle_morton_index_many(_ptr(q), len(q), int(bits), _ptr(out))
    return out


def morton_sort(pos, box, bits: int = 10):
    """(perm, keys_sorted) along the Morton curve, ties by input index."""
    pos, stride = _pos(pos)
    b = _box(box)
    n = len(pos)
    perm = np.empty(n, dtype=np.int32)
    keys = np.empty(n, dtype=np.uint32)
    lib().oracle_morton_sort(_ptr(pos), stride, n, _ptr(b), int(bits), _ptr(perm), _ptr(keys))
    return perm, keys


def hilbert_keys(pos, box, bits: int = 10) -> np.ndarray:
    pos, stride = _pos(pos)
    b = _box(box)
    keys = np.empty(len(pos), dtype=np.uint32)
    lib().oracle_hilbert_keys(_ptr(pos), stride, len(pos), _ptr(b), int(bits), _ptr(keys))
    return keys


def hilbert_sort(pos, box, bits: int = 10):
    """(perm, keys_sorted): stable order by key, ties by input index (C2)."""
    pos, stride = _pos(pos)
    b = _box(box)
    n = len(pos)
    perm = np.empty(n, dtype=np.int32)
    keys = np.empty(n, dtype=np.uint32)
    lib().oracle_hilbert_sort(_ptr(pos), stride, n, _ptr(b), int(bits), _ptr(perm), _ptr(keys))
    return perm, keys


def _neighbors(fn, pos, box, rc, skin, cap):
    pos, stride = _pos(pos)
    b = _box(box)
    n = len(pos)
    nbr = np.empty((n, cap), dtype=np.int32)
    counts = np.empty(n, dtype=np.int32)
    ov = fn(_ptr(pos), stride, n, _ptr(b), float(rc), float(skin), int(cap), _ptr(nbr), _ptr(counts))
    return nbr, counts, int(ov)


def neighbors_brute(pos, box, rc, skin, cap):
    """O(n^2) Verlet list (C3): (nbr [n,cap] sorted rows, -1 pads; counts; overflow)."""
    return _neighbors(lib().oracle_neighbors_brute, pos, box, rc, skin, cap)


def neighbors_cells(pos, box, rc, skin, cap):
    """Cell-list Verlet list (C3), same contract as neighbors_brute."""
    return _neighbors(lib().oracle_neighbors_cells, pos, box, rc, skin, cap)


def neighbors_of(pos, box, rc, skin, i: int) -> np.ndarray:
    """Sorted neighbor indices of atom i by brute force over all atoms."""
    pos, stride = _pos(pos)
    b = _box(box)
    buf = np.empty(4096, dtype=np.int32)
    m = lib().oracle_neighbors_of(_ptr(pos), stride, len(pos), _ptr(b), float(rc), float(skin), int(i), _ptr(buf), len(buf))
    if m > len(buf):
        buf = np.empty(int(m), dtype=np.int32)
        m = lib().oracle_neighbors_of(_ptr(pos), stride, len(pos), _ptr(b), float(rc), float(skin), int(i), _ptr(buf), len(buf))
    return buf[: int(m)].copy()


def neighbors_rows(pos, box, rc, skin, rows, cap):
    """Rows `rows` of the list by brute force (C3): (nbr [m, cap], counts [m])."""
    pos, stride = _pos(pos)
    b = _box(box)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    nbr = np.empty((len(rows), cap), dtype=np.int32)
    counts = np.empty(len(rows), dtype=np.int32)
    lib().oracle_neighbors_rows(_ptr(pos), stride, len(pos), _ptr(b), float(rc), float(skin), _ptr(rows), len(rows),
                                int(cap), _ptr(nbr), _ptr(counts))
    return nbr, counts


def edge_aggregate_rows(pos, box, rc, nbr, counts, feat, rows):
    """Aggregate (C5) of rows `rows` only: dict with out and out_abs [m, F]."""
    pos, stride = _pos(pos)
    b = _box(box)
    nbr = np.ascontiguousarray(nbr, dtype=np.int32)
    counts = np.ascontiguousarray(counts, dtype=np.int32)
    feat = np.ascontiguousarray(feat, dtype=np.float32)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    n, cap = nbr.shape
    F = feat.shape[1]
    out = np.empty((len(rows), F), dtype=np.float64)
    out_abs = np.empty((len(rows), F), dtype=np.float64)
    lib().oracle_edge_aggregate_rows(_ptr(pos), stride, n, _ptr(b), float(rc), _ptr(nbr), _ptr(counts), int(cap),
                                     _ptr(feat), int(F), _ptr(rows), len(rows), _ptr(out), _ptr(out_abs))
    return {"out": out, "out_abs": out_abs}


def pair_distances(pos, box, i, j) -> np.ndarray:
    """fp64 minimum-image distances of pairs (i[k], j[k])."""
    pos, stride = _pos(pos)
    b = _box(box)
    i = np.ascontiguousarray(i, dtype=np.int32)
    j = np.ascontiguousarray(j, dtype=np.int32)
    out = np.empty(len(i), dtype=np.float64)
    lib().oracle_pair_distances(_ptr(pos), stride, _ptr(b), _ptr(i), _ptr(j), len(i), _ptr(out))
    return out


def skin_check(pos, ref, box, skin):
    """(rebuild flag, max squared displacement in fp64) (C4)."""
    pos, stride = _pos(pos)
    ref, stride2 = _pos(ref)
    if stride2 != stride or ref.shape != pos.shape:
        raise ValueError("pos and ref must have the same layout")
    b = _box(box)
    m = ctypes.c_double(0.0)
    flag = lib().oracle_skin_check(_ptr(pos), _ptr(ref), stride, len(pos), _ptr(b), float(skin), ctypes.byref(m))
    return int(flag), float(m.value)


def cutoff(r: float, rc: float) -> float:
    """Smooth cosine cutoff f_c (C5)."""
    return float(lib().oracle_cutoff(float(r), float(rc)))


def edge_aggregate(pos, box, rc, nbr, counts, feat, edges: bool = False):
    """One-hop aggregation (C5).

    Returns a dict with ``out`` [n, F] (fp64), ``out_abs`` [n, F] (sum of
    f_c |h_j|, the per-element conditioning) and, if ``edges``, ``edge_vec``
    [n, cap, 4], ``edge_fc`` [n, cap], ``edge_unit`` [n, cap, 4] (fp64).
    """
    pos, stride = _pos(pos)
    b = _box(box)
    nbr = np.ascontiguousarray(nbr, dtype=np.int32)
    counts = np.ascontiguousarray(counts, dtype=np.int32)
    feat = np.ascontiguousarray(feat, dtype=np.float32)
    n, cap = nbr.shape
    F = feat.shape[1]
    out = np.empty((n, F), dtype=np.float64)
    out_abs = np.empty((n, F), dtype=np.float64)
    ev = ef = eu = None
    if edges:
        ev = np.empty((n, cap, 4), dtype=np.float64)
        ef = np.empty((n, cap), dtype=np.float64)
        eu = np.empty((n, cap, 4), dtype=np.float64)
    lib().oracle_edge_aggregate(_ptr(pos), stride, n, _ptr(b), float(rc), _ptr(nbr), _ptr(counts), int(cap),
                                _ptr(feat), int(F), _ptr(out), _ptr(out_abs), _ptr(ev), _ptr(ef), _ptr(eu))
    res = {"out": out, "out_abs": out_abs}
    if edges:
        res.update(edge_vec=ev, edge_fc=ef, edge_unit=eu)
    return res


def rebuild(pos3, box, rc, skin, cap, bits: int = 10, method: str = "cells"):
    """Full rebuild as the oracle sees it: Hilbert sort, then the list over
    the sorted positions.  Returns (perm, keys_sorted, pos_sorted [n,4],
    nbr, counts, overflow) in sorted-index space."""
    perm, keys = hilbert_sort(pos3, box, bits)
    p = np.ascontiguousarray(pos3, dtype=np.float32)[:, :3]
    ps = np.zeros((len(perm), 4), dtype=np.float32)
    ps[:, :3] = p[perm]
    fn = neighbors_cells if method == "cells" else neighbors_brute
    nbr, counts, ov = fn(ps, box, rc, skin, cap)
    return perm, keys, ps, nbr, counts, ov


def cutoff_deriv(r: float, rc: float) -> float:
    """d f_c / d r."""
    return float(lib().oracle_cutoff_deriv(float(r), float(rc)))


def edge_backward(pos, box, rc, nbr, counts, feat, grad_out):
    """VJP of the aggregation: (grad_feat [n, F], grad_pos [n, 3]) in fp64."""
    pos, stride = _pos(pos)
    b = _box(box)
    nbr = np.ascontiguousarray(nbr, dtype=np.int32)
    counts = np.ascontiguousarray(counts, dtype=np.int32)
    feat = np.ascontiguousarray(feat, dtype=np.float32)
    g = np.ascontiguousarray(grad_out, dtype=np.float32)
    n, cap = nbr.shape
    F = feat.shape[1]
    gf = np.empty((n, F), dtype=np.float64)
    gp = np.empty((n, 3), dtype=np.float64)
    lib().oracle_edge_backward(_ptr(pos), stride, n, _ptr(b), float(rc), _ptr(nbr), _ptr(counts), int(cap),
                               _ptr(feat), _ptr(g), int(F), _ptr(gf), _ptr(gp))
    return gf, gp


def min_pair(pos, box, nbr, counts):
    """Closest listed pair: (r2 fp64, i, j); (inf, -1, -1) when nothing is listed."""
    pos, stride = _pos(pos)
    b = _box(box)
    nbr = np.ascontiguousarray(nbr, dtype=np.int32)
    counts = np.ascontiguousarray(counts, dtype=np.int32)
    n, cap = nbr.shape
    r2 = ctypes.c_double(0.0)
    i = ctypes.c_int32(0)
    j = ctypes.c_int32(0)
    lib().oracle_min_pair(_ptr(pos), stride, n, _ptr(b), _ptr(nbr), _ptr(counts), int(cap), ctypes.byref(r2),
                          ctypes.byref(i), ctypes.byref(j))
    return float(r2.value), int(i.value), int(j.value)

