"""B200-native neighbor-rebuild library: Python binding of libtess.so.

The C ABI (``include/tess.h``) is the product; this module only marshals
arguments.  Every step of the path runs in the library's CUDA kernels on the
caller's current CUDA stream; PyTorch provides device memory and streams.

Two layers:
  * ``tess_*`` -- one-to-one ctypes bindings with the C names and arguments
    (raw device pointers as ints, ``tess_box`` as three floats).
  * ``hilbert_sort``, ``build_neighbors``, ``skin_check``, ``edge_aggregate``
    -- the same calls taking torch CUDA tensors; outputs and workspaces are
    allocated with torch when not given.

There is no CPU fallback: if the CUDA library is missing or a tensor is not
on a CUDA device, calls raise.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "TessError", "lib", "library_path", "Box",
    "tess_status_string", "tess_version", "tess_kernel_launch_count",
    "tess_hilbert_sort_workspace", "tess_hilbert_sort", "tess_hilbert_sort_static", "HILBERT_SORT_STATIC_MAX_N",
    "HILBERT_SORT_STATIC_BYTES",
    "tess_hilbert_resort_workspace", "tess_hilbert_resort", "hilbert_resort", "TESS_DEV_FULL_SORT",
    "tess_min_pair_distance_workspace", "tess_min_pair_distance", "min_pair_distance",
    "tess_step_graph_create", "tess_step_graph_launch", "tess_step_graph_request_rebuild", "tess_step_graph_destroy",
    "StepBuffers", "StepGraph",
    "tess_debug_lookback_timeout_workspace", "tess_debug_lookback_timeout",
    "tess_morton_sort", "morton_sort",
    "tess_build_neighbors_workspace", "tess_build_neighbors",
    "tess_skin_check", "tess_edge_aggregate", "tess_stage_timing", "tess_stage_times",
    "hilbert_sort", "build_neighbors", "skin_check", "edge_aggregate",
    "tess_edge_aggregate_backward", "edge_aggregate_backward",
    "TESS_DEV_OVERFLOW", "TESS_DEV_BAD_INPUT", "TESS_DEV_TIMEOUT", "TESS_NO_PAD_FILL", "TESS_LANE_SEARCH", "TESS_TILE_SEARCH", "TESS_LANE2_SEARCH", "STAGES",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
# TESS_LIBRARY selects another build of the same library (build.py variants)
library_path = os.environ.get("TESS_LIBRARY") or os.path.join(_HERE, "libtess.so")

TESS_DEV_OVERFLOW = 1
TESS_DEV_FULL_SORT = 8
TESS_DEV_BAD_INPUT = 2
TESS_DEV_TIMEOUT = 4
TESS_NO_PAD_FILL = 1
TESS_LANE_SEARCH = 2
TESS_TILE_SEARCH = 4
TESS_LANE2_SEARCH = 8
SEARCH_FLAGS = {"default": 0, "lane": TESS_LANE_SEARCH, "tile": TESS_TILE_SEARCH, "lane2": TESS_LANE2_SEARCH}
STAGES = ("hilbert_keys", "key_sort", "cell_binning", "pair_search", "skin_check", "edge_aggregate", "edge_backward",
          "resort", "min_pair")
_STATUS = {0: "ok", 1: "invalid argument", 2: "box too small", 3: "workspace too small", 4: "CUDA launch error",
           5: "n above the static scratch capacity"}
HILBERT_SORT_STATIC_MAX_N = 1 << 20
HILBERT_SORT_STATIC_BYTES = 21 << 20


class TessError(RuntimeError):
    """A library call returned a non-zero tess_status."""

    def __init__(self, fn: str, code: int):
        super().__init__("%s failed: %s (status %d)" % (fn, _STATUS.get(code, "unknown"), code))
        self.code = code


class Box(ctypes.Structure):
    _fields_ = [("lx", ctypes.c_float), ("ly", ctypes.c_float), ("lz", ctypes.c_float)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libtess.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(library_path):
        raise ImportError("libtess.so is not built (run `python space_filling_curve_b200/build.py` "
                          "or __graft_entry__.build()): there is no fallback path")
    L = ctypes.CDLL(library_path)
    P, i32, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    L.tess_status_string.argtypes = [i32]
    L.tess_status_string.restype = ctypes.c_char_p
    L.tess_version.restype = ctypes.c_char_p
    L.tess_kernel_launch_count.restype = ctypes.c_longlong
    L.tess_hilbert_sort_workspace.argtypes = [i32]
    L.tess_hilbert_sort_workspace.restype = sz
    L.tess_hilbert_sort.argtypes = [P, i32, Box, i32, P, sz, P, P, P, P, P]
    L.tess_hilbert_sort.restype = i32
    L.tess_step_graph_create.argtypes = [ctypes.POINTER(StepBuffers), P, ctypes.POINTER(P)]
    L.tess_step_graph_create.restype = i32
    L.tess_step_graph_launch.argtypes = [P, P]
    L.tess_step_graph_launch.restype = i32
    L.tess_step_graph_request_rebuild.argtypes = [ctypes.POINTER(StepBuffers), P]
    L.tess_step_graph_request_rebuild.restype = i32
    L.tess_step_graph_destroy.argtypes = [P]
    L.tess_step_graph_destroy.restype = None
    L.tess_debug_lookback_timeout_workspace.argtypes = []
    L.tess_debug_lookback_timeout_workspace.restype = sz
    L.tess_debug_lookback_timeout.argtypes = [P, sz, P, P]
    L.tess_debug_lookback_timeout.restype = i32
    L.tess_min_pair_distance_workspace.argtypes = []
    L.tess_min_pair_distance_workspace.restype = sz
    L.tess_min_pair_distance.argtypes = [P, i32, Box, P, P, i32, P, sz, P, P, P]
    L.tess_min_pair_distance.restype = i32
    L.tess_hilbert_resort_workspace.argtypes = [i32]
    L.tess_hilbert_resort_workspace.restype = sz
    L.tess_hilbert_resort.argtypes = [P, i32, Box, i32, P, P, P, sz, P, P, P, P, P]
    L.tess_hilbert_resort.restype = i32
    L.tess_morton_sort.argtypes = [P, i32, Box, i32, P, sz, P, P, P, P, P]
    L.tess_morton_sort.restype = i32
    L.tess_hilbert_sort_static.argtypes = [P, i32, Box, i32, P, P, P, P, P]
    L.tess_hilbert_sort_static.restype = i32
    L.tess_build_neighbors_workspace.argtypes = [i32, Box, f32, f32]
    L.tess_build_neighbors_workspace.restype = sz
    L.tess_build_neighbors.argtypes = [P, i32, Box, f32, f32, i32, i32, P, sz, P, P, P, P]
    L.tess_build_neighbors.restype = i32
    L.tess_skin_check.argtypes = [P, P, i32, Box, f32, P, P, P]
    L.tess_skin_check.restype = i32
    L.tess_edge_aggregate.argtypes = [P, i32, Box, f32, P, P, i32, P, i32, P, P, P, P, P]
    L.tess_edge_aggregate.restype = i32
    L.tess_edge_aggregate_backward.argtypes = [P, i32, Box, f32, P, P, i32, P, P, i32, P, P, P]
    L.tess_edge_aggregate_backward.restype = i32
    L.tess_stage_timing.argtypes = [i32]
    L.tess_stage_times.argtypes = [P, P, i32]
    L.tess_stage_times.restype = i32
    _lib = L
    return L


class StepBuffers(ctypes.Structure):
    """Mirror of tess_step_buffers (include/tess.h)."""
    _fields_ = [("n", ctypes.c_int), ("box", Box), ("rc", ctypes.c_float), ("skin", ctypes.c_float),
                ("max_neighbors", ctypes.c_int), ("bits", ctypes.c_int), ("F", ctypes.c_int), ("flags", ctypes.c_int),
                ("pos", ctypes.c_void_p), ("feat", ctypes.c_void_p), ("ws_sort", ctypes.c_void_p),
                ("ws_sort_bytes", ctypes.c_size_t), ("ws_list", ctypes.c_void_p), ("ws_list_bytes", ctypes.c_size_t),
                ("perm", ctypes.c_void_p), ("keys", ctypes.c_void_p), ("pos_sorted", ctypes.c_void_p),
                ("pos_cur", ctypes.c_void_p), ("nbr", ctypes.c_void_p), ("counts", ctypes.c_void_p),
                ("overflow", ctypes.c_void_p), ("sort_status", ctypes.c_void_p), ("rebuild", ctypes.c_void_p),
                ("max_disp2", ctypes.c_void_p), ("control", ctypes.c_void_p), ("out", ctypes.c_void_p)]


def _box(box) -> Box:
    if isinstance(box, Box):
        return box
    lx, ly, lz = (float(v) for v in box)
    return Box(lx, ly, lz)


# ------------------------------------------------------------------ raw C names


def tess_status_string(code: int) -> str:
    return lib().tess_status_string(int(code)).decode()


def tess_version() -> str:
    return lib().tess_version().decode()


def tess_kernel_launch_count() -> int:
    return int(lib().tess_kernel_launch_count())


def tess_hilbert_sort_workspace(n: int) -> int:
    return int(lib().tess_hilbert_sort_workspace(int(n)))


def tess_step_graph_create(buffers, stream, out) -> int:
    return int(lib().tess_step_graph_create(buffers, stream, out))


def tess_step_graph_launch(graph, stream) -> int:
    return int(lib().tess_step_graph_launch(graph, stream))


def tess_step_graph_request_rebuild(buffers, stream) -> int:
    return int(lib().tess_step_graph_request_rebuild(buffers, stream))


def tess_step_graph_destroy(graph) -> None:
    lib().tess_step_graph_destroy(graph)


def tess_debug_lookback_timeout_workspace() -> int:
    return int(lib().tess_debug_lookback_timeout_workspace())


def tess_debug_lookback_timeout(ws, ws_bytes, dev_status, stream) -> int:
    return int(lib().tess_debug_lookback_timeout(ws, ws_bytes, dev_status, stream))


def tess_min_pair_distance_workspace() -> int:
    return int(lib().tess_min_pair_distance_workspace())


def tess_min_pair_distance(pos, n, box, nbr, counts, max_neighbors, ws, ws_bytes, min_r2, min_pair, stream) -> int:
    return int(lib().tess_min_pair_distance(pos, n, _box(box), nbr, counts, max_neighbors, ws, ws_bytes, min_r2,
                                            min_pair, stream))


def tess_hilbert_resort_workspace(n: int) -> int:
    return int(lib().tess_hilbert_resort_workspace(int(n)))


def tess_hilbert_resort(pos, n, box, bits, perm_prev, keys_prev, ws, ws_bytes, perm, keys_sorted, pos_sorted,
                        dev_status, stream) -> int:
    return int(lib().tess_hilbert_resort(pos, n, _box(box), bits, perm_prev, keys_prev, ws, ws_bytes, perm,
                                         keys_sorted, pos_sorted, dev_status, stream))


def tess_hilbert_sort(pos, n, box, bits, ws, ws_bytes, perm, keys_sorted, pos_sorted, dev_status, stream) -> int:
    return int(lib().tess_hilbert_sort(pos, n, _box(box), bits, ws, ws_bytes, perm, keys_sorted, pos_sorted,
                                       dev_status, stream))


def tess_morton_sort(pos, n, box, bits, ws, ws_bytes, perm, keys_sorted, pos_sorted, dev_status, stream) -> int:
    return int(lib().tess_morton_sort(pos, n, _box(box), bits, ws, ws_bytes, perm, keys_sorted, pos_sorted,
                                      dev_status, stream))


def tess_hilbert_sort_static(pos, n, box, bits, perm, keys_sorted, pos_sorted, dev_status, stream) -> int:
    """Allocation-free Hilbert sort: the scratch lives inside the library
    (for up to HILBERT_SORT_STATIC_MAX_N atoms), for callers that cannot
    allocate device memory or lend a workspace."""
    return int(lib().tess_hilbert_sort_static(pos, n, _box(box), bits, perm, keys_sorted, pos_sorted, dev_status,
                                              stream))


def tess_build_neighbors_workspace(n, box, rc, skin) -> int:
    return int(lib().tess_build_neighbors_workspace(int(n), _box(box), float(rc), float(skin)))


def tess_build_neighbors(pos, n, box, rc, skin, max_neighbors, flags, ws, ws_bytes, nbr, counts, overflow,
                         stream) -> int:
    return int(lib().tess_build_neighbors(pos, n, _box(box), rc, skin, max_neighbors, flags, ws, ws_bytes, nbr,
                                          counts, overflow, stream))


def tess_skin_check(pos, pos_ref, n, box, skin, rebuild, max_disp2, stream) -> int:
    return int(lib().tess_skin_check(pos, pos_ref, n, _box(box), skin, rebuild, max_disp2, stream))


def tess_edge_aggregate(pos, n, box, rc, nbr, counts, max_neighbors, feat, F, out, edge_vec, edge_fc, edge_unit,
                        stream) -> int:
    return int(lib().tess_edge_aggregate(pos, n, _box(box), rc, nbr, counts, max_neighbors, feat, F, out, edge_vec,
                                         edge_fc, edge_unit, stream))


def tess_edge_aggregate_backward(pos, n, box, rc, nbr, counts, max_neighbors, feat, grad_out, F, grad_feat, grad_pos,
                                 stream) -> int:
    return int(lib().tess_edge_aggregate_backward(pos, n, _box(box), rc, nbr, counts, max_neighbors, feat, grad_out,
                                                  F, grad_feat, grad_pos, stream))


def tess_stage_timing(enable: bool) -> None:
    lib().tess_stage_timing(1 if enable else 0)


def tess_stage_times() -> dict:
    """{stage name: (total ms, calls)} since the last read (synchronises)."""
    ms = (ctypes.c_double * len(STAGES))()
    calls = (ctypes.c_longlong * len(STAGES))()
    k = lib().tess_stage_times(ctypes.cast(ms, ctypes.c_void_p), ctypes.cast(calls, ctypes.c_void_p), len(STAGES))
    return {STAGES[i]: (float(ms[i]), int(calls[i])) for i in range(k)}


# ------------------------------------------------------------------ torch layer


def _torch():
    import torch
    return torch


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need_cuda(name, t, dtype=None, shape_tail=None):
    torch = _torch()
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor (no CPU path)" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if dtype is not None and t.dtype != dtype:
        raise ValueError("%s must be %s" % (name, dtype))
    if shape_tail is not None and (t.dim() != 2 or t.shape[1] != shape_tail):
        raise ValueError("%s must be [n, %d]" % (name, shape_tail))


def _check(fn, code):
    if code != 0:
        raise TessError(fn, code)


def _workspace(nbytes, device, ws=None):
    torch = _torch()
    if ws is not None and ws.numel() * ws.element_size() >= nbytes:
        return ws
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


def hilbert_sort(pos, box, bits: int = 10, *, ws=None, perm=None, keys_sorted=None, pos_sorted=None,
                 dev_status=None, want_keys: bool = True, want_pos: bool = True, stream=None, curve: str = "hilbert"):
    """Order atoms along the 3-D Hilbert curve.  ``pos``: float32 [n, 3]
    CUDA tensor.  Returns (perm int32 [n], keys uint32->int32 view [n] or
    None, pos_sorted float32 [n, 4] or None, dev_status int32 [1])."""
    torch = _torch()
    _need_cuda("pos", pos, torch.float32, 3)
    n = pos.shape[0]
    dev = pos.device
    ws = _workspace(tess_hilbert_sort_workspace(n), dev, ws)
    perm = torch.empty(n, dtype=torch.int32, device=dev) if perm is None else perm
    if want_keys and keys_sorted is None:
        keys_sorted = torch.empty(n, dtype=torch.int32, device=dev)
    if want_pos and pos_sorted is None:
        pos_sorted = torch.empty((n, 4), dtype=torch.float32, device=dev)
    dev_status = torch.empty(1, dtype=torch.int32, device=dev) if dev_status is None else dev_status
    fn = tess_hilbert_sort if curve == "hilbert" else tess_morton_sort
    code = fn(_ptr(pos), n, box, bits, _ptr(ws), ws.numel() * ws.element_size(), _ptr(perm), _ptr(keys_sorted),
              _ptr(pos_sorted), _ptr(dev_status), _stream(stream))
    _check(fn.__name__, code)
    return perm, keys_sorted, pos_sorted, dev_status


def hilbert_resort(pos, box, perm_prev, keys_prev, bits: int = 10, *, ws=None, perm=None, keys_sorted=None,
                   pos_sorted=None, dev_status=None, want_pos: bool = True, stream=None):
    """Re-sort after the atoms moved, starting from an earlier sort's (perm,
    keys).  Same outputs as hilbert_sort for the same ``pos``; dev_status
    carries TESS_DEV_FULL_SORT when the full sort ran instead of the
    incremental one."""
    torch = _torch()
    _need_cuda("pos", pos, torch.float32, 3)
    _need_cuda("perm_prev", perm_prev, torch.int32)
    _need_cuda("keys_prev", keys_prev, torch.int32)
    n = pos.shape[0]
    dev = pos.device
    ws = _workspace(tess_hilbert_resort_workspace(n), dev, ws)
    perm = torch.empty(n, dtype=torch.int32, device=dev) if perm is None else perm
    keys_sorted = torch.empty(n, dtype=torch.int32, device=dev) if keys_sorted is None else keys_sorted
    if want_pos and pos_sorted is None:
        pos_sorted = torch.empty((n, 4), dtype=torch.float32, device=dev)
    dev_status = torch.empty(1, dtype=torch.int32, device=dev) if dev_status is None else dev_status
    code = tess_hilbert_resort(_ptr(pos), n, box, bits, _ptr(perm_prev), _ptr(keys_prev), _ptr(ws),
                               ws.numel() * ws.element_size(), _ptr(perm), _ptr(keys_sorted), _ptr(pos_sorted),
                               _ptr(dev_status), _stream(stream))
    _check("tess_hilbert_resort", code)
    return perm, keys_sorted, pos_sorted, dev_status


def morton_sort(pos, box, bits: int = 10, **kw):
    """Order atoms along the Morton (Z-order) curve; same outputs as hilbert_sort."""
    return hilbert_sort(pos, box, bits, curve="morton", **kw)


def build_neighbors(pos4, box, rc: float, skin: float, max_neighbors: int, *, pad_fill: bool = True,
                    search: str = "default", ws=None, nbr=None, counts=None, overflow=None, stream=None):
    """Padded Verlet list at rc + skin.  ``pos4``: float32 [n, 4] CUDA
    tensor.  Returns (nbr int32 [n, cap], counts int32 [n], overflow int32 [1])."""
    torch = _torch()
    _need_cuda("pos4", pos4, torch.float32, 4)
    n = pos4.shape[0]
    dev = pos4.device
    ws = _workspace(tess_build_neighbors_workspace(n, box, rc, skin), dev, ws)
    nbr = torch.empty((n, max_neighbors), dtype=torch.int32, device=dev) if nbr is None else nbr
    counts = torch.empty(n, dtype=torch.int32, device=dev) if counts is None else counts
    overflow = torch.empty(1, dtype=torch.int32, device=dev) if overflow is None else overflow
    flags = (0 if pad_fill else TESS_NO_PAD_FILL) | SEARCH_FLAGS[search]
    code = tess_build_neighbors(_ptr(pos4), n, box, float(rc), float(skin), int(max_neighbors), flags, _ptr(ws),
                                ws.numel() * ws.element_size(), _ptr(nbr), _ptr(counts), _ptr(overflow),
                                _stream(stream))
    _check("tess_build_neighbors", code)
    return nbr, counts, overflow


def skin_check(pos4, ref4, box, skin: float, *, rebuild=None, max_disp2=None, stream=None):
    """Rebuild flag (int32 [1]) and max squared displacement (float64 [1])."""
    torch = _torch()
    _need_cuda("pos4", pos4, torch.float32, 4)
    _need_cuda("ref4", ref4, torch.float32, 4)
    if pos4.shape != ref4.shape:
        raise ValueError("pos4 and ref4 must have the same shape")
    dev = pos4.device
    rebuild = torch.empty(1, dtype=torch.int32, device=dev) if rebuild is None else rebuild
    max_disp2 = torch.empty(1, dtype=torch.float64, device=dev) if max_disp2 is None else max_disp2
    code = tess_skin_check(_ptr(pos4), _ptr(ref4), pos4.shape[0], box, float(skin), _ptr(rebuild), _ptr(max_disp2),
                           _stream(stream))
    _check("tess_skin_check", code)
    return rebuild, max_disp2


def edge_aggregate(pos4, box, rc: float, nbr, counts, feat, *, out=None, edges: bool = False, stream=None):
    """out[i] = sum_j f_c(|r_ij|) feat[j] over row i.  With ``edges`` also
    returns edge_vec [n, cap, 4], edge_fc [n, cap], edge_unit [n, cap, 4]."""
    torch = _torch()
    _need_cuda("pos4", pos4, torch.float32, 4)
    _need_cuda("nbr", nbr, torch.int32)
    _need_cuda("counts", counts, torch.int32)
    _need_cuda("feat", feat, torch.float32)
    n, cap = nbr.shape
    F = feat.shape[1]
    dev = pos4.device
    out = torch.empty((n, F), dtype=torch.float32, device=dev) if out is None else out
    ev = ef = eu = None
    if edges:
        ev = torch.empty((n, cap, 4), dtype=torch.float32, device=dev)
        ef = torch.empty((n, cap), dtype=torch.float32, device=dev)
        eu = torch.empty((n, cap, 4), dtype=torch.float32, device=dev)
    code = tess_edge_aggregate(_ptr(pos4), n, box, float(rc), _ptr(nbr), _ptr(counts), cap, _ptr(feat), F,
                               _ptr(out), _ptr(ev), _ptr(ef), _ptr(eu), _stream(stream))
    _check("tess_edge_aggregate", code)
    if edges:
        return out, ev, ef, eu
    return out


def edge_aggregate_backward(pos4, box, rc: float, nbr, counts, feat, grad_out, *, grad_feat=None, grad_pos=None,
                            stream=None):
    """(dL/dfeat [n, F], dL/dpos [n, 3]) given dL/dout, for a full symmetric
    list without overflow (the output of build_neighbors)."""
    torch = _torch()
    _need_cuda("pos4", pos4, torch.float32, 4)
    _need_cuda("nbr", nbr, torch.int32)
    _need_cuda("counts", counts, torch.int32)
    _need_cuda("feat", feat, torch.float32)
    _need_cuda("grad_out", grad_out, torch.float32)
    n, cap = nbr.shape
    F = feat.shape[1]
    dev = pos4.device
    grad_feat = torch.empty((n, F), dtype=torch.float32, device=dev) if grad_feat is None else grad_feat
    grad_pos = torch.empty((n, 3), dtype=torch.float32, device=dev) if grad_pos is None else grad_pos
    code = tess_edge_aggregate_backward(_ptr(pos4), n, box, float(rc), _ptr(nbr), _ptr(counts), cap, _ptr(feat),
                                        _ptr(grad_out), F, _ptr(grad_feat), _ptr(grad_pos), _stream(stream))
    _check("tess_edge_aggregate_backward", code)
    return grad_feat, grad_pos


def min_pair_distance(pos4, box, nbr, counts, *, ws=None, stream=None):
    """Closest listed pair: (min_r2 float64 [1], pair int32 [2]) on the device;
    (+inf, (-1, -1)) when nothing is listed."""
    torch = _torch()
    _need_cuda("pos4", pos4, torch.float32, 4)
    _need_cuda("nbr", nbr, torch.int32)
    _need_cuda("counts", counts, torch.int32)
    n, cap = nbr.shape
    dev = pos4.device
    ws = _workspace(tess_min_pair_distance_workspace(), dev, ws)
    r2 = torch.empty(1, dtype=torch.float64, device=dev)
    pair = torch.empty(2, dtype=torch.int32, device=dev)
    code = tess_min_pair_distance(_ptr(pos4), n, box, _ptr(nbr), _ptr(counts), cap, _ptr(ws),
                                  ws.numel() * ws.element_size(), _ptr(r2), _ptr(pair), _stream(stream))
    _check("tess_min_pair_distance", code)
    return r2, pair


class StepGraph:
    """One time step as a CUDA graph whose rebuild branch is decided on the
    device (tess_step_graph_*).  Owns its buffers (torch tensors) and a
    stream; write the step's positions into ``pos`` ([n, 3], original order)
    before each ``launch``.  After a launch: ``rebuild`` (1 when the step
    rebuilt), ``perm``, ``nbr``, ``counts``, ``out`` and the rest hold that
    step's state; ``rebuilds`` reads the device's rebuild counter."""

    def __init__(self, pos, box, rc: float, skin: float, max_neighbors: int, feat, *, bits: int = 10,
                 pad_fill: bool = True, stream=None):
        torch = _torch()
        _need_cuda("pos", pos, torch.float32, 3)
        _need_cuda("feat", feat, torch.float32)
        n, F = pos.shape[0], feat.shape[1]
        dev = pos.device
        self.stream = torch.cuda.Stream(device=dev) if stream is None else stream
        self.pos = pos.clone()
        self.feat = feat
        self.ws_sort = _workspace(tess_hilbert_sort_workspace(n), dev)
        self.ws_list = _workspace(tess_build_neighbors_workspace(n, box, rc, skin), dev)
        e = lambda *shape, dtype=torch.int32: torch.zeros(shape, dtype=dtype, device=dev)
        self.perm, self.keys = e(n), e(n)
        self.pos_sorted, self.pos_cur = e(n, 4, dtype=torch.float32), e(n, 4, dtype=torch.float32)
        self.nbr, self.counts = e(n, max_neighbors), e(n)
        self.overflow, self.sort_status, self.rebuild = e(1), e(1), e(1)
        self.max_disp2 = e(1, dtype=torch.float64)
        self.control = e(2)
        self.out = e(n, F, dtype=torch.float32)
        b = StepBuffers()
        b.n, b.box, b.rc, b.skin = n, _box(box), float(rc), float(skin)
        b.max_neighbors, b.bits, b.F, b.flags = max_neighbors, bits, F, 0 if pad_fill else TESS_NO_PAD_FILL
        for name in ("pos", "feat", "ws_sort", "ws_list", "perm", "keys", "pos_sorted", "pos_cur", "nbr", "counts",
                     "overflow", "sort_status", "rebuild", "max_disp2", "control", "out"):
            setattr(b, name, getattr(self, name).data_ptr())
        b.ws_sort_bytes = self.ws_sort.numel()
        b.ws_list_bytes = self.ws_list.numel()
        self._b = b
        self._g = ctypes.c_void_p()
        torch.cuda.synchronize(dev)
        code = tess_step_graph_create(ctypes.byref(b), ctypes.c_void_p(self.stream.cuda_stream), ctypes.byref(self._g))
        _check("tess_step_graph_create", code)

    def launch(self):
        _check("tess_step_graph_launch", tess_step_graph_launch(self._g, ctypes.c_void_p(self.stream.cuda_stream)))

    def request_rebuild(self):
        _check("tess_step_graph_request_rebuild",
               tess_step_graph_request_rebuild(ctypes.byref(self._b), ctypes.c_void_p(self.stream.cuda_stream)))

    @property
    def rebuilds(self) -> int:
        """Rebuilds since create (waits for the graph's stream)."""
        self.stream.synchronize()
        return int(self.control[1].item())

    def close(self):
        if self._g:
            self.stream.synchronize()
            tess_step_graph_destroy(self._g)
            self._g = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

