"""Helpers shared by the GPU parity tests (test infrastructure)."""
from __future__ import annotations

import numpy as np

INT_MAX = np.iinfo(np.int32).max


def torch_cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch


def canon_rows(nbr: np.ndarray, counts: np.ndarray) -> np.ndarray:
    """Rows sorted ascending with -1 pads at the end (the oracle's form).
    Only the first min(count, cap) slots of a row are considered."""
    n, cap = nbr.shape
    m = np.minimum(counts, cap)
    slot = np.arange(cap)[None, :]
    g = np.where(slot < m[:, None], nbr, INT_MAX)
    g = np.sort(g, axis=1)
    return np.where(g == INT_MAX, -1, g).astype(np.int32)


def canon_rows_gpu(nbr, counts):
    """canon_rows computed with torch on the device, returned to the host."""
    torch = torch_cuda()
    n, cap = nbr.shape
    m = torch.clamp(counts, max=cap)
    slot = torch.arange(cap, device=nbr.device)[None, :]
    g = torch.where(slot < m[:, None], nbr, torch.full_like(nbr, INT_MAX))
    g, _ = torch.sort(g, dim=1)
    g = torch.where(g == INT_MAX, torch.full_like(g, -1), g)
    return g.cpu().numpy()


def agg_error(gpu_out: np.ndarray, ref: dict):
    """(worst condition-aware relative error, worst plain relative error over
    |ref| > 1e-3).  The condition-aware error divides by
    max(|ref|, sum_j f_c |h_j|), so that sums that cancel are not measured
    against their tiny result."""
    out = ref["out"]
    den = np.maximum(np.abs(out), ref["out_abs"])
    den = np.where(den == 0, 1.0, den)
    err = np.abs(gpu_out.astype(np.float64) - out) / den
    big = np.abs(out) > 1e-3
    plain = (np.abs(gpu_out.astype(np.float64) - out)[big] / np.abs(out[big])).max() if big.any() else 0.0
    return float(err.max()), float(plain)


def geometry_allowance(ref: dict, h: np.ndarray, nbr: np.ndarray, counts: np.ndarray, rc: float,
                       box) -> np.ndarray:
    """Per (row, feature): sum_j kappa_ij |h_j| with kappa_ij the change of
    f_c(r_ij) that the fp32 geometry of the list can cause.  In fp32 each
    minimum-image component carries up to 2^-23 L of rounding (the
    difference, then +-L), so r^2 carries up to 2^-22 (sqrt(3) r L + r^2) and
    f_c, whose slope in r^2 is f_c'(r) / (2 r), moves by up to
    |f_c'(r)| 2^-23 (sqrt(3) L + r).  r is the oracle's (fp64 from the fp32
    coordinates), f_c'(r) = -(pi / (2 rc)) sin(pi r / rc) for r < rc.
    Rows resting on edges just inside rc need this: there f_c -> 0 while
    its relative sensitivity to r grows without bound."""
    n, cap = nbr.shape
    r = ref["edge_vec"][..., 3]
    live = (np.arange(cap)[None, :] < np.minimum(counts, cap)[:, None]) & (nbr >= 0) & (r < rc)
    lmax = float(max(box))
    dfc = (np.pi / (2.0 * rc)) * np.abs(np.sin(np.pi * r / rc))
    kappa = np.where(live, dfc * 2.0 ** -23 * (np.sqrt(3.0) * lmax + r), 0.0)
    jj = np.where(live, nbr, 0)
    return (kappa[:, :, None] * np.abs(h.astype(np.float64))[jj]).sum(1)


def agg_error_geom(gpu_out: np.ndarray, ref: dict, allowance: np.ndarray):
    """agg_error after subtracting the fp32 geometry allowance from each
    element's difference (the 1e-5 bound then applies to what is left)."""
    out = ref["out"]
    den = np.maximum(np.abs(out), ref["out_abs"])
    den = np.where(den == 0, 1.0, den)
    diff = np.abs(gpu_out.astype(np.float64) - out)
    err = np.maximum(diff - allowance, 0.0) / den
    return float(err.max())
