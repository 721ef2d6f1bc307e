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
