"""Parity metric shared by the GPU tests, the smoke check and the benchmark.

Floating-point outputs are compared per token, normwise:
    rel_t = ||y_t - y_ref_t||_inf / ||y_ref_t||_inf,
gated at max_t rel_t <= TOL over tokens whose normalisation is well
conditioned (kappa_t = sum_s |w_ts| / |sum_s w_ts| <= KAPPA_MAX; the excluded
count is reported and expected to be 0).  Elementwise relative error is
ill-posed here because output components cross zero.

TOL = 2e-3 is the stated bar for bf16 inputs with fp32 accumulation.
"""
from __future__ import annotations

import numpy as np

TOL = 2e-3
KAPPA_MAX = 8.0


def token_rel_err(y, y_ref, kappa=None):
    """(max per-token normwise relative error, excluded token count, tensor-wise error)."""
    y = np.asarray(y, dtype=np.float64).reshape(-1, np.shape(y)[-1])
    r = np.asarray(y_ref, dtype=np.float64).reshape(-1, np.shape(y_ref)[-1])
    num = np.abs(y - r).max(axis=1)
    den = np.abs(r).max(axis=1)
    rel = num / den
    keep = np.ones(rel.shape, bool)
    if kappa is not None:
        keep = np.asarray(kappa).reshape(-1) <= KAPPA_MAX
    tensor = float(np.abs(y - r).max() / np.abs(r).max())
    worst = float(rel[keep].max()) if keep.any() else 0.0
    if not np.all(np.isfinite(y)):
        worst = float("inf")
    return worst, int((~keep).sum()), tensor


def tensor_rel_err(g, g_ref):
    """max |g - g_ref| / max |g_ref| over a whole tensor (the gradients' metric:
    per-token norms of a gradient can be arbitrarily small, so the error is taken
    relative to the tensor's largest entry)."""
    g = np.asarray(g, dtype=np.float64)
    r = np.asarray(g_ref, dtype=np.float64)
    if not np.all(np.isfinite(g)):
        return float("inf")
    scale = np.abs(r).max()
    if scale == 0.0:   # an exactly zero reference (e.g. dq, dk at P = 1): absolute error
        return float(np.abs(g).max())
    return float(np.abs(g - r).max() / scale)
