"""Parity rule between the GPU's fp16 output and the fp64 oracle.

An element passes iff |g - o| <= 2e-3 AND |g - o| / max(|o|, 1e-3) <= 1e-2
(max-abs 2e-3 and max-rel 1e-2 on fp16 outputs; the relative error is taken
against max(|o|, 1e-3) so that it stays defined for outputs near zero).
"""
from __future__ import annotations

import numpy as np

ABS_TOL = 2e-3
REL_TOL = 1e-2
REL_FLOOR = 1e-3


def parity_errors(gpu, ref):
    g = np.asarray(gpu, dtype=np.float64)
    o = np.asarray(ref, dtype=np.float64)
    assert g.shape == o.shape, (g.shape, o.shape)
    err = np.abs(g - o)
    rel = err / np.maximum(np.abs(o), REL_FLOOR)
    return err, rel


def assert_parity(gpu, ref, what=""):
    g = np.asarray(gpu, dtype=np.float64)
    assert np.all(np.isfinite(g)), f"{what}: non-finite GPU output"
    err, rel = parity_errors(gpu, ref)
    bad = (err > ABS_TOL) | (rel > REL_TOL)
    if bad.any():
        idx = np.unravel_index(np.argmax(rel), rel.shape)
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} elements out of tolerance; "
            f"max abs {err.max():.3e}, max rel {rel.max():.3e} at {idx} "
            f"(gpu {np.asarray(gpu, dtype=np.float64)[idx]:.6e}, oracle {np.asarray(ref)[idx]:.6e})")
    return float(err.max()) if err.size else 0.0, float(rel.max()) if rel.size else 0.0
