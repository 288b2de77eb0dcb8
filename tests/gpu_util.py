"""Helpers shared by the GPU tests (no method arithmetic here)."""
import numpy as np
import torch


def rel_err(x, ref) -> float:
    """max |x - ref| / max |ref| (fp64)."""
    x = np.asarray(x.detach().cpu().double().numpy() if hasattr(x, "detach") else x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    denom = np.abs(ref).max()
    return float(np.abs(x - ref).max() / (denom if denom > 0 else 1.0))


def assert_close_rel(x, ref, tol, what=""):
    e = rel_err(x, ref)
    assert e <= tol, f"{what}: max|err|/max|ref| = {e:.3e} > {tol:.1e}"
    return e
