"""GPU-vs-oracle comparison helpers (tests only).

The error metric: per output array and batch element, ||X_gpu - X_ref||_F /
||X_ref||_F; a test passes when the largest over elements and arrays is
within the tolerance (1e-9 float64, 1e-4 float32).  log det uses
|d| / max(1, |ref|).
"""
import numpy as np
import torch

TOL = {torch.float64: 1e-9, torch.float32: 1e-4}


def rel_per_element(x, ref, lead_ndim):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    axes = tuple(range(lead_ndim, ref.ndim))
    num = np.sqrt(((x - ref) ** 2).sum(axis=axes))
    den = np.sqrt((ref ** 2).sum(axis=axes))
    return np.where(den > 0, num / np.where(den > 0, den, 1), num)


def worst(x, ref, lead_ndim=1):
    r = rel_per_element(x, ref, lead_ndim)
    return float(np.max(r)) if r.size else 0.0


def logdet_err(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.max(np.abs(x - ref) / np.maximum(1.0, np.abs(ref)))) if ref.size else 0.0


def to_dev(a, dtype, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(a)).to(device=device, dtype=dtype)


def host(t):
    return t.detach().cpu().numpy()
