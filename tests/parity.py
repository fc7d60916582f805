"""GPU-vs-oracle comparison helpers (tests only).

The error metric is per block: every b x b block of a block array (the last
two axes) and every length-b segment of a vector (the last axis) is compared
with the oracle's on its own, ||X_blk - X_ref_blk||_F / den, where den is the
block's own Frobenius norm floored at FLOOR times the largest block norm of
the same batch element (blocks far from the diagonal of A^-1, or zero slots
such as a tree's root edge, would otherwise divide by almost nothing).  A test
passes when the largest ratio over blocks, batch elements and arrays is within
the tolerance (1e-9 float64, 1e-4 float32).  log det uses |d| / max(1, |ref|).
"""
import numpy as np
import torch

TOL = {torch.float64: 1e-9, torch.float32: 1e-4}
FLOOR = 1e-3


def rel_per_block(x, ref, lead_ndim=1, block_ndim=2):
    """Relative error of every block: array of shape lead + (blocks,)."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    assert ref.ndim >= lead_ndim + block_ndim, (ref.shape, lead_ndim, block_ndim)
    lead = ref.shape[:lead_ndim]
    bsz = int(np.prod(ref.shape[ref.ndim - block_ndim:]))
    nblk = int(np.prod(ref.shape[lead_ndim:ref.ndim - block_ndim]))
    d = (x - ref).reshape(lead + (nblk, bsz))
    r = ref.reshape(lead + (nblk, bsz))
    num = np.sqrt((d ** 2).sum(axis=-1))
    den = np.sqrt((r ** 2).sum(axis=-1))
    if nblk:
        den = np.maximum(den, FLOOR * den.max(axis=-1, keepdims=True))
    return np.where(den > 0, num / np.where(den > 0, den, 1), num)


def worst(x, ref, lead_ndim=1, block_ndim=2):
    """Largest per-block relative error; block_ndim=2 for b x b (or b x k)
    blocks, 1 for length-b segments of a vector."""
    r = rel_per_block(x, ref, lead_ndim, block_ndim)
    return float(np.max(r)) if r.size else 0.0


def worst_vec(x, ref, lead_ndim=1):
    """Largest per-segment relative error of a vector [lead..., L, b]."""
    return worst(x, ref, lead_ndim, block_ndim=1)


def logdet_err(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.max(np.abs(x - ref) / np.maximum(1.0, np.abs(ref)))) if ref.size else 0.0


def to_dev(a, dtype, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(a)).to(device=device, dtype=dtype)


def host(t):
    return t.detach().cpu().numpy()
