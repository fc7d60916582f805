"""Dense assembly of chain / tree matrices for brute-force checks (tests only)."""
import numpy as np


def sym_lower(D):
    """Full symmetric block from the lower triangle (the library's reading)."""
    return np.tril(D) + np.swapaxes(np.tril(D, -1), -1, -2)


def chain_dense(diag, lower):
    L, b = diag.shape[0], diag.shape[-1]
    A = np.zeros((L * b, L * b))
    for i in range(L):
        A[i * b:(i + 1) * b, i * b:(i + 1) * b] = sym_lower(diag[i])
    for i in range(L - 1):
        A[(i + 1) * b:(i + 2) * b, i * b:(i + 1) * b] = lower[i]
        A[i * b:(i + 1) * b, (i + 1) * b:(i + 2) * b] = lower[i].T
    return A


def tree_dense(parent, diag, edge):
    n, b = diag.shape[0], diag.shape[-1]
    A = np.zeros((n * b, n * b))
    for v in range(n):
        A[v * b:(v + 1) * b, v * b:(v + 1) * b] = sym_lower(diag[v])
        p = parent[v]
        if p >= 0:
            A[p * b:(p + 1) * b, v * b:(v + 1) * b] = edge[v]
            A[v * b:(v + 1) * b, p * b:(p + 1) * b] = edge[v].T
    return A


def blk(M, i, j, b):
    return M[i * b:(i + 1) * b, j * b:(j + 1) * b]


def rel(x, ref):
    """Frobenius-norm relative error (absolute when the reference is zero)."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    nr = np.linalg.norm(ref)
    d = np.linalg.norm(x - ref)
    return d / nr if nr > 0 else d


def balanced_parent(n, k=2):
    p = np.array([-1] + [(v - 1) // k for v in range(1, n)], dtype=np.int32)
    return p


def path_parent(n):
    return np.array([-1] + list(range(n - 1)), dtype=np.int32)


def star_parent(n):
    return np.array([-1] + [0] * (n - 1), dtype=np.int32)
