"""CPU oracle for the block selected inverse -- TEST INFRASTRUCTURE ONLY.

Plain double-precision C (``selinv_oracle.c``) behind a NumPy front end.
Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import this package; the product path never does, and
the oracle shares no code with the CUDA library.

What it computes follows gabp-sparse-inv 0.3.2 (PyPI page), "Implemented and
tested kernels" -> Chain and Tree, and the "Quickstart" conventions: the
on-pattern blocks of A^-1 (G_diag, G_lower / G_edge), log det A from the same
factorisation, and the chain solve x = A^-1 r; then the rows beyond them:
Gaussian draws from the factor ("Gaussian sampling"), the cotangents of the
selected inverse ("Differentiable selected inverse", written from the dense
definition Ab = -A^-1 Gbar A^-1), the block lower-bidiagonal non-symmetric
case and its cotangents ("Non-symmetric selected inverse"), and general
block-sparse SPD patterns ("General sparse selected inverse": its own
minimum-degree symbolic elimination, then the dense inverse read on the fill,
and its solve x = A^-1 r).
The C file states each recursion or definition and every reading taken where
the pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "selinv_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB = os.path.join(_BUILD, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/_build/liboracle.so`` with gcc."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        os.makedirs(_BUILD, exist_ok=True)
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _bind(path):
    """Load an oracle shared library and declare its signatures."""
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    lib.oracle_chain.argtypes = [P, P, I64, I64, ctypes.c_int, P, P, P, P, P, P, P]
    lib.oracle_chain.restype = ctypes.c_int
    lib.oracle_tree.argtypes = [P, I64, I64, ctypes.c_int, P, P, P, P, P, P]
    lib.oracle_tree.restype = ctypes.c_int
    lib.oracle_chain_sample.argtypes = [P, P, I64, I64, ctypes.c_int, P, P, P, P, P]
    lib.oracle_chain_sample.restype = ctypes.c_int
    lib.oracle_tree_sample.argtypes = [P, I64, I64, ctypes.c_int, P, P, P, P, P, P]
    lib.oracle_tree_sample.restype = ctypes.c_int
    lib.oracle_chain_backward.argtypes = [P, P, I64, I64, ctypes.c_int, P, P, P, P, P]
    lib.oracle_chain_backward.restype = ctypes.c_int
    lib.oracle_tree_backward.argtypes = [P, I64, I64, ctypes.c_int, P, P, P, P, P, P, P]
    lib.oracle_tree_backward.restype = ctypes.c_int
    lib.oracle_bidiag.argtypes = [P, P, I64, I64, ctypes.c_int, P, P, P]
    lib.oracle_bidiag.restype = ctypes.c_int
    lib.oracle_bidiag_backward.argtypes = [P, P, I64, I64, ctypes.c_int, P, P, P, P, P]
    lib.oracle_bidiag_backward.restype = ctypes.c_int
    lib.oracle_spd_inverse.argtypes = [P, ctypes.c_int, P, P]
    lib.oracle_spd_inverse.restype = ctypes.c_int
    lib.oracle_threads.argtypes = []
    lib.oracle_threads.restype = ctypes.c_int
    return lib


def _load(lib=None):
    global _lib
    if lib is not None:
        return lib
    if _lib is None:
        _lib = _bind(build())
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def threads() -> int:
    """Number of OpenMP threads the oracle's batch loop runs on."""
    return int(_load().oracle_threads())


def chain(diag, lower, rhs=None, want_g=True, lib=None):
    """Selected inverse of block-tridiagonal SPD chains.

    diag [..., L, b, b] (lower triangle read), lower [..., L-1, b, b] with
    lower[i] = A_{i+1,i}; optional rhs [..., L, b].
    Returns dict with G_diag [..., L, b, b], G_lower [..., L-1, b, b],
    logdet [...], x [..., L, b] (if rhs), info [...] (-1 ok, else the first
    block whose Schur complement is not positive definite) and asym [...]
    (largest |G - G^T| of a diagonal block before symmetrisation).
    """
    diag = _f64(diag)
    lead = diag.shape[:-3]
    L, b = diag.shape[-3], diag.shape[-1]
    batch = int(np.prod(lead)) if lead else 1
    if lower is None or L == 1:
        lower = np.zeros(lead + (max(L - 1, 0), b, b))
    lower = _f64(lower)
    assert lower.shape == lead + (L - 1, b, b)
    G_diag = np.empty(lead + (L, b, b)) if want_g else None
    G_lower = np.empty(lead + (L - 1, b, b)) if want_g else None
    logdet = np.empty(lead)
    info = np.empty(lead, dtype=np.int32)
    asym = np.zeros(lead)
    x = None
    if rhs is not None:
        rhs = _f64(rhs)
        assert rhs.shape == lead + (L, b)
        x = np.empty(lead + (L, b))
    rc = _load(lib).oracle_chain(_ptr(diag), _ptr(lower) if L > 1 else None, batch, L, b,
                              _ptr(G_diag), _ptr(G_lower), _ptr(logdet), _ptr(rhs), _ptr(x),
                              _ptr(info), _ptr(asym))
    if rc != 0:
        raise ValueError("oracle_chain: invalid arguments")
    return {"G_diag": G_diag, "G_lower": G_lower, "logdet": logdet, "x": x,
            "info": info, "asym": asym}


def chain_sample(diag, lower, z, rhs=None, lib=None):
    """Gaussian draw from the chain's own Cholesky factor A = L L^T:
    eta = L^-T z (+ A^-1 rhs when rhs is given).

    z [..., L, b] are the caller's standard normals.  Returns dict with eta
    [..., L, b], logdet [...] and info [...] (-1 ok, else the first block
    whose Schur complement is not positive definite).
    """
    diag = _f64(diag)
    lead = diag.shape[:-3]
    L, b = diag.shape[-3], diag.shape[-1]
    batch = int(np.prod(lead)) if lead else 1
    if lower is None or L == 1:
        lower = np.zeros(lead + (max(L - 1, 0), b, b))
    lower = _f64(lower)
    z = _f64(z)
    assert z.shape == lead + (L, b)
    if rhs is not None:
        rhs = _f64(rhs)
        assert rhs.shape == lead + (L, b)
    eta = np.empty(lead + (L, b))
    logdet = np.empty(lead)
    info = np.empty(lead, dtype=np.int32)
    rc = _load(lib).oracle_chain_sample(_ptr(diag), _ptr(lower) if L > 1 else None, batch, L, b,
                                        _ptr(rhs), _ptr(z), _ptr(eta), _ptr(logdet), _ptr(info))
    if rc != 0:
        raise ValueError("oracle_chain_sample: invalid arguments")
    return {"eta": eta, "logdet": logdet, "info": info}


def chain_backward(diag, lower, Gb_diag, Gb_lower, lib=None):
    """Cotangents of the chain's selected inverse: given the cotangents Gb_diag
    [..., L, b, b] on G_diag and Gb_lower [..., L-1, b, b] on G_lower, returns
    dict with Db [..., L, b, b] (lower-triangular: the forward reads only D's
    lower triangle), Bb [..., L-1, b, b] and info [...].  Dense definition,
    Ab = -A^-1 Gbar A^-1 (gabp-sparse-inv, "Differentiable selected inverse")."""
    diag = _f64(diag)
    lead = diag.shape[:-3]
    L, b = diag.shape[-3], diag.shape[-1]
    batch = int(np.prod(lead)) if lead else 1
    Gb_diag = _f64(Gb_diag)
    assert Gb_diag.shape == diag.shape
    Db = np.empty(lead + (L, b, b))
    info = np.empty(lead, dtype=np.int32)
    Bb = lower_ = None
    if L == 1:
        Gb_lower = None
    else:
        lower_ = _f64(lower)
        Gb_lower = _f64(Gb_lower)
        assert lower_.shape == lead + (L - 1, b, b) and Gb_lower.shape == lower_.shape
        Bb = np.empty(lead + (L - 1, b, b))
    rc = _load(lib).oracle_chain_backward(_ptr(diag), _ptr(lower_), batch, L, b, _ptr(Gb_diag),
                                          _ptr(Gb_lower), _ptr(Db), _ptr(Bb), _ptr(info))
    if rc != 0:
        raise ValueError("oracle_chain_backward: invalid arguments")
    return {"Db": Db, "Bb": Bb if Bb is not None else np.empty(lead + (0, b, b)), "info": info}


def tree_backward(parent, diag, edge, Gb_diag, Gb_edge, lib=None):
    """Cotangents of the tree selected inverse: from Gb_diag, Gb_edge [..., n, b, b]
    (cotangents of G_diag, G_edge; the root's edge slot is ignored), returns dict
    with Db (lower-triangular), Eb (root slot 0) and info [...].  Dense
    definition Ab = -A^-1 Gbar A^-1 (gabp-sparse-inv, "Differentiable selected
    inverse")."""
    parent = np.ascontiguousarray(parent, dtype=np.int32)
    diag, edge = _f64(diag), _f64(edge)
    Gb_diag, Gb_edge = _f64(Gb_diag), _f64(Gb_edge)
    lead = parent.shape[:-1]
    n = parent.shape[-1]
    b = diag.shape[-1]
    trees = int(np.prod(lead)) if lead else 1
    for a in (diag, edge, Gb_diag, Gb_edge):
        assert a.shape == lead + (n, b, b)
    Db = np.empty(lead + (n, b, b))
    Eb = np.empty(lead + (n, b, b))
    info = np.empty(lead, dtype=np.int32)
    rc = _load(lib).oracle_tree_backward(_ptr(parent), trees, n, b, _ptr(diag), _ptr(edge), _ptr(Gb_diag),
                                         _ptr(Gb_edge), _ptr(Db), _ptr(Eb), _ptr(info))
    if rc != 0:
        raise ValueError("oracle_tree_backward: invalid arguments")
    return {"Db": Db, "Eb": Eb, "info": info}


def bidiag(diag, lower, lib=None):
    """Selected inverse of block lower-bidiagonal matrices (general blocks):
    diag [..., L, b, b] = M_ii, lower [..., L-1, b, b] = M_{i+1,i}.  Returns
    dict with G_diag = (M^-1)_ii, G_lower = (M^-1)_{i+1,i} and info [...]
    (-1 ok, else the block of the first zero pivot).  Dense definition with
    partial pivoting (gabp-sparse-inv, "Non-symmetric selected inverse")."""
    diag = _f64(diag)
    lead = diag.shape[:-3]
    L, b = diag.shape[-3], diag.shape[-1]
    batch = int(np.prod(lead)) if lead else 1
    G_diag = np.empty(lead + (L, b, b))
    G_lower = np.empty(lead + (max(L - 1, 0), b, b))
    info = np.empty(lead, dtype=np.int32)
    lower = _f64(lower) if L > 1 else None
    if L > 1:
        assert lower.shape == lead + (L - 1, b, b)
    rc = _load(lib).oracle_bidiag(_ptr(diag), _ptr(lower), batch, L, b, _ptr(G_diag),
                                  _ptr(G_lower) if L > 1 else None, _ptr(info))
    if rc != 0:
        raise ValueError("oracle_bidiag: invalid arguments")
    return {"G_diag": G_diag, "G_lower": G_lower, "info": info}


def bidiag_backward(diag, lower, Gb_diag, Gb_lower, lib=None):
    """Cotangents of the non-symmetric chain: from Gb_diag, Gb_lower (cotangents
    of G_diag, G_lower) returns dict with Mb_diag, Mb_lower and info.  Dense
    definition Mb = -G^T Gbar G^T (gabp-sparse-inv, selinv_bidiag's backward)."""
    diag = _f64(diag)
    lead = diag.shape[:-3]
    L, b = diag.shape[-3], diag.shape[-1]
    batch = int(np.prod(lead)) if lead else 1
    Gb_diag = _f64(Gb_diag)
    assert Gb_diag.shape == diag.shape
    Mb_diag = np.empty(lead + (L, b, b))
    Mb_lower = np.empty(lead + (max(L - 1, 0), b, b))
    info = np.empty(lead, dtype=np.int32)
    lower_ = Gb_l = None
    if L > 1:
        lower_, Gb_l = _f64(lower), _f64(Gb_lower)
        assert lower_.shape == lead + (L - 1, b, b) and Gb_l.shape == lower_.shape
    rc = _load(lib).oracle_bidiag_backward(_ptr(diag), _ptr(lower_), batch, L, b, _ptr(Gb_diag), _ptr(Gb_l),
                                           _ptr(Mb_diag), _ptr(Mb_lower) if L > 1 else None, _ptr(info))
    if rc != 0:
        raise ValueError("oracle_bidiag_backward: invalid arguments")
    return {"Mb_diag": Mb_diag, "Mb_lower": Mb_lower, "info": info}


def junction_symbolic(n, edge_index, order=None):
    """Elimination order and filled pattern of a block graph (gabp-sparse-inv,
    "General sparse selected inverse (junction tree)": the pattern completed to
    its chordal fill S = pattern(L + L^T) by a min-degree elimination order).

    edge_index [2, m] holds the lower blocks (i, j), i > j.  Without `order`
    the order is greedy minimum degree on the elimination graph, ties going
    to the smaller node index.  Eliminating v joins its remaining neighbours
    into a clique.  Returns (order [n], S_index [2, nnz_S]) with S_index the
    pairs (i, j), i > j, of S sorted by j, then i."""
    ei = [int(x) for x in edge_index[0]]
    ej = [int(x) for x in edge_index[1]]
    adj = [set() for _ in range(n)]
    for i, j in zip(ei, ej):
        adj[i].add(j)
        adj[j].add(i)
    remaining = set(range(n))
    seq = []
    S = set((max(i, j), min(i, j)) for i, j in zip(ei, ej))
    given = None if order is None else [int(v) for v in order]
    for step in range(n):
        if given is None:
            v = min(remaining, key=lambda u: (len(adj[u]), u))
        else:
            v = given[step]
        nb = sorted(adj[v])
        for a in nb:                           # clique of the remaining neighbours
            for c in nb:
                if a < c and c not in adj[a]:
                    adj[a].add(c)
                    adj[c].add(a)
                    S.add((c, a))
        for a in nb:
            adj[a].discard(v)
        adj[v] = set()
        remaining.discard(v)
        seq.append(v)
    Sl = sorted(S, key=lambda p: (p[1], p[0]))
    return np.array(seq, dtype=np.int32), np.array(Sl, dtype=np.int64).T.reshape(2, -1)


def junction(diag, edge_index, edge_val, order=None, lib=None):
    """Selected inverse of a general block-sparse SPD matrix on its filled
    pattern S (gabp-sparse-inv, "General sparse selected inverse"): diag
    [..., n, b, b] (lower triangle read), edge_val [..., m, b, b] = A_{i,j} for
    the pairs (i, j), i > j, of edge_index.  Written from the definition: the
    dense A^-1 (textbook Cholesky) read on S.  Returns dict with G_diag,
    S_index, G_lower [..., nnz_S, b, b] (A^-1)_{i,j}, logdet, info (-1, or
    the node holding the first failing pivot in natural order)."""
    diag = _f64(diag)
    edge_val = _f64(edge_val)
    lead = diag.shape[:-3]
    n, b = diag.shape[-3], diag.shape[-1]
    ei = np.asarray(edge_index[0], dtype=np.int64)
    ej = np.asarray(edge_index[1], dtype=np.int64)
    _, S = junction_symbolic(n, np.stack([ei, ej]), order)
    batch = int(np.prod(lead)) if lead else 1
    d2 = diag.reshape(batch, n, b, b)
    e2 = edge_val.reshape(batch, len(ei), b, b)
    G_diag = np.zeros((batch, n, b, b))
    G_lower = np.zeros((batch, S.shape[1], b, b))
    logdet = np.zeros(batch)
    info = np.full(batch, -1, dtype=np.int32)
    N = n * b
    for e in range(batch):
        A = np.zeros((N, N))
        for v in range(n):
            A[v * b:(v + 1) * b, v * b:(v + 1) * b] = np.tril(d2[e, v]) + np.tril(d2[e, v], -1).T
        for k, (i, j) in enumerate(zip(ei, ej)):
            A[i * b:(i + 1) * b, j * b:(j + 1) * b] = e2[e, k]
            A[j * b:(j + 1) * b, i * b:(i + 1) * b] = e2[e, k].T
        A = np.ascontiguousarray(A)
        inv = np.empty((N, N))
        ld = np.zeros(1)
        rc = _load(lib).oracle_spd_inverse(_ptr(A), N, _ptr(inv), _ptr(ld))
        if rc != 0:
            info[e] = (rc - 1) // b
            continue
        logdet[e] = ld[0]
        for v in range(n):
            G_diag[e, v] = inv[v * b:(v + 1) * b, v * b:(v + 1) * b]
        for k in range(S.shape[1]):
            i, j = int(S[0, k]), int(S[1, k])
            G_lower[e, k] = inv[i * b:(i + 1) * b, j * b:(j + 1) * b]
    return {"G_diag": G_diag.reshape(lead + (n, b, b)), "S_index": S,
            "G_lower": G_lower.reshape(lead + (S.shape[1], b, b)), "logdet": logdet.reshape(lead),
            "info": info.reshape(lead)}


def junction_solve(diag, edge_index, edge_val, rhs, lib=None):
    """x = A^-1 r for general block-sparse SPD matrices (gabp-sparse-inv,
    "General sparse selected inverse": junction_solve from the same
    factorisation), written from the definition: the dense matrix assembled
    as in ``junction`` (D_v read on its lower triangle, A_{i,j} = edge_val[k]
    at (i, j) and transposed at (j, i)), its dense inverse by the textbook
    Cholesky route, times r.  diag [..., n, b, b], edge_val [..., m, b, b],
    rhs [..., n, b].  Returns dict with x [..., n, b], logdet, info (-1, or
    the node holding the first failing pivot in natural order)."""
    diag, edge_val, rhs = _f64(diag), _f64(edge_val), _f64(rhs)
    lead = diag.shape[:-3]
    n, b = diag.shape[-3], diag.shape[-1]
    ei = np.asarray(edge_index[0], dtype=np.int64)
    ej = np.asarray(edge_index[1], dtype=np.int64)
    batch = int(np.prod(lead)) if lead else 1
    d2 = diag.reshape(batch, n, b, b)
    e2 = edge_val.reshape(batch, len(ei), b, b)
    r2 = rhs.reshape(batch, n * b)
    x = np.zeros((batch, n * b))
    logdet = np.zeros(batch)
    info = np.full(batch, -1, dtype=np.int32)
    N = n * b
    for e in range(batch):
        A = np.zeros((N, N))
        for v in range(n):
            A[v * b:(v + 1) * b, v * b:(v + 1) * b] = np.tril(d2[e, v]) + np.tril(d2[e, v], -1).T
        for k, (i, j) in enumerate(zip(ei, ej)):
            A[i * b:(i + 1) * b, j * b:(j + 1) * b] = e2[e, k]
            A[j * b:(j + 1) * b, i * b:(i + 1) * b] = e2[e, k].T
        A = np.ascontiguousarray(A)
        inv = np.empty((N, N))
        ld = np.zeros(1)
        rc = _load(lib).oracle_spd_inverse(_ptr(A), N, _ptr(inv), _ptr(ld))
        if rc != 0:
            info[e] = (rc - 1) // b
            continue
        logdet[e] = ld[0]
        x[e] = inv @ r2[e]
    return {"x": x.reshape(lead + (n, b)), "logdet": logdet.reshape(lead), "info": info.reshape(lead)}


def junction_backward(diag, edge_index, edge_val, Gb_diag, Gb_lower, order=None, lib=None):
    """Cotangents of the general sparse selected inverse (gabp-sparse-inv,
    "General sparse selected inverse": selinv_junction's gradients reach diag
    and edge_val).  Gb_diag [..., n, b, b] and Gb_lower [..., nnz_S, b, b] are
    the cotangents of G_diag and of G_lower on S (junction_symbolic's S for the
    same order).  The dense definition Ab = -A^-1 Gbar A^-1 (Gbar holding
    Gb_lower[k] at (S_i[k], S_j[k])) is read back onto what the forward reads:
    Db = the lower-triangle projection of Ab_vv, and for input block k at
    (i, j), sitting at (i, j) and transposed at (j, i), Eb[k] = Ab_{i,j} +
    (Ab_{j,i})^T.  Returns dict with Db, Eb, info."""
    diag, edge_val = _f64(diag), _f64(edge_val)
    Gb_diag, Gb_lower = _f64(Gb_diag), _f64(Gb_lower)
    lead = diag.shape[:-3]
    n, b = diag.shape[-3], diag.shape[-1]
    ei = np.asarray(edge_index[0], dtype=np.int64)
    ej = np.asarray(edge_index[1], dtype=np.int64)
    _, S = junction_symbolic(n, np.stack([ei, ej]), order)
    batch = int(np.prod(lead)) if lead else 1
    d2 = diag.reshape(batch, n, b, b)
    e2 = edge_val.reshape(batch, len(ei), b, b)
    gd2 = Gb_diag.reshape(batch, n, b, b)
    gl2 = Gb_lower.reshape(batch, S.shape[1], b, b)
    Db = np.zeros((batch, n, b, b))
    Eb = np.zeros((batch, len(ei), b, b))
    info = np.full(batch, -1, dtype=np.int32)
    N = n * b
    for e in range(batch):
        A = np.zeros((N, N))
        Gbar = np.zeros((N, N))
        for v in range(n):
            A[v * b:(v + 1) * b, v * b:(v + 1) * b] = np.tril(d2[e, v]) + np.tril(d2[e, v], -1).T
            Gbar[v * b:(v + 1) * b, v * b:(v + 1) * b] = gd2[e, v]
        for k, (i, j) in enumerate(zip(ei, ej)):
            A[i * b:(i + 1) * b, j * b:(j + 1) * b] = e2[e, k]
            A[j * b:(j + 1) * b, i * b:(i + 1) * b] = e2[e, k].T
        for k in range(S.shape[1]):
            i, j = int(S[0, k]), int(S[1, k])
            Gbar[i * b:(i + 1) * b, j * b:(j + 1) * b] = gl2[e, k]
        A = np.ascontiguousarray(A)
        inv = np.empty((N, N))
        ld = np.zeros(1)
        rc = _load(lib).oracle_spd_inverse(_ptr(A), N, _ptr(inv), _ptr(ld))
        if rc != 0:
            info[e] = (rc - 1) // b
            continue
        Ab = -(inv @ Gbar @ inv)
        for v in range(n):
            blkv = Ab[v * b:(v + 1) * b, v * b:(v + 1) * b]
            Db[e, v] = np.tril(blkv + blkv.T, -1) + np.diag(np.diag(blkv))
        for k, (i, j) in enumerate(zip(ei, ej)):
            Eb[e, k] = Ab[i * b:(i + 1) * b, j * b:(j + 1) * b] + Ab[j * b:(j + 1) * b, i * b:(i + 1) * b].T
    return {"Db": Db.reshape(lead + (n, b, b)), "Eb": Eb.reshape(lead + (len(ei), b, b)),
            "info": info.reshape(lead)}


def tree(parent, diag, edge, lib=None):
    """Selected inverse of block-tree SPD matrices.

    parent [..., n] int (root = -1), diag [..., n, b, b], edge [..., n, b, b]
    with edge[v] = A_{parent(v),v} (root slot ignored).  Returns dict with
    G_diag, G_edge (root slot 0), logdet [...] and info [...] (-1 ok, node of
    a failing pivot, or -2 for a parent array that is not one rooted tree).
    """
    diag = _f64(diag)
    edge = _f64(edge)
    parent = np.ascontiguousarray(parent, dtype=np.int32)
    lead = parent.shape[:-1]
    n, b = diag.shape[-3], diag.shape[-1]
    trees = int(np.prod(lead)) if lead else 1
    assert diag.shape == lead + (n, b, b) and edge.shape == diag.shape
    G_diag = np.empty_like(diag)
    G_edge = np.empty_like(diag)
    logdet = np.empty(lead)
    info = np.empty(lead, dtype=np.int32)
    rc = _load(lib).oracle_tree(_ptr(parent), trees, n, b, _ptr(diag), _ptr(edge),
                             _ptr(G_diag), _ptr(G_edge), _ptr(logdet), _ptr(info))
    if rc != 0:
        raise ValueError("oracle_tree: invalid arguments")
    return {"G_diag": G_diag, "G_edge": G_edge, "logdet": logdet, "info": info}


def tree_sample(parent, diag, edge, z, lib=None):
    """Gaussian draw w = L^-T z on block trees (A = L L^T in the tree's own
    elimination order, children before parents).  parent [trees, n], diag /
    edge [trees, n, b, b], z [trees, n, b].  Returns dict with eta [trees, n, b],
    logdet [trees], info [trees] (-1 ok, a failing node, or -2 for a malformed tree)."""
    parent = np.ascontiguousarray(parent, dtype=np.int32)
    diag, edge, z = _f64(diag), _f64(edge), _f64(z)
    trees, n = parent.shape
    b = diag.shape[-1]
    assert diag.shape == (trees, n, b, b) and edge.shape == (trees, n, b, b) and z.shape == (trees, n, b)
    w = np.empty((trees, n, b))
    logdet = np.empty(trees)
    info = np.empty(trees, dtype=np.int32)
    rc = _load(lib).oracle_tree_sample(_ptr(parent), trees, n, b, _ptr(diag), _ptr(edge), _ptr(z), _ptr(w),
                                       _ptr(logdet), _ptr(info))
    if rc != 0:
        raise ValueError("oracle_tree_sample: invalid arguments")
    return {"eta": w, "logdet": logdet, "info": info}
