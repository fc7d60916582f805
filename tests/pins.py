"""Pins of the CPU oracle to facts outside itself (tests only).

Each pin returns an error that must stay below its tolerance.  They are
written so that a plausible slip in the oracle (a dropped term, a wrong sign
or index, a transposed operand) breaks at least one of them; the mutant test
plants such slips in copies of the oracle's C source and checks exactly that.

Sources:
  gabp-sparse-inv 0.3.2 (PyPI page)
    "Quickstart": G_diag[0] equals inv(A)[0:4,0:4] to 1e-10 for 8 blocks of
      size 4 with diag_load 2.0; tree G_diag[0] likewise; the path tree
      reproduces the chain block-for-block (the chain roots the path at its
      last node, the tree at node 0).
    "junction_solve" / "junction_logdet": solve and log det equal the dense
      ones.
    "Tests": every kernel against a dense fp64 oracle, symmetry / SPD
      properties, independent residuals, leading batch dimensions.
  sparsax (PyPI page) "Quick start": the 3 x 3 SPD example; "Factor once, do
    everything": sample_gaussian draws eta = A^-1 b + P^T L^-T z from the
    Cholesky factor (gabp-sparse-inv "Gaussian sampling": the covariance is
    exactly A^-1, checked on the standard basis).
"""
import json
import math
import os
from fractions import Fraction

import numpy as np

import oracle
from sparse_spd_selected_b200 import inputs
from tests.dense import (balanced_parent, blk, chain_dense, path_parent, rel,
                         star_parent, sym_lower, tree_dense)

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _chain_vs_dense(diag, lower, rhs, lib):
    """Max relative error of every oracle output against the dense route."""
    out = oracle.chain(diag, lower, rhs, lib=lib)
    lead = diag.shape[:-3]
    L, b = diag.shape[-3], diag.shape[-1]
    worst = 0.0
    for idx in np.ndindex(*lead) if lead else [()]:
        if out["info"][idx] != -1:
            return math.inf
        A = chain_dense(diag[idx], lower[idx])
        inv = np.linalg.inv(A)
        for i in range(L):
            worst = max(worst, rel(out["G_diag"][idx][i], blk(inv, i, i, b)))
        for i in range(L - 1):
            worst = max(worst, rel(out["G_lower"][idx][i], blk(inv, i + 1, i, b)))
        sign, ld = np.linalg.slogdet(A)
        worst = max(worst, abs(out["logdet"][idx] - ld) / max(1.0, abs(ld)), 0.0 if sign > 0 else math.inf)
        if rhs is not None:
            worst = max(worst, rel(out["x"][idx].ravel(), np.linalg.solve(A, rhs[idx].ravel())))
    return worst


def pin_tiny_chains_dense(lib=None):
    """Brute force: tiny random chains (with leading batch dims) vs dense inverse/slogdet/solve."""
    worst = 0.0
    for (L, b, lead) in [(1, 1, ()), (1, 3, (2,)), (2, 1, (3,)), (2, 2, ()), (3, 3, (2, 3)),
                         (5, 2, (2,)), (6, 4, ()), (4, 5, (2,))]:
        E = int(np.prod(lead)) if lead else 1
        d, l, r = inputs.chain_inputs(E, L, b, seed=100 + L * 10 + b, load=0.3, with_rhs=True)
        d = d.reshape(lead + d.shape[1:]) if lead else d[0]
        l = l.reshape(lead + l.shape[1:]) if lead else l[0]
        r = r.reshape(lead + r.shape[1:]) if lead else r[0]
        worst = max(worst, _chain_vs_dense(d, l, r, lib))
    return worst


def pin_quickstart(lib=None):
    """Quickstart fact: G_diag[0] == inv(A)[0:4,0:4] (atol 1e-10) on 8 blocks of 4, load 2.0."""
    w = inputs.WORKLOADS["chain_1x8_b4"]
    g = inputs.generate(w)
    out = oracle.chain(g["diag"], g["lower"], g["rhs"], lib=lib)
    inv = np.linalg.inv(chain_dense(g["diag"][0], g["lower"][0]))
    return float(np.abs(out["G_diag"][0, 0] - inv[0:4, 0:4]).max())


def _frac_inverse(M):
    """Exact inverse and determinant of a small rational matrix (Gauss-Jordan in Fractions)."""
    n = len(M)
    A = [[Fraction(x) for x in row] + [Fraction(int(i == j)) for j in range(n)]
         for i, row in enumerate(M)]
    det = Fraction(1)
    for k in range(n):
        p = next(i for i in range(k, n) if A[i][k] != 0)
        if p != k:
            A[k], A[p] = A[p], A[k]
            det = -det
        det *= A[k][k]
        piv = A[k][k]
        A[k] = [x / piv for x in A[k]]
        for i in range(n):
            if i != k and A[i][k] != 0:
                f = A[i][k]
                A[i] = [x - f * y for x, y in zip(A[i], A[k])]
    return [row[n:] for row in A], det


def pin_sparsax_3x3(lib=None):
    """sparsax 'Quick start' 3x3 SPD matrix as a b=1, L=3 chain vs exact rational arithmetic."""
    g = json.load(open(os.path.join(GOLDEN, "sparsax_quickstart_3x3.json")))
    n = g["n"]
    A = [[0.0] * n for _ in range(n)]
    for i, j, v in zip(g["Ai"], g["Aj"], g["Ax"]):
        if i <= j:                        # the page: entries with Ai <= Aj are used
            A[i][j] = v
            A[j][i] = v
    inv, det = _frac_inverse(A)
    bvec = [Fraction(x) for x in g["b"]]
    xs = [sum(inv[i][k] * bvec[k] for k in range(n)) for i in range(n)]
    diag = np.array([[[A[i][i]]] for i in range(n)])
    lower = np.array([[[A[i + 1][i]]] for i in range(n - 1)])
    out = oracle.chain(diag, lower, np.array(g["b"]).reshape(n, 1), lib=lib)
    errs = [abs(out["G_diag"][i, 0, 0] - float(inv[i][i])) for i in range(n)]
    errs += [abs(out["G_lower"][i, 0, 0] - float(inv[i + 1][i])) for i in range(n - 1)]
    errs += [abs(out["x"][i, 0] - float(xs[i])) for i in range(n)]
    errs += [abs(out["logdet"] - math.log(det))]
    return float(max(errs))


def _laplacian_inverse(m):
    """(T^-1)_{ij} = min(i,j) (m+1-max(i,j)) / (m+1), 1-based, for T = tridiag(-1,2,-1)."""
    i = np.arange(1, m + 1)
    return np.minimum.outer(i, i) * (m + 1 - np.maximum.outer(i, i)) / (m + 1)


def pin_laplacian_closed_form(lib=None):
    """b=1 1-D Laplacian and its rotated block version vs the closed-form inverse and det = m+1."""
    worst = 0.0
    for m in [1, 2, 3, 7, 30]:
        Tinv = _laplacian_inverse(m)
        out = oracle.chain(np.full((m, 1, 1), 2.0), np.full((m - 1, 1, 1), -1.0), lib=lib)
        worst = max(worst, rel(out["G_diag"][:, 0, 0], np.diag(Tinv)))
        if m > 1:
            worst = max(worst, rel(out["G_lower"][:, 0, 0], np.diag(Tinv, -1)))
        worst = max(worst, abs(out["logdet"] - math.log(m + 1)))
    # Rotated block Laplacian: D_i = 2I, B_i = -Q_i with Q_i = U_{i+1} U_i^T (U_i orthogonal).
    # Then A = U (T kron I) U^T, so G_ii = (T^-1)_ii I, G_{i+1,i} = (T^-1)_{i+1,i} Q_i,
    # log det A = b log(m+1) and x = U (T^-1 kron I) U^T r.
    rng = np.random.default_rng(7)
    for m, b in [(5, 3), (9, 4)]:
        U = np.stack([np.linalg.qr(rng.standard_normal((b, b)))[0] for _ in range(m)])
        Q = np.matmul(U[1:], np.swapaxes(U[:-1], 1, 2))
        r = rng.standard_normal((m, b))
        Tinv = _laplacian_inverse(m)
        out = oracle.chain(np.broadcast_to(2 * np.eye(b), (m, b, b)).copy(), -Q, r, lib=lib)
        for i in range(m):
            worst = max(worst, rel(out["G_diag"][i], Tinv[i, i] * np.eye(b)))
        for i in range(m - 1):
            worst = max(worst, rel(out["G_lower"][i], Tinv[i + 1, i] * Q[i]))
        worst = max(worst, abs(out["logdet"] - b * math.log(m + 1)))
        Ur = np.einsum("iba,ib->ia", U, r)                # U_i^T r_i
        x = np.einsum("iab,ib->ia", U, Tinv @ Ur)         # U_i sum_j T^-1_ij U_j^T r_j
        worst = max(worst, rel(out["x"], x))
    return worst


def pin_decoupled(lib=None):
    """B = 0: G_ii = D_i^-1, G_lower = 0, log det = sum log det D_i, x_i = D_i^-1 r_i."""
    d, _, r = inputs.chain_inputs(2, 6, 5, seed=11, load=0.5, with_rhs=True)
    lower = np.zeros((2, 5, 5, 5))
    out = oracle.chain(d, lower, r, lib=lib)
    worst = float(np.abs(out["G_lower"]).max())
    for e in range(2):
        for i in range(6):
            worst = max(worst, rel(out["G_diag"][e, i], np.linalg.inv(d[e, i])))
            worst = max(worst, rel(out["x"][e, i], np.linalg.solve(d[e, i], r[e, i])))
        ld = sum(np.linalg.slogdet(d[e, i])[1] for i in range(6))
        worst = max(worst, abs(out["logdet"][e] - ld) / abs(ld))
    return worst


def grid_closed_form(m, tau, r=None, rows=None):
    """Spectral closed form of the m x m grid precision T kron I + I kron T + tau I.

    With T = S diag(mu) S^T, s_j(i) = sqrt(2/(m+1)) sin(j pi (i+1)/(m+1)),
    lambda_jk = tau + mu_j + mu_k:
      G_ii      = S diag_k( sum_j s_j(i)^2        / lambda_jk ) S^T
      G_{i+1,i} = S diag_k( sum_j s_j(i+1) s_j(i) / lambda_jk ) S^T
      log det   = sum_jk log lambda_jk,   X = S ((S^T R S) / lambda) S^T.
    Returns (G_diag [rows], G_lower [rows], logdet, x) for the requested block rows.
    """
    j = np.arange(1, m + 1)
    i = np.arange(m)
    S = math.sqrt(2.0 / (m + 1)) * np.sin(np.outer(i + 1, j) * math.pi / (m + 1))
    mu = 4.0 * np.sin(j * math.pi / (2 * (m + 1))) ** 2
    lam = tau + mu[:, None] + mu[None, :]
    rows = range(m) if rows is None else rows
    Gd, Gl = {}, {}
    for row in rows:
        wk = (S[row] ** 2) @ (1.0 / lam)
        Gd[row] = (S * wk) @ S.T
        if row + 1 < m:
            wk = (S[row + 1] * S[row]) @ (1.0 / lam)
            Gl[row] = (S * wk) @ S.T
    x = None
    if r is not None:
        x = S @ ((S.T @ r @ S) / lam) @ S.T
    return Gd, Gl, float(np.log(lam).sum()), x


def pin_grid_closed_form(lib=None, m=12):
    """Grid precision chain (D = tridiag(-1,4+tau,-1), B = -I) vs its spectral closed form."""
    diag, lower, rhs, tau = inputs.grid_inputs(2, m, seed=21)
    out = oracle.chain(diag, lower, rhs, lib=lib)
    worst = 0.0
    for e in range(2):
        Gd, Gl, ld, x = grid_closed_form(m, tau[e], rhs[e])
        for i in range(m):
            worst = max(worst, rel(out["G_diag"][e, i], Gd[i]))
        for i in range(m - 1):
            worst = max(worst, rel(out["G_lower"][e, i], Gl[i]))
        worst = max(worst, abs(out["logdet"][e] - ld) / abs(ld), rel(out["x"][e], x))
    return worst


def block_row_residual(diag, lower, G_diag, G_lower):
    """max_v || A_vv G_vv + sum_u A_vu G_uv - I ||_F for a chain, from on-pattern blocks only."""
    L, b = diag.shape[0], diag.shape[-1]
    D = np.tril(diag) + np.swapaxes(np.tril(diag, -1), -1, -2)
    worst = 0.0
    for v in range(L):
        R = D[v] @ G_diag[v] - np.eye(b)
        if v > 0:    # A_{v,v-1} = B_{v-1}, G_{v-1,v} = G_lower[v-1]^T
            R += lower[v - 1] @ G_lower[v - 1].T
        if v + 1 < L:  # A_{v,v+1} = B_v^T, G_{v+1,v} = G_lower[v]
            R += lower[v].T @ G_lower[v]
        worst = max(worst, np.linalg.norm(R))
    return worst


def pin_block_row_identity(lib=None):
    """A G = I restricted to block rows (on-pattern blocks suffice) at b=16, L=64, plus solve residual."""
    d, l, r = inputs.chain_inputs(2, 64, 16, seed=31, load=2.0, with_rhs=True)
    out = oracle.chain(d, l, r, lib=lib)
    worst = 0.0
    for e in range(2):
        worst = max(worst, block_row_residual(d[e], l[e], out["G_diag"][e], out["G_lower"][e]))
        A = chain_dense(d[e], l[e])
        worst = max(worst, np.linalg.norm(A @ out["x"][e].ravel() - r[e].ravel()) / np.linalg.norm(r[e]))
        # G_ii symmetric positive definite (Cholesky succeeds)
        for i in range(64):
            np.linalg.cholesky(out["G_diag"][e, i])
    return worst


def _tree_vs_dense(parent, diag, edge, lib):
    out = oracle.tree(parent, diag, edge, lib=lib)
    worst = 0.0
    E, n, b = diag.shape[0], diag.shape[1], diag.shape[-1]
    for e in range(E):
        if out["info"][e] != -1:
            return math.inf
        A = tree_dense(parent[e], diag[e], edge[e])
        inv = np.linalg.inv(A)
        for v in range(n):
            worst = max(worst, rel(out["G_diag"][e, v], blk(inv, v, v, b)))
            p = parent[e, v]
            if p >= 0:
                worst = max(worst, rel(out["G_edge"][e, v], blk(inv, p, v, b)))
            else:
                worst = max(worst, float(np.abs(out["G_edge"][e, v]).max()))
        ld = np.linalg.slogdet(A)[1]
        worst = max(worst, abs(out["logdet"][e] - ld) / max(1.0, abs(ld)))
    return worst


def pin_tiny_trees_dense(lib=None):
    """Brute force: random / path / star / balanced / re-rooted trees vs the dense inverse."""
    worst = 0.0
    for n, b in [(1, 2), (2, 1), (5, 2), (12, 3), (17, 2)]:
        rng = np.random.default_rng(n * 100 + b)
        parents = [inputs.random_parent(rng, n), path_parent(n), star_parent(n),
                   balanced_parent(n, 2), balanced_parent(n, 3)]
        # a tree rooted at its last node, with parents drawn among later indices
        pr = np.full(n, -1, dtype=np.int32)
        for v in range(n - 1):
            pr[v] = rng.integers(v + 1, n)
        parents.append(pr)
        P = np.stack(parents)
        diag, edge = inputs.tree_inputs_from_parent(P, b, seed=n + b, load=0.3)
        worst = max(worst, _tree_vs_dense(P, diag, edge, lib))
    return worst


def pin_tree_quickstart(lib=None):
    """Tree quickstart shape (12 nodes, b=3, random kind): G_diag[0] == inv[0:3,0:3] to 1e-10."""
    P, diag, edge = inputs.tree_inputs(1, 12, 3, seed=0, load=2.0)
    out = oracle.tree(P, diag, edge, lib=lib)
    inv = np.linalg.inv(tree_dense(P[0], diag[0], edge[0]))
    return float(np.abs(out["G_diag"][0, 0] - inv[0:3, 0:3]).max())


def pin_root_invariance(lib=None):
    """Path tree rooted at node 0 (eliminated in the reverse order) == chain rooted at its last node."""
    L, b = 40, 6
    d, l, _ = inputs.chain_inputs(1, L, b, seed=41, load=0.5, with_rhs=False)
    ch = oracle.chain(d, l, lib=lib)
    parent = path_parent(L)[None]
    edge = np.zeros((1, L, b, b))
    edge[0, 1:] = np.swapaxes(l[0], 1, 2)       # edge[v] = A_{v-1,v} = lower[v-1]^T
    tr = oracle.tree(parent, d, edge, lib=lib)
    worst = max(rel(tr["G_diag"][0, i], ch["G_diag"][0, i]) for i in range(L))
    worst = max(worst, max(rel(tr["G_edge"][0, v].T, ch["G_lower"][0, v - 1]) for v in range(1, L)))
    worst = max(worst, abs(tr["logdet"][0] - ch["logdet"][0]) / abs(ch["logdet"][0]))
    return worst


def pin_not_spd(lib=None):
    """A non-positive-definite Schur complement is reported at the first failing block."""
    d, l, _ = inputs.chain_inputs(3, 7, 3, seed=51, load=1.0, with_rhs=False)
    d[1, 4] = -np.eye(3)
    d[2, 0, 1, 1] = np.nan
    out = oracle.chain(d, l, lib=lib)
    ok = list(out["info"]) == [-1, 4, 0]
    P, td, te = inputs.tree_inputs(2, 9, 2, seed=52, load=1.0)
    td[1, 5] = -np.eye(2)
    tout = oracle.tree(P, td, te, lib=lib)
    ok = ok and tout["info"][0] == -1 and tout["info"][1] >= 0
    bad = P.copy()
    bad[0, 3] = -1                               # two roots
    bad[1, 2] = 2                                # self loop
    ok = ok and list(oracle.tree(bad, td, te, lib=lib)["info"]) == [-2, -2]
    return 0.0 if ok else 1.0


def pin_sample_standard_basis(lib=None):
    """Draws for z = e_k, k = 1..N, are the columns of L^-T with L = numpy's
    Cholesky factor of the dense A (so W is upper triangular), and W W^T = A^-1:
    the check the pages name for their sampler (the covariance is exactly A^-1
    on the standard basis).  Log det against slogdet."""
    worst = 0.0
    for L, b, seed in [(3, 2, 61), (4, 3, 62), (1, 4, 63), (5, 1, 64)]:
        d, l, _ = inputs.chain_inputs(1, L, b, seed=seed, load=1.0, with_rhs=False)
        A = chain_dense(d[0], l[0])
        N = L * b
        Z = np.eye(N).reshape(N, L, b)
        out = oracle.chain_sample(np.repeat(d, N, 0), np.repeat(l, N, 0), Z, lib=lib)
        W = out["eta"].reshape(N, N).T
        worst = max(worst, rel(W, np.linalg.inv(np.linalg.cholesky(A)).T))
        worst = max(worst, rel(W @ W.T, np.linalg.inv(A)))
        worst = max(worst, abs(out["logdet"][0] - np.linalg.slogdet(A)[1]) / max(1.0, abs(np.linalg.slogdet(A)[1])))
        if (out["info"] != -1).any():
            return float("inf")
    return worst


def pin_sample_mean(lib=None):
    """z = 0 gives the solve A^-1 r; with both, eta = A^-1 r + L^-T z (numpy's
    solve and Cholesky on the dense A)."""
    d, l, r = inputs.chain_inputs(2, 5, 3, seed=65, load=0.8, with_rhs=True)
    z = np.random.default_rng(66).standard_normal(r.shape)
    zero = oracle.chain_sample(d, l, np.zeros_like(r), rhs=r, lib=lib)
    both = oracle.chain_sample(d, l, z, rhs=r, lib=lib)
    worst = 0.0
    for e in range(2):
        A = chain_dense(d[e], l[e])
        mean = np.linalg.solve(A, r[e].ravel())
        draw = np.linalg.inv(np.linalg.cholesky(A)).T @ z[e].ravel()
        worst = max(worst, rel(zero["eta"][e].ravel(), mean))
        worst = max(worst, rel(both["eta"][e].ravel(), mean + draw))
    return worst


def _children_first(parent):
    """Reverse breadth-first order of a rooted tree (every child before its parent)."""
    n = len(parent)
    kids = [[] for _ in range(n)]
    root = int(np.where(parent < 0)[0][0])
    for v in range(n):
        if parent[v] >= 0:
            kids[parent[v]].append(v)
    order, head = [root], 0
    while head < len(order):
        order.extend(kids[order[head]])
        head += 1
    return order[::-1]


def pin_tree_sample_standard_basis(lib=None):
    """Tree draws for z = e_k against numpy's dense Cholesky of A in a
    children-first order (mapped back to node order), and W W^T = A^-1;
    log det against slogdet.  Path, star, balanced and random trees."""
    worst = 0.0
    rng = np.random.default_rng(67)
    cases = [path_parent(5), star_parent(5), balanced_parent(7), inputs.random_parent(rng, 9)]
    for k, parent in enumerate(cases):
        b = 2 if k % 2 else 3
        n = len(parent)
        P = parent[None]
        d, e = inputs.tree_inputs_from_parent(P, b, seed=68 + k, load=1.0)
        A = tree_dense(parent, d[0], e[0])
        N = n * b
        z = np.eye(N).reshape(N, n, b)
        out = oracle.tree_sample(np.repeat(P, N, 0), np.repeat(d, N, 0), np.repeat(e, N, 0), z, lib=lib)
        if (out["info"] != -1).any():
            return float("inf")
        W = out["eta"].reshape(N, N).T
        idx = np.concatenate([np.arange(v * b, (v + 1) * b) for v in _children_first(parent)])
        Mp = np.linalg.inv(np.linalg.cholesky(A[np.ix_(idx, idx)])).T
        ref = np.empty_like(Mp)
        ref[np.ix_(idx, idx)] = Mp
        worst = max(worst, rel(W, ref), rel(W @ W.T, np.linalg.inv(A)))
        sl = np.linalg.slogdet(A)[1]
        worst = max(worst, abs(out["logdet"][0] - sl) / max(1.0, abs(sl)))
    return worst


def _proj_lower(M):
    """What the forward's lower-triangle read makes of a cotangent on a full
    diagonal block: M + M^T below the diagonal, M on it, zero above."""
    return np.tril(M + M.T, -1) + np.diag(np.diag(M))


def pin_backward_finite_differences(lib=None):
    """Cotangents against central differences of the (pinned) forward oracle,
    entry by entry, upper entries of D included (they must get zero)."""
    worst = 0.0
    for L, b, seed in [(3, 2, 31), (2, 3, 32), (1, 2, 33)]:
        d, l, _ = inputs.chain_inputs(1, L, b, seed=seed, load=1.0, with_rhs=False)
        rng = np.random.default_rng(seed)
        gd, gl = rng.standard_normal(d.shape), rng.standard_normal(l.shape)
        out = oracle.chain_backward(d, l, gd, gl, lib=lib)
        if (out["info"] != -1).any():
            return float("inf")

        def loss(dd, ll):
            o = oracle.chain(dd, ll, lib=lib)
            return float((o["G_diag"] * gd).sum() + (o["G_lower"] * gl).sum())

        h = 1e-5
        scale = max(1.0, float(np.abs(out["Db"]).max()), float(np.abs(out["Bb"]).max()) if L > 1 else 0.0)
        for idx in np.ndindex(*d.shape):
            dp, dm = d.copy(), d.copy()
            dp[idx] += h
            dm[idx] -= h
            worst = max(worst, abs((loss(dp, l) - loss(dm, l)) / (2 * h) - out["Db"][idx]) / scale)
        for idx in np.ndindex(*l.shape):
            lp, lm = l.copy(), l.copy()
            lp[idx] += h
            lm[idx] -= h
            worst = max(worst, abs((loss(d, lp) - loss(d, lm)) / (2 * h) - out["Bb"][idx]) / scale)
    return worst


def pin_backward_decoupled(lib=None):
    """B = 0: A^-1 is block diagonal (blocks D_i^-1), so -A^-1 Gbar A^-1 has
    diagonal blocks -D_i^-1 Gb_ii D_i^-1 and blocks -D_{i+1}^-1 Gb_{i+1,i} D_i^-1
    below them (none above: Gbar has nothing there), hence Db_i =
    proj(-D_i^-1 Gb_ii D_i^-1) and Bb_i = -D_{i+1}^-1 Gb_{i+1,i} D_i^-1."""
    L, b = 5, 4
    d, _, _ = inputs.chain_inputs(2, L, b, seed=34, load=0.5, with_rhs=False)
    lower = np.zeros((2, L - 1, b, b))
    rng = np.random.default_rng(34)
    gd, gl = rng.standard_normal(d.shape), rng.standard_normal(lower.shape)
    out = oracle.chain_backward(d, lower, gd, gl, lib=lib)
    worst = 0.0
    for e in range(2):
        inv = [np.linalg.inv(sym_lower(d[e, i])) for i in range(L)]
        for i in range(L):
            worst = max(worst, rel(out["Db"][e, i], _proj_lower(-inv[i] @ gd[e, i] @ inv[i])))
        for i in range(L - 1):
            worst = max(worst, rel(out["Bb"][e, i], -inv[i + 1] @ gl[e, i] @ inv[i]))
    return worst


def pin_backward_trace(lib=None):
    """Loss = tr A^-1 (Gb_ii = I, Gb_lower = 0): dL/dA = -A^-2, so Db_i =
    proj(-(A^-2)_ii) and Bb_i = -2 (A^-2)_{i+1,i}."""
    L, b = 6, 3
    d, l, _ = inputs.chain_inputs(2, L, b, seed=35, load=1.0, with_rhs=False)
    gd = np.broadcast_to(np.eye(b), d.shape).copy()
    out = oracle.chain_backward(d, l, gd, np.zeros(l.shape), lib=lib)
    worst = 0.0
    for e in range(2):
        A2 = np.linalg.matrix_power(np.linalg.inv(chain_dense(d[e], l[e])), 2)
        for i in range(L):
            worst = max(worst, rel(out["Db"][e, i], _proj_lower(-blk(A2, i, i, b))))
        for i in range(L - 1):
            worst = max(worst, rel(out["Bb"][e, i], -2.0 * blk(A2, i + 1, i, b)))
    return worst


def pin_tree_backward_finite_differences(lib=None):
    """Tree cotangents against central differences of the (pinned) tree forward
    oracle, every entry of diag and of the non-root edge slots."""
    worst = 0.0
    for parent, b, seed in [(np.array([-1, 0, 0, 0]), 2, 41), (np.array([2, 0, -1, 1, 1]), 2, 42)]:
        P = parent[None].astype(np.int32)
        d, e = inputs.tree_inputs_from_parent(P, b, seed=seed, load=1.0)
        rng = np.random.default_rng(seed)
        gd, ge = rng.standard_normal(d.shape), rng.standard_normal(e.shape)
        out = oracle.tree_backward(P, d, e, gd, ge, lib=lib)
        if (out["info"] != -1).any():
            return float("inf")

        def loss(dd, ee):
            o = oracle.tree(P, dd, ee, lib=lib)
            return float((o["G_diag"] * gd).sum() + (o["G_edge"] * ge).sum())

        h = 1e-5
        scale = max(1.0, float(np.abs(out["Db"]).max()), float(np.abs(out["Eb"]).max()))
        for idx in np.ndindex(*d.shape):
            dp, dm = d.copy(), d.copy()
            dp[idx] += h
            dm[idx] -= h
            worst = max(worst, abs((loss(dp, e) - loss(dm, e)) / (2 * h) - out["Db"][idx]) / scale)
        for idx in np.ndindex(*e.shape):
            if parent[idx[1]] < 0:
                worst = max(worst, abs(out["Eb"][idx]))      # the root slot gets nothing
                continue
            ep, em = e.copy(), e.copy()
            ep[idx] += h
            em[idx] -= h
            worst = max(worst, abs((loss(d, ep) - loss(d, em)) / (2 * h) - out["Eb"][idx]) / scale)
    return worst


def pin_tree_backward_path_is_chain(lib=None):
    """The path tree parent(i) = i + 1 is the chain (rooted at its last node):
    its cotangents equal the chain backward's block for block."""
    L, b = 7, 3
    d, l, _ = inputs.chain_inputs(2, L, b, seed=43, load=1.0, with_rhs=False)
    rng = np.random.default_rng(43)
    gd, gl = rng.standard_normal(d.shape), rng.standard_normal(l.shape)
    ref = oracle.chain_backward(d, l, gd, gl, lib=lib)
    parent = np.repeat(np.array(list(range(1, L)) + [-1], dtype=np.int32)[None], 2, 0)
    edge = np.zeros(d.shape)
    edge[:, :L - 1] = l
    ge = np.zeros(d.shape)
    ge[:, :L - 1] = gl
    ge[:, L - 1] = rng.standard_normal((2, b, b))        # the root slot's cotangent is ignored
    out = oracle.tree_backward(parent, d, edge, gd, ge, lib=lib)
    if (out["info"] != -1).any() or (ref["info"] != -1).any():
        return float("inf")
    return max(rel(out["Db"], ref["Db"]), rel(out["Eb"][:, :L - 1], ref["Bb"]),
               float(np.abs(out["Eb"][:, L - 1]).max()))


def _bidiag_dense(d, l):
    L, b = d.shape[0], d.shape[-1]
    M = np.zeros((L * b, L * b))
    for i in range(L):
        M[i * b:(i + 1) * b, i * b:(i + 1) * b] = d[i]
    for i in range(L - 1):
        M[(i + 1) * b:(i + 2) * b, i * b:(i + 1) * b] = l[i]
    return M


def pin_bidiag_dense(lib=None):
    """Non-symmetric chain blocks against numpy's inverse of the dense M, and
    against the pages' block formula G_{i+1,i} = -M_{i+1,i+1}^-1 M_{i+1,i} M_ii^-1;
    blocks with a zero diagonal force row exchanges."""
    worst = 0.0
    cases = [inputs.bidiag_inputs(2, 6, 3, seed=51, load=2.0), inputs.bidiag_inputs(1, 1, 4, seed=52, load=2.0)]
    d, l = inputs.bidiag_inputs(1, 4, 2, seed=53, load=0.0)
    d[0, :] = np.array([[0.0, 1.5], [-2.0, 0.3]])           # zero pivot in column 0 without exchanges
    cases.append((d, l))
    for d, l in cases:
        out = oracle.bidiag(d, l, lib=lib)
        if (out["info"] != -1).any():
            return float("inf")
        L, b = d.shape[1], d.shape[-1]
        for e in range(d.shape[0]):
            inv = np.linalg.inv(_bidiag_dense(d[e], l[e]))
            for i in range(L):
                worst = max(worst, rel(out["G_diag"][e, i], blk(inv, i, i, b)))
            for i in range(L - 1):
                worst = max(worst, rel(out["G_lower"][e, i], blk(inv, i + 1, i, b)))
                formula = -np.linalg.inv(d[e, i + 1]) @ l[e, i] @ np.linalg.inv(d[e, i])
                worst = max(worst, rel(out["G_lower"][e, i], formula))
    return worst


def pin_bidiag_scalar_exact(lib=None):
    """b = 1 in exact rationals: G_ii = 1/m_i, G_{i+1,i} = -l_i / (m_i m_{i+1})."""
    m = [Fraction(3), Fraction(-2), Fraction(5, 2), Fraction(7)]
    lo = [Fraction(1), Fraction(-4), Fraction(3, 2)]
    out = oracle.bidiag(np.array([[[[float(x)]] for x in m]]), np.array([[[[float(x)]] for x in lo]]), lib=lib)
    worst = 0.0
    for i, x in enumerate(m):
        worst = max(worst, abs(out["G_diag"][0, i, 0, 0] - float(1 / x)) / abs(float(1 / x)))
    for i, x in enumerate(lo):
        ref = float(-x / (m[i] * m[i + 1]))
        worst = max(worst, abs(out["G_lower"][0, i, 0, 0] - ref) / abs(ref))
    return worst


def pin_bidiag_singular(lib=None):
    """A singular diagonal block is reported as that block; others are fine."""
    d, l = inputs.bidiag_inputs(2, 5, 3, seed=54, load=2.0)
    d[1, 3] = np.array([[1.0, 2.0, 3.0], [2.0, 4.0, 6.0], [0.5, -1.0, 2.0]])   # rank 2
    out = oracle.bidiag(d, l, lib=lib)
    return 0.0 if (out["info"][0] == -1 and out["info"][1] == 3) else float("inf")


def pin_bidiag_backward_finite_differences(lib=None):
    """Non-symmetric chain cotangents against central differences of the
    (pinned) forward oracle, every entry of M_ii and M_{i+1,i}."""
    worst = 0.0
    for L, b, seed in [(3, 2, 61), (2, 3, 62), (1, 2, 63)]:
        d, l = inputs.bidiag_inputs(1, L, b, seed=seed, load=2.0)
        rng = np.random.default_rng(seed)
        gd, gl = rng.standard_normal(d.shape), rng.standard_normal(l.shape)
        out = oracle.bidiag_backward(d, l, gd, gl, lib=lib)
        if (out["info"] != -1).any():
            return float("inf")

        def loss(dd, ll):
            o = oracle.bidiag(dd, ll, lib=lib)
            return float((o["G_diag"] * gd).sum() + (o["G_lower"] * gl).sum())

        h = 1e-5
        scale = max(1.0, float(np.abs(out["Mb_diag"]).max()))
        for idx in np.ndindex(*d.shape):
            dp, dm = d.copy(), d.copy()
            dp[idx] += h
            dm[idx] -= h
            worst = max(worst, abs((loss(dp, l) - loss(dm, l)) / (2 * h) - out["Mb_diag"][idx]) / scale)
        for idx in np.ndindex(*l.shape):
            lp, lm = l.copy(), l.copy()
            lp[idx] += h
            lm[idx] -= h
            worst = max(worst, abs((loss(d, lp) - loss(d, lm)) / (2 * h) - out["Mb_lower"][idx]) / scale)
    return worst


def pin_bidiag_backward_scalar_exact(lib=None):
    """b = 1 in exact rationals: with g_i = 1/m_i and h_i = -l_i g_i g_{i+1},
    Mb_ii = -(g_i^2 Gd_i + h_i Gl_i g_i + g_i Gl_{i-1} h_{i-1}) and
    Mb_{i+1,i} = -g_{i+1} Gl_i g_i (dG = -G dM G, written out by hand)."""
    m = [Fraction(3), Fraction(-2), Fraction(5, 2)]
    lo = [Fraction(1), Fraction(-4)]
    gd = [Fraction(1, 2), Fraction(-3), Fraction(2)]
    gl = [Fraction(5), Fraction(1, 3)]
    g = [1 / x for x in m]
    h = [-lo[i] * g[i] * g[i + 1] for i in range(2)]
    out = oracle.bidiag_backward(np.array([[[[float(x)]] for x in m]]), np.array([[[[float(x)]] for x in lo]]),
                                 np.array([[[[float(x)]] for x in gd]]), np.array([[[[float(x)]] for x in gl]]),
                                 lib=lib)
    worst = 0.0
    for i in range(3):
        ref = -(g[i] * g[i] * gd[i] + (h[i] * gl[i] * g[i] if i < 2 else 0) +
                (g[i] * gl[i - 1] * h[i - 1] if i > 0 else 0))
        worst = max(worst, abs(out["Mb_diag"][0, i, 0, 0] - float(ref)) / abs(float(ref)))
    for i in range(2):
        ref = -g[i + 1] * gl[i] * g[i]
        worst = max(worst, abs(out["Mb_lower"][0, i, 0, 0] - float(ref)) / abs(float(ref)))
    return worst


def _graph_dense(n, b, ei, ej, d, e):
    A = np.zeros((n * b, n * b))
    for v in range(n):
        A[v * b:(v + 1) * b, v * b:(v + 1) * b] = sym_lower(d[v])
    for k, (i, j) in enumerate(zip(ei, ej)):
        A[i * b:(i + 1) * b, j * b:(j + 1) * b] = e[k]
        A[j * b:(j + 1) * b, i * b:(i + 1) * b] = e[k].T
    return A


def pin_junction_dense(lib=None):
    """General sparse SPD (the pages' 3 x 3 grid with blocks of 2, a random
    graph): every block on S against numpy's inverse, log det against slogdet,
    and S strictly larger than the input pattern (fill)."""
    worst = 0.0
    rng = np.random.default_rng(71)
    cases = [(9, 2, inputs.grid_edges(3, 3))]
    pairs = sorted({(max(a, c), min(a, c)) for a, c in rng.integers(0, 12, (20, 2)) if a != c})
    cases.append((12, 3, np.array(pairs).T))
    for n, b, E in cases:
        d, e = inputs.graph_inputs(2, n, b, E, seed=72, load=1.0)
        out = oracle.junction(d, E, e, lib=lib)
        if (out["info"] != -1).any() or out["S_index"].shape[1] <= E.shape[1]:
            return float("inf")
        for k in range(2):
            A = _graph_dense(n, b, E[0], E[1], d[k], e[k])
            inv = np.linalg.inv(A)
            for v in range(n):
                worst = max(worst, rel(out["G_diag"][k, v], blk(inv, v, v, b)))
            for s_, (i, j) in enumerate(out["S_index"].T):
                worst = max(worst, rel(out["G_lower"][k, s_], blk(inv, int(i), int(j), b)))
            sl = np.linalg.slogdet(A)[1]
            worst = max(worst, abs(out["logdet"][k] - sl) / abs(sl))
    return worst


def pin_junction_symbolic(lib=None):
    """Minimum-degree elimination and fill on graphs worked by hand: the 4-cycle
    (all degrees 2: node 0 first, joining 1 and 3: one fill block (3, 1)); a
    star (leaves first, no fill); a path (no fill)."""
    o, S = oracle.junction_symbolic(4, np.array([[1, 2, 3, 3], [0, 1, 2, 0]]))
    bad = o.tolist() != [0, 1, 2, 3] or S.T.tolist() != [[1, 0], [3, 0], [2, 1], [3, 1], [3, 2]]
    o, S = oracle.junction_symbolic(6, np.array([[1, 2, 3, 4, 5], [0, 0, 0, 0, 0]]))
    bad |= o.tolist() != [1, 2, 3, 4, 0, 5] or S.shape[1] != 5
    o, S = oracle.junction_symbolic(5, np.array([[1, 2, 3, 4], [0, 1, 2, 3]]))
    bad |= o.tolist() != [0, 1, 2, 3, 4] or S.shape[1] != 4
    return float("inf") if bad else 0.0


def pin_junction_tree_and_order(lib=None):
    """Zero fill on a tree: S is the input pattern and the blocks equal the
    (pinned) tree oracle's; another elimination order changes S but not the
    blocks of A^-1 on the input pattern."""
    parent = np.array([-1, 0, 0, 1, 1, 2, 5, 5])
    n, b = parent.size, 3
    P = parent[None].astype(np.int32)
    d, edge = inputs.tree_inputs_from_parent(P, b, seed=73, load=1.0)
    kids = [v for v in range(n) if parent[v] >= 0]
    E = np.array([[max(v, parent[v]) for v in kids], [min(v, parent[v]) for v in kids]])
    # edge[v] = A_{p(v), v}; the junction input holds A_{i,j} with i > j
    vals = np.stack([edge[0, v] if parent[v] > v else edge[0, v].T for v in kids])[None]
    out = oracle.junction(d, E, vals, lib=lib)
    ref = oracle.tree(P, d, edge, lib=lib)
    worst = rel(out["G_diag"], ref["G_diag"])
    if out["S_index"].shape[1] != E.shape[1]:
        return float("inf")
    for s_, (i, j) in enumerate(out["S_index"].T):
        v = int(i) if parent[int(i)] == int(j) else int(j)          # the child of the pair
        g = ref["G_edge"][0, v]                                      # (A^-1)_{p(v), v}
        worst = max(worst, rel(out["G_lower"][0, s_], g if parent[v] > v else g.T))
    rev = oracle.junction(d, E, vals, order=np.arange(n)[::-1], lib=lib)
    worst = max(worst, rel(rev["G_diag"], out["G_diag"]))
    Sr = {(int(i), int(j)): s_ for s_, (i, j) in enumerate(rev["S_index"].T)}
    for s_, (i, j) in enumerate(out["S_index"].T):
        worst = max(worst, rel(rev["G_lower"][0, Sr[(int(i), int(j))]], out["G_lower"][0, s_]))
    return worst


def pin_junction_backward_finite_differences(lib=None):
    """General sparse cotangents against central differences of the (pinned)
    junction forward oracle on the pages' 3 x 3 grid; the fill blocks of S
    carry cotangents too."""
    E = inputs.grid_edges(3, 3)
    d, e = inputs.graph_inputs(1, 9, 2, E, seed=81, load=1.0)
    _, S = oracle.junction_symbolic(9, E)
    rng = np.random.default_rng(81)
    gd, gl = rng.standard_normal(d.shape), rng.standard_normal((1, S.shape[1], 2, 2))
    out = oracle.junction_backward(d, E, e, gd, gl, lib=lib)
    if (out["info"] != -1).any():
        return float("inf")

    def loss(dd, ee):
        o = oracle.junction(dd, E, ee, lib=lib)
        return float((o["G_diag"] * gd).sum() + (o["G_lower"] * gl).sum())

    h = 1e-5
    scale = max(1.0, float(np.abs(out["Db"]).max()), float(np.abs(out["Eb"]).max()))
    worst = 0.0
    for idx in np.ndindex(*d.shape):
        dp, dm = d.copy(), d.copy()
        dp[idx] += h
        dm[idx] -= h
        worst = max(worst, abs((loss(dp, e) - loss(dm, e)) / (2 * h) - out["Db"][idx]) / scale)
    for idx in np.ndindex(*e.shape):
        ep, em = e.copy(), e.copy()
        ep[idx] += h
        em[idx] -= h
        worst = max(worst, abs((loss(d, ep) - loss(d, em)) / (2 * h) - out["Eb"][idx]) / scale)
    return worst


def pin_junction_backward_path_is_chain(lib=None):
    """On a path pattern (pairs (i + 1, i)) the general sparse cotangents are
    the (pinned) chain backward's."""
    L, b = 6, 3
    cd, cl, _ = inputs.chain_inputs(1, L, b, seed=82, load=1.0, with_rhs=False)
    rng = np.random.default_rng(82)
    cgd, cgl = rng.standard_normal(cd.shape), rng.standard_normal(cl.shape)
    P = np.array([np.arange(1, L), np.arange(L - 1)])
    jb = oracle.junction_backward(cd, P, cl, cgd, cgl, lib=lib)
    cb = oracle.chain_backward(cd, cl, cgd, cgl, lib=lib)
    return max(rel(jb["Db"], cb["Db"]), rel(jb["Eb"], cb["Bb"]))


def pin_junction_solve(lib=None):
    """The general sparse solve x = A^-1 r: on a path pattern (pairs (i + 1,
    i)) it is the (pinned) chain oracle's solve; without edges each block row
    is its own system, x_v = D_v^-1 r_v (numpy's solve of each symmetric
    D_v); on a random pattern the block residual sum_u A_vu x_u - r_v
    vanishes and log det equals the (pinned) selected inverse's."""
    worst = 0.0
    L, b = 7, 3
    cd, cl, cr = inputs.chain_inputs(2, L, b, seed=83, load=1.0)
    P = np.array([np.arange(1, L), np.arange(L - 1)])
    js = oracle.junction_solve(cd, P, cl, cr, lib=lib)
    ch = oracle.chain(cd, cl, cr, want_g=False, lib=lib)
    worst = max(worst, rel(js["x"], ch["x"]), float(np.max(np.abs(js["logdet"] - ch["logdet"]))))
    n = 5
    d, e = inputs.graph_inputs(1, n, b, np.zeros((2, 0), dtype=np.int64), seed=84, load=1.0)
    r = np.random.default_rng(84).standard_normal((1, n, b))
    js = oracle.junction_solve(d, np.zeros((2, 0), dtype=np.int64), e, r, lib=lib)
    for v in range(n):
        Dv = np.tril(d[0, v]) + np.tril(d[0, v], -1).T
        worst = max(worst, rel(js["x"][0, v], np.linalg.solve(Dv, r[0, v])))
    n, m = 12, 25
    rng = np.random.default_rng(85)
    pairs = sorted({(max(a, c), min(a, c)) for a, c in rng.integers(0, n, (m, 2)) if a != c})
    E = np.array(pairs, dtype=np.int64).T
    d, e = inputs.graph_inputs(2, n, b, E, seed=85, load=1.0)
    r = rng.standard_normal((2, n, b))
    js = oracle.junction_solve(d, E, e, r, lib=lib)
    full = oracle.junction(d, E, e, lib=lib)
    for k in range(2):
        res = np.einsum("vab,vb->va", np.tril(d[k]) + np.swapaxes(np.tril(d[k], -1), -1, -2), js["x"][k]) - r[k]
        np.add.at(res, E[0], np.einsum("kab,kb->ka", e[k], js["x"][k][E[1]]))
        np.add.at(res, E[1], np.einsum("kba,kb->ka", e[k], js["x"][k][E[0]]))
        worst = max(worst, float(np.linalg.norm(res) / np.linalg.norm(r[k])))
    worst = max(worst, float(np.max(np.abs(js["logdet"] - full["logdet"]))))
    return worst


# name -> (function, tolerance)
PINS = {
    "tiny_chains_dense": (pin_tiny_chains_dense, 1e-12),
    "quickstart": (pin_quickstart, 1e-10),
    "sparsax_3x3": (pin_sparsax_3x3, 1e-14),
    "laplacian_closed_form": (pin_laplacian_closed_form, 1e-12),
    "decoupled": (pin_decoupled, 1e-12),
    "grid_closed_form": (pin_grid_closed_form, 1e-12),
    "block_row_identity": (pin_block_row_identity, 1e-12),
    "tiny_trees_dense": (pin_tiny_trees_dense, 1e-12),
    "tree_quickstart": (pin_tree_quickstart, 1e-10),
    "root_invariance": (pin_root_invariance, 1e-11),
    "sample_standard_basis": (pin_sample_standard_basis, 1e-12),
    "sample_mean": (pin_sample_mean, 1e-12),
    "tree_sample_standard_basis": (pin_tree_sample_standard_basis, 1e-12),
    "not_spd": (pin_not_spd, 0.5),
    "backward_finite_differences": (pin_backward_finite_differences, 1e-7),
    "backward_decoupled": (pin_backward_decoupled, 1e-12),
    "backward_trace": (pin_backward_trace, 1e-11),
    "tree_backward_finite_differences": (pin_tree_backward_finite_differences, 1e-7),
    "tree_backward_path_is_chain": (pin_tree_backward_path_is_chain, 1e-12),
    "bidiag_dense": (pin_bidiag_dense, 1e-12),
    "bidiag_scalar_exact": (pin_bidiag_scalar_exact, 1e-15),
    "bidiag_singular": (pin_bidiag_singular, 0.5),
    "bidiag_backward_finite_differences": (pin_bidiag_backward_finite_differences, 1e-7),
    "bidiag_backward_scalar_exact": (pin_bidiag_backward_scalar_exact, 1e-14),
    "junction_dense": (pin_junction_dense, 1e-11),
    "junction_symbolic": (pin_junction_symbolic, 0.5),
    "junction_tree_and_order": (pin_junction_tree_and_order, 1e-12),
    "junction_backward_finite_differences": (pin_junction_backward_finite_differences, 1e-7),
    "junction_backward_path_is_chain": (pin_junction_backward_path_is_chain, 1e-12),
    "junction_solve": (pin_junction_solve, 1e-11),
}
