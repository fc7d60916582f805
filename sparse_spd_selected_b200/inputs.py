"""Seeded synthetic inputs shared by the oracle side and the GPU side.

This module holds no arithmetic of the selected-inverse method: it only draws
random blocks and assembles SPD test matrices.  Every batch element has its
own generator, ``numpy.random.default_rng([seed, element])`` (PCG64), so any
subset of a batch can be regenerated alone, bit-for-bit equal to the same
elements of the full batch; that is how full-size runs are checked against the
CPU oracle on sampled elements.

Recipes (the workloads are the pages' problem shapes with synthetic values):

chain   per element draw, in order: B ~ N(0,1)/sqrt(b)  [L-1,b,b],
        C ~ N(0,1) [L,b,b], then (if a right-hand side is asked for)
        r ~ N(0,1) [L,b].  D_i = C_i C_i^T / b + (load + delta_i) I with
        delta_i = max_r ( sum_c |A_{i,i-1}[r,c]| + sum_c |A_{i,i+1}[r,c]| ),
        A_{i,i-1} = B_{i-1}, A_{i,i+1} = B_i^T, absent neighbours 0.
tree    per tree draw u ~ U[0,1) [n-1] and set parent[v] = floor(u_v * v)
        (uniform in [0, v), root 0 has parent -1); then edge ~ N(0,1)/sqrt(b)
        for v = 1..n-1 (root slot 0); then C ~ N(0,1) [n,b,b].
        D_v = C_v C_v^T / b + (load + delta_v) I with
        delta_v = ||edge[v]^T||_inf (0 at the root) + sum_{c in ch(v)} ||edge[c]||_inf.
grid    per element draw tau ~ U(0.01, 1), then r ~ N(0,1) [m, m]:
        the m x m grid Laplacian ordered by rows plus tau I as a chain with
        D_i = tridiag(-1, 4 + tau, -1), B_i = -I (stored dense).

Both additive terms make the off-diagonal part strictly block-row dominant
while C C^T / b is positive semidefinite, so every matrix is SPD with
smallest eigenvalue at least ``load`` (grid: at least tau).
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Iterable, Optional, Sequence

import numpy as np


def _rng(seed: int, element: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(element)])


def _chain_element(rng, L, b, load, with_rhs):
    B = rng.standard_normal((L - 1, b, b)) / math.sqrt(b)
    C = rng.standard_normal((L, b, b))
    r = rng.standard_normal((L, b)) if with_rhs else None
    absB = np.abs(B)
    row_left = np.zeros((L, b))            # sum_c |A_{i,i-1}[r,c]| = row sums of |B_{i-1}|
    row_right = np.zeros((L, b))           # sum_c |A_{i,i+1}[r,c]| = column sums of |B_i|
    if L > 1:
        row_left[1:] = absB.sum(axis=2)
        row_right[:-1] = absB.sum(axis=1)
    delta = (row_left + row_right).max(axis=1)
    D = np.matmul(C, np.swapaxes(C, 1, 2)) / b
    D += (load + delta)[:, None, None] * np.eye(b)
    return D, B, r


def chain_inputs(batch: int, L: int, b: int, seed: int, load: float,
                 with_rhs: bool = True, elements: Optional[Sequence[int]] = None):
    """Block-tridiagonal SPD chains: returns (diag [E,L,b,b], lower [E,L-1,b,b], rhs [E,L,b] or None).

    E = batch, or len(elements) when a subset of the batch is asked for.
    """
    idx = range(batch) if elements is None else list(elements)
    E = len(idx)
    diag = np.empty((E, L, b, b))
    lower = np.empty((E, L - 1, b, b))
    rhs = np.empty((E, L, b)) if with_rhs else None
    for k, e in enumerate(idx):
        D, B, r = _chain_element(_rng(seed, e), L, b, load, with_rhs)
        diag[k] = D
        lower[k] = B
        if with_rhs:
            rhs[k] = r
    return diag, lower, rhs


def random_parent(rng, n: int) -> np.ndarray:
    """parent[0] = -1, parent[v] uniform in [0, v) (a random recursive tree)."""
    u = rng.random(n - 1)
    parent = np.empty(n, dtype=np.int32)
    parent[0] = -1
    parent[1:] = np.floor(u * np.arange(1, n)).astype(np.int32)
    return parent


def _tree_element(rng, n, b, load):
    parent = random_parent(rng, n)
    edge = np.zeros((n, b, b))
    edge[1:] = rng.standard_normal((n - 1, b, b)) / math.sqrt(b)
    C = rng.standard_normal((n, b, b))
    absE = np.abs(edge)
    up = absE.sum(axis=1).max(axis=1)          # ||edge[v]^T||_inf (max column sum of |edge[v]|)
    down = absE.sum(axis=2).max(axis=1)        # ||edge[c]||_inf (max row sum of |edge[c]|)
    up[0] = 0.0
    delta = up.copy()
    np.add.at(delta, parent[1:], down[1:])
    D = np.matmul(C, np.swapaxes(C, 1, 2)) / b
    D += (load + delta)[:, None, None] * np.eye(b)
    return parent, D, edge


def tree_inputs(trees: int, n: int, b: int, seed: int, load: float,
                elements: Optional[Sequence[int]] = None):
    """Random block trees: returns (parent [E,n] int32, diag [E,n,b,b], edge [E,n,b,b])."""
    idx = range(trees) if elements is None else list(elements)
    E = len(idx)
    parent = np.empty((E, n), dtype=np.int32)
    diag = np.empty((E, n, b, b))
    edge = np.empty((E, n, b, b))
    for k, t in enumerate(idx):
        parent[k], diag[k], edge[k] = _tree_element(_rng(seed, t), n, b, load)
    return parent, diag, edge


def tree_inputs_from_parent(parent: np.ndarray, b: int, seed: int, load: float):
    """Blocks for given parent arrays [E,n] (edges and diagonals drawn as in ``tree_inputs``)."""
    parent = np.asarray(parent, dtype=np.int32)
    E, n = parent.shape
    diag = np.empty((E, n, b, b))
    edge = np.zeros((E, n, b, b))
    for k in range(E):
        rng = _rng(seed, k)
        p = parent[k]
        nonroot = p >= 0
        edge[k][nonroot] = rng.standard_normal((int(nonroot.sum()), b, b)) / math.sqrt(b)
        C = rng.standard_normal((n, b, b))
        absE = np.abs(edge[k])
        up = absE.sum(axis=1).max(axis=1)
        up[~nonroot] = 0.0
        down = absE.sum(axis=2).max(axis=1)
        delta = up.copy()
        np.add.at(delta, p[nonroot], down[nonroot])
        diag[k] = np.matmul(C, np.swapaxes(C, 1, 2)) / b + (load + delta)[:, None, None] * np.eye(b)
    return diag, edge


def grid_taus(batch: int, seed: int, elements: Optional[Iterable[int]] = None):
    idx = range(batch) if elements is None else list(elements)
    return np.array([_rng(seed, e).uniform(0.01, 1.0) for e in idx])


def grid_inputs(batch: int, m: int, seed: int, with_rhs: bool = True,
                elements: Optional[Sequence[int]] = None):
    """Row-ordered m x m grid precision as a chain of L = m blocks of size m.

    Returns (diag [E,m,m,m], lower [E,m-1,m,m], rhs [E,m,m] or None, tau [E]).
    """
    idx = range(batch) if elements is None else list(elements)
    E = len(idx)
    diag = np.zeros((E, m, m, m))
    lower = np.zeros((E, m - 1, m, m))
    rhs = np.empty((E, m, m)) if with_rhs else None
    tau = np.empty(E)
    off = np.eye(m, k=-1) + np.eye(m, k=1)
    for k, e in enumerate(idx):
        rng = _rng(seed, e)
        tau[k] = rng.uniform(0.01, 1.0)
        if with_rhs:
            rhs[k] = rng.standard_normal((m, m))
        diag[k] = (4.0 + tau[k]) * np.eye(m) - off
        lower[k] = -np.eye(m)
    return diag, lower, rhs, tau


def grid_inputs_torch(batch: int, m: int, seed: int, device, dtype=None, with_rhs: bool = True):
    """The ``grid_inputs`` batch assembled directly in device memory (same values).

    The only random numbers (tau and the right-hand sides) come from the same
    per-element generators; the blocks are written with torch on ``device``.
    """
    import torch
    dtype = dtype or torch.float64
    taus = torch.tensor(grid_taus(batch, seed), dtype=dtype, device=device)
    eye = torch.eye(m, dtype=dtype, device=device)
    off = torch.diag(torch.ones(m - 1, dtype=dtype, device=device), -1)
    off = off + off.T
    diag = torch.empty((batch, m, m, m), dtype=dtype, device=device)
    diag.copy_(((4.0 + taus)[:, None, None, None] * eye - off).expand(batch, m, m, m))
    lower = torch.empty((batch, m - 1, m, m), dtype=dtype, device=device)
    lower.copy_((-eye).expand(batch, m - 1, m, m))
    rhs = None
    if with_rhs:
        r = np.stack([_grid_rhs(seed, e, m) for e in range(batch)])
        rhs = torch.from_numpy(r).to(device=device, dtype=dtype)
    return diag, lower, rhs, taus


def _grid_rhs(seed, e, m):
    rng = _rng(seed, e)
    rng.uniform(0.01, 1.0)
    return rng.standard_normal((m, m))


@dataclass(frozen=True)
class Workload:
    """One synthetic workload: its kind, sizes, seed and value recipe."""
    name: str
    kind: str              # "chain", "tree" or "grid"
    batch: int             # chains, trees or grid elements
    L: int                 # chain blocks, or tree nodes n
    b: int
    seed: int
    load: float = 0.0      # diagonal load (chain, tree)
    solve: bool = False    # one right-hand side per element
    dtypes: tuple = ("f64",)

    @property
    def nodes(self) -> int:
        return self.batch * self.L


# The five workloads of the problem statement, named by what they are, and a
# lattice for the general sparse case.
WORKLOADS = {
    w.name: w for w in [
        Workload("chain_1x8_b4", "chain", 1, 8, 4, seed=0, load=2.0, solve=True),
        Workload("chain_4096x64_b16", "chain", 4096, 64, 16, seed=1, load=2.0, solve=True),
        Workload("chain_64x4096_b32", "chain", 64, 4096, 32, seed=2, load=0.5,
                 dtypes=("f64", "f32")),
        Workload("forest_8x32768_b16", "tree", 8, 32768, 16, seed=3, load=1.0),
        Workload("grid_256x128_b128", "grid", 256, 128, 128, seed=4, solve=True),
        # general sparse SPD on a loopy pattern (the pages' grid-graph example):
        # 64 matrices on a 32 x 32 lattice of 8 x 8 blocks
        Workload("lattice_64x1024_b8", "junction", 64, 1024, 8, seed=5, load=1.0),
    ]
}


def standard_normals(batch: int, L: int, b: int, seed: int, elements: Optional[Sequence[int]] = None):
    """Standard normals z [n, L, b] for Gaussian draws: batch element e uses its
    own generator default_rng([seed, e, 1]), a stream apart from its matrix."""
    elements = range(batch) if elements is None else elements
    return np.stack([np.random.default_rng([int(seed), int(e), 1]).standard_normal((L, b)) for e in elements])


def grid_edges(rows: int, cols: int) -> np.ndarray:
    """Lower pairs (i, j), i > j, of a rows x cols 4-neighbour lattice, node r*cols + c."""
    E = []
    for r in range(rows):
        for c in range(cols):
            v = r * cols + c
            if c + 1 < cols:
                E.append((v + 1, v))
            if r + 1 < rows:
                E.append((v + cols, v))
    return np.array(E, dtype=np.int64).T.reshape(2, -1)


def graph_inputs(batch: int, n: int, b: int, edge_index: np.ndarray, seed: int, load: float,
                 elements: Optional[Sequence[int]] = None):
    """Block-sparse SPD matrices on a given pattern (the pages' random_spd_graph
    shape): edge blocks A_{i,j} = B / sqrt(b), diagonals C C^T / b + (load +
    delta_v) I with delta_v the sum over v's incident blocks of their largest
    absolute row sum as they sit in block row v (strict block-row dominance,
    hence SPD).  Element e draws from default_rng([seed, e, 4])."""
    elements = range(batch) if elements is None else elements
    ei, ej = np.asarray(edge_index[0]), np.asarray(edge_index[1])
    m = ei.size
    diag, edge = [], []
    for e in elements:
        rng = np.random.default_rng([int(seed), int(e), 4])
        E = rng.standard_normal((m, b, b)) / math.sqrt(b)
        C = rng.standard_normal((n, b, b))
        delta = np.zeros(n)
        absE = np.abs(E)
        np.add.at(delta, ei, absE.sum(axis=2).max(axis=1))      # A_{i,j} in block row i
        np.add.at(delta, ej, absE.sum(axis=1).max(axis=1))      # A_{j,i} = A_{i,j}^T in block row j
        diag.append(np.matmul(C, np.swapaxes(C, 1, 2)) / b + (load + delta)[:, None, None] * np.eye(b))
        edge.append(E)
    return np.stack(diag), np.stack(edge)


def bidiag_inputs(batch: int, L: int, b: int, seed: int, load: float,
                  elements: Optional[Sequence[int]] = None):
    """Block lower-bidiagonal matrices with general blocks: M_ii = C_i / sqrt(b)
    + load I and M_{i+1,i} = B_i / sqrt(b), C_i and B_i standard normal (the
    pages' random_nonsym_bidiag shape with its diag_load); element e draws from
    default_rng([seed, e, 3])."""
    elements = range(batch) if elements is None else elements
    diag, lower = [], []
    for e in elements:
        rng = np.random.default_rng([int(seed), int(e), 3])
        lower.append(rng.standard_normal((L - 1, b, b)) / math.sqrt(b))
        diag.append(rng.standard_normal((L, b, b)) / math.sqrt(b) + load * np.eye(b))
    return np.stack(diag), np.stack(lower)


def cotangents(batch: int, L: int, b: int, seed: int, elements: Optional[Sequence[int]] = None):
    """Standard-normal cotangents (Gb_diag [n, L, b, b], Gb_lower [n, L-1, b, b])
    of a loss on a chain's selected inverse: element e draws from
    default_rng([seed, e, 2]), a stream apart from its matrix and draws."""
    elements = range(batch) if elements is None else elements
    gd, gl = [], []
    for e in elements:
        rng = np.random.default_rng([int(seed), int(e), 2])
        gd.append(rng.standard_normal((L, b, b)))
        gl.append(rng.standard_normal((L - 1, b, b)))
    return np.stack(gd), np.stack(gl)


def tree_cotangents(trees: int, n: int, b: int, seed: int, elements: Optional[Sequence[int]] = None):
    """Standard-normal cotangents (Gb_diag, Gb_edge [n_trees, n, b, b]) of a loss
    on a tree's selected inverse, tree e drawing from default_rng([seed, e, 2])."""
    elements = range(trees) if elements is None else elements
    gd, ge = [], []
    for e in elements:
        rng = np.random.default_rng([int(seed), int(e), 2])
        gd.append(rng.standard_normal((n, b, b)))
        ge.append(rng.standard_normal((n, b, b)))
    return np.stack(gd), np.stack(ge)


def generate(w: Workload, elements: Optional[Sequence[int]] = None):
    """Host (NumPy) inputs of a workload, or of a subset of its batch elements."""
    if w.kind == "chain":
        diag, lower, rhs = chain_inputs(w.batch, w.L, w.b, w.seed, w.load, w.solve, elements)
        return {"diag": diag, "lower": lower, "rhs": rhs}
    if w.kind == "tree":
        parent, diag, edge = tree_inputs(w.batch, w.L, w.b, w.seed, w.load, elements)
        return {"parent": parent, "diag": diag, "edge": edge}
    if w.kind == "grid":
        diag, lower, rhs, tau = grid_inputs(w.batch, w.b, w.seed, w.solve, elements)
        return {"diag": diag, "lower": lower, "rhs": rhs, "tau": tau}
    if w.kind == "junction":
        side = int(round(math.sqrt(w.L)))
        E = grid_edges(side, w.L // side)
        diag, edge = graph_inputs(w.batch, w.L, w.b, E, w.seed, w.load, elements)
        return {"diag": diag, "edge_val": edge, "edge_index": E}
    raise ValueError(w.kind)
