"""General block-sparse SPD matrices on the GPU (selinv_junction, b <= 16)
against the oracle: the plan's elimination order and filled pattern S must
equal the oracle's symbolic elimination exactly, and every block of A^-1 on
S its dense inverse, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from sparse_spd_selected_b200 import inputs, selinv
from tests.parity import TOL, host, logdet_err, to_dev, worst

pytestmark = pytest.mark.gpu


def random_pattern(n, m, seed):
    rng = np.random.default_rng(seed)
    pairs = sorted({(max(a, c), min(a, c)) for a, c in rng.integers(0, n, (m, 2)) if a != c})
    return np.array(pairs, dtype=np.int64).T.reshape(2, -1)


def run(n, E, b, seed, dtype, lead=(2,), order=None, load=1.0):
    batch = int(np.prod(lead))
    d, e = inputs.graph_inputs(batch, n, b, E, seed=seed, load=load)
    d = d.reshape(lead + (n, b, b))
    e = e.reshape(lead + (E.shape[1], b, b))
    plan = selinv.JunctionPlan(n, E, order)
    o_ref, S_ref = oracle.junction_symbolic(n, E, order)
    assert plan.order.tolist() == o_ref.tolist()
    assert np.array_equal(plan.S_index, S_ref)
    dd, ee = to_dev(d, dtype), to_dev(e, dtype)
    out = selinv.junction(plan, dd, ee)
    ref = oracle.junction(host(dd), E, host(ee), order)
    assert (ref["info"] == -1).all()
    nl = len(lead)
    assert worst(host(out["G_diag"]), ref["G_diag"], nl) <= TOL[dtype]
    if plan.nnz:
        assert worst(host(out["G_lower"]), ref["G_lower"], nl) <= TOL[dtype]
    assert logdet_err(host(out["logdet"]), ref["logdet"]) <= TOL[dtype]
    assert (host(out["info"]) == -1).all()
    return plan


@pytest.mark.parametrize("b", [1, 2, 5, 16])
def test_junction_grid_3x3(cuda_ok, b):
    """The pages' loopy 3 x 3 grid: S grows past the input pattern."""
    E = inputs.grid_edges(3, 3)
    plan = run(9, E, b, 11000 + b, torch.float64)
    assert plan.nnz > E.shape[1]


@pytest.mark.parametrize("b", [1, 3, 8, 16])
@pytest.mark.parametrize("n,m", [(12, 20), (40, 90)])
def test_junction_random_graphs(cuda_ok, b, n, m):
    run(n, random_pattern(n, m, 11100 + n + b), b, 11200 + n + b, torch.float64)


def test_junction_given_order_tree_and_single_node(cuda_ok):
    E = inputs.grid_edges(4, 5)
    run(20, E, 4, 11300, torch.float64, order=np.arange(20)[::-1].copy())
    parent = inputs.random_parent(np.random.default_rng(5), 30)
    T = np.array([[max(v, p) for v, p in enumerate(parent) if p >= 0],
                  [min(v, p) for v, p in enumerate(parent) if p >= 0]])
    plan = run(30, T, 6, 11301, torch.float64)
    assert plan.nnz == T.shape[1]                       # a tree has no fill
    run(1, np.zeros((2, 0), dtype=np.int64), 7, 11302, torch.float64)


def test_junction_f32_and_leading_dims(cuda_ok):
    run(16, inputs.grid_edges(4, 4), 16, 11400, torch.float32, lead=(3,), load=2.0)
    run(16, inputs.grid_edges(4, 4), 8, 11402, torch.float32, lead=(3,), load=2.0)      # the 8 x 8 tile path
    run(12, random_pattern(12, 25, 3), 4, 11401, torch.float64, lead=(2, 3))


def test_junction_grid_16x16(cuda_ok):
    """A 16 x 16 lattice of blocks of 4 (N = 1024), three matrices."""
    run(256, inputs.grid_edges(16, 16), 4, 11500, torch.float64, lead=(3,))


def test_junction_not_spd(cuda_ok):
    E = inputs.grid_edges(3, 4)
    d, e = inputs.graph_inputs(2, 12, 3, E, seed=11600, load=1.0)
    d[1, 5] = -np.eye(3)
    plan = selinv.JunctionPlan(12, E)
    out = selinv.junction(plan, to_dev(d, torch.float64), to_dev(e, torch.float64), check=False)
    info = host(out["info"])
    assert info[0] == -1 and info[1] >= 0
    with pytest.raises(selinv.NotSPDError):
        selinv.junction(plan, to_dev(d, torch.float64), to_dev(e, torch.float64))


def test_junction_lattice_benchmark_size(cuda_ok):
    """The benchmarked launch: 64 matrices on a 32 x 32 lattice of 8 x 8 blocks
    (N = 8192 each).  Every matrix: the diagonal block rows of A G = I, which
    use only blocks on S (the pattern is inside S), sum_u A_vu G_uv = I.  One
    sampled matrix: every block on S and log det against the dense inverse
    (numpy's LAPACK on the same matrix, read on S)."""
    w = inputs.WORKLOADS["lattice_64x1024_b8"]
    g = inputs.generate(w)
    E = g["edge_index"]
    n, b = w.L, w.b
    plan = selinv.JunctionPlan(n, E)
    out = selinv.junction(plan, to_dev(g["diag"], torch.float64), to_dev(g["edge_val"], torch.float64))
    Gd, Gl = host(out["G_diag"]), host(out["G_lower"])
    Si, Sj = plan.S_index
    slot = {(int(i), int(j)): k for k, (i, j) in enumerate(zip(Si, Sj))}
    ei, ej = E
    sym = lambda D: np.tril(D) + np.swapaxes(np.tril(D, -1), -1, -2)
    # block row v of A G, diagonal block: D_v G_vv + sum over pattern neighbours u of A_vu G_uv
    ki = np.array([slot[(int(i), int(j))] for i, j in zip(ei, ej)])
    for e in range(w.batch):
        R = np.einsum("vab,vbc->vac", sym(g["diag"][e]), Gd[e]) - np.eye(b)
        Aij = g["edge_val"][e]                       # A_{i,j}, i > j
        Gij = Gl[e][ki]                              # (A^-1)_{i,j}
        np.add.at(R, ei, Aij @ np.swapaxes(Gij, -1, -2))       # row i: A_ij G_ji = A_ij G_ij^T
        np.add.at(R, ej, np.swapaxes(Aij, -1, -2) @ Gij)       # row j: A_ji G_ij = A_ij^T G_ij
        assert float(np.abs(R).max()) <= 1e-9, e
    # one matrix against the dense inverse
    e = 17
    N = n * b
    A = np.zeros((N, N))
    for v in range(n):
        A[v * b:(v + 1) * b, v * b:(v + 1) * b] = sym(g["diag"][e, v])
    for k, (i, j) in enumerate(zip(ei, ej)):
        A[i * b:(i + 1) * b, j * b:(j + 1) * b] = g["edge_val"][e, k]
        A[j * b:(j + 1) * b, i * b:(i + 1) * b] = g["edge_val"][e, k].T
    inv = np.linalg.inv(A)
    ref_d = np.stack([inv[v * b:(v + 1) * b, v * b:(v + 1) * b] for v in range(n)])
    ref_l = np.stack([inv[i * b:(i + 1) * b, j * b:(j + 1) * b] for i, j in zip(Si, Sj)])
    assert worst(Gd[e][None], ref_d[None]) <= 1e-9
    assert worst(Gl[e][None], ref_l[None]) <= 1e-9
    assert logdet_err(host(out["logdet"])[e], np.linalg.slogdet(A)[1]) <= 1e-9


def test_junction_graph_replay_reads_new_values(cuda_ok):
    """Calls with the same buffers replay the launch sequence recorded by the
    first one (the plan's graph cache): new values written into those buffers
    give the new matrices' results; other buffers, another batch size or
    another block size record their own; a replay inside the caller's own
    stream capture still works."""
    E = inputs.grid_edges(6, 6)
    n, b = 36, 8
    plan = selinv.JunctionPlan(n, E)
    d1, e1 = inputs.graph_inputs(3, n, b, E, seed=11700, load=1.0)
    d2, e2 = inputs.graph_inputs(3, n, b, E, seed=11701, load=1.0)
    dd, ee = to_dev(d1, torch.float64), to_dev(e1, torch.float64)
    out = {"G_diag": torch.empty_like(dd), "G_lower": torch.empty((3, plan.nnz, b, b), dtype=torch.float64, device="cuda"),
           "logdet": torch.empty(3, dtype=torch.float64, device="cuda"),
           "info": torch.empty(3, dtype=torch.int32, device="cuda")}
    ws = torch.empty(plan.workspace_size(torch.float64, b, 3), dtype=torch.uint8, device="cuda")
    for d, e in ((d1, e1), (d2, e2), (d1, e1)):
        dd.copy_(to_dev(d, torch.float64))
        ee.copy_(to_dev(e, torch.float64))
        r = selinv.junction(plan, dd, ee, out=out, workspace=ws)
        ref = oracle.junction(d, E, e)
        assert worst(host(r["G_diag"]), ref["G_diag"]) <= 1e-9
        assert worst(host(r["G_lower"]), ref["G_lower"]) <= 1e-9
        assert logdet_err(host(r["logdet"]), ref["logdet"]) <= 1e-9
    fresh = selinv.junction(plan, dd, ee)                          # other buffers: its own recording
    assert torch.equal(fresh["G_diag"], out["G_diag"]) and torch.equal(fresh["G_lower"], out["G_lower"])
    one = selinv.junction(plan, dd[:1].contiguous(), ee[:1].contiguous())   # another batch size
    assert torch.equal(one["G_diag"], out["G_diag"][:1])
    d5, e5 = inputs.graph_inputs(2, n, 5, E, seed=11702, load=1.0)  # another block size
    r5 = selinv.junction(plan, to_dev(d5, torch.float64), to_dev(e5, torch.float64))
    assert worst(host(r5["G_diag"]), oracle.junction(d5, E, e5)["G_diag"]) <= 1e-9
    # inside the caller's own capture the launches go straight into that graph
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        selinv.junction(plan, dd, ee, check=False, out=out, workspace=ws)
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=s):
        selinv.junction(plan, dd, ee, check=False, out=out, workspace=ws)
    out["G_diag"].zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out["G_diag"], fresh["G_diag"])


def solve_both(n, E, b, seed, dtype, lead=(2,), load=1.0):
    batch = int(np.prod(lead))
    d, e = inputs.graph_inputs(batch, n, b, E, seed=seed, load=load)
    r = np.random.default_rng([seed, 7]).standard_normal((batch, n, b))
    d, e, r = d.reshape(lead + (n, b, b)), e.reshape(lead + (E.shape[1], b, b)), r.reshape(lead + (n, b))
    plan = selinv.JunctionPlan(n, E)
    dd, ee, rr = to_dev(d, dtype), to_dev(e, dtype), to_dev(r, dtype)
    x, ld, info = selinv.junction_solve(plan, dd, ee, rr)
    ref = oracle.junction_solve(host(dd), E, host(ee), host(rr))
    nl = len(lead)
    assert (host(info) == -1).all()
    assert worst(host(x), ref["x"], nl, block_ndim=1) <= TOL[dtype]
    assert logdet_err(host(ld), ref["logdet"]) <= TOL[dtype]
    return plan, dd, ee, rr, x


@pytest.mark.parametrize("b", [1, 3, 8, 16])
def test_junction_solve_matches_oracle(cuda_ok, b):
    """x = A^-1 r on the pages' 3 x 3 grid and on random patterns (fill)."""
    solve_both(9, inputs.grid_edges(3, 3), b, 11800 + b, torch.float64)
    solve_both(30, random_pattern(30, 70, 11810 + b), b, 11820 + b, torch.float64)


def test_junction_solve_f32_leading_dims_and_selinv_consistency(cuda_ok):
    solve_both(16, inputs.grid_edges(4, 4), 8, 11900, torch.float32, lead=(3,), load=2.0)
    solve_both(16, inputs.grid_edges(4, 4), 16, 11901, torch.float32, lead=(2, 2), load=2.0)
    plan, dd, ee, rr, x = solve_both(20, inputs.grid_edges(4, 5), 5, 11902, torch.float64, lead=(3,))
    # the same factorisation: the log det of the selected-inverse call is identical
    full = selinv.junction(plan, dd, ee)
    _, ld, _ = selinv.junction_solve(plan, dd, ee, rr)
    assert torch.equal(ld, full["logdet"])


def test_junction_solve_lattice_benchmark_size(cuda_ok):
    """64 matrices on the 32 x 32 lattice of 8 x 8 blocks: the block residual
    sum_u A_vu x_u - r_v of every matrix, against the right-hand side."""
    w = inputs.WORKLOADS["lattice_64x1024_b8"]
    g = inputs.generate(w)
    E = g["edge_index"]
    n, b = w.L, w.b
    r = np.random.default_rng(11950).standard_normal((w.batch, n, b))
    plan = selinv.JunctionPlan(n, E)
    x, _, info = selinv.junction_solve(plan, to_dev(g["diag"], torch.float64), to_dev(g["edge_val"], torch.float64),
                                       to_dev(r, torch.float64))
    x = host(x)
    assert (host(info) == -1).all()
    ei, ej = E
    sym = lambda D: np.tril(D) + np.swapaxes(np.tril(D, -1), -1, -2)
    for e in range(w.batch):
        res = np.einsum("vab,vb->va", sym(g["diag"][e]), x[e]) - r[e]
        np.add.at(res, ei, np.einsum("kab,kb->ka", g["edge_val"][e], x[e][ej]))
        np.add.at(res, ej, np.einsum("kba,kb->ka", g["edge_val"][e], x[e][ei]))
        assert float(np.linalg.norm(res) / np.linalg.norm(r[e])) <= 1e-12, e


def test_junction_solve_not_spd(cuda_ok):
    E = inputs.grid_edges(3, 4)
    d, e = inputs.graph_inputs(2, 12, 3, E, seed=11960, load=1.0)
    d[1, 5] = -np.eye(3)
    plan = selinv.JunctionPlan(12, E)
    r = to_dev(np.ones((2, 12, 3)), torch.float64)
    _, _, info = selinv.junction_solve(plan, to_dev(d, torch.float64), to_dev(e, torch.float64), r, check=False)
    assert host(info)[0] == -1 and host(info)[1] >= 0
    with pytest.raises(selinv.NotSPDError):
        selinv.junction_solve(plan, to_dev(d, torch.float64), to_dev(e, torch.float64), r)
