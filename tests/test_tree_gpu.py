"""GPU tree kernels (level-set schedule) vs the CPU oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from sparse_spd_selected_b200 import inputs, selinv
from tests.dense import balanced_parent, path_parent, star_parent
from tests.parity import TOL, host, logdet_err, to_dev, worst

pytestmark = pytest.mark.gpu


def compare(P, diag, edge, dtype=torch.float64):
    d_dev, e_dev = to_dev(diag, dtype), to_dev(edge, dtype)
    plan = selinv.TreePlan(P)
    out = selinv.selinv_tree(plan, d_dev, e_dev)
    ref = oracle.tree(P, host(d_dev), host(e_dev))
    assert (ref["info"] == -1).all()
    return {
        "G_diag": worst(host(out["G_diag"]), ref["G_diag"]),
        "G_edge": worst(host(out["G_edge"]), ref["G_edge"]),
        "logdet": logdet_err(host(out["logdet"]), ref["logdet"]),
    }, out, plan


@pytest.mark.parametrize("b", [1, 3, 4, 8, 13, 16])
def test_topologies(cuda_ok, b):
    n = 37
    rng = np.random.default_rng(b)
    pr = np.full(n, -1, dtype=np.int32)
    for v in range(n - 1):
        pr[v] = rng.integers(v + 1, n)
    P = np.stack([inputs.random_parent(rng, n), path_parent(n), star_parent(n), balanced_parent(n, 2),
                  balanced_parent(n, 5), pr])
    diag, edge = inputs.tree_inputs_from_parent(P, b, seed=10 + b, load=0.5)
    errs, out, _ = compare(P, diag, edge)
    assert max(errs.values()) <= TOL[torch.float64], errs
    assert not out["G_edge"][:5, 0].any()          # trees 0-4 are rooted at node 0
    assert not out["G_edge"][5, n - 1].any()       # tree 5 is rooted at its last node


def test_single_node_and_f32(cuda_ok):
    P = np.array([[-1]], dtype=np.int32)
    diag, edge = inputs.tree_inputs_from_parent(P, 16, seed=5, load=1.0)
    errs, _, _ = compare(P, diag, edge)
    assert max(errs.values()) <= 1e-9
    P, diag, edge = inputs.tree_inputs(3, 200, 16, seed=6, load=1.0)
    errs, _, _ = compare(P, diag, edge, torch.float32)
    assert max(errs.values()) <= TOL[torch.float32], errs


def test_path_tree_equals_chain(cuda_ok):
    """Root invariance: the path rooted at node 0 reproduces the chain (rooted at its last node)."""
    L, b = 50, 16
    d, l, _ = inputs.chain_inputs(2, L, b, seed=7, load=0.5, with_rhs=False)
    ch = selinv.selinv_chain(to_dev(d, torch.float64), to_dev(l, torch.float64))
    P = np.stack([path_parent(L)] * 2)
    edge = np.zeros((2, L, b, b))
    edge[:, 1:] = np.swapaxes(l, -1, -2)
    tr = selinv.selinv_tree(selinv.TreePlan(P), to_dev(d, torch.float64), to_dev(edge, torch.float64))
    assert worst(host(tr["G_diag"]), host(ch["G_diag"])) <= 1e-10
    assert worst(np.swapaxes(host(tr["G_edge"])[:, 1:], -1, -2), host(ch["G_lower"])) <= 1e-10
    assert logdet_err(host(tr["logdet"]), host(ch["logdet"])) <= 1e-12


def test_full_size_forest_sampled(cuda_ok):
    """8 random trees of 32768 nodes, b = 16 (the benchmark launch); oracle on two trees."""
    w = inputs.WORKLOADS["forest_8x32768_b16"]
    g = inputs.generate(w)
    plan = selinv.TreePlan(g["parent"])
    out = selinv.selinv_tree(plan, to_dev(g["diag"], torch.float64), to_dev(g["edge"], torch.float64))
    pick = [0, 7]
    ref = oracle.tree(g["parent"][pick], g["diag"][pick], g["edge"][pick])
    assert worst(host(out["G_diag"][pick]), ref["G_diag"]) <= 1e-9
    assert worst(host(out["G_edge"][pick]), ref["G_edge"]) <= 1e-9
    assert logdet_err(host(out["logdet"][pick]), ref["logdet"]) <= 1e-9
    Gd = out["G_diag"]
    assert torch.equal(Gd, Gd.transpose(-1, -2))


def test_tree_not_spd_and_determinism(cuda_ok):
    P, diag, edge = inputs.tree_inputs(2, 40, 16, seed=9, load=1.0)
    d2 = diag.copy()
    d2[1, 17] = -np.eye(16)
    plan = selinv.TreePlan(P)
    with pytest.raises(selinv.NotSPDError) as ei:
        selinv.selinv_tree(plan, to_dev(d2, torch.float64), to_dev(edge, torch.float64))
    assert ei.value.info[0] == -1 and ei.value.info[1] >= 0
    a = selinv.selinv_tree(plan, to_dev(diag, torch.float64), to_dev(edge, torch.float64))
    b = selinv.selinv_tree(plan, to_dev(diag, torch.float64), to_dev(edge, torch.float64))
    for k in ("G_diag", "G_edge", "logdet"):
        assert torch.equal(a[k], b[k])


def _held_node(P, tree):
    """A non-root node of `tree` with children (its children wait on its flag)."""
    par = P[tree]
    kids = np.bincount(par[par >= 0], minlength=P.shape[1])
    cand = [v for v in range(P.shape[1]) if par[v] >= 0 and kids[v] > 0]
    return tree * P.shape[1] + cand[len(cand) // 2]


@pytest.mark.parametrize("b", [16, 5])
def test_bounded_wait_gives_up_on_an_unpublished_parent(cuda_ok, b):
    """A node whose completion flag is never published (the plan's test hook):
    its children give up after the spin limit, its tree reports info = -2
    (WaitTimeoutError with check=True), the failure reaches the descendants at
    once, the other trees are exact, and the next call on the same plan and
    context is correct.  Forward sweep, draw and backward (all three waits)."""
    import time
    P, diag, edge = inputs.tree_inputs(3, 300, b, seed=41 + b, load=1.0)
    plan = selinv.TreePlan(P)
    dd, ee = to_dev(diag, torch.float64), to_dev(edge, torch.float64)
    ref = oracle.tree(P, diag, edge)
    plan.set_wait(spin_limit=4096, withhold=_held_node(P, 1))
    t0 = time.perf_counter()
    out = selinv.selinv_tree(plan, dd, ee, check=False)
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 10.0
    assert host(out["info"]).tolist() == [-1, -2, -1]
    ok = [0, 2]
    assert worst(host(out["G_diag"])[ok], ref["G_diag"][ok]) <= 1e-9
    assert worst(host(out["G_edge"])[ok], ref["G_edge"][ok]) <= 1e-9
    with pytest.raises(selinv.WaitTimeoutError):
        selinv.selinv_tree(plan, dd, ee)
    # draw: the vector recurrence waits on the same flags
    z = to_dev(np.random.default_rng(5).standard_normal((3, 300, b)), torch.float64)
    dr = selinv.tree_sample(plan, dd, ee, z, check=False)
    torch.cuda.synchronize()
    assert host(dr["info"]).tolist() == [-1, -2, -1]
    # backward: its parents-first pass waits on the same flags
    plan.set_wait()
    fwd = selinv.selinv_tree(plan, dd, ee)
    gd = to_dev(np.random.default_rng(6).standard_normal(diag.shape), torch.float64)
    bw_ok = selinv.tree_backward(plan, dd, ee, fwd["G_diag"], fwd["G_edge"], gd, None)
    plan.set_wait(spin_limit=4096, withhold=_held_node(P, 1))
    bw = selinv.tree_backward(plan, dd, ee, fwd["G_diag"], fwd["G_edge"], gd, None, check=False)
    torch.cuda.synchronize()
    assert host(bw["info"]).tolist() == [-1, -2, -1]
    assert torch.equal(bw["Db"][ok], bw_ok["Db"][ok]) and torch.equal(bw["Eb"][ok], bw_ok["Eb"][ok])
    # the hook off again: the same plan and context give the exact answer
    plan.set_wait()
    again = selinv.selinv_tree(plan, dd, ee)
    assert (host(again["info"]) == -1).all()
    assert worst(host(again["G_diag"]), ref["G_diag"]) <= 1e-9
    assert worst(host(again["G_edge"]), ref["G_edge"]) <= 1e-9


def test_tree_validate_reports_non_finite_inputs(cuda_ok):
    """validate=True on trees: info = -3 - v for the first node v whose D_v
    (lower triangle) or edge slot holds a non-finite entry; root edge slots and
    upper triangles are not read, hence not checked."""
    P, diag, edge = inputs.tree_inputs(4, 60, 16, seed=77, load=1.0)
    diag[1, 40, 5, 2] = np.nan
    v2 = int(np.nonzero(P[2] >= 0)[0][10])
    edge[2, v2, 3, 3] = -np.inf
    edge[3, 0] = np.nan                      # root slot of tree 3 (root is node 0): not read
    diag[3, 7, 0, 9] = np.nan                # upper triangle: not read
    plan = selinv.TreePlan(P)
    out = selinv.selinv_tree(plan, to_dev(diag, torch.float64), to_dev(edge, torch.float64), check=False,
                             validate=True)
    assert host(out["info"]).tolist() == [-1, -3 - 40, -3 - v2, -1]
    with pytest.raises(selinv.NonFiniteInputError):
        selinv.selinv_tree(plan, to_dev(diag, torch.float64), to_dev(edge, torch.float64), validate=True)
