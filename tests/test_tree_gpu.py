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
