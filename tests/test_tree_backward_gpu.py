"""Cotangents of the tree selected inverse on the GPU (selinv_tree_backward,
b <= 16) against the oracle's dense definition Ab = -A^-1 Gbar A^-1, through
the C ABI, and the autograd wrapper built on it (the pages' selinv_tree)."""
import numpy as np
import pytest
import torch

import oracle
from sparse_spd_selected_b200 import inputs, selinv
from tests.dense import balanced_parent, path_parent, star_parent
from tests.parity import TOL, host, to_dev, worst

pytestmark = pytest.mark.gpu


def random_parent(n, seed):
    return inputs.random_parent(np.random.default_rng(seed), n)


def run(parents, b, seed, dtype, load=1.0):
    P = np.stack(parents).astype(np.int32)
    d, e = inputs.tree_inputs_from_parent(P, b, seed=seed, load=load)
    rng = np.random.default_rng([seed, 5])
    gd, ge = rng.standard_normal(d.shape), rng.standard_normal(e.shape)
    plan = selinv.TreePlan(P)
    dd, ee = to_dev(d, dtype), to_dev(e, dtype)
    fwd = selinv.selinv_tree(plan, dd, ee)
    out = selinv.tree_backward(plan, dd, ee, fwd["G_diag"], fwd["G_edge"], to_dev(gd, dtype), to_dev(ge, dtype))
    ref = oracle.tree_backward(P, host(dd), host(ee), host(to_dev(gd, dtype)), host(to_dev(ge, dtype)))
    assert (ref["info"] == -1).all()
    return out, ref


@pytest.mark.parametrize("b", [1, 3, 8, 13, 16])
def test_tree_backward_topologies(cuda_ok, b):
    n = 23
    parents = [path_parent(n), star_parent(n), balanced_parent(n), random_parent(n, 7 + b)]
    out, ref = run(parents, b, 9600 + b, torch.float64)
    assert worst(host(out["Db"]), ref["Db"]) <= TOL[torch.float64]
    assert worst(host(out["Eb"]), ref["Eb"]) <= TOL[torch.float64]
    assert (host(out["info"]) == -1).all()


def test_tree_backward_single_node_and_f32(cuda_ok):
    out, ref = run([np.array([-1])], 16, 9700, torch.float64)
    assert worst(host(out["Db"]), ref["Db"]) <= TOL[torch.float64]
    assert np.all(host(out["Eb"]) == 0.0)
    out, ref = run([random_parent(40, 3), balanced_parent(40)], 16, 9701, torch.float32, load=2.0)
    assert worst(host(out["Db"]), ref["Db"]) <= TOL[torch.float32]
    assert worst(host(out["Eb"]), ref["Eb"]) <= TOL[torch.float32]


def test_tree_autograd_matches_oracle(cuda_ok):
    """loss = <Wd, G_diag> + <We, G_edge> through selinv_tree_ad."""
    P = np.stack([random_parent(30, 11), balanced_parent(30)]).astype(np.int32)
    d, e = inputs.tree_inputs_from_parent(P, 4, seed=9800, load=1.0)
    rng = np.random.default_rng(9800)
    wd, we = rng.standard_normal(d.shape), rng.standard_normal(e.shape)
    plan = selinv.TreePlan(P)
    dd = to_dev(d, torch.float64).requires_grad_(True)
    ee = to_dev(e, torch.float64).requires_grad_(True)
    Gd, Ge = selinv.selinv_tree_ad(plan, dd, ee)
    loss = (Gd * to_dev(wd, torch.float64)).sum() + (Ge * to_dev(we, torch.float64)).sum()
    loss.backward()
    ref = oracle.tree_backward(P, d, e, wd, we)
    assert worst(host(dd.grad), ref["Db"]) <= TOL[torch.float64]
    assert worst(host(ee.grad), ref["Eb"]) <= TOL[torch.float64]


def test_tree_backward_forest_sampled(cuda_ok):
    """The forest workload's shape (8 random trees of 32768 nodes, b = 16).  The
    dense oracle is out of reach there, so (1) trees of 32 nodes drawn the same
    way are checked against it at full precision, and (2) on the forest itself
    the cotangents must reproduce a directional derivative of the loss
    <Gb_diag, G_diag> + <Gb_edge, G_edge>, taken by central differences of the
    forward (a property that holds at any size)."""
    sub, ref = run([inputs.random_parent(np.random.default_rng(12), 32),
                    inputs.random_parent(np.random.default_rng(13), 32)], 16, 9901, torch.float64)
    assert worst(host(sub["Db"]), ref["Db"]) <= TOL[torch.float64]
    assert worst(host(sub["Eb"]), ref["Eb"]) <= TOL[torch.float64]

    w = inputs.WORKLOADS["forest_8x32768_b16"]
    g = inputs.generate(w)
    plan = selinv.TreePlan(g["parent"])
    rng = np.random.default_rng(9900)
    gd = to_dev(rng.standard_normal(g["diag"].shape), torch.float64)
    ge = to_dev(rng.standard_normal(g["edge"].shape), torch.float64)
    dd, ee = to_dev(g["diag"], torch.float64), to_dev(g["edge"], torch.float64)
    fwd = selinv.selinv_tree(plan, dd, ee)
    out = selinv.tree_backward(plan, dd, ee, fwd["G_diag"], fwd["G_edge"], gd, ge)
    assert (host(out["info"]) == -1).all()
    dD = torch.tril(to_dev(rng.standard_normal(g["diag"].shape), torch.float64))
    dE = to_dev(rng.standard_normal(g["edge"].shape), torch.float64)
    root = torch.from_numpy(g["parent"] < 0).to("cuda")
    dE[root] = 0.0

    def loss(eps):
        o = selinv.selinv_tree(plan, dd + eps * dD, ee + eps * dE)
        return float((o["G_diag"] * gd).sum() + (o["G_edge"] * ge).sum())

    h = 1e-4
    fd = (loss(h) - loss(-h)) / (2 * h)
    an = float((out["Db"] * dD).sum() + (out["Eb"] * dE).sum())
    assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (fd, an)


def test_tree_backward_not_spd(cuda_ok):
    P = np.stack([random_parent(12, 1), random_parent(12, 2)]).astype(np.int32)
    d, e = inputs.tree_inputs_from_parent(P, 4, seed=9950, load=1.0)
    d[1, 5] = -np.eye(4)
    plan = selinv.TreePlan(P)
    dd, ee = to_dev(d, torch.float64), to_dev(e, torch.float64)
    fwd = selinv.selinv_tree(plan, dd, ee, check=False)
    out = selinv.tree_backward(plan, dd, ee, fwd["G_diag"], fwd["G_edge"], check=False)
    info = host(out["info"])
    assert info[0] == -1 and info[1] >= 0
