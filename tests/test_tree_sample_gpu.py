"""Gaussian draws on block trees, eta = L^-T z in the tree's elimination order,
on the GPU against the oracle's draws from the same z, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from sparse_spd_selected_b200 import inputs, selinv
from tests.dense import balanced_parent, path_parent, star_parent
from tests.parity import TOL, host, logdet_err, to_dev, worst, worst_vec

pytestmark = pytest.mark.gpu


def draws(P, diag, edge, z, dtype=torch.float64):
    plan = selinv.TreePlan(P)
    out = selinv.tree_sample(plan, to_dev(diag, dtype), to_dev(edge, dtype), to_dev(z, dtype))
    ref = oracle.tree_sample(P, host(to_dev(diag, dtype)), host(to_dev(edge, dtype)), host(to_dev(z, dtype)))
    assert (ref["info"] == -1).all()
    return out, ref


@pytest.mark.parametrize("b", [1, 3, 8, 13, 16])
def test_tree_sample_topologies(cuda_ok, b):
    n = 37
    rng = np.random.default_rng(100 + b)
    pr = np.full(n, -1, dtype=np.int32)
    for v in range(n - 1):
        pr[v] = rng.integers(v + 1, n)
    P = np.stack([inputs.random_parent(rng, n), path_parent(n), star_parent(n), balanced_parent(n, 3), pr])
    diag, edge = inputs.tree_inputs_from_parent(P, b, seed=200 + b, load=0.5)
    z = rng.standard_normal((5, n, b))
    out, ref = draws(P, diag, edge, z)
    assert worst_vec(host(out["eta"]), ref["eta"]) <= TOL[torch.float64]
    assert logdet_err(host(out["logdet"]), ref["logdet"]) <= TOL[torch.float64]
    assert (host(out["info"]) == -1).all()


def test_tree_sample_single_node_and_f32(cuda_ok):
    P = np.array([[-1]], dtype=np.int32)
    diag, edge = inputs.tree_inputs_from_parent(P, 16, seed=300, load=1.0)
    z = np.random.default_rng(301).standard_normal((1, 1, 16))
    out, ref = draws(P, diag, edge, z)
    assert worst_vec(host(out["eta"]), ref["eta"]) <= TOL[torch.float64]
    rng = np.random.default_rng(302)
    P = np.stack([inputs.random_parent(rng, 50) for _ in range(3)])
    diag, edge = inputs.tree_inputs_from_parent(P, 16, seed=303, load=1.0)
    z = rng.standard_normal((3, 50, 16))
    out, ref = draws(P, diag, edge, z, torch.float32)
    assert worst_vec(host(out["eta"]), ref["eta"]) <= TOL[torch.float32]


def test_tree_sample_full_size_forest(cuda_ok):
    """8 random trees of 32768 nodes, b = 16; oracle on two trees."""
    w = inputs.WORKLOADS["forest_8x32768_b16"]
    g = inputs.generate(w)
    z = inputs.standard_normals(w.batch, w.L, w.b, w.seed)
    plan = selinv.TreePlan(g["parent"])
    out = selinv.tree_sample(plan, to_dev(g["diag"], torch.float64), to_dev(g["edge"], torch.float64),
                             to_dev(z, torch.float64))
    pick = [0, 7]
    ref = oracle.tree_sample(g["parent"][pick], g["diag"][pick], g["edge"][pick], z[pick])
    assert worst_vec(host(out["eta"][pick]), ref["eta"]) <= TOL[torch.float64]
    assert logdet_err(host(out["logdet"][pick]), ref["logdet"]) <= TOL[torch.float64]


def test_tree_sample_not_spd(cuda_ok):
    rng = np.random.default_rng(400)
    P = np.stack([inputs.random_parent(rng, 20) for _ in range(3)])
    diag, edge = inputs.tree_inputs_from_parent(P, 4, seed=401, load=1.0)
    diag[1, 7] = -np.eye(4)
    z = rng.standard_normal((3, 20, 4))
    plan = selinv.TreePlan(P)
    out = selinv.tree_sample(plan, to_dev(diag, torch.float64), to_dev(edge, torch.float64),
                             to_dev(z, torch.float64), check=False)
    info = host(out["info"]).tolist()
    assert info[0] == -1 and info[2] == -1 and info[1] >= 0
