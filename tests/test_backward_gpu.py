"""Cotangents of the chain selected inverse on the GPU (selinv_chain_backward,
b <= 16) against the oracle's dense definition Ab = -A^-1 Gbar A^-1, through
the C ABI, and the autograd wrapper built on it."""
import numpy as np
import pytest
import torch

import oracle
from sparse_spd_selected_b200 import inputs, selinv
from tests.parity import TOL, host, to_dev, worst

pytestmark = pytest.mark.gpu


def case(lead, L, b, seed, dtype, load=1.0, null_lower_cot=False):
    batch = int(np.prod(lead))
    d, l, _ = inputs.chain_inputs(batch, L, b, seed=seed, load=load, with_rhs=False)
    d = d.reshape(lead + (L, b, b))
    l = l.reshape(lead + (L - 1, b, b))
    rng = np.random.default_rng([seed, 7])
    gd = rng.standard_normal(d.shape)
    gl = np.zeros(l.shape) if null_lower_cot else rng.standard_normal(l.shape)
    dd, ll = to_dev(d, dtype), to_dev(l, dtype)
    fwd = selinv.selinv_chain(dd, ll)
    out = selinv.chain_backward(dd, ll, fwd["G_diag"], fwd["G_lower"], to_dev(gd, dtype),
                                None if null_lower_cot else to_dev(gl, dtype))
    ref = oracle.chain_backward(host(dd), host(ll), host(to_dev(gd, dtype)), host(to_dev(gl, dtype)))
    assert (ref["info"] == -1).all()
    return out, ref


@pytest.mark.parametrize("b", [1, 3, 8, 13, 16])
@pytest.mark.parametrize("L", [1, 2, 5, 19])
def test_backward_f64(cuda_ok, b, L):
    out, ref = case((3,), L, b, 9000 + 10 * b + L, torch.float64)
    assert worst(host(out["Db"]), ref["Db"]) <= TOL[torch.float64]
    if L > 1:
        assert worst(host(out["Bb"]), ref["Bb"]) <= TOL[torch.float64]
    assert (host(out["info"]) == -1).all()
    assert np.all(np.triu(host(out["Db"]), 1) == 0.0)          # nothing above the diagonal


@pytest.mark.parametrize("b,L", [(16, 9), (5, 12)])
def test_backward_f32(cuda_ok, b, L):
    out, ref = case((4,), L, b, 9100 + b, torch.float32, load=2.0)
    assert worst(host(out["Db"]), ref["Db"]) <= TOL[torch.float32]
    assert worst(host(out["Bb"]), ref["Bb"]) <= TOL[torch.float32]


def test_backward_null_cotangent_and_leading_dims(cuda_ok):
    """Gb_lower = None is a zero cotangent; leading batch dimensions flatten."""
    out, ref = case((2, 3), 7, 16, 9200, torch.float64, null_lower_cot=True)
    assert worst(host(out["Db"]), ref["Db"], 2) <= TOL[torch.float64]
    assert worst(host(out["Bb"]), ref["Bb"], 2) <= TOL[torch.float64]


def test_autograd_matches_oracle(cuda_ok):
    """loss = <Wd, G_diag> + <Wl, G_lower> through selinv_chain_ad; the gradients
    of diag and lower are the oracle's cotangents for (Wd, Wl)."""
    L, b = 6, 4
    d, l, _ = inputs.chain_inputs(2, L, b, seed=9300, load=1.0, with_rhs=False)
    rng = np.random.default_rng(9300)
    wd, wl = rng.standard_normal(d.shape), rng.standard_normal(l.shape)
    dd = to_dev(d, torch.float64).requires_grad_(True)
    ll = to_dev(l, torch.float64).requires_grad_(True)
    Gd, Gl = selinv.selinv_chain_ad(dd, ll)
    loss = (Gd * to_dev(wd, torch.float64)).sum() + (Gl * to_dev(wl, torch.float64)).sum()
    loss.backward()
    ref = oracle.chain_backward(d, l, wd, wl)
    assert worst(host(dd.grad), ref["Db"]) <= TOL[torch.float64]
    assert worst(host(ll.grad), ref["Bb"]) <= TOL[torch.float64]


def test_backward_full_size_sampled(cuda_ok):
    """4096 chains x 64 blocks of 16 (the b = 16 chain workload's shape); the
    oracle's dense definition on two of them."""
    w = inputs.WORKLOADS["chain_4096x64_b16"]
    g = inputs.generate(w)
    rng = np.random.default_rng(9400)
    gd = rng.standard_normal(g["diag"].shape)
    gl = rng.standard_normal(g["lower"].shape)
    dd, ll = to_dev(g["diag"], torch.float64), to_dev(g["lower"], torch.float64)
    fwd = selinv.selinv_chain(dd, ll)
    out = selinv.chain_backward(dd, ll, fwd["G_diag"], fwd["G_lower"], to_dev(gd, torch.float64),
                                to_dev(gl, torch.float64))
    assert (host(out["info"]) == -1).all()
    pick = [0, w.batch - 1]
    ref = oracle.chain_backward(g["diag"][pick], g["lower"][pick], gd[pick], gl[pick])
    assert worst(host(out["Db"])[pick], ref["Db"]) <= TOL[torch.float64]
    assert worst(host(out["Bb"])[pick], ref["Bb"]) <= TOL[torch.float64]


def test_backward_not_spd_reports_block(cuda_ok):
    L, b = 6, 4
    d, l, _ = inputs.chain_inputs(2, L, b, seed=9500, load=1.0, with_rhs=False)
    d[1, 3] = -np.eye(b)                       # block 3 of chain 1 is not positive definite
    dd, ll = to_dev(d, torch.float64), to_dev(l, torch.float64)
    fwd = selinv.selinv_chain(dd, ll, check=False)
    out = selinv.chain_backward(dd, ll, fwd["G_diag"], fwd["G_lower"], fwd["G_diag"], fwd["G_lower"],
                                check=False)
    info = host(out["info"])
    assert info[0] == -1 and info[1] == host(fwd["info"])[1] >= 0
    with pytest.raises(selinv.NotSPDError):
        selinv.chain_backward(dd, ll, fwd["G_diag"], fwd["G_lower"], fwd["G_diag"], fwd["G_lower"])
