"""Selected inverse of block lower-bidiagonal matrices with general blocks on
the GPU (selinv_bidiag, b <= 16) against the oracle's dense pivoted inverse,
through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from sparse_spd_selected_b200 import inputs, selinv
from tests.parity import TOL, host, to_dev, worst

pytestmark = pytest.mark.gpu


def check(d, l, dtype, lead_ndim=1):
    dd, ll = to_dev(d, dtype), to_dev(l, dtype)
    out = selinv.bidiag(dd, ll)
    ref = oracle.bidiag(host(dd), host(ll))
    assert (ref["info"] == -1).all()
    assert worst(host(out["G_diag"]), ref["G_diag"], lead_ndim) <= TOL[dtype]
    if d.shape[-3] > 1:
        assert worst(host(out["G_lower"]), ref["G_lower"], lead_ndim) <= TOL[dtype]
    assert (host(out["info"]) == -1).all()


@pytest.mark.parametrize("b", [1, 2, 5, 11, 16])
@pytest.mark.parametrize("L", [1, 2, 7, 33])
def test_bidiag_f64(cuda_ok, b, L):
    d, l = inputs.bidiag_inputs(5, L, b, seed=10000 + 10 * b + L, load=2.0)   # odd batch: a half-warp idles
    check(d, l, torch.float64)


@pytest.mark.parametrize("b,L", [(16, 9), (6, 12)])
def test_bidiag_f32(cuda_ok, b, L):
    d, l = inputs.bidiag_inputs(4, L, b, seed=10100 + b, load=3.0)
    check(d, l, torch.float32)


def test_bidiag_needs_pivoting_and_leading_dims(cuda_ok):
    """Blocks with a zero diagonal (no elimination order without row exchanges
    starts on the diagonal) and ill-scaled rows; leading batch dimensions."""
    d, l = inputs.bidiag_inputs(6, 5, 4, seed=10200, load=0.0)
    rng = np.random.default_rng(10200)
    for e in range(6):
        for i in range(5):
            perm = rng.permutation(4)
            d[e, i] = np.eye(4)[perm] * rng.uniform(0.5, 2.0, 4)[:, None] + 0.1 * d[e, i]
            d[e, i][np.arange(4), np.arange(4)] = 0.0
    check(d.reshape(2, 3, 5, 4, 4), l.reshape(2, 3, 4, 4, 4), torch.float64, lead_ndim=2)


def test_bidiag_full_size_sampled(cuda_ok):
    """4096 chains x 64 blocks of 16 (the b = 16 chain workload's shape with
    general blocks); the oracle's dense inverse on two of them."""
    d, l = inputs.bidiag_inputs(4096, 64, 16, seed=10300, load=2.0)
    out = selinv.bidiag(to_dev(d, torch.float64), to_dev(l, torch.float64))
    pick = [0, 4095]
    ref = oracle.bidiag(d[pick], l[pick])
    assert worst(host(out["G_diag"])[pick], ref["G_diag"]) <= TOL[torch.float64]
    assert worst(host(out["G_lower"])[pick], ref["G_lower"]) <= TOL[torch.float64]
    assert (host(out["info"]) == -1).all()


def test_bidiag_singular_block(cuda_ok):
    d, l = inputs.bidiag_inputs(3, 6, 3, seed=10400, load=2.0)
    d[1, 4] = np.array([[1.0, 2.0, 3.0], [2.0, 4.0, 6.0], [0.5, -1.0, 2.0]])   # rank 2
    out = selinv.bidiag(to_dev(d, torch.float64), to_dev(l, torch.float64), check=False)
    assert host(out["info"]).tolist() == [-1, 4, -1]
    with pytest.raises(selinv.SingularBlockError):
        selinv.bidiag(to_dev(d, torch.float64), to_dev(l, torch.float64))


def check_backward(d, l, dtype, lead_ndim=1, null_lower=False):
    dd, ll = to_dev(d, dtype), to_dev(l, dtype)
    fwd = selinv.bidiag(dd, ll)
    rng = np.random.default_rng(int(d.size) % 1000)
    gd = rng.standard_normal(d.shape)
    gl = np.zeros(l.shape) if null_lower else rng.standard_normal(l.shape)
    out = selinv.bidiag_backward(fwd["G_diag"], fwd["G_lower"], to_dev(gd, dtype),
                                 None if null_lower else to_dev(gl, dtype))
    ref = oracle.bidiag_backward(host(dd), host(ll), host(to_dev(gd, dtype)), host(to_dev(gl, dtype)))
    assert (ref["info"] == -1).all()
    assert worst(host(out["Mb_diag"]), ref["Mb_diag"], lead_ndim) <= TOL[dtype]
    if d.shape[-3] > 1:
        assert worst(host(out["Mb_lower"]), ref["Mb_lower"], lead_ndim) <= TOL[dtype]


@pytest.mark.parametrize("b", [1, 3, 8, 16])
@pytest.mark.parametrize("L", [1, 2, 9])
def test_bidiag_backward_f64(cuda_ok, b, L):
    d, l = inputs.bidiag_inputs(3, L, b, seed=10500 + 10 * b + L, load=2.0)
    check_backward(d, l, torch.float64)


def test_bidiag_backward_f32_null_and_leading_dims(cuda_ok):
    d, l = inputs.bidiag_inputs(4, 7, 16, seed=10600, load=3.0)
    check_backward(d, l, torch.float32)
    d, l = inputs.bidiag_inputs(6, 5, 5, seed=10601, load=2.0)
    check_backward(d.reshape(2, 3, 5, 5, 5), l.reshape(2, 3, 4, 5, 5), torch.float64, lead_ndim=2, null_lower=True)


def test_bidiag_autograd_matches_oracle(cuda_ok):
    d, l = inputs.bidiag_inputs(2, 6, 4, seed=10700, load=2.0)
    rng = np.random.default_rng(10700)
    wd, wl = rng.standard_normal(d.shape), rng.standard_normal(l.shape)
    dd = to_dev(d, torch.float64).requires_grad_(True)
    ll = to_dev(l, torch.float64).requires_grad_(True)
    Gd, Gl = selinv.bidiag_ad(dd, ll)
    ((Gd * to_dev(wd, torch.float64)).sum() + (Gl * to_dev(wl, torch.float64)).sum()).backward()
    ref = oracle.bidiag_backward(d, l, wd, wl)
    assert worst(host(dd.grad), ref["Mb_diag"]) <= TOL[torch.float64]
    assert worst(host(ll.grad), ref["Mb_lower"]) <= TOL[torch.float64]


def test_bidiag_backward_full_size_sampled(cuda_ok):
    d, l = inputs.bidiag_inputs(4096, 64, 16, seed=10800, load=2.0)
    dd, ll = to_dev(d, torch.float64), to_dev(l, torch.float64)
    fwd = selinv.bidiag(dd, ll)
    rng = np.random.default_rng(10800)
    gd, gl = rng.standard_normal(d.shape), rng.standard_normal(l.shape)
    out = selinv.bidiag_backward(fwd["G_diag"], fwd["G_lower"], to_dev(gd, torch.float64), to_dev(gl, torch.float64))
    pick = [0, 4095]
    ref = oracle.bidiag_backward(d[pick], l[pick], gd[pick], gl[pick])
    assert worst(host(out["Mb_diag"])[pick], ref["Mb_diag"]) <= TOL[torch.float64]
    assert worst(host(out["Mb_lower"])[pick], ref["Mb_lower"]) <= TOL[torch.float64]
