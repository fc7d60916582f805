"""Gaussian draws eta = A^-1 r + L^-T z on the GPU against the oracle's draws
from the same standard normals z, through the C ABI (b <= 16 chains)."""
import numpy as np
import pytest
import torch

import oracle
from sparse_spd_selected_b200 import inputs, selinv
from tests.dense import chain_dense, rel
from tests.parity import TOL, host, logdet_err, to_dev, worst, worst_vec

pytestmark = pytest.mark.gpu


def draw(batch, L, b, seed, with_rhs, dtype, load=1.0):
    d, l, r = inputs.chain_inputs(batch, L, b, seed=seed, load=load, with_rhs=True)
    z = np.random.default_rng([seed, 99]).standard_normal(r.shape)
    dd, ll, zz = to_dev(d, dtype), to_dev(l, dtype), to_dev(z, dtype)
    rr = to_dev(r, dtype) if with_rhs else None
    out = selinv.chain_sample(dd, ll, zz, rr)
    ref = oracle.chain_sample(host(dd), host(ll), host(zz), rhs=host(rr) if with_rhs else None)
    assert (ref["info"] == -1).all()
    return out, ref


@pytest.mark.parametrize("b", [1, 2, 4, 7, 16])
@pytest.mark.parametrize("L", [1, 2, 5, 17])
@pytest.mark.parametrize("with_rhs", [False, True])
def test_sample_f64(cuda_ok, b, L, with_rhs):
    out, ref = draw(3, L, b, 8000 + 10 * b + L, with_rhs, torch.float64)
    assert worst_vec(host(out["eta"]), ref["eta"]) <= TOL[torch.float64]
    assert logdet_err(host(out["logdet"]), ref["logdet"]) <= TOL[torch.float64]
    assert (host(out["info"]) == -1).all()


@pytest.mark.parametrize("b,L", [(16, 9), (5, 12)])
def test_sample_f32(cuda_ok, b, L):
    out, ref = draw(4, L, b, 8100 + b, True, torch.float32)
    assert worst_vec(host(out["eta"]), ref["eta"]) <= TOL[torch.float32]


def test_sample_standard_basis_is_the_cholesky_factor(cuda_ok):
    """Draws for z = e_k are the columns of L^-T, L = numpy's Cholesky factor of
    the dense A: upper triangular, and W W^T = A^-1 (the pages' covariance check)."""
    L, b = 4, 3
    N = L * b
    d, l, _ = inputs.chain_inputs(1, L, b, seed=8200, load=1.0, with_rhs=False)
    A = chain_dense(d[0], l[0])
    z = np.eye(N).reshape(N, L, b)
    out = selinv.chain_sample(to_dev(np.repeat(d, N, 0), torch.float64), to_dev(np.repeat(l, N, 0), torch.float64),
                              to_dev(z, torch.float64))
    W = host(out["eta"]).reshape(N, N).T
    assert rel(W, np.linalg.inv(np.linalg.cholesky(A)).T) <= 1e-12
    assert rel(W @ W.T, np.linalg.inv(A)) <= 1e-12


def test_sample_with_zero_z_is_the_solve(cuda_ok):
    """z = 0 leaves the mean: bitwise the solve-only call's x."""
    d, l, r = inputs.chain_inputs(64, 20, 16, seed=8300, load=1.0, with_rhs=True)
    dd, ll, rr = (to_dev(a, torch.float64) for a in (d, l, r))
    out = selinv.chain_sample(dd, ll, torch.zeros_like(rr), rr)
    x, ld, _ = selinv.chain_solve(dd, ll, rr)
    assert torch.equal(out["eta"], x) and torch.equal(out["logdet"], ld)


def test_sample_full_size_b16(cuda_ok):
    """4096 chains of 64 blocks of 16 (the headline chain workload's shape)."""
    w = inputs.WORKLOADS["chain_4096x64_b16"]
    g = inputs.generate(w)
    z = np.random.default_rng([w.seed, 98]).standard_normal(g["rhs"].shape)
    dd, ll, rr, zz = (to_dev(g[k] if k != "z" else z, torch.float64) for k in ("diag", "lower", "rhs", "z"))
    out = selinv.chain_sample(dd, ll, zz, rr)
    pick = [0, 1, 2047, 4095]
    ref = oracle.chain_sample(g["diag"][pick], g["lower"][pick], z[pick], rhs=g["rhs"][pick])
    assert worst_vec(host(out["eta"][pick]), ref["eta"]) <= TOL[torch.float64]
    assert logdet_err(host(out["logdet"][pick]), ref["logdet"]) <= TOL[torch.float64]


def test_sample_not_spd_and_unsupported(cuda_ok):
    d, l, r = inputs.chain_inputs(3, 6, 4, seed=8400, load=1.0, with_rhs=True)
    d[1, 3] = -np.eye(4)
    z = np.zeros_like(r)
    out = selinv.chain_sample(to_dev(d, torch.float64), to_dev(l, torch.float64), to_dev(z, torch.float64),
                              check=False)
    assert host(out["info"]).tolist() == [-1, 3, -1]
    with pytest.raises(selinv.NotSPDError):
        selinv.chain_sample(to_dev(d, torch.float64), to_dev(l, torch.float64), to_dev(z, torch.float64))
    d2, l2, r2 = inputs.chain_inputs(1, 3, 20, seed=8401, load=1.0, with_rhs=True)
    with pytest.raises(selinv.SelinvError):          # float32 draws stop at b = 16
        selinv.chain_sample(to_dev(d2, torch.float32), to_dev(l2, torch.float32), to_dev(r2, torch.float32))


@pytest.mark.parametrize("b", [17, 32, 40, 64, 100, 128])
@pytest.mark.parametrize("L", [1, 3, 6])
def test_sample_large_blocks_f64(cuda_ok, b, L):
    """Draws through the CTA kernel (R_i z_i met inside its blocked inverse)."""
    out, ref = draw(2, L, b, 8500 + b + L, L != 3, torch.float64)
    assert worst_vec(host(out["eta"]), ref["eta"]) <= TOL[torch.float64]
    assert logdet_err(host(out["logdet"]), ref["logdet"]) <= TOL[torch.float64]


def test_sample_grid_sampled(cuda_ok):
    """The grid workload's shape (256 chains of 128 blocks of 128): a Gibbs step
    eta = A^-1 r + L^-T z on all chains, two of them against the oracle."""
    d, l, r, _ = inputs.grid_inputs_torch(256, 128, 4, "cuda", torch.float64, True)
    z = torch.from_numpy(inputs.standard_normals(256, 128, 128, 4)).cuda()
    out = selinv.chain_sample(d, l, z, r)
    pick = [0, 255]
    ref = oracle.chain_sample(host(d[pick]), host(l[pick]), host(z[pick]), rhs=host(r[pick]))
    assert worst_vec(host(out["eta"][pick]), ref["eta"]) <= TOL[torch.float64]
    assert logdet_err(host(out["logdet"][pick]), ref["logdet"]) <= TOL[torch.float64]
