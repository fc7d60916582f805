"""Several right-hand sides from one factorisation, X = A^-1 R (b <= 16), on the
GPU against the oracle's solve column by column, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from sparse_spd_selected_b200 import inputs, selinv
from tests.parity import TOL, host, logdet_err, to_dev, worst

pytestmark = pytest.mark.gpu


def ref_solve(d, l, R):
    cols = [oracle.chain(d, l, R[..., c], want_g=False) for c in range(R.shape[-1])]
    return np.stack([c["x"] for c in cols], axis=-1), cols[0]["logdet"]


@pytest.mark.parametrize("b,L,k", [(16, 9, 1), (16, 9, 16), (16, 9, 5), (7, 6, 3), (4, 17, 33),
                                   (1, 5, 2), (16, 1, 4), (12, 3, 17)])
def test_multi_rhs_f64(cuda_ok, b, L, k):
    d, l, _ = inputs.chain_inputs(3, L, b, seed=9000 + 7 * b + L + k, load=1.0, with_rhs=False)
    R = np.random.default_rng([9000, b, L, k]).standard_normal((3, L, b, k))
    dd, ll, rr = (to_dev(a, torch.float64) for a in (d, l, R))
    x, ld, info = selinv.chain_solve_multi(dd, ll, rr)
    ref_x, ref_ld = ref_solve(host(dd), host(ll), R)
    assert x.shape == (3, L, b, k)
    assert worst(host(x), ref_x) <= TOL[torch.float64]
    assert logdet_err(host(ld), ref_ld) <= TOL[torch.float64]
    assert (host(info) == -1).all()


def test_multi_rhs_f32(cuda_ok):
    d, l, _ = inputs.chain_inputs(4, 10, 16, seed=9100, load=1.0, with_rhs=False)
    R = np.random.default_rng(9101).standard_normal((4, 10, 16, 20))
    dd, ll, rr = (to_dev(a, torch.float32) for a in (d, l, R))
    x, _, _ = selinv.chain_solve_multi(dd, ll, rr)
    ref_x, _ = ref_solve(host(dd), host(ll), host(rr))
    assert worst(host(x), ref_x) <= TOL[torch.float32]


def test_multi_rhs_full_size(cuda_ok):
    """4096 chains of 64 blocks of 16 with 16 right-hand sides, sampled chains."""
    w = inputs.WORKLOADS["chain_4096x64_b16"]
    g = inputs.generate(w)
    R = np.random.default_rng(9200).standard_normal((w.batch, w.L, w.b, 16))
    dd, ll, rr = (to_dev(a, torch.float64) for a in (g["diag"], g["lower"], R))
    x, ld, _ = selinv.chain_solve_multi(dd, ll, rr)
    pick = [0, 777, 4095]
    ref_x, ref_ld = ref_solve(g["diag"][pick], g["lower"][pick], R[pick])
    assert worst(host(x[pick]), ref_x) <= TOL[torch.float64]
    assert logdet_err(host(ld[pick]), ref_ld) <= TOL[torch.float64]


def test_multi_rhs_errors(cuda_ok):
    d, l, _ = inputs.chain_inputs(2, 4, 20, seed=9300, load=1.0, with_rhs=False)
    R = np.zeros((2, 4, 20, 3))
    with pytest.raises(selinv.SelinvError):        # b > 16 not supported here
        selinv.chain_solve_multi(to_dev(d, torch.float64), to_dev(l, torch.float64), to_dev(R, torch.float64))
    d, l, _ = inputs.chain_inputs(2, 4, 8, seed=9301, load=1.0, with_rhs=False)
    with pytest.raises(ValueError):                 # wrong rhs shape
        selinv.chain_solve_multi(to_dev(d, torch.float64), to_dev(l, torch.float64),
                                 to_dev(np.zeros((2, 4, 7, 3)), torch.float64))
