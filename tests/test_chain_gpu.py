"""GPU chain kernels vs the CPU oracle, called through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from sparse_spd_selected_b200 import inputs, selinv
from tests.parity import TOL, host, logdet_err, to_dev, worst, worst_vec

pytestmark = pytest.mark.gpu


def run_both(diag, lower, rhs, dtype, lead_ndim=1):
    """GPU (inputs rounded to dtype) vs oracle on the same rounded inputs."""
    d_dev, l_dev = to_dev(diag, dtype), to_dev(lower, dtype)
    r_dev = to_dev(rhs, dtype) if rhs is not None else None
    out = selinv.selinv_chain(d_dev, l_dev, r_dev)
    ref = oracle.chain(host(d_dev), host(l_dev), host(r_dev) if rhs is not None else None)
    assert (ref["info"] == -1).all()
    errs = {
        "G_diag": worst(host(out["G_diag"]), ref["G_diag"], lead_ndim),
        "G_lower": worst(host(out["G_lower"]), ref["G_lower"], lead_ndim) if diag.shape[-3] > 1 else 0.0,
        "logdet": logdet_err(host(out["logdet"]), ref["logdet"]),
    }
    if rhs is not None:
        errs["x"] = worst_vec(host(out["x"]), ref["x"], lead_ndim)
    assert (host(out["info"]) == -1).all()
    return errs, out


@pytest.mark.parametrize("b", [1, 2, 3, 4, 5, 7, 8, 9, 12, 15, 16])
@pytest.mark.parametrize("L", [1, 2, 3, 5, 17])
def test_small_blocks_f64(cuda_ok, b, L):
    diag, lower, rhs = inputs.chain_inputs(6, L, b, seed=1000 + 17 * b + L, load=0.5)
    errs, _ = run_both(diag, lower, rhs, torch.float64)
    assert max(errs.values()) <= TOL[torch.float64], errs


@pytest.mark.parametrize("b,L", [(4, 9), (16, 33), (11, 6)])
def test_small_blocks_f32(cuda_ok, b, L):
    diag, lower, rhs = inputs.chain_inputs(5, L, b, seed=2000 + b, load=2.0)
    errs, _ = run_both(diag, lower, rhs, torch.float32)
    assert max(errs.values()) <= TOL[torch.float32], errs


def test_leading_batch_dims(cuda_ok):
    diag, lower, rhs = inputs.chain_inputs(6, 7, 16, seed=3001, load=1.0)
    shp = (2, 3)
    errs, out = run_both(diag.reshape(shp + diag.shape[1:]), lower.reshape(shp + lower.shape[1:]),
                         rhs.reshape(shp + rhs.shape[1:]), torch.float64, lead_ndim=2)
    assert out["G_diag"].shape == (2, 3, 7, 16, 16) and out["logdet"].shape == (2, 3)
    assert max(errs.values()) <= 1e-9, errs


def test_quickstart_fact(cuda_ok):
    """G_diag[0] == inv(A)[0:4, 0:4] to 1e-10 on 8 blocks of 4 with diag_load 2.0."""
    w = inputs.WORKLOADS["chain_1x8_b4"]
    g = inputs.generate(w)
    out = selinv.selinv_chain(to_dev(g["diag"][0], torch.float64), to_dev(g["lower"][0], torch.float64),
                              to_dev(g["rhs"][0], torch.float64))
    from tests.dense import chain_dense
    inv = np.linalg.inv(chain_dense(g["diag"][0], g["lower"][0]))
    assert np.abs(host(out["G_diag"])[0] - inv[0:4, 0:4]).max() <= 1e-10
    errs, _ = run_both(g["diag"], g["lower"], g["rhs"], torch.float64)
    assert max(errs.values()) <= 1e-9, errs


def test_full_size_b16_sampled(cuda_ok):
    """4096 chains x 64 blocks of 16 (the benchmark launch), checked on sampled chains."""
    w = inputs.WORKLOADS["chain_4096x64_b16"]
    g = inputs.generate(w)
    d, l, r = (to_dev(g[k], torch.float64) for k in ("diag", "lower", "rhs"))
    out = selinv.selinv_chain(d, l, r)
    pick = [0, 1, 2, 777, 2048, 4094, 4095]
    ref = oracle.chain(g["diag"][pick], g["lower"][pick], g["rhs"][pick])
    assert worst(host(out["G_diag"][pick]), ref["G_diag"]) <= 1e-9
    assert worst(host(out["G_lower"][pick]), ref["G_lower"]) <= 1e-9
    assert worst_vec(host(out["x"][pick]), ref["x"]) <= 1e-9
    assert logdet_err(host(out["logdet"][pick]), ref["logdet"]) <= 1e-9
    # properties that hold for every chain: exact symmetry of G_ii, positive diagonal
    Gd = out["G_diag"]
    assert torch.equal(Gd, Gd.transpose(-1, -2))
    assert bool((torch.diagonal(Gd, dim1=-2, dim2=-1) > 0).all())


def test_upper_triangle_of_diag_is_not_read(cuda_ok):
    diag, lower, rhs = inputs.chain_inputs(3, 6, 16, seed=3100, load=1.0)
    d_dev = to_dev(diag, torch.float64)
    ref = selinv.selinv_chain(d_dev, to_dev(lower, torch.float64), to_dev(rhs, torch.float64))
    junk = d_dev.clone()
    iu = torch.triu_indices(16, 16, 1)
    junk[..., iu[0], iu[1]] = float("nan")
    out = selinv.selinv_chain(junk, to_dev(lower, torch.float64), to_dev(rhs, torch.float64))
    for k in ("G_diag", "G_lower", "logdet", "x"):
        assert torch.equal(out[k], ref[k]), k


def test_not_spd_reports_first_failing_block(cuda_ok):
    diag, lower, _ = inputs.chain_inputs(3, 7, 16, seed=3200, load=1.0)
    diag[1, 4] = -np.eye(16)
    diag[2, 0, 3, 3] = np.nan
    with pytest.raises(selinv.NotSPDError) as ei:
        selinv.selinv_chain(to_dev(diag, torch.float64), to_dev(lower, torch.float64))
    assert ei.value.info == [-1, 4, 0]
    out = selinv.selinv_chain(to_dev(diag, torch.float64), to_dev(lower, torch.float64), check=False)
    assert host(out["info"]).tolist() == [-1, 4, 0]


def test_deterministic(cuda_ok):
    diag, lower, rhs = inputs.chain_inputs(64, 20, 16, seed=3300, load=1.0)
    args = [to_dev(a, torch.float64) for a in (diag, lower, rhs)]
    a = selinv.selinv_chain(*args)
    b = selinv.selinv_chain(*args)
    for k in ("G_diag", "G_lower", "logdet", "x"):
        assert torch.equal(a[k], b[k]), k


def test_solve_only_and_logdet_only(cuda_ok):
    diag, lower, rhs = inputs.chain_inputs(9, 12, 16, seed=3400, load=1.0)
    d, l, r = (to_dev(a, torch.float64) for a in (diag, lower, rhs))
    full = selinv.selinv_chain(d, l, r)
    x, ld, info = selinv.chain_solve(d, l, r)
    assert torch.equal(x, full["x"]) and torch.equal(ld, full["logdet"])
    only = selinv.selinv_chain(d, l, want_g=False)
    assert torch.equal(only["logdet"], full["logdet"]) and only["G_diag"] is None


def test_workspace_too_small_is_rejected(cuda_ok):
    diag, lower, _ = inputs.chain_inputs(2, 5, 16, seed=3500, load=1.0)
    ws = torch.empty(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(ValueError):
        selinv.selinv_chain(to_dev(diag, torch.float64), to_dev(lower, torch.float64), workspace=ws)


def test_empty_batch(cuda_ok):
    d = torch.empty((0, 5, 16, 16), dtype=torch.float64, device="cuda")
    l = torch.empty((0, 4, 16, 16), dtype=torch.float64, device="cuda")
    out = selinv.selinv_chain(d, l)
    assert out["G_diag"].shape == (0, 5, 16, 16)


# ---------------- 16 < b <= 128: one CTA per chain ----------------

@pytest.mark.parametrize("b", [17, 24, 32, 33, 48, 64, 65, 100, 128])
@pytest.mark.parametrize("L", [1, 2, 5])
def test_large_blocks_f64(cuda_ok, b, L):
    diag, lower, rhs = inputs.chain_inputs(3, L, b, seed=4000 + 7 * b + L, load=0.5)
    errs, _ = run_both(diag, lower, rhs, torch.float64)
    assert max(errs.values()) <= TOL[torch.float64], errs


@pytest.mark.parametrize("b,L", [(32, 20), (64, 6), (128, 4), (40, 7)])
def test_large_blocks_f32(cuda_ok, b, L):
    diag, lower, rhs = inputs.chain_inputs(3, L, b, seed=5000 + b, load=2.0)
    errs, _ = run_both(diag, lower, rhs, torch.float32)
    assert max(errs.values()) <= TOL[torch.float32], errs


def test_large_solve_only_and_logdet_only(cuda_ok):
    diag, lower, rhs = inputs.chain_inputs(4, 9, 64, seed=5100, load=1.0)
    d, l, r = (to_dev(a, torch.float64) for a in (diag, lower, rhs))
    full = selinv.selinv_chain(d, l, r)
    x, ld, _ = selinv.chain_solve(d, l, r)
    assert torch.equal(x, full["x"]) and torch.equal(ld, full["logdet"])
    only = selinv.selinv_chain(d, l, want_g=False)
    assert torch.equal(only["logdet"], full["logdet"])
    Gd = full["G_diag"]
    assert torch.equal(Gd, Gd.transpose(-1, -2))


def test_grid_full_size_sampled(cuda_ok):
    """256 grid precisions (128 x 128 grid as 128 blocks of 128), checked on two elements
    against the oracle and against the spectral closed form."""
    from tests.pins import grid_closed_form
    w = inputs.WORKLOADS["grid_256x128_b128"]
    diag, lower, rhs, taus = inputs.grid_inputs_torch(w.batch, w.b, w.seed, "cuda")
    out = selinv.selinv_chain(diag, lower, rhs)
    pick = [0, 255]
    g = inputs.generate(w, elements=pick)
    ref = oracle.chain(g["diag"], g["lower"], g["rhs"])
    assert worst(host(out["G_diag"][pick]), ref["G_diag"]) <= 1e-9
    assert worst(host(out["G_lower"][pick]), ref["G_lower"]) <= 1e-9
    assert worst_vec(host(out["x"][pick]), ref["x"]) <= 1e-9
    assert logdet_err(host(out["logdet"][pick]), ref["logdet"]) <= 1e-9
    for k, e in enumerate(pick):
        Gd, Gl, ld, x = grid_closed_form(w.b, g["tau"][k], g["rhs"][k], rows=[0, 63, 127])
        for i in (0, 63, 127):
            assert worst(host(out["G_diag"][e, i])[None], Gd[i][None]) <= 1e-9
        for i in (0, 63):
            assert worst(host(out["G_lower"][e, i])[None], Gl[i][None]) <= 1e-9
        assert abs(host(out["logdet"][e]) - ld) / abs(ld) <= 1e-9
        assert worst_vec(host(out["x"][e])[None], x[None]) <= 1e-9


@pytest.mark.parametrize("dtype", [torch.float64, torch.float32])
def test_long_chains_full_size_sampled(cuda_ok, dtype):
    """64 chains of 4096 blocks of 32 (diag load 0.5), float64 and float32, sampled chains."""
    w = inputs.WORKLOADS["chain_64x4096_b32"]
    g = inputs.generate(w)
    d, l = to_dev(g["diag"], dtype), to_dev(g["lower"], dtype)
    out = selinv.selinv_chain(d, l)
    pick = [0, 63]
    ref = oracle.chain(host(d[pick]), host(l[pick]))
    tol = TOL[dtype]
    assert worst(host(out["G_diag"][pick]), ref["G_diag"]) <= tol
    assert worst(host(out["G_lower"][pick]), ref["G_lower"]) <= tol
    assert logdet_err(host(out["logdet"][pick]), ref["logdet"]) <= tol


def test_pivot_reciprocal_against_cuda_division(cuda_ok):
    """A 1 x 1 block's inverse is the kernel's pivot reciprocal (Newton-refined
    hardware estimate): it must agree with CUDA's IEEE division to a few ulp
    over a wide range of magnitudes, and log det with log."""
    rng = np.random.default_rng(123)
    d = np.exp(rng.uniform(-40.0, 40.0, size=200_000))
    dev = torch.from_numpy(d).cuda().reshape(-1, 1, 1, 1)
    out = selinv.selinv_chain(dev, None)
    ref = 1.0 / dev
    ulp = torch.abs(out["G_diag"] - ref) / (torch.finfo(torch.float64).eps * torch.abs(ref))
    assert float(ulp.max()) <= 4.0
    assert float(torch.max(torch.abs(out["logdet"] - torch.log(dev.reshape(-1))))) <= 1e-12


def test_pivot_reciprocal_at_the_ends_of_the_range(cuda_ok):
    """Pivots near the ends of the float64 range: in [2^-1022, 2^1022) the
    kernel's Newton-refined reciprocal agrees with CUDA's 1/d to a few ulp;
    outside it (subnormal pivots, pivots whose reciprocal would be subnormal,
    pivots whose reciprocal overflows) the fast reciprocal would flush, so the
    block is reported in info like a non-positive pivot."""
    rng = np.random.default_rng(321)
    small = 2.0 ** rng.uniform(-1022.0, -1000.0, 4000)
    large = 2.0 ** rng.uniform(1000.0, 1021.9, 4000)
    out_of_range = np.concatenate([
        2.0 ** rng.uniform(1022.0, 1023.9, 100),                 # reciprocal below 2^-1022
        2.0 ** np.array([-1022.25, -1023.0, -1030.0, -1060.0]),  # subnormal pivots
        np.array([5e-324])])
    d = np.concatenate([small, large, out_of_range])
    dev = torch.from_numpy(d).cuda().reshape(-1, 1, 1, 1)
    out = selinv.selinv_chain(dev, None, check=False)
    G = out["G_diag"].reshape(-1)
    ref = 1.0 / dev.reshape(-1)
    info = host(out["info"])
    n1 = small.size + large.size
    ulp = torch.abs(G[:n1] - ref[:n1]) / (torch.finfo(torch.float64).eps * torch.abs(ref[:n1]))
    assert float(ulp.max()) <= 4.0
    assert (info[:n1] == -1).all()
    assert (info[n1:] == 0).all()
    with pytest.raises(selinv.NotSPDError):
        selinv.selinv_chain(dev[n1:], None)


# ---------------- 16 < b <= 32 without a right-hand side: two-ended kernel ----------------

@pytest.mark.parametrize("b", [17, 20, 24, 31, 32])
@pytest.mark.parametrize("L", [1, 2, 3, 4, 5, 8, 33])
def test_two_ended_blocks_f64(cuda_ok, b, L):
    diag, lower, _ = inputs.chain_inputs(3, L, b, seed=6000 + 3 * b + L, load=0.5, with_rhs=False)
    errs, out = run_both(diag, lower, None, torch.float64)
    assert max(errs.values()) <= TOL[torch.float64], errs
    Gd = out["G_diag"]
    assert torch.equal(Gd, Gd.transpose(-1, -2))


@pytest.mark.parametrize("b,L", [(32, 40), (24, 9)])
def test_two_ended_blocks_f32(cuda_ok, b, L):
    diag, lower, _ = inputs.chain_inputs(3, L, b, seed=6100 + b, load=1.0, with_rhs=False)
    errs, _ = run_both(diag, lower, None, torch.float32)
    assert max(errs.values()) <= TOL[torch.float32], errs


def test_two_ended_logdet_only_and_not_spd(cuda_ok):
    diag, lower, _ = inputs.chain_inputs(4, 12, 32, seed=6200, load=1.0, with_rhs=False)
    d, l = to_dev(diag, torch.float64), to_dev(lower, torch.float64)
    full = selinv.selinv_chain(d, l)
    only = selinv.selinv_chain(d, l, want_g=False)
    assert torch.equal(only["logdet"], full["logdet"])
    bad = diag.copy()
    bad[1, 3] = -np.eye(32)          # top half
    bad[2, 10] = -np.eye(32)         # bottom half
    out = selinv.selinv_chain(to_dev(bad, torch.float64), l, check=False)
    info = host(out["info"]).tolist()
    assert info[0] == -1 and info[3] == -1 and info[1] >= 0 and info[2] >= 0


@pytest.mark.parametrize("batch,L,b", [(2, 600, 32), (3, 200, 20), (1, 96, 32), (5, 401, 17)])
def test_segmented_chains_f64(cuda_ok, batch, L, b):
    """Chains cut into segments (separators eliminated last) against the oracle's
    sequential elimination: every block of G, log det."""
    assert selinv.chain_segments(batch, L, b) >= 3
    diag, lower, _ = inputs.chain_inputs(batch, L, b, seed=7000 + L + b, load=0.5, with_rhs=False)
    errs, out = run_both(diag, lower, None, torch.float64)
    assert max(errs.values()) <= TOL[torch.float64], errs
    Gd = out["G_diag"]
    assert torch.equal(Gd, Gd.transpose(-1, -2))


def test_segmented_chains_f32(cuda_ok):
    assert selinv.chain_segments(2, 300, 32) >= 3
    diag, lower, _ = inputs.chain_inputs(2, 300, 32, seed=7100, load=1.0, with_rhs=False)
    errs, _ = run_both(diag, lower, None, torch.float32)
    assert max(errs.values()) <= TOL[torch.float32], errs


def test_segmented_logdet_only_and_not_spd(cuda_ok):
    """Log det without G (two-ended kernel) agrees with the segmented call; a
    chain that is not positive definite is reported, its neighbours are not."""
    diag, lower, _ = inputs.chain_inputs(3, 300, 32, seed=7200, load=1.0, with_rhs=False)
    d, l = to_dev(diag, torch.float64), to_dev(lower, torch.float64)
    assert selinv.chain_segments(3, 300, 32) >= 3 and selinv.chain_segments(3, 300, 32, want_g=False) == 0
    full = selinv.selinv_chain(d, l)
    only = selinv.selinv_chain(d, l, want_g=False)
    assert logdet_err(host(only["logdet"]), host(full["logdet"])) <= 1e-12
    bad = diag.copy()
    bad[1, 150] = -np.eye(32)
    bad[2, [7, 100, 299]] = -np.eye(32)
    out = selinv.selinv_chain(to_dev(bad, torch.float64), l, check=False)
    info = host(out["info"]).tolist()
    assert info[0] == -1 and info[1] >= 0 and info[2] >= 0
    with pytest.raises(selinv.NotSPDError):
        selinv.selinv_chain(to_dev(bad, torch.float64), l)


def test_segmented_deterministic_and_leading_dims(cuda_ok):
    """The segmented path gives bitwise identical results on repeated calls, and
    takes leading batch dimensions like every other chain path."""
    diag, lower, _ = inputs.chain_inputs(4, 160, 32, seed=7300, load=0.8, with_rhs=False)
    assert selinv.chain_segments(4, 160, 32) >= 3
    d, l = to_dev(diag, torch.float64), to_dev(lower, torch.float64)
    a = selinv.selinv_chain(d, l)
    b = selinv.selinv_chain(d, l)
    for k in ("G_diag", "G_lower", "logdet", "info"):
        assert torch.equal(a[k], b[k]), k
    shp = (2, 2)
    errs, out = run_both(diag.reshape(shp + diag.shape[1:]), lower.reshape(shp + lower.shape[1:]), None,
                         torch.float64, lead_ndim=2)
    assert out["G_diag"].shape == (2, 2, 160, 32, 32) and out["logdet"].shape == (2, 2)
    assert max(errs.values()) <= TOL[torch.float64], errs


@pytest.mark.parametrize("b", [5, 16, 32, 64])
def test_validate_reports_non_finite_inputs(cuda_ok, b):
    """validate=True (SELINV_CHECK): an element whose read entries hold a NaN or
    an infinity reports info = -3 - k for the first such block k; entries the
    call does not read (the upper triangle of D) are not checked; clean
    elements are untouched; check=True raises NonFiniteInputError."""
    diag, lower, rhs = inputs.chain_inputs(5, 7, b, seed=3500 + b, load=1.0)
    diag[1, 3, b - 1, 0] = np.nan            # lower triangle of D_3
    lower[2, 2, 0, b - 1] = np.inf           # B_2
    rhs[3, 5, 0] = np.nan                    # r_5
    diag[4, 1, 0, b - 1] = np.nan            # upper triangle of D_1: not read
    d, l, r = (to_dev(a, torch.float64) for a in (diag, lower, rhs))
    out = selinv.selinv_chain(d, l, r, check=False, validate=True)
    info = host(out["info"]).tolist()
    assert info[0] == -1 and info[4] == -1
    assert info[1] == -3 - 3 and info[2] == -3 - 2 and info[3] == -3 - 5
    ref = oracle.chain(diag[[0]], lower[[0]], rhs[[0]])
    assert worst(host(out["G_diag"])[[0]], ref["G_diag"]) <= 1e-9
    with pytest.raises(selinv.NonFiniteInputError):
        selinv.selinv_chain(d, l, r, validate=True)
    clean = selinv.selinv_chain(d[[0, 4]], l[[0, 4]], r[[0, 4]], validate=True)
    assert (host(clean["info"]) == -1).all()


@pytest.mark.parametrize("b", [1, 3, 4, 7, 8])
@pytest.mark.parametrize("L", [1, 2, 8, 16])
def test_short_chains_of_small_blocks(cuda_ok, b, L):
    """float64, b <= 8, L <= 16: the shared-memory kernel with 8 x 8 tiles.
    Against the oracle; the solve-only and log-det-only calls agree with the
    full one; the upper triangle of D is not read; a failing block is named."""
    diag, lower, rhs = inputs.chain_inputs(6, L, b, seed=3600 + 10 * b + L, load=0.5)
    errs, full = run_both(diag, lower, rhs, torch.float64)
    assert max(errs.values()) <= TOL[torch.float64], errs
    d, l, r = (to_dev(a, torch.float64) for a in (diag, lower, rhs))
    x, ld, _ = selinv.chain_solve(d, l, r)
    assert torch.equal(x, full["x"]) and torch.equal(ld, full["logdet"])
    only = selinv.selinv_chain(d, l, None, want_g=False)
    assert torch.equal(only["logdet"], full["logdet"])
    junk = d.clone()
    if b > 1:
        iu = torch.triu_indices(b, b, 1)
        junk[..., iu[0], iu[1]] = float("nan")
    again = selinv.selinv_chain(junk, l, r)
    for k in ("G_diag", "G_lower", "logdet", "x"):
        assert torch.equal(again[k], full[k]), k
    bad = diag.copy()
    bad[2, L - 1] = -np.eye(b)
    out = selinv.selinv_chain(to_dev(bad, torch.float64), l, check=False)
    info = host(out["info"]).tolist()
    assert info[2] == L - 1 and all(v == -1 for k, v in enumerate(info) if k != 2)


# ---------------- b <= 16, more chains than the GPU holds at once ----------------

BIG_BATCH = 5000      # above the 2368 chains a B200 holds at once (one per CTA, 16 per SM)


@pytest.mark.parametrize("b,L,dtype", [(16, 8, torch.float64), (16, 9, torch.float64), (5, 12, torch.float64),
                                       (16, 10, torch.float32)])
def test_batch_beyond_one_round(cuda_ok, b, L, dtype):
    """Chains started in the first round and in the last one, sampled against
    the oracle; G, x and log det the same from every entry point."""
    diag, lower, rhs = inputs.chain_inputs(BIG_BATCH, L, b, seed=8100 + 7 * b + L, load=1.0)
    d, l, r = to_dev(diag, dtype), to_dev(lower, dtype), to_dev(rhs, dtype)
    out = selinv.selinv_chain(d, l, r)
    assert bool((out["info"] == -1).all())
    pick = [0, 1, 2500, 3900, 4300, 4998, 4999]
    ref = oracle.chain(host(d)[pick], host(l)[pick], host(r)[pick])
    tol = TOL[dtype]
    assert worst(host(out["G_diag"][pick]), ref["G_diag"]) <= tol
    assert worst(host(out["G_lower"][pick]), ref["G_lower"]) <= tol
    assert worst_vec(host(out["x"][pick]), ref["x"]) <= tol
    assert logdet_err(host(out["logdet"][pick]), ref["logdet"]) <= tol
    Gd = out["G_diag"]
    assert torch.equal(Gd, Gd.transpose(-1, -2))
    again = selinv.selinv_chain(d, l, r)
    for k in ("G_diag", "G_lower", "x", "logdet"):
        assert torch.equal(again[k], out[k]), k
    g_only = selinv.selinv_chain(d, l)
    assert torch.equal(g_only["G_diag"], out["G_diag"]) and torch.equal(g_only["G_lower"], out["G_lower"])
    x, ld, info = selinv.chain_solve(d, l, r)
    assert torch.equal(x, out["x"]) and torch.equal(ld, out["logdet"])


def test_batch_beyond_one_round_not_spd(cuda_ok):
    diag, lower, _ = inputs.chain_inputs(BIG_BATCH, 8, 16, seed=8200, load=1.0, with_rhs=False)
    diag[BIG_BATCH - 1, 2] = -np.eye(16)
    diag[BIG_BATCH - 2, 6] = -np.eye(16)
    out = selinv.selinv_chain(to_dev(diag, torch.float64), to_dev(lower, torch.float64), check=False)
    info = host(out["info"])
    assert (info[:BIG_BATCH - 2] == -1).all()
    assert info[BIG_BATCH - 1] == 2 and info[BIG_BATCH - 2] == 6
