"""selinv_chain_noalloc: the b <= 16 chain path for callers that cannot allocate.

Some callers run inside another framework's execution hook (an inference
plugin's enqueue, a compiler runtime's custom call) where device allocation is
forbidden or would stall the device; this entry point takes only inputs and
outputs and uses a scratch array the library owns.  Its results must match
the CPU oracle and the workspace-taking entry point, on two calls in a row
(the shared scratch keeps the previous call's contents), for every choice of
outputs (G and x, G only, x only, log det only).  This file is collected last
on purpose.
"""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import oracle
from sparse_spd_selected_b200 import inputs, selinv
from tests.parity import TOL, host, logdet_err, to_dev, worst, worst_vec

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_cap():
    """SELINV_CHAIN_NOALLOC_MAX_BYTES as include/selinv.h defines it."""
    src = open(os.path.join(ROOT, "include", "selinv.h")).read()
    m = re.search(r"#define\s+SELINV_CHAIN_NOALLOC_MAX_BYTES\s+\(\(size_t\)(\d+)\s*<<\s*(\d+)\)", src)
    assert m, "SELINV_CHAIN_NOALLOC_MAX_BYTES not found in the header"
    return int(m.group(1)) << int(m.group(2))


def _noalloc_fn():
    lib = selinv.lib()
    fn = lib.selinv_chain_noalloc
    P = ctypes.c_void_p
    fn.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32,
                   P, P, P, P, P, P, P, P, P]
    fn.restype = ctypes.c_int
    return fn


def _call(fn, d, l, r, dtype, want_g, want_x):
    lead = d.shape[:-3]
    L, b = d.shape[-3], d.shape[-1]
    G = torch.full_like(d, float("nan")) if want_g else None
    Gl = torch.full_like(l, float("nan")) if want_g else None
    x = torch.full_like(r, float("nan")) if want_x else None
    ld = torch.full(lead, float("nan"), dtype=torch.float64, device=d.device)
    info = torch.full(lead, 7, dtype=torch.int32, device=d.device)
    p = lambda t: ctypes.c_void_p(t.data_ptr()) if t is not None else None
    st = fn(selinv.F64 if dtype == torch.float64 else selinv.F32, d.shape[0], L, b, p(d), p(l), p(G), p(Gl),
            p(ld), p(r if want_x else None), p(x), p(info),
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == selinv.OK, selinv.status_string(st)
    torch.cuda.synchronize()
    return {"G_diag": G, "G_lower": Gl, "x": x, "logdet": ld, "info": info}


@pytest.mark.parametrize("want_g,want_x", [(True, True), (True, False), (False, True), (False, False)])
@pytest.mark.parametrize("dtype", [torch.float64, torch.float32])
def test_noalloc_matches_oracle_and_workspace_entry_point(cuda_ok, dtype, want_g, want_x):
    fn = _noalloc_fn()
    tol = TOL[dtype]
    for call, (batch, L, b, seed) in enumerate([(40, 33, 16, 71), (25, 17, 11, 72)]):   # two calls in a row
        diag, lower, rhs = inputs.chain_inputs(batch, L, b, seed=seed, load=1.0)
        d, l, r = (to_dev(a, dtype) for a in (diag, lower, rhs))
        got = _call(fn, d, l, r, dtype, want_g, want_x)
        ref = oracle.chain(host(d), host(l), host(r) if want_x else None, want_g=want_g)
        ws = selinv.selinv_chain(d, l, r if want_x else None, want_g=want_g)
        assert (host(got["info"]) == -1).all()
        if want_g:
            for k in ("G_diag", "G_lower"):
                assert worst(host(got[k]), ref[k]) <= tol, (call, k)
                assert worst(host(got[k]), host(ws[k])) <= tol, (call, k)
        if want_x:
            assert worst_vec(host(got["x"]), ref["x"]) <= tol, call
            assert worst_vec(host(got["x"]), host(ws["x"])) <= tol, call
        assert logdet_err(host(got["logdet"]), ref["logdet"]) <= tol, call
        assert logdet_err(host(got["logdet"]), host(ws["logdet"])) <= tol, call


def test_noalloc_rejects_requests_beyond_its_scratch(cuda_ok):
    fn = _noalloc_fn()
    cap = header_cap()
    slot = 192 * 8
    d = torch.empty((1, 64, 16, 16), dtype=torch.float64, device="cuda")   # never read: rejected first
    p = ctypes.c_void_p(d.data_ptr())
    batch = cap // (slot * 63) + 1                  # just beyond the scratch for L = 64
    assert fn(selinv.F64, batch, 64, 16, p, p, p, p, None, None, None, p, None) == selinv.ERR_WORKSPACE
    # products that wrap 64 bits must not slip under the limit
    assert fn(selinv.F64, 1 << 61, 64, 16, p, p, p, p, None, None, None, p, None) == selinv.ERR_WORKSPACE
    assert fn(selinv.F64, 3, (1 << 62) + 1, 16, p, p, p, p, None, None, None, p, None) == selinv.ERR_WORKSPACE
