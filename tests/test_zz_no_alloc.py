"""selinv_chain_noalloc: the b <= 16 chain path for callers that cannot allocate.

Some callers run inside another framework's execution hook (an inference
plugin's enqueue, a compiler runtime's custom call) where device allocation is
forbidden or would stall the device; this entry point takes only inputs and
outputs and uses a scratch array the library owns.  Its results must match
the workspace-taking entry point, on two calls in a row (the shared scratch
keeps the previous call's contents).  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from sparse_spd_selected_b200 import inputs, selinv
from tests.parity import TOL, host, logdet_err, to_dev, worst

pytestmark = pytest.mark.gpu

MAX_BYTES = 16 << 20      # SELINV_CHAIN_NOALLOC_MAX_BYTES in include/selinv.h


def _noalloc_fn():
    lib = selinv.lib()
    fn = lib.selinv_chain_noalloc
    P = ctypes.c_void_p
    fn.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32,
                   P, P, P, P, P, P, P, P, P]
    fn.restype = ctypes.c_int
    return fn, MAX_BYTES


def _call(fn, d, l, r, dtype):
    lead = d.shape[:-3]
    L, b = d.shape[-3], d.shape[-1]
    G = torch.empty_like(d)
    Gl = torch.empty_like(l)
    x = torch.empty_like(r)
    ld = torch.empty(lead, dtype=torch.float64, device=d.device)
    info = torch.empty(lead, dtype=torch.int32, device=d.device)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    st = fn(selinv.F64 if dtype == torch.float64 else selinv.F32, d.shape[0], L, b, p(d), p(l), p(G), p(Gl),
            p(ld), p(r), p(x), p(info), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == selinv.OK, selinv.status_string(st)
    torch.cuda.synchronize()
    return {"G_diag": G, "G_lower": Gl, "x": x, "logdet": ld, "info": info}


@pytest.mark.parametrize("dtype", [torch.float64, torch.float32])
def test_noalloc_matches_workspace_entry_point(cuda_ok, dtype):
    fn, cap = _noalloc_fn()
    tol = TOL[dtype]
    for call, (batch, L, b, seed) in enumerate([(40, 33, 16, 71), (25, 17, 11, 72)]):   # two calls in a row
        diag, lower, rhs = inputs.chain_inputs(batch, L, b, seed=seed, load=1.0)
        d, l, r = (to_dev(a, dtype) for a in (diag, lower, rhs))
        ref = selinv.selinv_chain(d, l, r)
        got = _call(fn, d, l, r, dtype)
        assert (host(got["info"]) == -1).all()
        for k in ("G_diag", "G_lower", "x"):
            assert worst(host(got[k]), host(ref[k])) <= tol, (call, k)
        assert logdet_err(host(got["logdet"]), host(ref["logdet"])) <= tol, call


def test_noalloc_rejects_requests_beyond_its_scratch(cuda_ok):
    fn, cap = _noalloc_fn()
    slot = 192 * 8
    batch = cap // (slot * 63) + 1                  # just beyond the scratch for L = 64
    d = torch.empty((1, 64, 16, 16), dtype=torch.float64, device="cuda")   # never read: rejected first
    p = ctypes.c_void_p(d.data_ptr())
    st = fn(selinv.F64, batch, 64, 16, p, p, p, p, None, None, None, p, None)
    assert st == selinv.ERR_WORKSPACE
