"""The C-ABI library loads, exports every entry point include/selinv.h declares,
and rejects bad arguments synchronously (no GPU needed: nothing is launched)."""
import ctypes
import os
import re

import numpy as np
import pytest

from sparse_spd_selected_b200 import build, selinv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return selinv.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "selinv.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"\b([a-z_][a-z0-9_]*)\s*\(", src)
    keywords = {"if", "sizeof", "while", "for", "return"}
    return sorted({n for n in names if n not in keywords and n.startswith(("selinv_", "chain_"))})


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert "selinv_chain" in names and "chain_solve" in names and "selinv_tree" in names
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings_and_limits(lib):
    for code in range(9):
        assert selinv.status_string(code) and selinv.status_string(code) != "unknown status"
    assert selinv.max_block() == 128
    assert lib.selinv_version() >= 100


FAKE = ctypes.c_void_p(1 << 20)     # never dereferenced: validation fails first


def call_chain(lib, dtype=0, batch=1, L=4, b=4, diag=FAKE, lower=FAKE, G=FAKE, Gl=FAKE, ld=None,
               rhs=None, x=None, info=FAKE, ws=FAKE, ws_bytes=1 << 30, flags=0):
    return lib.selinv_chain(dtype, batch, L, b, diag, lower, G, Gl, ld, rhs, x, info, ws, ws_bytes, flags, None)


def test_chain_argument_errors(lib):
    assert call_chain(lib, dtype=7) == selinv.ERR_INVALID_ARG
    assert call_chain(lib, L=0) == selinv.ERR_INVALID_ARG
    assert call_chain(lib, b=0) == selinv.ERR_INVALID_ARG
    assert call_chain(lib, batch=-1) == selinv.ERR_INVALID_ARG
    assert call_chain(lib, b=129) == selinv.ERR_UNSUPPORTED
    assert call_chain(lib, diag=None) == selinv.ERR_INVALID_ARG
    assert call_chain(lib, lower=None) == selinv.ERR_INVALID_ARG
    assert call_chain(lib, info=None) == selinv.ERR_INVALID_ARG
    assert call_chain(lib, diag=ctypes.c_void_p((1 << 20) + 4)) == selinv.ERR_INVALID_ARG   # misaligned f64
    assert call_chain(lib, Gl=None) == selinv.ERR_INVALID_ARG                              # G_diag without G_lower
    assert call_chain(lib, rhs=FAKE) == selinv.ERR_INVALID_ARG                              # rhs without x
    assert call_chain(lib, ws=None) == selinv.ERR_WORKSPACE
    assert call_chain(lib, ws_bytes=16) == selinv.ERR_WORKSPACE
    assert call_chain(lib, batch=0) == selinv.OK                                            # nothing to do


def test_workspace_sizes(lib):
    f = lib.selinv_chain_workspace_size
    assert f(0, 10, 8, 16, 0, 0) == 0                       # log det only: no workspace
    small = f(0, 10, 8, 16, 1, 0)
    assert small >= 10 * 7 * 192 * 8 and small % 256 == 0
    assert f(1, 10, 8, 16, 1, 0) < small                     # float32 slots are half the size
    assert f(0, 10, 1, 16, 1, 1) == 0                        # one block: nothing kept between sweeps


def test_tree_plan_rejects_malformed_parents(lib):
    def plan(parent):
        p = np.ascontiguousarray(np.asarray(parent, dtype=np.int32))
        h = ctypes.c_void_p()
        trees, n = (1, p.size) if p.ndim == 1 else p.shape
        return lib.selinv_tree_plan(p.ctypes.data_as(ctypes.c_void_p), trees, n, ctypes.byref(h))
    assert plan([-1, 0, -1]) == selinv.ERR_BAD_TREE          # two roots
    assert plan([0, 0, 1]) == selinv.ERR_BAD_TREE            # no root (self loop at 0)
    assert plan([1, 2, 0, -1]) == selinv.ERR_BAD_TREE        # cycle 0 -> 1 -> 2 -> 0
    assert plan([-1, 5, 0]) == selinv.ERR_BAD_TREE           # out of range
    assert plan([[-1, 0, 1], [-1, -1, 0]]) == selinv.ERR_BAD_TREE   # second tree has two roots
    assert lib.selinv_tree_plan(None, 1, 3, ctypes.byref(ctypes.c_void_p())) == selinv.ERR_INVALID_ARG


def test_segment_rules(lib):
    """Only 16 < b <= 32 chains with G, no solve, L >= 96 and a small batch are cut."""
    f = lib.selinv_chain_segments
    f.restype = ctypes.c_int32
    f.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32]
    assert f(2, 600, 32, 1, 0) >= 3
    assert f(2, 600, 16, 1, 0) == 0          # warp kernel
    assert f(2, 600, 33, 1, 0) == 0          # CTA kernel
    assert f(2, 600, 32, 0, 0) == 0          # log det only: two-ended kernel
    assert f(2, 600, 32, 1, 1) == 0          # with a solve
    assert f(2, 95, 32, 1, 0) == 0           # too short
    assert f(100000, 4096, 32, 1, 0) == 0    # batch fills the GPU
    assert f(1, 10 ** 6, 32, 1, 0) == 16     # at most 16 segments


def test_sample_and_multi_argument_errors(lib):
    """The draw and the several-right-hand-side solve reject bad arguments before any launch."""
    s = lib.selinv_chain_sample
    # dtype, batch, L, b, diag, lower, rhs, z, eta, logdet, info, ws, ws_bytes, stream
    assert s(0, 1, 4, 4, FAKE, FAKE, None, None, FAKE, None, FAKE, FAKE, 1 << 30, None) == selinv.ERR_INVALID_ARG
    assert s(0, 1, 4, 4, FAKE, FAKE, None, FAKE, None, None, FAKE, FAKE, 1 << 30, None) == selinv.ERR_INVALID_ARG
    assert s(1, 1, 4, 20, FAKE, FAKE, None, FAKE, FAKE, None, FAKE, FAKE, 1 << 30, None) == selinv.ERR_UNSUPPORTED
    assert s(0, 1, 4, 129, FAKE, FAKE, None, FAKE, FAKE, None, FAKE, FAKE, 1 << 30, None) == selinv.ERR_UNSUPPORTED
    assert s(0, 1, 4, 4, FAKE, FAKE, None, FAKE, FAKE, None, FAKE, FAKE, 16, None) == selinv.ERR_WORKSPACE
    assert s(0, 0, 4, 4, FAKE, FAKE, None, FAKE, FAKE, None, FAKE, FAKE, 1 << 30, None) == selinv.OK
    m = lib.chain_solve_multi
    # dtype, batch, L, b, nrhs, diag, lower, rhs, x, logdet, info, ws, ws_bytes, stream
    assert m(0, 1, 4, 4, 0, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, 1 << 30, None) == selinv.ERR_INVALID_ARG
    assert m(0, 1, 4, 4, 3, FAKE, FAKE, None, FAKE, None, FAKE, FAKE, 1 << 30, None) == selinv.ERR_INVALID_ARG
    assert m(0, 1, 4, 20, 3, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, 1 << 30, None) == selinv.ERR_UNSUPPORTED
    assert m(0, 1, 4, 4, 3, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, 16, None) == selinv.ERR_WORKSPACE
    assert m(0, 0, 4, 4, 3, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, 1 << 30, None) == selinv.OK


def test_backward_argument_errors(lib):
    """The backward rejects bad arguments before any launch."""
    f = lib.selinv_chain_backward
    ws = lib.selinv_chain_backward_workspace_size
    ws.restype = ctypes.c_size_t
    ws.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32]
    assert ws(0, 3, 5, 16) >= 3 * 5 * 2 * 256 * 8 and ws(0, 3, 5, 16) % 256 == 0
    assert ws(0, 3, 5, 17) == 0

    # dtype, batch, L, b, diag, lower, G_diag, G_lower, Gb_diag, Gb_lower, Db, Bb, info, ws, ws_bytes, stream
    def call(**kw):
        args = dict(dtype=0, batch=1, L=4, b=4, diag=FAKE, lower=FAKE, Gd=FAKE, Gl=FAKE, Gbd=FAKE, Gbl=FAKE,
                    Db=FAKE, Bb=FAKE, info=FAKE, ws=FAKE, nbytes=1 << 30)
        args.update(kw)
        return f(args["dtype"], args["batch"], args["L"], args["b"], args["diag"], args["lower"], args["Gd"],
                 args["Gl"], args["Gbd"], args["Gbl"], args["Db"], args["Bb"], args["info"], args["ws"],
                 args["nbytes"], None)
    assert call(b=17) == selinv.ERR_UNSUPPORTED
    assert call(Gd=None) == selinv.ERR_INVALID_ARG
    assert call(Db=None) == selinv.ERR_INVALID_ARG
    assert call(Bb=None) == selinv.ERR_INVALID_ARG
    assert call(Gl=None) == selinv.ERR_INVALID_ARG
    assert call(nbytes=16) == selinv.ERR_WORKSPACE
    assert call(ws=None) == selinv.ERR_WORKSPACE
    assert call(batch=0) == selinv.OK


def test_tree_backward_argument_errors(lib):
    """Without a GPU no plan can be built; a null plan is rejected before any launch."""
    ws = lib.selinv_tree_backward_workspace_size
    ws.restype = ctypes.c_size_t
    ws.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int32]
    assert ws(None, 0, 16) == 0
    f = lib.selinv_tree_backward
    # plan, dtype, b, diag, edge, G_diag, G_edge, Gb_diag, Gb_edge, Db, Eb, info, ws, ws_bytes, stream
    assert f(None, 0, 4, FAKE, FAKE, FAKE, FAKE, None, None, FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == \
        selinv.ERR_INVALID_ARG


def test_bidiag_argument_errors(lib):
    f = lib.selinv_bidiag
    # dtype, batch, L, b, diag, lower, G_diag, G_lower, info, stream
    assert f(0, 1, 4, 17, FAKE, FAKE, FAKE, FAKE, FAKE, None) == selinv.ERR_UNSUPPORTED
    assert f(0, 1, 4, 4, FAKE, None, FAKE, FAKE, FAKE, None) == selinv.ERR_INVALID_ARG
    assert f(0, 1, 4, 4, FAKE, FAKE, None, FAKE, FAKE, None) == selinv.ERR_INVALID_ARG
    assert f(0, 1, 4, 4, FAKE, FAKE, FAKE, None, FAKE, None) == selinv.ERR_INVALID_ARG
    assert f(0, 0, 4, 4, FAKE, FAKE, FAKE, FAKE, FAKE, None) == selinv.OK


def test_bidiag_backward_argument_errors(lib):
    f = lib.selinv_bidiag_backward
    # dtype, batch, L, b, G_diag, G_lower, Gb_diag, Gb_lower, Mb_diag, Mb_lower, stream
    assert f(0, 1, 4, 17, FAKE, FAKE, None, None, FAKE, FAKE, None) == selinv.ERR_UNSUPPORTED
    assert f(0, 1, 4, 4, None, FAKE, None, None, FAKE, FAKE, None) == selinv.ERR_INVALID_ARG
    assert f(0, 1, 4, 4, FAKE, FAKE, None, None, FAKE, None, None) == selinv.ERR_INVALID_ARG
    assert f(0, 0, 4, 4, FAKE, FAKE, None, None, FAKE, FAKE, None) == selinv.OK


def test_junction_plan_rejects_bad_patterns(lib):
    """Pattern and order checks run on the host before anything touches a device."""
    def plan(ei, ej, n, order=None):
        a = np.ascontiguousarray(np.asarray(ei, dtype=np.int32))
        c = np.ascontiguousarray(np.asarray(ej, dtype=np.int32))
        o = None if order is None else np.ascontiguousarray(np.asarray(order, dtype=np.int32))
        h = ctypes.c_void_p()
        return lib.selinv_junction_plan(n, a.size, a.ctypes.data_as(ctypes.c_void_p), c.ctypes.data_as(ctypes.c_void_p),
                                        None if o is None else o.ctypes.data_as(ctypes.c_void_p), ctypes.byref(h))
    assert plan([0], [1], 3) == selinv.ERR_INVALID_ARG             # i < j
    assert plan([1], [1], 3) == selinv.ERR_INVALID_ARG             # diagonal
    assert plan([3], [0], 3) == selinv.ERR_INVALID_ARG             # out of range
    assert plan([2, 2], [1, 1], 3) == selinv.ERR_INVALID_ARG       # repeated block
    assert plan([1], [0], 3, order=[0, 0, 1]) == selinv.ERR_INVALID_ARG   # not a permutation
    assert lib.selinv_junction(None, 0, 4, 1, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, 1 << 30, None) == \
        selinv.ERR_INVALID_ARG


def test_noalloc_rejects_oversized_requests_before_any_device_call(lib):
    """The allocation-free chain entry point checks its request against the
    built-in scratch by division, so products that wrap 64 bits are refused."""
    f = lib.selinv_chain_noalloc
    P = ctypes.c_void_p
    f.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32] + [P] * 9
    f.restype = ctypes.c_int
    # dtype, batch, L, b, diag, lower, G_diag, G_lower, logdet, rhs, x, info, stream
    assert f(0, 1 << 61, 64, 16, FAKE, FAKE, FAKE, FAKE, None, None, None, FAKE, None) == selinv.ERR_WORKSPACE
    assert f(0, 3, (1 << 62) + 1, 16, FAKE, FAKE, FAKE, FAKE, None, None, None, FAKE, None) == selinv.ERR_WORKSPACE
    assert f(1, 1 << 40, 1 << 40, 4, FAKE, FAKE, None, None, None, FAKE, FAKE, FAKE, None) == selinv.ERR_WORKSPACE
    assert f(0, 1, 4, 17, FAKE, FAKE, FAKE, FAKE, None, None, None, FAKE, None) == selinv.ERR_UNSUPPORTED
    assert f(0, 1, 4, 4, FAKE, FAKE, FAKE, None, None, None, None, FAKE, None) == selinv.ERR_INVALID_ARG
    assert f(0, 0, 4, 4, FAKE, FAKE, FAKE, FAKE, None, None, None, FAKE, None) == selinv.OK


def test_tree_set_wait_argument_errors(lib):
    assert lib.selinv_tree_plan_set_wait(None, 10, -1) == selinv.ERR_INVALID_ARG
    assert selinv.status_string(selinv.ERR_TIMEOUT) != "unknown status"


def test_flags_are_validated_before_any_launch(lib):
    """SELINV_WANT_LOGDET / SELINV_WANT_SOLVE insist on their pointers; unknown bits are refused."""
    assert call_chain(lib, batch=0, flags=selinv.CHECK) == selinv.OK
    assert call_chain(lib, flags=1 << 7) == selinv.ERR_INVALID_ARG
    assert call_chain(lib, flags=selinv.WANT_LOGDET) == selinv.ERR_INVALID_ARG          # logdet NULL
    assert call_chain(lib, flags=selinv.WANT_SOLVE) == selinv.ERR_INVALID_ARG           # rhs, x NULL
    assert call_chain(lib, batch=0, ld=FAKE, rhs=FAKE, x=FAKE,
                      flags=selinv.WANT_LOGDET | selinv.WANT_SOLVE | selinv.CHECK) == selinv.OK
    f = lib.selinv_tree
    assert f(None, 0, 4, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, 1 << 30, 0, None) == selinv.ERR_INVALID_ARG


def test_junction_solve_argument_errors(lib):
    f = lib.selinv_junction_solve
    # plan, dtype, b, batch, diag, edge_val, rhs, x, logdet, info, workspace, ws_bytes, stream
    assert f(None, 0, 4, 1, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, 1 << 30, None) == selinv.ERR_INVALID_ARG
