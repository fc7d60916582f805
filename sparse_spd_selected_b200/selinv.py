"""ctypes binding of libselinv (the C ABI in include/selinv.h).

Argument marshalling only: tensors are checked for device, dtype and
contiguity, outputs and the workspace are allocated with torch, and every
step of the computation runs in the library's CUDA kernels on the current
torch stream.  There is no CPU fallback: if ``libselinv.so`` is missing or no
CUDA device is present, calls raise.

The calls follow the problem statement of gabp-sparse-inv 0.3.2 (PyPI page,
"Quickstart"): inputs ``[..., L, b, b]`` with optional leading batch
dimensions, outputs only the on-pattern blocks of A^-1 (never the dense
inverse), plus log det A and A^-1 r from the same factorisation.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("SELINV_LIB") or os.path.join(_HERE, "libselinv.so")

(OK, ERR_INVALID_ARG, ERR_NOT_SPD, ERR_BAD_TREE, ERR_CUDA, ERR_WORKSPACE, ERR_UNSUPPORTED, ERR_HOST_MEMORY,
 ERR_TIMEOUT) = range(9)
F64, F32 = 0, 1
WANT_LOGDET, WANT_SOLVE, CHECK = 1, 2, 4          # flags of selinv_chain / selinv_tree

_lib = None


class SelinvError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


class NotSPDError(SelinvError):
    def __init__(self, info):
        self.info = info
        super().__init__(ERR_NOT_SPD, f"first failing block per batch element: {info}")


class WaitTimeoutError(SelinvError):
    """A bounded dependency wait of a tree sweep gave up (info = -2 for that tree)."""

    def __init__(self, info):
        self.info = info
        super().__init__(ERR_TIMEOUT, f"info per tree: {info}")


class NonFiniteInputError(SelinvError):
    """An input entry the call reads is not finite (validate=True: SELINV_CHECK)."""

    def __init__(self, info):
        self.info = info
        blocks = [(-3 - v) if v <= -3 else None for v in info]
        super().__init__(ERR_INVALID_ARG, f"first block with a non-finite entry per batch element: {blocks}")


class SingularBlockError(SelinvError):
    """A diagonal block of a non-symmetric chain is singular."""

    def __init__(self, info):
        self.info = info
        super().__init__(ERR_NOT_SPD, f"first singular diagonal block per batch element: {info}")


def lib():
    """The loaded libselinv.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m sparse_spd_selected_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, I32, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
        L.selinv_status_string.argtypes = [ctypes.c_int]
        L.selinv_status_string.restype = ctypes.c_char_p
        L.selinv_version.restype = I32
        L.selinv_max_block.restype = I32
        L.selinv_chain_workspace_size.argtypes = [ctypes.c_int, I64, I64, I32, I32, I32]
        L.selinv_chain_workspace_size.restype = SZ
        L.selinv_chain_segments.argtypes = [I64, I64, I32, I32, I32]
        L.selinv_chain_segments.restype = I32
        L.selinv_chain.argtypes = [ctypes.c_int, I64, I64, I32, P, P, P, P, P, P, P, P, P, SZ, ctypes.c_uint32, P]
        L.selinv_chain.restype = ctypes.c_int
        L.chain_solve_multi.argtypes = [ctypes.c_int, I64, I64, I32, I32, P, P, P, P, P, P, P, SZ, P]
        L.chain_solve_multi.restype = ctypes.c_int
        L.selinv_chain_sample.argtypes = [ctypes.c_int, I64, I64, I32, P, P, P, P, P, P, P, P, SZ, P]
        L.selinv_chain_sample.restype = ctypes.c_int
        L.chain_solve.argtypes = [ctypes.c_int, I64, I64, I32, P, P, P, P, P, P, P, SZ, P]
        L.chain_solve.restype = ctypes.c_int
        L.selinv_bidiag.argtypes = [ctypes.c_int, I64, I64, I32, P, P, P, P, P, P]
        L.selinv_bidiag.restype = ctypes.c_int
        L.selinv_bidiag_backward.argtypes = [ctypes.c_int, I64, I64, I32, P, P, P, P, P, P, P]
        L.selinv_bidiag_backward.restype = ctypes.c_int
        L.selinv_chain_backward_workspace_size.argtypes = [ctypes.c_int, I64, I64, I32]
        L.selinv_chain_backward_workspace_size.restype = SZ
        L.selinv_chain_backward.argtypes = [ctypes.c_int, I64, I64, I32, P, P, P, P, P, P, P, P, P, P, SZ, P]
        L.selinv_chain_backward.restype = ctypes.c_int
        L.selinv_tree_backward_workspace_size.argtypes = [P, ctypes.c_int, I32]
        L.selinv_tree_backward_workspace_size.restype = SZ
        L.selinv_tree_backward.argtypes = [P, ctypes.c_int, I32, P, P, P, P, P, P, P, P, P, P, SZ, P]
        L.selinv_tree_backward.restype = ctypes.c_int
        L.selinv_junction_plan.argtypes = [I64, I64, P, P, P, ctypes.POINTER(P)]
        L.selinv_junction_plan.restype = ctypes.c_int
        L.selinv_junction_plan_free.argtypes = [P]
        L.selinv_junction_plan_free.restype = None
        L.selinv_junction_plan_info.argtypes = [P, ctypes.POINTER(I64), ctypes.POINTER(I32), ctypes.POINTER(I32)]
        L.selinv_junction_plan_info.restype = ctypes.c_int
        L.selinv_junction_plan_pattern.argtypes = [P, P, P, P]
        L.selinv_junction_plan_pattern.restype = ctypes.c_int
        L.selinv_junction_symbolic.argtypes = [I64, I64, P, P, P, ctypes.POINTER(I64), P, P, I64, P]
        L.selinv_junction_symbolic.restype = ctypes.c_int
        L.selinv_junction_plan_launches.argtypes = [P]
        L.selinv_junction_plan_launches.restype = I64
        L.selinv_junction_workspace_size.argtypes = [P, ctypes.c_int, I32, I64]
        L.selinv_junction_workspace_size.restype = SZ
        L.selinv_junction.argtypes = [P, ctypes.c_int, I32, I64, P, P, P, P, P, P, P, SZ, P]
        L.selinv_junction.restype = ctypes.c_int
        L.selinv_junction_solve.argtypes = [P, ctypes.c_int, I32, I64, P, P, P, P, P, P, P, SZ, P]
        L.selinv_junction_solve.restype = ctypes.c_int
        L.selinv_tree_plan.argtypes = [P, I64, I64, ctypes.POINTER(P)]
        L.selinv_tree_plan.restype = ctypes.c_int
        L.selinv_tree_plan_free.argtypes = [P]
        L.selinv_tree_plan_free.restype = None
        L.selinv_tree_plan_set_wait.argtypes = [P, I32, I64]
        L.selinv_tree_plan_set_wait.restype = ctypes.c_int
        L.selinv_tree_plan_levels.argtypes = [P, ctypes.POINTER(I32), ctypes.POINTER(I32)]
        L.selinv_tree_plan_levels.restype = ctypes.c_int
        L.selinv_tree_workspace_size.argtypes = [P, ctypes.c_int, I32]
        L.selinv_tree_workspace_size.restype = SZ
        L.selinv_tree.argtypes = [P, ctypes.c_int, I32, P, P, P, P, P, P, P, SZ, ctypes.c_uint32, P]
        L.selinv_tree_sample.argtypes = [P, ctypes.c_int, I32, P, P, P, P, P, P, P, SZ, P]
        L.selinv_tree_sample.restype = ctypes.c_int
        L.selinv_tree.restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().selinv_status_string(int(status)).decode()


def max_block() -> int:
    return int(lib().selinv_max_block())


def _code(dtype) -> int:
    if dtype == torch.float64:
        return F64
    if dtype == torch.float32:
        return F32
    raise TypeError(f"libselinv computes in float64 or float32, not {dtype}")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _cuda_contig(name, t, dtype=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must have dtype {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _stream_handle(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(status, what):
    if status != OK:
        raise SelinvError(status, what)


def chain_workspace_size(dtype, batch, L, b, want_g=True, want_x=False) -> int:
    return int(lib().selinv_chain_workspace_size(_code(dtype), batch, L, b, int(want_g), int(want_x)))


def chain_segments(batch, L, b, want_g=True, want_x=False) -> int:
    """Segments per chain selinv_chain uses for these sizes on the current device (0: none)."""
    return int(lib().selinv_chain_segments(batch, L, b, int(want_g), int(want_x)))


def _workspace(nbytes, device, workspace):
    if nbytes == 0:
        return None
    if workspace is not None:
        if workspace.numel() * workspace.element_size() < nbytes:
            raise ValueError(f"workspace needs {nbytes} bytes")
        return workspace
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def _raise_on_info(info, check):
    if check:
        host = info.cpu()
        if bool((host <= -3).any()):
            raise NonFiniteInputError(host.tolist())
        if bool((host == -2).any()):
            raise WaitTimeoutError(host.tolist())
        if bool((host >= 0).any()):
            raise NotSPDError(host.tolist())


def selinv_chain(diag: torch.Tensor, lower: Optional[torch.Tensor] = None, rhs: Optional[torch.Tensor] = None,
                 *, want_g: bool = True, check: bool = True, validate: bool = False, out=None, workspace=None,
                 stream=None):
    """Selected inverse (+ log det, + optional solve) of block-tridiagonal SPD chains.

    diag [..., L, b, b], lower [..., L-1, b, b] (lower[i] = A_{i+1,i}),
    rhs [..., L, b] optional.  Returns a dict with G_diag, G_lower, logdet
    (float64), x (if rhs) and info (int32, -1 = ok).  With check=True the
    call synchronises once to read info and raises NotSPDError on failure.
    validate=True adds the library's on-device input check (SELINV_CHECK):
    an element with a non-finite entry among those read reports info
    -3 - k, raised as NonFiniteInputError when check=True.
    ``out`` may hold preallocated output tensors under the same keys.
    """
    _cuda_contig("diag", diag)
    dt = diag.dtype
    code = _code(dt)
    if diag.dim() < 3 or diag.shape[-1] != diag.shape[-2]:
        raise ValueError("diag must be [..., L, b, b]")
    lead = tuple(diag.shape[:-3])
    L, b = int(diag.shape[-3]), int(diag.shape[-1])
    batch = 1
    for d in lead:
        batch *= int(d)
    if L > 1:
        if lower is None:
            raise ValueError("lower is required when L > 1")
        _cuda_contig("lower", lower, dt)
        if tuple(lower.shape) != lead + (L - 1, b, b):
            raise ValueError(f"lower must be {lead + (L - 1, b, b)}, got {tuple(lower.shape)}")
    else:
        lower = None
    if rhs is not None:
        _cuda_contig("rhs", rhs, dt)
        if tuple(rhs.shape) != lead + (L, b):
            raise ValueError(f"rhs must be {lead + (L, b)}")
    dev = diag.device
    out = dict(out or {})
    G_diag = G_lower = x = None
    if want_g:
        G_diag = out.get("G_diag")
        if G_diag is None:
            G_diag = torch.empty(lead + (L, b, b), dtype=dt, device=dev)
        G_lower = out.get("G_lower")
        if G_lower is None:
            G_lower = torch.empty(lead + (max(L - 1, 0), b, b), dtype=dt, device=dev)
    if rhs is not None:
        x = out.get("x")
        if x is None:
            x = torch.empty(lead + (L, b), dtype=dt, device=dev)
    logdet = out.get("logdet")
    if logdet is None:
        logdet = torch.empty(lead, dtype=torch.float64, device=dev)
    info = out.get("info")
    if info is None:
        info = torch.empty(lead, dtype=torch.int32, device=dev)
    nbytes = chain_workspace_size(dt, batch, L, b, want_g, rhs is not None)
    ws = _workspace(nbytes, dev, workspace)
    with torch.cuda.device(dev):
        st = lib().selinv_chain(code, batch, L, b, _ptr(diag), _ptr(lower),
                                _ptr(G_diag), _ptr(G_lower if L > 1 else None), _ptr(logdet),
                                _ptr(rhs), _ptr(x), _ptr(info), _ptr(ws), nbytes, CHECK if validate else 0,
                                _stream_handle(stream))
    _check(st, "selinv_chain")
    _raise_on_info(info, check)
    return {"G_diag": G_diag, "G_lower": G_lower, "logdet": logdet, "x": x, "info": info}


def chain_solve(diag, lower, rhs, *, check=True, workspace=None, stream=None):
    """x = A^-1 r for block-tridiagonal SPD chains (no G blocks formed); returns (x, logdet, info)."""
    r = selinv_chain(diag, lower, rhs, want_g=False, check=False, workspace=workspace, stream=stream)
    _raise_on_info(r["info"], check)
    return r["x"], r["logdet"], r["info"]


def chain_solve_multi(diag, lower, rhs, *, check=True, out=None, workspace=None, stream=None):
    """X = A^-1 R for block-tridiagonal SPD chains with several right-hand sides
    (b <= 16): rhs [..., L, b, k].  Returns (x [..., L, b, k], logdet, info)."""
    _cuda_contig("diag", diag)
    dt = diag.dtype
    if diag.dim() < 3 or diag.shape[-1] != diag.shape[-2]:
        raise ValueError("diag must be [..., L, b, b]")
    lead = tuple(diag.shape[:-3])
    L, b = int(diag.shape[-3]), int(diag.shape[-1])
    batch = 1
    for d in lead:
        batch *= int(d)
    if L > 1:
        if lower is None:
            raise ValueError("lower is required when L > 1")
        _cuda_contig("lower", lower, dt)
        if tuple(lower.shape) != lead + (L - 1, b, b):
            raise ValueError(f"lower must be {lead + (L - 1, b, b)}, got {tuple(lower.shape)}")
    else:
        lower = None
    _cuda_contig("rhs", rhs, dt)
    if rhs.dim() != len(lead) + 3 or tuple(rhs.shape[:-1]) != lead + (L, b):
        raise ValueError(f"rhs must be {lead + (L, b)} + (k,)")
    k = int(rhs.shape[-1])
    dev = diag.device
    out = dict(out or {})
    x = out.get("x")
    if x is None:
        x = torch.empty(lead + (L, b, k), dtype=dt, device=dev)
    logdet = out.get("logdet")
    if logdet is None:
        logdet = torch.empty(lead, dtype=torch.float64, device=dev)
    info = out.get("info")
    if info is None:
        info = torch.empty(lead, dtype=torch.int32, device=dev)
    nbytes = chain_workspace_size(dt, batch, L, b, False, True)
    ws = _workspace(nbytes, dev, workspace)
    with torch.cuda.device(dev):
        st = lib().chain_solve_multi(_code(dt), batch, L, b, k, _ptr(diag), _ptr(lower), _ptr(rhs), _ptr(x),
                                     _ptr(logdet), _ptr(info), _ptr(ws), nbytes, _stream_handle(stream))
    _check(st, "chain_solve_multi")
    _raise_on_info(info, check)
    return x, logdet, info


def chain_sample(diag, lower, z, rhs=None, *, check=True, out=None, workspace=None, stream=None):
    """Gaussian draw from the chain's own Cholesky factor A = L L^T (b <= 16; float64 up to b = 128):
    eta = L^-T z, plus A^-1 rhs when rhs is given, so eta ~ N(A^-1 rhs, A^-1)
    for standard normal z [..., L, b] supplied by the caller.  Returns a dict
    with eta, logdet (float64) and info (int32, -1 = ok)."""
    _cuda_contig("diag", diag)
    dt = diag.dtype
    if diag.dim() < 3 or diag.shape[-1] != diag.shape[-2]:
        raise ValueError("diag must be [..., L, b, b]")
    lead = tuple(diag.shape[:-3])
    L, b = int(diag.shape[-3]), int(diag.shape[-1])
    batch = 1
    for d in lead:
        batch *= int(d)
    if L > 1:
        if lower is None:
            raise ValueError("lower is required when L > 1")
        _cuda_contig("lower", lower, dt)
        if tuple(lower.shape) != lead + (L - 1, b, b):
            raise ValueError(f"lower must be {lead + (L - 1, b, b)}, got {tuple(lower.shape)}")
    else:
        lower = None
    _cuda_contig("z", z, dt)
    if tuple(z.shape) != lead + (L, b):
        raise ValueError(f"z must be {lead + (L, b)}")
    if rhs is not None:
        _cuda_contig("rhs", rhs, dt)
        if tuple(rhs.shape) != lead + (L, b):
            raise ValueError(f"rhs must be {lead + (L, b)}")
    dev = diag.device
    out = dict(out or {})
    eta = out.get("eta")
    if eta is None:
        eta = torch.empty(lead + (L, b), dtype=dt, device=dev)
    logdet = out.get("logdet")
    if logdet is None:
        logdet = torch.empty(lead, dtype=torch.float64, device=dev)
    info = out.get("info")
    if info is None:
        info = torch.empty(lead, dtype=torch.int32, device=dev)
    nbytes = chain_workspace_size(dt, batch, L, b, False, True)
    ws = _workspace(nbytes, dev, workspace)
    with torch.cuda.device(dev):
        st = lib().selinv_chain_sample(_code(dt), batch, L, b, _ptr(diag), _ptr(lower), _ptr(rhs), _ptr(z),
                                       _ptr(eta), _ptr(logdet), _ptr(info), _ptr(ws), nbytes,
                                       _stream_handle(stream))
    _check(st, "selinv_chain_sample")
    _raise_on_info(info, check)
    return {"eta": eta, "logdet": logdet, "info": info}


def bidiag(diag, lower=None, *, check=True, out=None, stream=None):
    """Selected inverse of block lower-bidiagonal matrices with general blocks
    (b <= 16): diag [..., L, b, b] = M_ii, lower [..., L-1, b, b] = M_{i+1,i}.
    Returns a dict with G_diag = (M^-1)_ii, G_lower = (M^-1)_{i+1,i} and info
    (int32, -1 = ok, else the first singular diagonal block)."""
    _cuda_contig("diag", diag)
    dt = diag.dtype
    if diag.dim() < 3 or diag.shape[-1] != diag.shape[-2]:
        raise ValueError("diag must be [..., L, b, b]")
    lead = tuple(diag.shape[:-3])
    L, b = int(diag.shape[-3]), int(diag.shape[-1])
    batch = 1
    for d in lead:
        batch *= int(d)
    if L > 1:
        if lower is None:
            raise ValueError("lower is required when L > 1")
        _cuda_contig("lower", lower, dt)
        if tuple(lower.shape) != lead + (L - 1, b, b):
            raise ValueError(f"lower must be {lead + (L - 1, b, b)}")
    else:
        lower = None
    dev = diag.device
    out = dict(out or {})
    G_diag = out.get("G_diag")
    if G_diag is None:
        G_diag = torch.empty_like(diag)
    G_lower = out.get("G_lower")
    if G_lower is None:
        G_lower = torch.empty(lead + (max(L - 1, 0), b, b), dtype=dt, device=dev)
    info = out.get("info")
    if info is None:
        info = torch.empty(lead, dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        st = lib().selinv_bidiag(_code(dt), batch, L, b, _ptr(diag), _ptr(lower), _ptr(G_diag),
                                 _ptr(G_lower if L > 1 else None), _ptr(info), _stream_handle(stream))
    _check(st, "selinv_bidiag")
    if check:
        host = info.cpu()
        if bool((host >= 0).any()):
            raise SingularBlockError(host.tolist())
    return {"G_diag": G_diag, "G_lower": G_lower, "info": info}


def bidiag_backward(G_diag, G_lower, Gb_diag=None, Gb_lower=None, *, out=None, stream=None):
    """Cotangents of bidiag (b <= 16) from its outputs G_diag, G_lower and their
    cotangents (None = zero): returns a dict with Mb_diag and Mb_lower."""
    _cuda_contig("G_diag", G_diag)
    dt = G_diag.dtype
    if G_diag.dim() < 3 or G_diag.shape[-1] != G_diag.shape[-2]:
        raise ValueError("G_diag must be [..., L, b, b]")
    lead = tuple(G_diag.shape[:-3])
    L, b = int(G_diag.shape[-3]), int(G_diag.shape[-1])
    batch = 1
    for d in lead:
        batch *= int(d)
    shape_l = lead + (max(L - 1, 0), b, b)
    if Gb_diag is not None:
        _cuda_contig("Gb_diag", Gb_diag, dt)
        if Gb_diag.shape != G_diag.shape:
            raise ValueError("Gb_diag must have G_diag's shape")
    if L > 1:
        _cuda_contig("G_lower", G_lower, dt)
        if tuple(G_lower.shape) != shape_l:
            raise ValueError(f"G_lower must be {shape_l}")
        if Gb_lower is not None:
            _cuda_contig("Gb_lower", Gb_lower, dt)
            if tuple(Gb_lower.shape) != shape_l:
                raise ValueError(f"Gb_lower must be {shape_l}")
    else:
        G_lower = Gb_lower = None
    out = dict(out or {})
    Mb_diag = out.get("Mb_diag")
    if Mb_diag is None:
        Mb_diag = torch.empty_like(G_diag)
    Mb_lower = out.get("Mb_lower")
    if Mb_lower is None:
        Mb_lower = torch.empty(shape_l, dtype=dt, device=G_diag.device)
    with torch.cuda.device(G_diag.device):
        st = lib().selinv_bidiag_backward(_code(dt), batch, L, b, _ptr(G_diag), _ptr(G_lower), _ptr(Gb_diag),
                                          _ptr(Gb_lower), _ptr(Mb_diag), _ptr(Mb_lower if L > 1 else None),
                                          _stream_handle(stream))
    _check(st, "selinv_bidiag_backward")
    return {"Mb_diag": Mb_diag, "Mb_lower": Mb_lower}


class _BidiagFn(torch.autograd.Function):
    """G_diag, G_lower = bidiag(diag, lower) with its analytic backward."""

    @staticmethod
    def forward(ctx, diag, lower):
        out = bidiag(diag, lower)
        ctx.save_for_backward(out["G_diag"], out["G_lower"])
        return out["G_diag"], out["G_lower"]

    @staticmethod
    def backward(ctx, gb_diag, gb_lower):
        G_diag, G_lower = ctx.saved_tensors
        r = bidiag_backward(G_diag, G_lower, None if gb_diag is None else gb_diag.contiguous(),
                            None if gb_lower is None else gb_lower.contiguous())
        return r["Mb_diag"], r["Mb_lower"]


def bidiag_ad(diag, lower):
    """Differentiable selected inverse of block lower-bidiagonal matrices (the
    pages' selinv_bidiag, b <= 16): returns (G_diag, G_lower)."""
    return _BidiagFn.apply(diag, lower)


def chain_backward_workspace_size(dtype, batch, L, b) -> int:
    return int(lib().selinv_chain_backward_workspace_size(_code(dtype), batch, L, b))


def chain_backward(diag, lower, G_diag, G_lower, Gb_diag=None, Gb_lower=None, *, check=True, out=None,
                   workspace=None, stream=None):
    """Cotangents of selinv_chain (b <= 16): from the cotangents Gb_diag, Gb_lower
    of its outputs G_diag, G_lower (None = zero), the cotangents Db of diag
    (lower-triangular: only D's lower triangle is read) and Bb of lower.
    Returns a dict with Db, Bb and info (int32, -1 = ok)."""
    _cuda_contig("diag", diag)
    dt = diag.dtype
    if diag.dim() < 3 or diag.shape[-1] != diag.shape[-2]:
        raise ValueError("diag must be [..., L, b, b]")
    lead = tuple(diag.shape[:-3])
    L, b = int(diag.shape[-3]), int(diag.shape[-1])
    batch = 1
    for d in lead:
        batch *= int(d)
    _cuda_contig("G_diag", G_diag, dt)
    if Gb_diag is not None:
        _cuda_contig("Gb_diag", Gb_diag, dt)
    for name, t in (("G_diag", G_diag), ("Gb_diag", Gb_diag)):
        if t is not None and tuple(t.shape) != tuple(diag.shape):
            raise ValueError(f"{name} must have diag's shape")
    shape_l = lead + (L - 1, b, b)
    if L > 1:
        for name, t in (("lower", lower), ("G_lower", G_lower)):
            if t is None:
                raise ValueError(f"{name} is required when L > 1")
            _cuda_contig(name, t, dt)
            if tuple(t.shape) != shape_l:
                raise ValueError(f"{name} must be {shape_l}")
        if Gb_lower is not None:
            _cuda_contig("Gb_lower", Gb_lower, dt)
            if tuple(Gb_lower.shape) != shape_l:
                raise ValueError(f"Gb_lower must be {shape_l}")
    else:
        lower = G_lower = Gb_lower = None
    dev = diag.device
    out = dict(out or {})
    Db = out.get("Db")
    if Db is None:
        Db = torch.empty_like(diag)
    Bb = out.get("Bb")
    if Bb is None:
        Bb = torch.empty(shape_l, dtype=dt, device=dev)
    info = out.get("info")
    if info is None:
        info = torch.empty(lead, dtype=torch.int32, device=dev)
    nbytes = chain_backward_workspace_size(dt, batch, L, b)
    ws = _workspace(nbytes, dev, workspace)
    with torch.cuda.device(dev):
        st = lib().selinv_chain_backward(_code(dt), batch, L, b, _ptr(diag), _ptr(lower), _ptr(G_diag),
                                         _ptr(G_lower), _ptr(Gb_diag), _ptr(Gb_lower), _ptr(Db),
                                         _ptr(Bb if L > 1 else None), _ptr(info), _ptr(ws), nbytes,
                                         _stream_handle(stream))
    _check(st, "selinv_chain_backward")
    _raise_on_info(info, check)
    return {"Db": Db, "Bb": Bb, "info": info}


class _SelinvChainFn(torch.autograd.Function):
    """G_diag, G_lower = selinv_chain(diag, lower) with its analytic backward."""

    @staticmethod
    def forward(ctx, diag, lower):
        out = selinv_chain(diag, lower)
        ctx.save_for_backward(diag, lower, out["G_diag"], out["G_lower"])
        return out["G_diag"], out["G_lower"]

    @staticmethod
    def backward(ctx, gb_diag, gb_lower):
        diag, lower, G_diag, G_lower = ctx.saved_tensors
        r = chain_backward(diag, lower, G_diag, G_lower,
                           None if gb_diag is None else gb_diag.contiguous(),
                           None if gb_lower is None else gb_lower.contiguous())
        return r["Db"], r["Bb"]


def selinv_chain_ad(diag, lower):
    """Differentiable selected inverse of chains (b <= 16): returns (G_diag,
    G_lower); gradients reach diag (its lower triangle: the forward reads no
    other entry) and lower through chain_backward."""
    return _SelinvChainFn.apply(diag, lower)


def junction_symbolic(n, edge_index, order=None):
    """The junction plan's symbolic phase on the host (no device): returns
    (order [n], S_index [2, nnz_S]) exactly as JunctionPlan would."""
    import numpy as np
    ei = np.ascontiguousarray(np.asarray(edge_index[0], dtype=np.int32))
    ej = np.ascontiguousarray(np.asarray(edge_index[1], dtype=np.int32))
    o = None if order is None else np.ascontiguousarray(np.asarray(order, dtype=np.int32))
    args = (int(n), ei.size, ei.ctypes.data_as(ctypes.c_void_p), ej.ctypes.data_as(ctypes.c_void_p),
            None if o is None else o.ctypes.data_as(ctypes.c_void_p))
    nnz = ctypes.c_int64()
    _check(lib().selinv_junction_symbolic(*args, ctypes.byref(nnz), None, None, 0, None), "selinv_junction_symbolic")
    si = np.empty(max(nnz.value, 1), dtype=np.int32)
    sj = np.empty(max(nnz.value, 1), dtype=np.int32)
    od = np.empty(int(n), dtype=np.int32)
    _check(lib().selinv_junction_symbolic(*args, ctypes.byref(nnz), si.ctypes.data_as(ctypes.c_void_p),
                                          sj.ctypes.data_as(ctypes.c_void_p), nnz.value,
                                          od.ctypes.data_as(ctypes.c_void_p)), "selinv_junction_symbolic")
    return od, np.stack([si[:nnz.value], sj[:nnz.value]]).astype(np.int64)


class JunctionPlan:
    """Symbolic analysis of a block-sparse SPD pattern, cached on the device:
    elimination order (greedy minimum degree unless given), filled pattern S,
    elimination tree and its levels.  edge_index [2, m] holds the lower blocks
    (i, j), i > j.  After construction: .order [n] and .S_index [2, nnz_S]
    (pairs (i, j), i > j, sorted by j then i)."""

    def __init__(self, n, edge_index, order=None):
        import numpy as np
        ei = np.ascontiguousarray(np.asarray(edge_index[0], dtype=np.int32))
        ej = np.ascontiguousarray(np.asarray(edge_index[1], dtype=np.int32))
        if ei.shape != ej.shape or ei.ndim != 1:
            raise ValueError("edge_index must be [2, m]")
        o = None if order is None else np.ascontiguousarray(np.asarray(order, dtype=np.int32))
        h = ctypes.c_void_p()
        st = lib().selinv_junction_plan(int(n), ei.size, ei.ctypes.data_as(ctypes.c_void_p),
                                        ej.ctypes.data_as(ctypes.c_void_p),
                                        None if o is None else o.ctypes.data_as(ctypes.c_void_p), ctypes.byref(h))
        _check(st, "selinv_junction_plan")
        self._h = h
        self.n, self.m = int(n), int(ei.size)
        nnz, lc, ld = ctypes.c_int64(), ctypes.c_int32(), ctypes.c_int32()
        _check(lib().selinv_junction_plan_info(h, ctypes.byref(nnz), ctypes.byref(lc), ctypes.byref(ld)),
               "selinv_junction_plan_info")
        self.nnz = int(nnz.value)
        self.levels = (int(lc.value), int(ld.value))
        si = np.empty(max(self.nnz, 1), dtype=np.int32)
        sj = np.empty(max(self.nnz, 1), dtype=np.int32)
        od = np.empty(self.n, dtype=np.int32)
        _check(lib().selinv_junction_plan_pattern(h, si.ctypes.data_as(ctypes.c_void_p),
                                                  sj.ctypes.data_as(ctypes.c_void_p),
                                                  od.ctypes.data_as(ctypes.c_void_p)), "selinv_junction_plan_pattern")
        self.S_index = np.stack([si[:self.nnz], sj[:self.nnz]]).astype(np.int64)
        self.order = od
        self.launches = int(lib().selinv_junction_plan_launches(h))

    @property
    def handle(self):
        return self._h

    def workspace_size(self, dtype, b, batch) -> int:
        return int(lib().selinv_junction_workspace_size(self._h, _code(dtype), b, batch))

    def close(self):
        if getattr(self, "_h", None) and _lib is not None:
            _lib.selinv_junction_plan_free(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def junction_solve(plan: JunctionPlan, diag, edge_val, rhs, *, check=True, out=None, workspace=None, stream=None):
    """x = A^-1 r for general block-sparse SPD matrices on the plan's pattern
    (b <= 16), from the same factorisation: diag [..., n, b, b], edge_val
    [..., m, b, b], rhs [..., n, b].  Returns (x, logdet, info)."""
    _cuda_contig("diag", diag)
    dt = diag.dtype
    if diag.dim() < 3 or diag.shape[-1] != diag.shape[-2] or int(diag.shape[-3]) != plan.n:
        raise ValueError(f"diag must be [..., {plan.n}, b, b]")
    lead = tuple(diag.shape[:-3])
    b = int(diag.shape[-1])
    batch = 1
    for d in lead:
        batch *= int(d)
    _cuda_contig("edge_val", edge_val, dt)
    if tuple(edge_val.shape) != lead + (plan.m, b, b):
        raise ValueError(f"edge_val must be {lead + (plan.m, b, b)}")
    _cuda_contig("rhs", rhs, dt)
    if tuple(rhs.shape) != lead + (plan.n, b):
        raise ValueError(f"rhs must be {lead + (plan.n, b)}")
    dev = diag.device
    out = dict(out or {})
    x = out.get("x")
    if x is None:
        x = torch.empty_like(rhs)
    logdet = out.get("logdet")
    if logdet is None:
        logdet = torch.empty(lead, dtype=torch.float64, device=dev)
    info = out.get("info")
    if info is None:
        info = torch.empty(lead, dtype=torch.int32, device=dev)
    nbytes = plan.workspace_size(dt, b, batch)
    ws = _workspace(nbytes, dev, workspace)
    with torch.cuda.device(dev):
        st = lib().selinv_junction_solve(plan.handle, _code(dt), b, batch, _ptr(diag), _ptr(edge_val), _ptr(rhs),
                                         _ptr(x), _ptr(logdet), _ptr(info), _ptr(ws), nbytes, _stream_handle(stream))
    _check(st, "selinv_junction_solve")
    _raise_on_info(info, check)
    return x, logdet, info


def junction(plan: JunctionPlan, diag, edge_val, *, check=True, out=None, workspace=None, stream=None):
    """Selected inverse of general block-sparse SPD matrices on the plan's
    filled pattern (b <= 16): diag [..., n, b, b], edge_val [..., m, b, b].
    Returns dict with G_diag, G_lower [..., nnz_S, b, b] on plan.S_index,
    logdet and info."""
    _cuda_contig("diag", diag)
    dt = diag.dtype
    if diag.dim() < 3 or diag.shape[-1] != diag.shape[-2] or int(diag.shape[-3]) != plan.n:
        raise ValueError(f"diag must be [..., {plan.n}, b, b]")
    lead = tuple(diag.shape[:-3])
    b = int(diag.shape[-1])
    batch = 1
    for d in lead:
        batch *= int(d)
    _cuda_contig("edge_val", edge_val, dt)
    if tuple(edge_val.shape) != lead + (plan.m, b, b):
        raise ValueError(f"edge_val must be {lead + (plan.m, b, b)}")
    dev = diag.device
    out = dict(out or {})
    G_diag = out.get("G_diag")
    if G_diag is None:
        G_diag = torch.empty_like(diag)
    G_lower = out.get("G_lower")
    if G_lower is None:
        G_lower = torch.empty(lead + (plan.nnz, b, b), dtype=dt, device=dev)
    logdet = out.get("logdet")
    if logdet is None:
        logdet = torch.empty(lead, dtype=torch.float64, device=dev)
    info = out.get("info")
    if info is None:
        info = torch.empty(lead, dtype=torch.int32, device=dev)
    nbytes = plan.workspace_size(dt, b, batch)
    ws = _workspace(nbytes, dev, workspace)
    with torch.cuda.device(dev):
        st = lib().selinv_junction(plan.handle, _code(dt), b, batch, _ptr(diag), _ptr(edge_val), _ptr(G_diag),
                                   _ptr(G_lower), _ptr(logdet), _ptr(info), _ptr(ws), nbytes, _stream_handle(stream))
    _check(st, "selinv_junction")
    _raise_on_info(info, check)
    return {"G_diag": G_diag, "G_lower": G_lower, "S_index": plan.S_index, "logdet": logdet, "info": info}


class TreePlan:
    """Validated level-set schedule of `trees` parent arrays of n nodes each (cached on the device)."""

    def __init__(self, parent):
        import numpy as np
        p = np.ascontiguousarray(np.asarray(parent, dtype=np.int32))
        if p.ndim == 1:
            p = p[None]
        if p.ndim != 2:
            raise ValueError("parent must be [n] or [trees, n]")
        self.trees, self.n = int(p.shape[0]), int(p.shape[1])
        h = ctypes.c_void_p()
        st = lib().selinv_tree_plan(p.ctypes.data_as(ctypes.c_void_p), self.trees, self.n, ctypes.byref(h))
        _check(st, "selinv_tree_plan")
        self._h = h

    @property
    def handle(self):
        return self._h

    def levels(self):
        c, d = ctypes.c_int32(), ctypes.c_int32()
        _check(lib().selinv_tree_plan_levels(self._h, ctypes.byref(c), ctypes.byref(d)), "levels")
        return c.value, d.value

    def set_wait(self, spin_limit: int = 0, withhold: int = -1):
        """Bound of the sweeps' dependency waits (polls; 0 = the default) and a
        node whose completion is never published (-1 = none; a test hook)."""
        _check(lib().selinv_tree_plan_set_wait(self._h, int(spin_limit), int(withhold)), "selinv_tree_plan_set_wait")

    def workspace_size(self, dtype, b) -> int:
        return int(lib().selinv_tree_workspace_size(self._h, _code(dtype), b))

    def backward_workspace_size(self, dtype, b) -> int:
        return int(lib().selinv_tree_backward_workspace_size(self._h, _code(dtype), b))

    def close(self):
        if getattr(self, "_h", None) and _lib is not None:
            _lib.selinv_tree_plan_free(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def selinv_tree(plan: TreePlan, diag: torch.Tensor, edge: torch.Tensor, *, check=True, validate=False, out=None,
                workspace=None, stream=None):
    """Selected inverse and log det of block-tree SPD matrices.

    diag, edge [trees, n, b, b] (or [n, b, b] for one tree) with
    edge[v] = A_{parent(v), v}.  Returns dict with G_diag, G_edge (root slot
    zero), logdet [trees] float64 and info [trees].  check and validate as in
    selinv_chain (info -3 - v: node v holds a non-finite entry).
    """
    _cuda_contig("diag", diag)
    dt = diag.dtype
    code = _code(dt)
    _cuda_contig("edge", edge, dt)
    single = diag.dim() == 3
    d4 = diag[None] if single else diag
    e4 = edge[None] if single else edge
    if d4.dim() != 4 or tuple(d4.shape[:2]) != (plan.trees, plan.n) or d4.shape[-1] != d4.shape[-2]:
        raise ValueError(f"diag must be [{plan.trees}, {plan.n}, b, b]")
    if e4.shape != d4.shape:
        raise ValueError("edge must have diag's shape")
    b = int(d4.shape[-1])
    dev = diag.device
    out = dict(out or {})
    G_diag = out.get("G_diag")
    if G_diag is None:
        G_diag = torch.empty_like(d4)
    G_edge = out.get("G_edge")
    if G_edge is None:
        G_edge = torch.empty_like(d4)
    logdet = out.get("logdet")
    if logdet is None:
        logdet = torch.empty(plan.trees, dtype=torch.float64, device=dev)
    info = out.get("info")
    if info is None:
        info = torch.empty(plan.trees, dtype=torch.int32, device=dev)
    nbytes = plan.workspace_size(dt, b)
    ws = _workspace(nbytes, dev, workspace)
    with torch.cuda.device(dev):
        st = lib().selinv_tree(plan.handle, code, b, _ptr(d4), _ptr(e4), _ptr(G_diag), _ptr(G_edge),
                               _ptr(logdet), _ptr(info), _ptr(ws), nbytes, CHECK if validate else 0,
                               _stream_handle(stream))
    _check(st, "selinv_tree")
    _raise_on_info(info, check)
    if single:
        G_diag, G_edge = G_diag[0], G_edge[0]
    return {"G_diag": G_diag, "G_edge": G_edge, "logdet": logdet, "info": info}


def tree_backward(plan: TreePlan, diag, edge, G_diag, G_edge, Gb_diag=None, Gb_edge=None, *, check=True, out=None,
                  workspace=None, stream=None):
    """Cotangents of selinv_tree (b <= 16): from the cotangents Gb_diag, Gb_edge
    of its outputs G_diag, G_edge (None = zero; the root's edge slot is
    ignored), the cotangents Db of diag (lower-triangular: only D's lower
    triangle is read) and Eb of edge (root slot 0).  Returns a dict with Db,
    Eb and info."""
    _cuda_contig("diag", diag)
    dt = diag.dtype
    single = diag.dim() == 3
    lift = (lambda x: None if x is None else (x[None] if single else x))
    d4, e4, gd4, ge4 = lift(diag), lift(edge), lift(G_diag), lift(G_edge)
    gbd4, gbe4 = lift(Gb_diag), lift(Gb_edge)
    if d4.dim() != 4 or tuple(d4.shape[:2]) != (plan.trees, plan.n) or d4.shape[-1] != d4.shape[-2]:
        raise ValueError(f"diag must be [{plan.trees}, {plan.n}, b, b]")
    for name, x in (("edge", e4), ("G_diag", gd4), ("G_edge", ge4), ("Gb_diag", gbd4), ("Gb_edge", gbe4)):
        if x is None:
            if name in ("edge", "G_diag", "G_edge"):
                raise ValueError(f"{name} is required")
            continue
        _cuda_contig(name, x, dt)
        if x.shape != d4.shape:
            raise ValueError(f"{name} must have diag's shape")
    b = int(d4.shape[-1])
    dev = diag.device
    out = dict(out or {})
    Db = out.get("Db")
    if Db is None:
        Db = torch.empty_like(d4)
    Eb = out.get("Eb")
    if Eb is None:
        Eb = torch.empty_like(d4)
    info = out.get("info")
    if info is None:
        info = torch.empty(plan.trees, dtype=torch.int32, device=dev)
    nbytes = plan.backward_workspace_size(dt, b)
    ws = _workspace(nbytes, dev, workspace)
    with torch.cuda.device(dev):
        st = lib().selinv_tree_backward(plan.handle, _code(dt), b, _ptr(d4), _ptr(e4), _ptr(gd4), _ptr(ge4),
                                        _ptr(gbd4), _ptr(gbe4), _ptr(Db), _ptr(Eb), _ptr(info), _ptr(ws), nbytes,
                                        _stream_handle(stream))
    _check(st, "selinv_tree_backward")
    _raise_on_info(info, check)
    if single:
        Db, Eb = Db[0], Eb[0]
    return {"Db": Db, "Eb": Eb, "info": info}


class _SelinvTreeFn(torch.autograd.Function):
    """G_diag, G_edge = selinv_tree(plan, diag, edge) with its analytic backward."""

    @staticmethod
    def forward(ctx, diag, edge, plan):
        out = selinv_tree(plan, diag, edge)
        ctx.plan = plan
        ctx.save_for_backward(diag, edge, out["G_diag"], out["G_edge"])
        return out["G_diag"], out["G_edge"]

    @staticmethod
    def backward(ctx, gb_diag, gb_edge):
        diag, edge, G_diag, G_edge = ctx.saved_tensors
        r = tree_backward(ctx.plan, diag, edge, G_diag, G_edge,
                          None if gb_diag is None else gb_diag.contiguous(),
                          None if gb_edge is None else gb_edge.contiguous())
        return r["Db"], r["Eb"], None


def selinv_tree_ad(plan: TreePlan, diag, edge):
    """Differentiable selected inverse of block trees (b <= 16): returns
    (G_diag, G_edge); gradients reach diag (its lower triangle) and edge
    through tree_backward -- the pages' selinv_tree."""
    return _SelinvTreeFn.apply(diag, edge, plan)


def tree_sample(plan: TreePlan, diag: torch.Tensor, edge: torch.Tensor, z: torch.Tensor, *, check=True, out=None,
                workspace=None, stream=None):
    """Gaussian draw on block trees: eta = L^-T z for A = L L^T in the tree's own
    elimination order (children before parents), z [trees, n, b] the caller's
    standard normals (b <= 16).  Returns dict with eta, logdet and info."""
    _cuda_contig("diag", diag)
    dt = diag.dtype
    _cuda_contig("edge", edge, dt)
    _cuda_contig("z", z, dt)
    single = diag.dim() == 3
    d4 = diag[None] if single else diag
    e4 = edge[None] if single else edge
    z3 = z[None] if single else z
    if d4.dim() != 4 or tuple(d4.shape[:2]) != (plan.trees, plan.n) or d4.shape[-1] != d4.shape[-2]:
        raise ValueError(f"diag must be [{plan.trees}, {plan.n}, b, b]")
    if e4.shape != d4.shape:
        raise ValueError("edge must have diag's shape")
    b = int(d4.shape[-1])
    if tuple(z3.shape) != (plan.trees, plan.n, b):
        raise ValueError(f"z must be [{plan.trees}, {plan.n}, {b}]")
    dev = diag.device
    out = dict(out or {})
    eta = out.get("eta")
    if eta is None:
        eta = torch.empty_like(z3)
    logdet = out.get("logdet")
    if logdet is None:
        logdet = torch.empty(plan.trees, dtype=torch.float64, device=dev)
    info = out.get("info")
    if info is None:
        info = torch.empty(plan.trees, dtype=torch.int32, device=dev)
    nbytes = plan.workspace_size(dt, b)
    ws = _workspace(nbytes, dev, workspace)
    with torch.cuda.device(dev):
        st = lib().selinv_tree_sample(plan.handle, _code(dt), b, _ptr(d4), _ptr(e4), _ptr(z3), _ptr(eta),
                                      _ptr(logdet), _ptr(info), _ptr(ws), nbytes, _stream_handle(stream))
    _check(st, "selinv_tree_sample")
    _raise_on_info(info, check)
    return {"eta": eta[0] if single else eta, "logdet": logdet, "info": info}
