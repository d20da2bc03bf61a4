"""Thin Python binding over libssm_scan.so (the C ABI declared in include/ssm_scan.h).

Argument marshalling only: every step of the selective scan runs in the library's CUDA
kernels.  PyTorch provides device memory and the current CUDA stream.  If the shared
library has not been built, loading raises -- there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

from .build import LIB_PATH, build  # noqa: F401  (build is re-exported for convenience)

SSM_OK = 0
_STATUS = {0: "SSM_OK", 1: "SSM_ERR_INVALID_ARG", 2: "SSM_ERR_UNSUPPORTED", 3: "SSM_ERR_CUDA",
           4: "SSM_ERR_BAD_SLOT", 5: "SSM_ERR_TIMEOUT", 6: "SSM_ERR_WORKSPACE"}
SSM_F32, SSM_BF16 = 0, 1
ABI_VERSION = 5
DISC_EULER, DISC_ZOH = 0, 1  # ssm_discretization_t
ALGO_AUTO, ALGO_CHUNKED, ALGO_SEQUENTIAL = 0, 1, 2  # ssm_algorithm_t
_ALGO = {"auto": ALGO_AUTO, "chunked": ALGO_CHUNKED, "sequential": ALGO_SEQUENTIAL}

# Every function the header declares; tests check the library exports all of them.
EXPORTED = ("ssm_scan_fwd", "ssm_scan_fwd_varlen", "ssm_state_update", "ssm_scan_workspace_size",
            "ssm_get_device_status", "ssm_status_string", "ssm_abi_version", "ssm_scan_fwd_noalloc",
            "ssm_scan_fwd_varlen_pool", "ssm_test_drop_first_handoff", "ssm_scan_bwd",
            "ssm_scan_bwd_workspace_size", "ssm_ssd_fwd")
NOALLOC_SCRATCH_BYTES = 4 << 20  # SSM_NOALLOC_SCRATCH_BYTES


class SSMError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {_STATUS.get(code, code)}")


class ScanParams(ctypes.Structure):
    """Mirror of ssm_scan_params."""
    _fields_ = [
        ("dtype", ctypes.c_int), ("y_fp32", ctypes.c_int32),
        ("batch", ctypes.c_int64), ("dim", ctypes.c_int64), ("dstate", ctypes.c_int64),
        ("seqlen", ctypes.c_int64),
        ("x_batch_stride", ctypes.c_int64), ("x_dim_stride", ctypes.c_int64),
        ("bc_batch_stride", ctypes.c_int64), ("bc_state_stride", ctypes.c_int64),
        ("u", ctypes.c_void_p), ("delta", ctypes.c_void_p), ("z", ctypes.c_void_p),
        ("B", ctypes.c_void_p), ("C", ctypes.c_void_p),
        ("A", ctypes.c_void_p), ("Dskip", ctypes.c_void_p), ("delta_bias", ctypes.c_void_p),
        ("h0", ctypes.c_void_p), ("y", ctypes.c_void_p), ("h_last", ctypes.c_void_p),
        ("ngroups", ctypes.c_int64), ("bc_group_stride", ctypes.c_int64), ("discretization", ctypes.c_int32),
        ("algorithm", ctypes.c_int32),
    ]


class SsdParams(ctypes.Structure):
    """Mirror of ssm_ssd_params."""
    _fields_ = [("batch", ctypes.c_int64), ("nheads", ctypes.c_int64), ("headdim", ctypes.c_int64),
                ("dstate", ctypes.c_int64), ("seqlen", ctypes.c_int64)] + \
               [(n, ctypes.c_void_p) for n in ("x", "dt", "A", "B", "C", "h0", "y", "h_last")]


class ScanGrads(ctypes.Structure):
    """Mirror of ssm_scan_grads."""
    _fields_ = [(n, ctypes.c_void_p) for n in ("dy", "dh_last", "du", "ddelta", "dz", "dB", "dC", "dA", "dDskip",
                                                 "ddelta_bias", "dh0")]


_lib = None


def load(path: str | None = None) -> ctypes.CDLL:
    """Load the built library.  Raises FileNotFoundError if it has not been built."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise FileNotFoundError(
            f"{p} is missing: build the CUDA library first (python -m selective_state_space_15_b200.build)")
    lib = ctypes.CDLL(p)
    P, I64, S = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
    pp = ctypes.POINTER(ScanParams)
    lib.ssm_scan_fwd.argtypes = [pp, P, S, P]
    lib.ssm_scan_fwd_noalloc.argtypes = [pp, P]
    lib.ssm_scan_fwd_noalloc.restype = ctypes.c_int
    lib.ssm_scan_fwd_varlen.argtypes = [pp, P, I64, P, S, P]
    lib.ssm_scan_fwd_varlen_pool.argtypes = [pp, P, I64, P, I64, P, P, S, P]
    lib.ssm_state_update.argtypes = [P, I64, P, I64, pp, P]
    lib.ssm_scan_workspace_size.argtypes = [pp, I64]
    lib.ssm_scan_workspace_size.restype = S
    lib.ssm_scan_bwd.argtypes = [pp, ctypes.POINTER(ScanGrads), P, S, P]
    lib.ssm_scan_bwd_workspace_size.argtypes = [pp]
    lib.ssm_ssd_fwd.argtypes = [ctypes.POINTER(SsdParams), P]
    lib.ssm_scan_bwd_workspace_size.restype = S
    lib.ssm_get_device_status.argtypes = [P]
    lib.ssm_status_string.argtypes = [ctypes.c_int]
    lib.ssm_status_string.restype = ctypes.c_char_p
    lib.ssm_abi_version.argtypes = []
    lib.ssm_test_drop_first_handoff.argtypes = []
    lib.ssm_test_drop_first_handoff.restype = None
    for f in ("ssm_scan_fwd", "ssm_scan_fwd_varlen", "ssm_scan_fwd_varlen_pool", "ssm_state_update",
              "ssm_get_device_status", "ssm_scan_bwd", "ssm_ssd_fwd"):
        getattr(lib, f).restype = ctypes.c_int
    if lib.ssm_abi_version() != ABI_VERSION:
        raise RuntimeError(f"libssm_scan ABI {lib.ssm_abi_version()} != binding ABI {ABI_VERSION}")
    if path is None:
        _lib = lib
    return lib


# ----------------------------------------------------------------------------- helpers

def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return SSM_BF16
    if t.dtype == torch.float32:
        return SSM_F32
    raise TypeError(f"unsupported input dtype {t.dtype} (bfloat16 or float32)")


def _check(code: int, where: str):
    if code != SSM_OK:
        raise SSMError(code, where)


def _y_fp32(u, y):
    """1 when y is float32 while the inputs are bf16 (the float32-output option)."""
    import torch
    if y is None or y.dtype == u.dtype:
        return 0
    if y.dtype == torch.float32:
        return 1
    raise TypeError("y must have the input dtype or float32")


def _time_contig(*ts):
    for t in ts:
        if t is not None and t.stride(-1) != 1:
            raise ValueError("the time (last) axis must have stride 1")


def _algo(algorithm) -> int:
    """ssm_algorithm_t code for 'auto' / 'chunked' / 'sequential' (or the code itself)."""
    if isinstance(algorithm, str):
        if algorithm not in _ALGO:
            raise ValueError(f"algorithm must be one of {sorted(_ALGO)}")
        return _ALGO[algorithm]
    return int(algorithm)


def _f32(t):
    import torch
    if t is not None and (t.dtype != torch.float32 or not t.is_contiguous()):
        raise ValueError("A, Dskip, delta_bias and states must be contiguous float32")
    return t


# ----------------------------------------------------------------------------- scans

def scan_params(u, delta, B, C, A, Dskip=None, delta_bias=None, z=None, h0=None, y=None, h_last=None, zoh=False,
                algorithm="auto"):
    """Fill ScanParams for the fixed-length layout u/delta/z/y [b, D, L], B/C [b, N, L] (or
    [b, G, N, L]: G channel groups, channel d reading group d // (D / G))."""
    bsz, dim, L = u.shape
    N = A.shape[1]
    _time_contig(u, delta, z, B, C, y)
    for t in (delta, z, y):
        if t is not None and (t.shape != u.shape or t.stride() != u.stride()):
            raise ValueError("delta, z and y must match u's shape and strides")
    G = B.shape[1] if B.dim() == 4 else 1
    want = (bsz, G, N, L) if B.dim() == 4 else (bsz, N, L)
    if B.shape != want or C.shape != B.shape or C.stride() != B.stride():
        raise ValueError("B and C must be [batch, (groups,) dstate, seqlen] with equal strides")
    for t in (A, Dskip, delta_bias, h0, h_last):
        _f32(t)
    p = ScanParams()
    p.dtype = _dtype_code(u)
    p.y_fp32 = _y_fp32(u, y)
    p.batch, p.dim, p.dstate, p.seqlen = bsz, dim, N, L
    p.x_batch_stride, p.x_dim_stride = u.stride(0), u.stride(1)
    p.bc_batch_stride, p.bc_state_stride = B.stride(0), B.stride(-2)
    if B.dim() == 4:
        p.ngroups, p.bc_group_stride = G, B.stride(1)
    p.u, p.delta, p.z, p.B, p.C = _ptr(u), _ptr(delta), _ptr(z), _ptr(B), _ptr(C)
    p.A, p.Dskip, p.delta_bias, p.h0 = _ptr(A), _ptr(Dskip), _ptr(delta_bias), _ptr(h0)
    p.y, p.h_last = _ptr(y), _ptr(h_last)
    p.discretization = DISC_ZOH if zoh else DISC_EULER
    p.algorithm = _algo(algorithm)
    return p


def scan_fwd(u, delta, B, C, A, Dskip=None, delta_bias=None, z=None, h0=None, y=None, h_last=None,
             return_last_state=True, stream=None, y_dtype=None, zoh=False, algorithm="auto"):
    """Selective scan over a fixed-length batch.  Returns (y, h_last).

    y is allocated in ``y_dtype`` (default: the input dtype; float32 is also accepted).
    ``zoh``: zero-order-hold input matrix instead of Bbar = Delta B.  ``algorithm``: 'auto',
    'chunked' or 'sequential' (ssm_algorithm_t)."""
    import torch
    y = torch.empty_like(u, dtype=y_dtype or u.dtype) if y is None else y
    if h_last is None and return_last_state:
        h_last = torch.empty((u.shape[0], u.shape[1], A.shape[1]), device=u.device, dtype=torch.float32)
    p = scan_params(u, delta, B, C, A, Dskip, delta_bias, z, h0, y, h_last, zoh, algorithm)
    lib = load()
    ws = lib.ssm_scan_workspace_size(ctypes.byref(p), 0)
    wbuf = torch.empty(ws, device=u.device, dtype=torch.uint8) if ws else None
    _check(lib.ssm_scan_fwd(ctypes.byref(p), _ptr(wbuf), ws, _stream(stream)), "ssm_scan_fwd")
    return y, h_last


def varlen_params(u, delta, B, C, A, Dskip=None, delta_bias=None, z=None, h0=None, y=None, h_last=None,
                  total=None, zoh=False, algorithm="auto"):
    """ScanParams for the packed layout u/delta/z/y [D, T(+pad)], B/C [N, T(+pad)] (or
    [G, N, T(+pad)]: G channel groups).

    ``total`` is the number of packed tokens T when the rows are padded beyond it.
    """
    dim, width = u.shape
    T = width if total is None else int(total)
    N = A.shape[1]
    _time_contig(u, delta, z, B, C, y)
    for t in (delta, z, y):
        if t is not None and (t.shape != u.shape or t.stride() != u.stride()):
            raise ValueError("delta, z and y must match u's shape and strides")
    if B.shape[-2] != N or C.shape != B.shape or C.stride() != B.stride() or B.shape[-1] < T or B.dim() > 3:
        raise ValueError("B and C must be [(groups,) dstate, >=T] with equal strides")
    for t in (A, Dskip, delta_bias, h0, h_last):
        _f32(t)
    p = ScanParams()
    p.dtype = _dtype_code(u)
    p.y_fp32 = _y_fp32(u, y)
    p.batch, p.dim, p.dstate, p.seqlen = 1, dim, N, T
    p.x_batch_stride, p.x_dim_stride = 0, u.stride(0)
    p.bc_batch_stride, p.bc_state_stride = 0, B.stride(-2)
    if B.dim() == 3:
        p.ngroups, p.bc_group_stride = B.shape[0], B.stride(0)
    p.u, p.delta, p.z, p.B, p.C = _ptr(u), _ptr(delta), _ptr(z), _ptr(B), _ptr(C)
    p.A, p.Dskip, p.delta_bias, p.h0 = _ptr(A), _ptr(Dskip), _ptr(delta_bias), _ptr(h0)
    p.y, p.h_last = _ptr(y), _ptr(h_last)
    p.discretization = DISC_ZOH if zoh else DISC_EULER
    p.algorithm = _algo(algorithm)
    return p


def scan_bwd(u, delta, B, C, A, dy, Dskip=None, delta_bias=None, z=None, h0=None, dh_last=None, stream=None,
             zoh=False, grad_dtype=None, want_dh0=True):
    """Gradients of scan_fwd (fixed-length batch) given dy (and optionally dh_last).

    Returns a dict with du, ddelta, dz (None without z) [b, D, L] in ``grad_dtype`` (default: the
    input dtype; float32 is also accepted), dB, dC [b, N, L], dA [D, N], dDskip, dbias [D] and
    dh0 [b, D, N] (float32)."""
    import torch
    gdt = grad_dtype or u.dtype
    if dy.dtype != gdt:
        raise TypeError("dy must have the gradient dtype")
    bsz, dim, L = u.shape
    N = A.shape[1]
    out = {"du": torch.empty_like(u, dtype=gdt), "ddelta": torch.empty_like(u, dtype=gdt),
           "dz": torch.empty_like(u, dtype=gdt) if z is not None else None,
           "dB": torch.empty((bsz, N, L), device=u.device, dtype=torch.float32),
           "dC": torch.empty((bsz, N, L), device=u.device, dtype=torch.float32),
           "dA": torch.empty((dim, N), device=u.device, dtype=torch.float32),
           "dDskip": torch.empty(dim, device=u.device, dtype=torch.float32) if Dskip is not None else None,
           "dbias": torch.empty(dim, device=u.device, dtype=torch.float32) if delta_bias is not None else None,
           "dh0": torch.empty((bsz, dim, N), device=u.device, dtype=torch.float32) if want_dh0 else None}
    for t in (dy, out["du"], out["ddelta"], out["dz"]):
        if t is not None and t.stride() != u.stride():
            raise ValueError("dy and the per-step gradients must have u's strides")
    p = scan_params(u, delta, B, C, A, Dskip, delta_bias, z, h0, None, None, zoh)
    p.y_fp32 = 1 if (gdt == torch.float32 and u.dtype != torch.float32) else 0
    _f32(dh_last)
    g = ScanGrads()
    g.dy, g.dh_last = _ptr(dy), _ptr(dh_last)
    g.du, g.ddelta, g.dz = _ptr(out["du"]), _ptr(out["ddelta"]), _ptr(out["dz"])
    g.dB, g.dC, g.dA = _ptr(out["dB"]), _ptr(out["dC"]), _ptr(out["dA"])
    g.dDskip, g.ddelta_bias, g.dh0 = _ptr(out["dDskip"]), _ptr(out["dbias"]), _ptr(out["dh0"])
    lib = load()
    ws = lib.ssm_scan_bwd_workspace_size(ctypes.byref(p))
    wbuf = torch.empty(ws, device=u.device, dtype=torch.uint8) if ws else None
    _check(lib.ssm_scan_bwd(ctypes.byref(p), ctypes.byref(g), _ptr(wbuf), ws, _stream(stream)), "ssm_scan_bwd")
    return out


def ssd_fwd(x, dt, A, B, C, h0=None, y=None, h_last=None, return_last_state=True, stream=None):
    """SSD chunked form (tensor cores): x [b, H, P, L] bf16, dt [b, H, L] float32 (the step, > 0),
    A [H] float32, B, C [b, N, L] bf16, h0 [b, H, P, N] float32 or None.  Returns (y, h_last)."""
    import torch
    bsz, H, P, L = x.shape
    N = B.shape[1]
    for t in (x, B, C):
        if t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("x, B and C must be contiguous bfloat16")
    for t in (dt, A, h0, h_last):
        _f32(t)
    if tuple(dt.shape) != (bsz, H, L) or tuple(B.shape) != (bsz, N, L) or C.shape != B.shape:
        raise ValueError("dt must be [b, H, L] and B, C [b, N, L]")
    y = torch.empty_like(x) if y is None else y
    if h_last is None and return_last_state:
        h_last = torch.empty((bsz, H, P, N), device=x.device, dtype=torch.float32)
    p = SsdParams()
    p.batch, p.nheads, p.headdim, p.dstate, p.seqlen = bsz, H, P, N, L
    p.x, p.dt, p.A, p.B, p.C = _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C)
    p.h0, p.y, p.h_last = _ptr(h0), _ptr(y), _ptr(h_last)
    _check(load().ssm_ssd_fwd(ctypes.byref(p), _stream(stream)), "ssm_ssd_fwd")
    return y, h_last


def scan_fwd_varlen(u, delta, B, C, A, cu_seqlens, Dskip=None, delta_bias=None, z=None, h0=None, y=None,
                    h_last=None, total=None, return_last_state=True, stream=None, y_dtype=None, zoh=False,
                    algorithm="auto"):
    """Packed variable-length scan.  cu_seqlens: int32 device tensor [nseq+1].  Returns (y, h_last)."""
    import torch
    if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_contiguous():
        raise ValueError("cu_seqlens must be a contiguous int32 tensor")
    nseq = cu_seqlens.shape[0] - 1
    y = torch.empty_like(u, dtype=y_dtype or u.dtype) if y is None else y
    if h_last is None and return_last_state:
        h_last = torch.empty((nseq, u.shape[0], A.shape[1]), device=u.device, dtype=torch.float32)
    p = varlen_params(u, delta, B, C, A, Dskip, delta_bias, z, h0, y, h_last, total, zoh, algorithm)
    lib = load()
    ws = lib.ssm_scan_workspace_size(ctypes.byref(p), nseq)
    wbuf = torch.empty(ws, device=u.device, dtype=torch.uint8) if ws else None
    _check(lib.ssm_scan_fwd_varlen(ctypes.byref(p), _ptr(cu_seqlens), nseq, _ptr(wbuf), ws, _stream(stream)),
           "ssm_scan_fwd_varlen")
    return y, h_last


def scan_fwd_varlen_pool(u, delta, B, C, A, cu_seqlens, pool, slot_ids, Dskip=None, delta_bias=None, z=None,
                         y=None, total=None, stream=None, y_dtype=None, zoh=False, algorithm="auto"):
    """Packed prefill into a state pool: sequence i starts from pool[slot_ids[i]] and its final
    state is written back there.  pool: float32 [S, D, N]; slot_ids: int32 [nseq].  Returns y."""
    import torch
    if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_contiguous():
        raise ValueError("cu_seqlens must be a contiguous int32 tensor")
    if slot_ids.dtype != torch.int32 or not slot_ids.is_contiguous():
        raise ValueError("slot_ids must be a contiguous int32 tensor")
    _f32(pool)
    nseq = cu_seqlens.shape[0] - 1
    if slot_ids.shape[0] != nseq:
        raise ValueError("one slot id per sequence")
    if tuple(pool.shape[1:]) != (u.shape[0], A.shape[1]):
        raise ValueError("pool must be [S, dim, dstate]")
    y = torch.empty_like(u, dtype=y_dtype or u.dtype) if y is None else y
    p = varlen_params(u, delta, B, C, A, Dskip, delta_bias, z, None, y, None, total, zoh, algorithm)
    lib = load()
    ws = lib.ssm_scan_workspace_size(ctypes.byref(p), nseq)
    wbuf = torch.empty(ws, device=u.device, dtype=torch.uint8) if ws else None
    _check(lib.ssm_scan_fwd_varlen_pool(ctypes.byref(p), _ptr(cu_seqlens), nseq, _ptr(pool), pool.shape[0],
                                        _ptr(slot_ids), _ptr(wbuf), ws, _stream(stream)),
           "ssm_scan_fwd_varlen_pool")
    return y


def state_update(pool, slot_ids, u, delta, B, C, A, Dskip=None, delta_bias=None, z=None, y=None, stream=None,
                 y_dtype=None, zoh=False):
    """One decode step in place on ``pool`` [S, D, N] float32.  u/delta/z [R, D]; B/C [R, N]."""
    import torch
    if slot_ids.dtype != torch.int32 or not slot_ids.is_contiguous():
        raise ValueError("slot_ids must be a contiguous int32 tensor")
    S, dim, N = pool.shape
    R = slot_ids.shape[0]
    _f32(pool)
    for t in (A, Dskip, delta_bias):
        _f32(t)
    _time_contig(u, delta, z, B, C)
    y = torch.empty_like(u, dtype=y_dtype or u.dtype) if y is None else y
    p = ScanParams()
    p.dtype = _dtype_code(u)
    p.y_fp32 = _y_fp32(u, y)
    p.batch, p.dim, p.dstate, p.seqlen = R, dim, N, 1
    p.x_batch_stride, p.x_dim_stride = u.stride(0), 0
    p.bc_batch_stride, p.bc_state_stride = B.stride(0), 0
    for t in (delta, z, y):
        if t is not None and t.stride(0) != u.stride(0):
            raise ValueError("u, delta, z and y must share the row stride")
    if C.stride(0) != B.stride(0):
        raise ValueError("B and C must share the row stride")
    p.u, p.delta, p.z, p.B, p.C = _ptr(u), _ptr(delta), _ptr(z), _ptr(B), _ptr(C)
    p.A, p.Dskip, p.delta_bias, p.y = _ptr(A), _ptr(Dskip), _ptr(delta_bias), _ptr(y)
    p.discretization = DISC_ZOH if zoh else DISC_EULER
    _check(load().ssm_state_update(_ptr(pool), S, _ptr(slot_ids), R, ctypes.byref(p), _stream(stream)),
           "ssm_state_update")
    return y


def device_status(stream=None) -> int:
    """Synchronise the stream, then read-and-clear the library's device status word."""
    return load().ssm_get_device_status(_stream(stream))


def status_string(code: int) -> str:
    return load().ssm_status_string(code).decode()
