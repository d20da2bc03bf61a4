"""fp64 CPU oracle for the selective scan -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline leg and its
``--impl reference`` arm) may import this package.  The CUDA library never does, and this
package imports nothing from it.

The arithmetic lives in ``ssm_oracle.c`` (scalar fp64, libm ``exp``/``log1p``, ``-O2`` without
fast-math).  This module only compiles it with gcc, loads it with ctypes and marshals numpy
arrays.  Inputs are converted to float64 exactly (fp32 and bf16 values are representable), so
the oracle sees precisely the values the GPU sees.

Definitions followed (cited by page title and section; see ``ssm_oracle.c`` for the full list):
  * ufo.work "会议长序列建模状态空间模型加速…" §1.1 -- h_t = exp(Δ_t A) h_{t-1} + Δ_t B_t x_t,
    y_t = C_t h_t;
  * discosf.com "企业官网建设流程全解析" §1.1 (skip term D x) and §1.3 (Δ = softplus(·));
  * ufo.work §4.2 -- packed sequences restart from h = 0 at each cu_seqlens boundary;
  * ufo.work §4.1 -- single-token update of a persistent per-request state;
  * discosf.com §1.2 -- the zero-order-hold input matrix Bbar = (ΔA)^-1 (exp(ΔA) - I) ΔB,
    chosen with ``zoh=True`` (default: Bbar = ΔB);
  * ufo.work §2.2 -- the training backward pass; ``scan_bwd`` returns the gradients that the
    forward definition fixes (reverse-mode derivative of ``scan``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssm_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_build", "libssm_oracle.so")
_lib = None
_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile ssm_oracle.c into a shared object (gcc -O2, no fast-math). Returns its path."""
    os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared",
               "-o", tmp, _SRC, "-lm", "-lpthread"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I = ctypes.c_int64
            lib.oracle_scan.argtypes = [I, I, I, I] + [P] * 13 + [ctypes.c_int, ctypes.c_int]
            lib.oracle_scan.restype = ctypes.c_int
            lib.oracle_scan_varlen.argtypes = [I, I, I] + [P] * 8 + [P, I] + [P] * 4 + [ctypes.c_int, ctypes.c_int]
            lib.oracle_scan_varlen.restype = ctypes.c_int
            lib.oracle_state_update.argtypes = [I, I, I, P, P, P, I] + [P] * 10 + [ctypes.c_int]
            lib.oracle_state_update.restype = ctypes.c_int
            lib.oracle_scan_bwd.argtypes = [I, I, I, I] + [P] * 20 + [ctypes.c_int, ctypes.c_int]
            lib.oracle_scan_bwd.restype = ctypes.c_int
            _lib = lib
    return _lib


def _f64(a):
    if a is None:
        return None
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def scan(u, delta, B, C, A, Dskip=None, bias=None, z=None, h0=None, nthreads: int = 1, zoh: bool = False):
    """Fixed-length batch scan.

    u, delta, z: [batch, dim, L]; B, C: [batch, N, L]; A: [dim, N]; Dskip, bias: [dim];
    h0: [batch, dim, N] or None (zero state).
    B, C may also be [batch, G, N, L]: G groups of dim/G consecutive channels, each group
    with its own B and C (channels are independent, ufo.work page §3.2, so a grouped scan is
    the scan of each group's channels with that group's B and C).
    ``zoh``: zero-order-hold input matrix instead of Bbar = Δ B.
    Returns dict with y [batch, dim, L], h_last [batch, dim, N] and the magnitudes
    y_mag, h_mag used to scale errors.
    """
    if np.ndim(B) == 4:
        G = B.shape[1]
        dim = np.shape(u)[1]
        assert dim % G == 0 and np.shape(C) == np.shape(B)
        dg = dim // G
        parts = []
        for g in range(G):
            sl = slice(g * dg, (g + 1) * dg)
            sub = lambda x, ax=1: None if x is None else np.asarray(x)[(slice(None),) * ax + (sl,)]  # noqa: E731
            parts.append(scan(sub(u), sub(delta), np.asarray(B)[:, g], np.asarray(C)[:, g], np.asarray(A)[sl],
                              sub(Dskip, 0), sub(bias, 0), sub(z), sub(h0), nthreads=nthreads, zoh=zoh))
        return {k: np.concatenate([r[k] for r in parts], axis=1) for k in parts[0]}
    u, delta, B, C, A = (_f64(x) for x in (u, delta, B, C, A))
    z, Dskip, bias, h0 = (_f64(x) for x in (z, Dskip, bias, h0))
    batch, dim, L = u.shape
    N = A.shape[1]
    assert delta.shape == u.shape and B.shape == (batch, N, L) and C.shape == B.shape
    assert A.shape == (dim, N)
    if z is not None:
        assert z.shape == u.shape
    if h0 is not None:
        assert h0.shape == (batch, dim, N)
    y = np.empty((batch, dim, L))
    y_mag = np.empty_like(y)
    h_last = np.empty((batch, dim, N))
    h_mag = np.empty_like(h_last)
    rc = _load().oracle_scan(batch, dim, N, L, _ptr(u), _ptr(delta), _ptr(z), _ptr(B), _ptr(C),
                             _ptr(A), _ptr(Dskip), _ptr(bias), _ptr(h0), _ptr(y), _ptr(h_last),
                             _ptr(y_mag), _ptr(h_mag), int(bool(zoh)), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_scan rejected its arguments (code {rc})")
    return {"y": y, "h_last": h_last, "y_mag": y_mag, "h_mag": h_mag}


def scan_varlen(u, delta, B, C, A, cu_seqlens, Dskip=None, bias=None, z=None, nthreads: int = 1,
                zoh: bool = False):
    """Packed varlen scan. u, delta, z: [dim, T]; B, C: [N, T] (or [G, N, T]: channel groups as
    in scan()); cu_seqlens: [nseq+1].

    Every sequence starts from h = 0.  Returns y [dim, T], h_last [nseq, dim, N] and magnitudes.
    """
    if np.ndim(B) == 3:
        G = B.shape[0]
        dim = np.shape(u)[0]
        assert dim % G == 0 and np.shape(C) == np.shape(B)
        dg = dim // G
        parts = []
        for g in range(G):
            sl = slice(g * dg, (g + 1) * dg)
            sub = lambda x: None if x is None else np.asarray(x)[sl]  # noqa: E731
            parts.append(scan_varlen(sub(u), sub(delta), np.asarray(B)[g], np.asarray(C)[g], np.asarray(A)[sl],
                                     cu_seqlens, sub(Dskip), sub(bias), sub(z), nthreads=nthreads, zoh=zoh))
        return {"y": np.concatenate([r["y"] for r in parts], axis=0),
                "y_mag": np.concatenate([r["y_mag"] for r in parts], axis=0),
                "h_last": np.concatenate([r["h_last"] for r in parts], axis=1),
                "h_mag": np.concatenate([r["h_mag"] for r in parts], axis=1)}
    u, delta, B, C, A = (_f64(x) for x in (u, delta, B, C, A))
    z, Dskip, bias = (_f64(x) for x in (z, Dskip, bias))
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    dim, T = u.shape
    N = A.shape[1]
    nseq = cu.shape[0] - 1
    assert B.shape == (N, T) and C.shape == (N, T) and delta.shape == u.shape
    y = np.empty((dim, T))
    y_mag = np.empty_like(y)
    h_last = np.empty((nseq, dim, N))
    h_mag = np.empty_like(h_last)
    rc = _load().oracle_scan_varlen(dim, N, T, _ptr(u), _ptr(delta), _ptr(z), _ptr(B), _ptr(C),
                                    _ptr(A), _ptr(Dskip), _ptr(bias), _ptr(cu), nseq, _ptr(y),
                                    _ptr(h_last), _ptr(y_mag), _ptr(h_mag), int(bool(zoh)), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_scan_varlen rejected its arguments (code {rc})")
    return {"y": y, "h_last": h_last, "y_mag": y_mag, "h_mag": h_mag}


def scan_varlen_pool(u, delta, B, C, A, cu_seqlens, pool, slot_ids, Dskip=None, bias=None, z=None,
                     pool_mag=None, nthreads: int = 1, zoh: bool = False):
    """Packed prefill into a state pool, in place on ``pool`` (float64 [S, dim, N]).

    The serving flow of the ufo.work page's second article, §4.2 (a prompt is prefilled in
    chunks into the per-request state of the §4.1 pool): sequence i of the packed batch is the
    fixed-length scan of its columns started from pool[slot_ids[i]], and its final state
    replaces pool[slot_ids[i]].  An id outside [0, S) starts from zero and writes nothing back.
    ``pool_mag`` (same shape, optional) carries the magnitude bound of the pool entries and is
    updated alongside.  Returns y [dim, T] and y_mag.
    """
    u, delta, B, C, A = (_f64(x) for x in (u, delta, B, C, A))
    z, Dskip, bias = (_f64(x) for x in (z, Dskip, bias))
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    dim, T = u.shape
    N = A.shape[1]
    S = pool.shape[0]
    assert pool.shape == (S, dim, N) and pool.dtype == np.float64
    y = np.zeros((dim, T))
    y_mag = np.zeros_like(y)
    for i in range(cu.shape[0] - 1):
        lo, hi, slot = int(cu[i]), int(cu[i + 1]), int(slot_ids[i])
        if hi == lo:
            continue
        ok = 0 <= slot < S
        h0 = pool[slot][None] if ok else np.zeros((1, dim, N))
        col = slice(lo, hi)
        r = scan(u[None, :, col], delta[None, :, col], B[None, :, col], C[None, :, col], A, Dskip, bias,
                 None if z is None else z[None, :, col], h0, nthreads=nthreads, zoh=zoh)
        y[:, col] = r["y"][0]
        y_mag[:, col] = r["y_mag"][0]
        if pool_mag is not None and ok:
            # scan() starts its magnitude recursion from |h0|; the recursion is linear in its
            # start, so the bound from pool_mag adds the decayed excess pool_mag - |h0| (>= 0),
            # run as a scan with no input (u = 0, B = 0)
            excess = np.maximum(pool_mag[slot] - np.abs(pool[slot]), 0.0)[None]
            r_ex = scan(np.zeros((1, dim, hi - lo)), delta[None, :, col], np.zeros((1, N, hi - lo)),
                        C[None, :, col], A, None, bias, None if z is None else z[None, :, col], excess,
                        nthreads=nthreads, zoh=zoh)
            y_mag[:, col] += r_ex["y_mag"][0]
            pool_mag[slot] = r["h_mag"][0] + r_ex["h_mag"][0]
        if ok:
            pool[slot] = r["h_last"][0]
    return {"y": y, "y_mag": y_mag}


def state_update(pool, slot_ids, u, delta, B, C, A, Dskip=None, bias=None, z=None, pool_mag=None,
                 zoh: bool = False):
    """One decode step, in place on ``pool`` (float64 array [S, dim, N]).

    slot_ids: [R]; u, delta, z: [R, dim]; B, C: [R, N].  ``pool_mag`` (same shape as pool, or
    None) carries the magnitude recursion across steps.  Returns dict with y [R, dim], y_mag.
    """
    assert pool.dtype == np.float64 and pool.flags.c_contiguous
    if pool_mag is not None:
        assert pool_mag.dtype == np.float64 and pool_mag.flags.c_contiguous and pool_mag.shape == pool.shape
    u, delta, B, C, A = (_f64(x) for x in (u, delta, B, C, A))
    z, Dskip, bias = (_f64(x) for x in (z, Dskip, bias))
    ids = np.ascontiguousarray(np.asarray(slot_ids, dtype=np.int64))
    S, dim, N = pool.shape
    R = ids.shape[0]
    assert u.shape == (R, dim) and B.shape == (R, N)
    y = np.empty((R, dim))
    y_mag = np.empty_like(y)
    rc = _load().oracle_state_update(S, dim, N, _ptr(pool), _ptr(pool_mag), _ptr(ids), R, _ptr(u),
                                     _ptr(delta), _ptr(z), _ptr(B), _ptr(C), _ptr(A), _ptr(Dskip),
                                     _ptr(bias), _ptr(y), _ptr(y_mag), int(bool(zoh)))
    if rc != 0:
        raise ValueError(f"oracle_state_update rejected its arguments (code {rc})")
    return {"y": y, "y_mag": y_mag}


def scan_bwd(u, delta, B, C, A, dy, Dskip=None, bias=None, z=None, h0=None, dh_last=None, nthreads: int = 1,
             zoh: bool = False):
    """Gradients of the fixed-length batch scan (the reverse-mode derivative of ``scan``).

    Given dy = dL/dy [batch, dim, L] and optionally dh_last = dL/dh_last [batch, dim, N],
    returns du, ddelta, dz (None without z) [batch, dim, L]; dB, dC [batch, N, L];
    dA [dim, N]; dDskip, dbias [dim]; dh0 [batch, dim, N] (the gradient for the initial state,
    whether or not one is given).  The ufo.work page, §2.2, describes how training keeps or
    recomputes the states for this pass; the values are fixed by the forward definition.
    """
    u, delta, B, C, A, dy = (_f64(x) for x in (u, delta, B, C, A, dy))
    z, Dskip, bias, h0, dh_last = (_f64(x) for x in (z, Dskip, bias, h0, dh_last))
    batch, dim, L = u.shape
    N = A.shape[1]
    assert delta.shape == u.shape and dy.shape == u.shape and B.shape == (batch, N, L) and C.shape == B.shape
    assert A.shape == (dim, N)
    for x, shape in ((z, u.shape), (h0, (batch, dim, N)), (dh_last, (batch, dim, N))):
        assert x is None or x.shape == shape
    out = {"du": np.empty_like(u), "ddelta": np.empty_like(u), "dz": np.empty_like(u) if z is not None else None,
           "dB": np.empty_like(B), "dC": np.empty_like(C), "dA": np.empty_like(A),
           "dDskip": np.empty(dim), "dbias": np.empty(dim), "dh0": np.empty((batch, dim, N))}
    rc = _load().oracle_scan_bwd(batch, dim, N, L, _ptr(u), _ptr(delta), _ptr(z), _ptr(B), _ptr(C), _ptr(A),
                                 _ptr(Dskip), _ptr(bias), _ptr(h0), _ptr(dy), _ptr(dh_last),
                                 _ptr(out["du"]), _ptr(out["ddelta"]), _ptr(out["dz"]), _ptr(out["dB"]),
                                 _ptr(out["dC"]), _ptr(out["dA"]), _ptr(out["dDskip"]), _ptr(out["dbias"]),
                                 _ptr(out["dh0"]), int(bool(zoh)), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_scan_bwd rejected its arguments (code {rc})")
    return out


def scaled_error(x, ref, mag) -> float:
    """max_i |x_i - ref_i| / mag_i, where mag is the oracle's magnitude bound (|ref| <= mag).

    Non-finite values in x give +inf.  Where mag == 0 the reference is exactly zero and any
    nonzero x counts as an infinite error.
    """
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    mag = np.asarray(mag, dtype=np.float64)
    if not np.all(np.isfinite(x)):
        return float("inf")
    diff = np.abs(x - ref)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.where(mag > 0, diff / np.where(mag > 0, mag, 1.0), np.where(diff > 0, np.inf, 0.0))
    return float(r.max()) if r.size else 0.0
