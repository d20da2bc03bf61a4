"""Chunk-checkpointed backward of the scan -- TEST INFRASTRUCTURE ONLY.

Only ``tests/`` use this module; the CUDA library never does.  It is the training-side
schedule the pages describe for the backward pass, written as plainly as possible so that a
kernel following it can be checked step by step: the ufo.work page, §2.2 (strategy B:
checkpoints plus recomputation), and its second article, §3.1 (chunk-level checkpoints: keep
only the state at every chunk boundary, and recompute the inside of a chunk from its boundary
during the backward pass).

    forward:  run the scan, keeping only H[c] = the state entering chunk c
    backward: for c = last .. first:
                recompute h_t for t in chunk c from H[c]
                run the reverse recurrence dh_t = C_t dyraw_t + a_{t+1} dh_{t+1} inside the
                chunk, starting from the dh handed back by chunk c+1, and accumulate the
                gradients of every input from (h_{t-1}, dh_t)
                hand dh (now the gradient of the state entering chunk c) to chunk c-1

It must equal ``oracle.scan_bwd`` (the unchunked reverse-mode derivative) for every chunk
size.  fp64 numpy, vectorised over the states only.
"""
from __future__ import annotations

import numpy as np


def _softplus(x):
    return np.logaddexp(0.0, x)


def _coef(dt, A, zoh):
    """Input coefficient per state (and its partial derivatives in Delta and A)."""
    if not zoh:
        return np.full_like(A, dt), np.ones_like(A), np.zeros_like(A)
    x = dt * A
    small = np.abs(x) < 1e-2
    xs = np.where(small, 1.0, x)
    c = np.where(x == 0.0, dt, np.expm1(xs) / xs * dt)
    series = sum(k * x ** (k - 1) / np.prod(np.arange(1, k + 2, dtype=np.float64)) for k in range(1, 9))
    dphi = np.where(small, series, (xs * np.exp(xs) - np.expm1(xs)) / (xs * xs))
    return c, np.exp(x), dt * dt * dphi


def scan_bwd_chunked(u, delta, B, C, A, dy, Dskip=None, bias=None, z=None, h0=None, dh_last=None, chunk=64,
                     zoh=False):
    """Same arguments and results as ``oracle.scan_bwd``; ``chunk`` is the checkpoint spacing."""
    u, delta, B, C, A, dy = (np.asarray(v, dtype=np.float64) for v in (u, delta, B, C, A, dy))
    b, D, L = u.shape
    N = A.shape[1]
    Dk = np.zeros(D) if Dskip is None else np.asarray(Dskip, dtype=np.float64)
    bi = np.zeros(D) if bias is None else np.asarray(bias, dtype=np.float64)
    out = {"du": np.zeros_like(u), "ddelta": np.zeros_like(u), "dz": None if z is None else np.zeros_like(u),
           "dB": np.zeros_like(B), "dC": np.zeros_like(C), "dA": np.zeros_like(A), "dDskip": np.zeros(D),
           "dbias": np.zeros(D), "dh0": np.zeros((b, D, N))}
    starts = list(range(0, L, chunk))
    for bb in range(b):
        for d in range(D):
            Ad = A[d]
            dt = _softplus(delta[bb, d] + bi[d])
            # forward: only the chunk-boundary states are kept
            h = np.zeros(N) if h0 is None else np.asarray(h0, dtype=np.float64)[bb, d].copy()
            bound = []
            for c0 in starts:
                bound.append(h.copy())
                for t in range(c0, min(c0 + chunk, L)):
                    h = np.exp(dt[t] * Ad) * h + _coef(dt[t], Ad, zoh)[0] * B[bb, :, t] * u[bb, d, t]
            # backward, chunk by chunk from the end
            dh = np.zeros(N) if dh_last is None else np.asarray(dh_last, dtype=np.float64)[bb, d].copy()
            for ci in range(len(starts) - 1, -1, -1):
                c0, c1 = starts[ci], min(starts[ci] + chunk, L)
                hs = [bound[ci]]                                  # hs[k] = state before step c0 + k
                for t in range(c0, c1):
                    hs.append(np.exp(dt[t] * Ad) * hs[-1] + _coef(dt[t], Ad, zoh)[0] * B[bb, :, t] * u[bb, d, t])
                for t in range(c1 - 1, c0 - 1, -1):
                    k = t - c0
                    ht, hp = hs[k + 1], hs[k]
                    yraw = C[bb, :, t] @ ht + Dk[d] * u[bb, d, t]
                    dyraw = dy[bb, d, t]
                    if z is not None:
                        zz = z[bb, d, t]
                        sg = 1.0 / (1.0 + np.exp(-zz))
                        out["dz"][bb, d, t] = dyraw * yraw * sg * (1.0 + zz * (1.0 - sg))
                        dyraw *= zz * sg
                    out["dDskip"][d] += dyraw * u[bb, d, t]
                    dh = dh + dyraw * C[bb, :, t]
                    out["dC"][bb, :, t] += dyraw * ht
                    a = np.exp(dt[t] * Ad)
                    c, dc_ddt, dc_da = _coef(dt[t], Ad, zoh)
                    out["dB"][bb, :, t] += dh * c * u[bb, d, t]
                    out["du"][bb, d, t] = dyraw * Dk[d] + np.sum(dh * c * B[bb, :, t])
                    da = dh * hp
                    dcoef = dh * B[bb, :, t] * u[bb, d, t]
                    ddt = np.sum(da * a * Ad + dcoef * dc_ddt)
                    out["dA"][d] += da * a * dt[t] + dcoef * dc_da
                    dd = ddt / (1.0 + np.exp(-(delta[bb, d, t] + bi[d])))
                    out["ddelta"][bb, d, t] = dd
                    out["dbias"][d] += dd
                    dh = dh * a
            out["dh0"][bb, d] = dh
    return out
