"""Closed-form brute force of the selective scan in 50-digit decimal -- TEST INFRASTRUCTURE ONLY.

This is a second, independent statement of the same mathematics, used to pin the fp64 oracle.
Instead of stepping the recurrence it unrolls it (ufo.work "…状态空间模型加速" §1.1 gives the
recurrence; the kj168168.com page "突破算力边界…" §三.2 writes the unrolled sum of decayed inputs):

    h_t[n] = (prod_{s=0..t} abar_s[n]) h0[n] + sum_{k=0..t} (prod_{s=k+1..t} abar_s[n]) Δ_k B_k[n] u_k
    y_t    = g(z_t) (sum_n C_t[n] h_t[n] + D u_t)

with abar_s[n] = exp(Δ_s A[n]), Δ_s = ln(1 + e^(δ_s + bias)) and g(z) = z / (1 + e^-z).
Every product is formed afresh for each (t, k): O(L^2 N) decimal operations, so use it only on
tiny inputs (L <= ~16).
"""
from __future__ import annotations

from decimal import Decimal, getcontext

import numpy as np

getcontext().prec = 50


def _D(x) -> Decimal:
    return Decimal(float(x))  # exact conversion of the binary64 value


def _softplus(x: Decimal) -> Decimal:
    return (Decimal(1) + x.exp()).ln()


def _silu(z: Decimal) -> Decimal:
    return z / (Decimal(1) + (-z).exp())


def scan_channel(u, delta, B, C, A_row, dskip=0.0, bias=0.0, z=None, h0=None):
    """One channel. u, delta, z: [L]; B, C: [N, L]; A_row: [N]; h0: [N] or None.

    Returns (y [L], h_last [N]) as float64 arrays rounded from the decimal results.
    """
    L = len(u)
    N = len(A_row)
    dt = [_softplus(_D(delta[t]) + _D(bias)) for t in range(L)]
    abar = [[(dt[t] * _D(A_row[n])).exp() for t in range(L)] for n in range(N)]
    bx = [[dt[t] * _D(B[n][t]) * _D(u[t]) for t in range(L)] for n in range(N)]
    y = np.empty(L)
    h_last = np.empty(N)
    for t in range(L):
        acc = Decimal(0)
        for n in range(N):
            hn = Decimal(0)
            for k in range(t + 1):
                p = Decimal(1)
                for s in range(k + 1, t + 1):
                    p *= abar[n][s]
                hn += p * bx[n][k]
            if h0 is not None:
                p = Decimal(1)
                for s in range(t + 1):
                    p *= abar[n][s]
                hn += p * _D(h0[n])
            acc += _D(C[n][t]) * hn
            if t == L - 1:
                h_last[n] = float(hn)
        yt = acc + _D(dskip) * _D(u[t])
        if z is not None:
            yt *= _silu(_D(z[t]))
        y[t] = float(yt)
    return y, h_last


def scan(u, delta, B, C, A, Dskip=None, bias=None, z=None, h0=None):
    """Batch form with the oracle's layouts: u [b, D, L]; B, C [b, N, L]; A [D, N]."""
    u = np.asarray(u, dtype=np.float64)
    bsz, dim, L = u.shape
    N = A.shape[1]
    y = np.empty((bsz, dim, L))
    h = np.empty((bsz, dim, N))
    for b in range(bsz):
        for d in range(dim):
            y[b, d], h[b, d] = scan_channel(
                u[b, d], delta[b, d], B[b], C[b], A[d],
                0.0 if Dskip is None else Dskip[d], 0.0 if bias is None else bias[d],
                None if z is None else z[b, d], None if h0 is None else h0[b, d])
    return y, h
