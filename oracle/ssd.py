"""Chunked SSD (state-space duality) form of the scan, scalar A per head -- TEST INFRASTRUCTURE ONLY.

Only ``tests/`` use this module; the CUDA library never does.  It is a second statement of
the scan for the case the ufo.work page's second article ("Mamba-2/SSD架构下的矩阵化加速范式…")
works with: a scalar decay A_h per head and a step Δ_h,t shared by the head's P channels.
§1.1 of that article writes the scan as masked attention, Y = (mask ∘ (Q Kᵀ)) V, with
Q = C, K = B and V = Δ x; §2.2 gives the masked score with its input-dependent decay,
S_ts = C_t · B_s · exp(A Σ_{k=s+1..t} Δ_k) for s ≤ t (0 above the diagonal), computed from a
prefix sum of ΔA.  Over a long sequence the product is taken chunk by chunk, with the state
H [P, N] carried between chunks (the chunk-boundary states of its §3.1 checkpointing):

    cum_t   = Σ_{k=c0..t} Δ_k A                          (prefix sum inside the chunk)
    Y[:, t] = Σ_{s=c0..t} S_ts V[:, s] + exp(cum_t) H_in C_t
    H_out   = exp(cum_last) H_in + Σ_s exp(cum_last - cum_s) V[:, s] B_sᵀ

No skip term or gate: those act elementwise on y exactly as in the scan.  fp64, numpy
matrix products, no reassociation beyond the chunking above.
"""
from __future__ import annotations

import numpy as np


def ssd_chunked(x, dt, A, B, C, chunk, h0=None):
    """x: [H, P, L] (head h, channel p of the head, step t); dt: [H, L] (Δ, already positive);
    A: [H] (scalar decay per head); B, C: [N, L] shared by all heads; h0: [H, P, N] or None.

    Returns (y [H, P, L], h_last [H, P, N])."""
    x, dt, A, B, C = (np.asarray(v, dtype=np.float64) for v in (x, dt, A, B, C))
    H, P, L = x.shape
    N = B.shape[0]
    assert dt.shape == (H, L) and A.shape == (H,) and B.shape == (N, L) and C.shape == (N, L) and chunk >= 1
    y = np.zeros((H, P, L))
    state = np.zeros((H, P, N)) if h0 is None else np.array(h0, dtype=np.float64)
    for h in range(H):
        Hs = state[h]
        for c0 in range(0, L, chunk):
            sl = slice(c0, min(c0 + chunk, L))
            d = dt[h, sl]
            cum = np.cumsum(d * A[h])                              # [T]
            V = x[h][:, sl] * d[None, :]                           # [P, T]
            T = d.shape[0]
            lower = np.tril(np.ones((T, T), dtype=bool))
            with np.errstate(over="ignore"):
                decay = np.where(lower, np.exp(np.where(lower, cum[:, None] - cum[None, :], 0.0)), 0.0)
            S = (C[:, sl].T @ B[:, sl]) * decay                    # [T, T]: S[t, s]
            y[h][:, sl] = V @ S.T + (Hs @ C[:, sl]) * np.exp(cum)[None, :]
            Hs = np.exp(cum[-1]) * Hs + (V * np.exp(cum[-1] - cum)[None, :]) @ B[:, sl].T
        state[h] = Hs
    return y, state
