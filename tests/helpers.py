"""Shared test helpers: device upload of workload arrays and oracle comparison."""
from __future__ import annotations

import numpy as np

import oracle

TOL = {"f32": 1e-4, "bf16": 3e-3}   # max error scaled by the oracle magnitude bound

# A bf16 output is rounded to nearest once, at the store.  bf16 carries an 8-bit significand,
# so that rounding alone moves a value by up to 2^-8 (3.9e-3) of itself -- more than the 3e-3
# gate.  The gate therefore bounds the arithmetic error, and a bf16 *output* is allowed its
# own half-ulp on top: |y - ref| <= tol*mag + 2^-8 (|ref| + tol*mag).  float32 outputs
# (including bf16 inputs with float32 y) get no allowance.
BF16_UNIT_ROUNDOFF = 2.0 ** -8


def torch_dtype(name):
    import torch
    return torch.bfloat16 if name == "bf16" else torch.float32


def dev(x, dtype="f32", device="cuda", pitch=None):
    """Upload a float32 numpy array (bf16-exact values when dtype == 'bf16').

    ``pitch`` pads the last axis to that many elements (the padding holds NaN so that any
    read of it would show up in the outputs)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    if pitch is not None and pitch != x.shape[-1]:
        pad = torch.full(x.shape[:-1] + (pitch,), float("nan"), dtype=torch.float32)
        pad[..., : x.shape[-1]] = t
        t = pad
    return t.to(device=device, dtype=torch_dtype(dtype))


def host(t, width=None):
    """Device tensor -> float64 numpy (optionally cut to `width` columns)."""
    if width is not None:
        t = t[..., :width]
    return t.float().cpu().numpy().astype(np.float64)


def scaled_error(x, ref, mag, tol=0.0, rounding=0.0):
    """oracle.scaled_error after removing an output-rounding allowance rounding*(|ref|+tol*mag)."""
    if rounding == 0.0:
        return oracle.scaled_error(x, ref, mag)
    x = np.asarray(x, dtype=np.float64)
    if not np.all(np.isfinite(x)):
        return float("inf")
    ref = np.asarray(ref, dtype=np.float64)
    mag = np.asarray(mag, dtype=np.float64)
    diff = np.maximum(np.abs(x - ref) - rounding * (np.abs(ref) + tol * mag), 0.0)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.where(mag > 0, diff / np.where(mag > 0, mag, 1.0), np.where(diff > 0, np.inf, 0.0))
    return float(r.max()) if r.size else 0.0


def check(name, x, ref, mag, tol, out_dtype="f32"):
    """Assert the scaled error is within tol; a bf16 output gets its half-ulp allowance."""
    rounding = BF16_UNIT_ROUNDOFF if out_dtype == "bf16" else 0.0
    err = scaled_error(x, ref, mag, tol, rounding)
    assert err <= tol, f"{name}: scaled error {err:.3e} > {tol:.1e}"
    return err


def round_up(x, m):
    return (x + m - 1) // m * m
