"""Seeded synthetic inputs for the selective-scan workloads.

This module only draws random numbers and rounds them to the storage dtype; it holds none of
the scan's arithmetic.  It is the one piece shared by the CUDA-side tests/bench and the fp64
oracle, so both see bit-identical inputs.

Recipe (the same for every workload): u, δ, z, B, C ~ N(0, 1) drawn in float32 and then
rounded to the storage dtype (bf16 with round-to-nearest-even where the workload is bf16);
A[d, n] = -(n + 1); D[d] = 1; a per-channel step size dt is drawn log-uniformly in
[1e-3, 1e-1] and bias[d] = log(expm1(dt)) so that softplus(bias) = dt (the Δ initialisation
range of discosf.com "企业官网建设流程全解析" §1.2).  A, D and bias are float32.
B and C are shared by all channels of a sequence ([batch, N, L] / [N, T]).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

# name -> shape/dtype/seed.  Sizes follow the five workloads the scan is specified on.
CONFIGS = {
    "tiny_f32": dict(kind="batch", batch=1, dim=16, dstate=16, seqlen=256, dtype="f32", seed=0),
    "batch_f32": dict(kind="batch", batch=2, dim=1536, dstate=16, seqlen=2048, dtype="f32", seed=1),
    "varlen_bf16": dict(kind="varlen", nseq=16, len_lo=256, len_hi=4096, dim=2048, dstate=16,
                        dtype="bf16", seed=2),
    "long_bf16": dict(kind="batch", batch=1, dim=2560, dstate=16, seqlen=131072, dtype="bf16", seed=3),
    "long_n128_bf16": dict(kind="batch", batch=1, dim=1024, dstate=128, seqlen=32768, dtype="bf16",
                           seed=3),
    "decode_bf16": dict(kind="decode", num_slots=1024, dim=5120, dstate=16, R=256, steps=1000,
                        dtype="bf16", seed=4),
}


def round_to_bf16(x) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returned as float32."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) & np.uint32(0xFFFF0000)
    return r.view(np.float32)


def _store(x: np.ndarray, dtype: str) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    return round_to_bf16(x) if dtype == "bf16" else x


def _normal(rng, shape, dtype):
    return _store(rng.standard_normal(shape, dtype=np.float32), dtype)


def channel_params(rng, dim: int, dstate: int):
    """A[d,n] = -(n+1), D = 1, bias = log(expm1(dt)) with dt log-uniform in [1e-3, 1e-1]."""
    A = np.ascontiguousarray(np.broadcast_to(-(np.arange(dstate, dtype=np.float32) + 1.0), (dim, dstate)))
    Dskip = np.ones(dim, dtype=np.float32)
    dt = np.exp(rng.uniform(np.log(1e-3), np.log(1e-1), size=dim))
    bias = np.log(np.expm1(dt)).astype(np.float32)
    return A, Dskip, bias


@dataclass
class ScanInputs:
    """Host arrays (float32 holding exact storage-dtype values) for one scan problem."""
    dtype: str
    u: np.ndarray
    delta: np.ndarray
    z: np.ndarray | None
    B: np.ndarray
    C: np.ndarray
    A: np.ndarray
    Dskip: np.ndarray | None
    bias: np.ndarray | None
    h0: np.ndarray | None = None
    cu_seqlens: np.ndarray | None = None      # varlen only, int32 [nseq+1]
    meta: dict = field(default_factory=dict)


def batch_inputs(batch, dim, dstate, seqlen, dtype="f32", seed=0, gate=True, h0=False) -> ScanInputs:
    """Fixed-length batch: u, δ, z [batch, dim, L]; B, C [batch, N, L]."""
    rng = np.random.default_rng(seed)
    u = _normal(rng, (batch, dim, seqlen), dtype)
    delta = _normal(rng, (batch, dim, seqlen), dtype)
    z = _normal(rng, (batch, dim, seqlen), dtype)
    B = _normal(rng, (batch, dstate, seqlen), dtype)
    C = _normal(rng, (batch, dstate, seqlen), dtype)
    A, Dskip, bias = channel_params(rng, dim, dstate)
    h = rng.standard_normal((batch, dim, dstate), dtype=np.float32) if h0 else None
    return ScanInputs(dtype, u, delta, z if gate else None, B, C, A, Dskip, bias, h0=h,
                      meta=dict(kind="batch", batch=batch, dim=dim, dstate=dstate, seqlen=seqlen, seed=seed))


def varlen_lengths(nseq, len_lo, len_hi, seed) -> np.ndarray:
    rng = np.random.default_rng([seed, 7])
    return rng.integers(len_lo, len_hi + 1, size=nseq).astype(np.int64)


def varlen_inputs(lengths, dim, dstate, dtype="bf16", seed=2, gate=True) -> ScanInputs:
    """Packed varlen: u, δ, z [dim, T]; B, C [N, T]; cu_seqlens int32 [nseq+1]."""
    lengths = np.asarray(lengths, dtype=np.int64)
    cu = np.zeros(len(lengths) + 1, dtype=np.int64)
    cu[1:] = np.cumsum(lengths)
    T = int(cu[-1])
    rng = np.random.default_rng(seed)
    u = _normal(rng, (dim, T), dtype)
    delta = _normal(rng, (dim, T), dtype)
    z = _normal(rng, (dim, T), dtype)
    B = _normal(rng, (dstate, T), dtype)
    C = _normal(rng, (dstate, T), dtype)
    A, Dskip, bias = channel_params(rng, dim, dstate)
    return ScanInputs(dtype, u, delta, z if gate else None, B, C, A, Dskip, bias,
                      cu_seqlens=cu.astype(np.int32),
                      meta=dict(kind="varlen", nseq=len(lengths), dim=dim, dstate=dstate, total=T, seed=seed))


@dataclass
class DecodeProblem:
    dtype: str
    pool0: np.ndarray         # float32 [S, dim, N]
    slot_ids: np.ndarray      # int32 [R], distinct
    A: np.ndarray
    Dskip: np.ndarray
    bias: np.ndarray
    seed: int
    R: int
    dim: int
    dstate: int


def decode_problem(num_slots, dim, dstate, R, dtype="bf16", seed=4) -> DecodeProblem:
    rng = np.random.default_rng([seed, 1_000_000])
    pool0 = rng.standard_normal((num_slots, dim, dstate), dtype=np.float32)
    slots = np.random.default_rng([seed, 1_000_001]).choice(num_slots, size=R, replace=False).astype(np.int32)
    A, Dskip, bias = channel_params(np.random.default_rng([seed, 1_000_002]), dim, dstate)
    return DecodeProblem(dtype, pool0, slots, A, Dskip, bias, seed, R, dim, dstate)


def decode_step_inputs(prob: DecodeProblem, step: int, channels=None):
    """Fresh per-step token inputs: u, δ, z [R, dim]; B, C [R, N]; seeded by (seed, step).

    ``channels`` (optional index array) returns only those columns of u, δ, z -- the draws are
    the same as for the full width, so a channel subset is an exact slice.
    """
    rng = np.random.default_rng([prob.seed, step])
    u = _normal(rng, (prob.R, prob.dim), prob.dtype)
    delta = _normal(rng, (prob.R, prob.dim), prob.dtype)
    z = _normal(rng, (prob.R, prob.dim), prob.dtype)
    B = _normal(rng, (prob.R, prob.dstate), prob.dtype)
    C = _normal(rng, (prob.R, prob.dstate), prob.dtype)
    if channels is not None:
        u, delta, z = u[:, channels], delta[:, channels], z[:, channels]
    return dict(u=u, delta=delta, z=z, B=B, C=C)


def config_inputs(name: str):
    """Inputs for a named workload (decode returns a DecodeProblem)."""
    c = CONFIGS[name]
    if c["kind"] == "batch":
        return batch_inputs(c["batch"], c["dim"], c["dstate"], c["seqlen"], c["dtype"], c["seed"])
    if c["kind"] == "varlen":
        lens = varlen_lengths(c["nseq"], c["len_lo"], c["len_hi"], c["seed"])
        return varlen_inputs(lens, c["dim"], c["dstate"], c["dtype"], c["seed"])
    return decode_problem(c["num_slots"], c["dim"], c["dstate"], c["R"], c["dtype"], c["seed"])


@dataclass
class SsdInputs:
    """Host arrays for one SSD (scalar-A-per-head) problem: x [b, H, P, L] and B, C [b, N, L]
    bf16-exact float32; dt [b, H, L] > 0, A [H] < 0 and h0 [b, H, P, N] float32."""
    x: np.ndarray
    dt: np.ndarray
    A: np.ndarray
    B: np.ndarray
    C: np.ndarray
    h0: np.ndarray | None
    meta: dict = field(default_factory=dict)


def ssd_inputs(batch, nheads, headdim, dstate, seqlen, seed=5, h0=False) -> SsdInputs:
    """x, B, C ~ N(0, 1) rounded to bf16; dt log-uniform in [1e-3, 1e-1] per (sequence, head,
    step); A[h] = -exp(U[log 0.5, log 16]) per head (slow and fast decays); h0 ~ N(0, 1) when
    asked for."""
    rng = np.random.default_rng([seed, 55])
    x = _normal(rng, (batch, nheads, headdim, seqlen), "bf16")
    B = _normal(rng, (batch, dstate, seqlen), "bf16")
    C = _normal(rng, (batch, dstate, seqlen), "bf16")
    dt = np.exp(rng.uniform(np.log(1e-3), np.log(1e-1), size=(batch, nheads, seqlen))).astype(np.float32)
    A = (-np.exp(rng.uniform(np.log(0.5), np.log(16.0), size=nheads))).astype(np.float32)
    hz = rng.standard_normal((batch, nheads, headdim, dstate), dtype=np.float32) if h0 else None
    return SsdInputs(x, dt, A, B, C, hz, meta=dict(batch=batch, nheads=nheads, headdim=headdim, dstate=dstate,
                                                   seqlen=seqlen, seed=seed))
