"""GPU parity of the lane-sequential scan kernel (algorithm = 'sequential') against the fp64 oracle.

Same error metric and gates as test_scan_gpu.py: max |x - x_oracle| / m with m the oracle's
magnitude bound, 1e-4 for float32 inputs and 3e-3 for bf16 inputs (bf16 outputs get their
half-ulp allowance).  The shapes cover several 64/32-channel tiles with a ragged tail tile,
sequences that are not a multiple of the chunk, length 0 and 1, packed sequences starting
mid-vector, more than 64 packed sequences (no length ranking), initial states, the pool
prefill, channel groups and the float32-output option.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle  # noqa: E402
import selective_state_space_15_b200 as ssm  # noqa: E402
import workloads  # noqa: E402
from helpers import TOL, check, dev, host, round_up  # noqa: E402

NTHREADS = oracle.default_threads()
SEQ = "sequential"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ssm.load()


def _batch(inp, dtype, h0=None, gate=True, y_dtype=None, algorithm=SEQ):
    """Rows padded to a 16-byte pitch (NaN in the padding) when L is not a multiple of 8: the
    sequential kernel takes 16-byte aligned rows only."""
    L = inp.u.shape[-1]
    pitch = round_up(L, 8)
    u, dl = dev(inp.u, dtype, pitch=pitch)[..., :L], dev(inp.delta, dtype, pitch=pitch)[..., :L]
    z = dev(inp.z, dtype, pitch=pitch)[..., :L] if gate else None
    B, C = dev(inp.B, dtype, pitch=pitch)[..., :L], dev(inp.C, dtype, pitch=pitch)[..., :L]
    A, D, bias = (torch.from_numpy(x).cuda() for x in (inp.A, inp.Dskip, inp.bias))
    h0t = torch.from_numpy(h0).cuda() if h0 is not None else None
    y = torch.empty(u.shape[:-1] + (pitch,), device="cuda", dtype=y_dtype or u.dtype)[..., :L]
    y, hl = ssm.scan_fwd(u, dl, B, C, A, D, bias, z, h0t, y=y, algorithm=algorithm)
    torch.cuda.synchronize()
    return host(y), host(hl)


def _varlen(inp, dtype, h0=None, y_dtype=None, algorithm=SEQ):
    T = inp.meta["total"]
    pitch = round_up(T, 8)
    u, dl, z, B, C = (dev(x, dtype, pitch=pitch) for x in (inp.u, inp.delta, inp.z, inp.B, inp.C))
    A, D, bias = (torch.from_numpy(x).cuda() for x in (inp.A, inp.Dskip, inp.bias))
    cu = torch.from_numpy(inp.cu_seqlens).cuda()
    h0t = torch.from_numpy(h0).cuda() if h0 is not None else None
    y, hl = ssm.scan_fwd_varlen(u, dl, B, C, A, cu, D, bias, z, h0t, total=T, y_dtype=y_dtype, algorithm=algorithm)
    torch.cuda.synchronize()
    return host(y, T), host(hl)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [
    (1, 16, 16, 256),     # one tile, part-filled
    (2, 200, 16, 1000),   # 4 tiles of 64 channels, the last ragged; L not a multiple of the chunk
    (3, 70, 16, 1),       # single step
    (1, 8, 16, 37),       # one partial chunk
    (2, 72, 32, 515),     # dstate 32 (32-channel tiles)
    (1, 33, 32, 64),
])
def test_batch_full(shape, dtype):
    b, D, N, L = shape
    inp = workloads.batch_inputs(b, D, N, L, dtype, seed=400 + L + D)
    y, hl = _batch(inp, dtype)
    ref = oracle.scan(inp.u, inp.delta, inp.B, inp.C, inp.A, inp.Dskip, inp.bias, inp.z, nthreads=NTHREADS)
    check("y", y, ref["y"], ref["y_mag"], TOL[dtype], dtype)
    check("h_last", hl, ref["h_last"], ref["h_mag"], TOL[dtype])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_batch_initial_state_no_gate(dtype):
    inp = workloads.batch_inputs(2, 80, 16, 600, dtype, seed=7, gate=False, h0=True)
    y, hl = _batch(inp, dtype, h0=inp.h0, gate=False)
    ref = oracle.scan(inp.u, inp.delta, inp.B, inp.C, inp.A, inp.Dskip, inp.bias, None, inp.h0, nthreads=NTHREADS)
    check("y", y, ref["y"], ref["y_mag"], TOL[dtype], dtype)
    check("h_last", hl, ref["h_last"], ref["h_mag"], TOL[dtype])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N,lengths", [
    (16, [5, 1, 17, 0, 300, 9, 64, 1000]),   # empty and length-1 sequences, unaligned starts
    (16, [4096, 256, 1024, 33]),
    (32, [100, 0, 37, 300, 1]),
])
def test_varlen_full(N, lengths, dtype):
    D = 96
    inp = workloads.varlen_inputs(lengths, D, N, dtype, seed=500 + len(lengths) + N)
    y, hl = _varlen(inp, dtype)
    ref = oracle.scan_varlen(inp.u, inp.delta, inp.B, inp.C, inp.A, inp.cu_seqlens, inp.Dskip, inp.bias, inp.z,
                             nthreads=NTHREADS)
    check("y", y, ref["y"], ref["y_mag"], TOL[dtype], dtype)
    check("h_last", hl, ref["h_last"], ref["h_mag"], TOL[dtype])


def test_varlen_many_sequences_unranked():
    """More packed sequences than the kernel ranks by length (64): units in sequence order."""
    rng = np.random.default_rng(79)
    lengths = [int(x) for x in rng.integers(0, 60, size=150)]
    lengths[3], lengths[100] = 0, 200
    inp = workloads.varlen_inputs(lengths, 40, 16, "bf16", seed=80)
    y, hl = _varlen(inp, "bf16")
    ref = oracle.scan_varlen(inp.u, inp.delta, inp.B, inp.C, inp.A, inp.cu_seqlens, inp.Dskip, inp.bias, inp.z,
                             nthreads=NTHREADS)
    check("y", y, ref["y"], ref["y_mag"], TOL["bf16"], "bf16")
    check("h_last", hl, ref["h_last"], ref["h_mag"], TOL["bf16"])


def test_varlen_initial_states_float32_output():
    lengths = [100, 0, 37, 400]
    D, N = 70, 16
    inp = workloads.varlen_inputs(lengths, D, N, "bf16", seed=3)
    h0 = np.random.default_rng(1).standard_normal((len(lengths), D, N)).astype(np.float32)
    y, hl = _varlen(inp, "bf16", h0=h0, y_dtype=torch.float32)
    cu = inp.cu_seqlens
    for s in range(len(lengths)):
        sl = slice(cu[s], cu[s + 1])
        ref = oracle.scan(inp.u[None, :, sl], inp.delta[None, :, sl], inp.B[None, :, sl], inp.C[None, :, sl],
                          inp.A, inp.Dskip, inp.bias, inp.z[None, :, sl], h0[s][None])
        check(f"y[{s}]", y[:, sl], ref["y"][0], ref["y_mag"][0], TOL["bf16"], "f32")
        check(f"h[{s}]", hl[s], ref["h_last"][0], ref["h_mag"][0], TOL["bf16"])


@pytest.mark.parametrize("algorithm", ["sequential", "chunked"])
def test_varlen_workload_both_kernels(algorithm):
    """The full varlen workload (16 sequences, D=2048) through each kernel, sampled channels."""
    inp = workloads.config_inputs("varlen_bf16")
    y, hl = _varlen(inp, "bf16", algorithm=algorithm)
    ch = np.arange(7, inp.u.shape[0], 41)
    ref = oracle.scan_varlen(inp.u[ch], inp.delta[ch], inp.B, inp.C, inp.A[ch], inp.cu_seqlens, inp.Dskip[ch],
                             inp.bias[ch], inp.z[ch], nthreads=NTHREADS)
    check("y", y[ch], ref["y"], ref["y_mag"], TOL["bf16"], "bf16")
    check("h_last", hl[:, ch], ref["h_last"], ref["h_mag"], TOL["bf16"])
    assert np.all(np.isfinite(y))


def test_pool_prefill_sequential():
    lengths = [300, 0, 77, 1000, 5]
    D, N, S = 64, 16, 9
    inp = workloads.varlen_inputs(lengths, D, N, "bf16", seed=600)
    T = inp.meta["total"]
    pool0 = np.random.default_rng(601).standard_normal((S, D, N)).astype(np.float32)
    slots = np.array([4, 0, 8, 2, 6], dtype=np.int32)
    pitch = round_up(T, 8)
    u, dl, z, B, C = (dev(x, "bf16", pitch=pitch) for x in (inp.u, inp.delta, inp.z, inp.B, inp.C))
    A, Dk, bias = (torch.from_numpy(x).cuda() for x in (inp.A, inp.Dskip, inp.bias))
    pool = torch.from_numpy(pool0.copy()).cuda()
    y = ssm.scan_fwd_varlen_pool(u, dl, B, C, A, torch.from_numpy(inp.cu_seqlens).cuda(), pool,
                                 torch.from_numpy(slots).cuda(), Dk, bias, z, total=T, algorithm=SEQ)
    torch.cuda.synchronize()
    pool_ref = pool0.astype(np.float64)
    ref = oracle.scan_varlen_pool(inp.u, inp.delta, inp.B, inp.C, inp.A, inp.cu_seqlens, pool_ref, slots,
                                  inp.Dskip, inp.bias, inp.z)
    check("y", host(y, T), ref["y"], ref["y_mag"], TOL["bf16"], "bf16")
    got = host(pool)
    for i, sl in enumerate(slots):
        lo, hi = inp.cu_seqlens[i], inp.cu_seqlens[i + 1]
        if hi == lo:
            assert np.array_equal(got[sl], pool0[sl])   # an empty sequence leaves its slot as it was
        else:
            r = oracle.scan(inp.u[None, :, lo:hi], inp.delta[None, :, lo:hi], inp.B[None, :, lo:hi],
                            inp.C[None, :, lo:hi], inp.A, inp.Dskip, inp.bias, inp.z[None, :, lo:hi],
                            pool0[sl][None])
            check(f"pool[{sl}]", got[sl], r["h_last"][0], r["h_mag"][0], TOL["bf16"])
    untouched = [s for s in range(S) if s not in set(slots.tolist())]
    assert np.array_equal(got[untouched], pool0[untouched])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_channel_groups_sequential(dtype):
    b, D, N, L, G = 2, 128, 16, 512, 2
    inp = workloads.batch_inputs(b, D, N, L, dtype, seed=700)
    rng = np.random.default_rng(701)
    B4, C4 = (workloads._store(rng.standard_normal((b, G, N, L)).astype(np.float32), dtype) for _ in range(2))
    u, dl, z = (dev(x, dtype) for x in (inp.u, inp.delta, inp.z))
    A, Dk, bias = (torch.from_numpy(x).cuda() for x in (inp.A, inp.Dskip, inp.bias))
    y, hl = ssm.scan_fwd(u, dl, dev(B4, dtype), dev(C4, dtype), A, Dk, bias, z, algorithm=SEQ)
    torch.cuda.synchronize()
    ref = oracle.scan(inp.u, inp.delta, B4, C4, inp.A, inp.Dskip, inp.bias, inp.z, nthreads=NTHREADS)
    check("y", host(y), ref["y"], ref["y_mag"], TOL[dtype], dtype)
    check("h_last", host(hl), ref["h_last"], ref["h_mag"], TOL[dtype])


def test_large_step_sequential():
    inp = workloads.batch_inputs(1, 64, 16, 300, "f32", seed=4)
    inp.delta[:] = 40.0
    inp.bias[:] = 0.0
    y, hl = _batch(inp, "f32")
    ref = oracle.scan(inp.u, inp.delta, inp.B, inp.C, inp.A, inp.Dskip, inp.bias, inp.z)
    assert np.all(np.isfinite(y)) and np.all(np.isfinite(hl))
    check("y", y, ref["y"], ref["y_mag"], TOL["f32"])


def test_sequential_rejections_and_workspace():
    """Cases the sequential kernel does not take are refused before anything runs; its
    workspace (the unit ticket) is reported and enforced."""
    lib = ssm.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    inp = workloads.batch_inputs(1, 64, 64, 128, "bf16", seed=9)
    u, dl, z, B, C = (dev(x, "bf16") for x in (inp.u, inp.delta, inp.z, inp.B, inp.C))
    A = torch.from_numpy(inp.A).cuda()
    y = torch.empty_like(u)
    p = ssm.scan_params(u, dl, B, C, A, z=z, y=y, algorithm=SEQ)               # dstate 64
    assert lib.ssm_scan_fwd(ctypes.byref(p), None, 0, stream) == 2            # SSM_ERR_UNSUPPORTED
    inp = workloads.batch_inputs(1, 64, 16, 128, "bf16", seed=10)
    u, dl, z, B, C = (dev(x, "bf16") for x in (inp.u, inp.delta, inp.z, inp.B, inp.C))
    A = torch.from_numpy(inp.A).cuda()
    y = torch.empty_like(u)
    p = ssm.scan_params(u, dl, B, C, A, z=z, y=y, zoh=True, algorithm=SEQ)     # zero-order hold
    assert lib.ssm_scan_fwd(ctypes.byref(p), None, 0, stream) == 2
    p = ssm.scan_params(u, dl, B, C, A, z=z, y=y, algorithm=SEQ)
    need = lib.ssm_scan_workspace_size(ctypes.byref(p), 0)
    assert need == 16
    assert lib.ssm_scan_fwd(ctypes.byref(p), None, 0, stream) == 6            # SSM_ERR_WORKSPACE
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    for _ in range(2):                                                         # the ticket is re-zeroed
        assert lib.ssm_scan_fwd(ctypes.byref(p), ctypes.c_void_p(ws.data_ptr()), need, stream) == 0
    torch.cuda.synchronize()
    ref = oracle.scan(inp.u, inp.delta, inp.B, inp.C, inp.A, z=inp.z)
    check("y", host(y), ref["y"], ref["y_mag"], TOL["bf16"], "bf16")
    assert ssm.device_status() == 0
