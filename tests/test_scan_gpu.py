"""GPU parity: the CUDA scans (through the C ABI) against the fp64 oracle.

Error metric: max |x - x_oracle| / m, with m the oracle's absolute-value bound (|x_oracle| <= m);
gates 1e-4 for float32 inputs and 3e-3 for bf16 inputs (the latter includes the 2^-9 rounding
of the bf16 output).  Full-size workloads are checked on sampled channels: channels are
independent, so the oracle run on a channel subset is exact for those channels.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle  # noqa: E402
import selective_state_space_15_b200 as ssm  # noqa: E402
import workloads  # noqa: E402
from helpers import TOL, check, dev, host, round_up  # noqa: E402

NTHREADS = oracle.default_threads()


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ssm.load()


def run_batch(inp, dtype, h0=None, gate=True, with_last=True, y_dtype=None):
    u, dl = dev(inp.u, dtype), dev(inp.delta, dtype)
    z = dev(inp.z, dtype) if (gate and inp.z is not None) else None
    B, C = dev(inp.B, dtype), dev(inp.C, dtype)
    A, D, bias = (torch.from_numpy(x).cuda() for x in (inp.A, inp.Dskip, inp.bias))
    h0t = torch.from_numpy(h0).cuda() if h0 is not None else None
    y, hl = ssm.scan_fwd(u, dl, B, C, A, D, bias, z, h0t, return_last_state=with_last, y_dtype=y_dtype)
    torch.cuda.synchronize()
    return host(y), (host(hl) if hl is not None else None)


def oracle_batch(inp, channels=None, h0=None, gate=True):
    sl = slice(None) if channels is None else channels
    return oracle.scan(inp.u[:, sl], inp.delta[:, sl], inp.B, inp.C, inp.A[sl], inp.Dskip[sl], inp.bias[sl],
                       inp.z[:, sl] if (gate and inp.z is not None) else None,
                       None if h0 is None else h0[:, sl], nthreads=NTHREADS)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [
    (1, 16, 16, 256),     # the tiny workload's shape
    (2, 40, 16, 1000),    # several chunks, tail channel tile (40 = 5 tiles of 8)
    (1, 8, 16, 1),        # single step
    (3, 9, 16, 777),      # odd everything
    (1, 24, 32, 515),
    (1, 12, 64, 300),
    (1, 10, 128, 200),
    (2, 20, 256, 160),    # N=256: 8 warps split the states of an 8-channel tile
    (1, 9, 256, 77),      # N=256, element-wise staging, tail tile
])
def test_batch_small_full(shape, dtype):
    b, D, N, L = shape
    inp = workloads.batch_inputs(b, D, N, L, dtype, seed=100 + L)
    y, hl = run_batch(inp, dtype)
    ref = oracle_batch(inp)
    check("y", y, ref["y"], ref["y_mag"], TOL[dtype], dtype)
    check("h_last", hl, ref["h_last"], ref["h_mag"], TOL[dtype])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_batch_with_initial_state_no_gate(dtype):
    b, D, N, L = 2, 16, 16, 600
    inp = workloads.batch_inputs(b, D, N, L, dtype, seed=7, gate=False, h0=True)
    y, hl = run_batch(inp, dtype, h0=inp.h0, gate=False)
    ref = oracle_batch(inp, h0=inp.h0, gate=False)
    check("y", y, ref["y"], ref["y_mag"], TOL[dtype], dtype)
    check("h_last", hl, ref["h_last"], ref["h_mag"], TOL[dtype])


def test_optional_terms_absent():
    # no z, no Dskip, no bias, no h_last output
    inp = workloads.batch_inputs(1, 16, 16, 300, "f32", seed=9, gate=False)
    u, dl, B, C = (dev(x) for x in (inp.u, inp.delta, inp.B, inp.C))
    A = torch.from_numpy(inp.A).cuda()
    y, hl = ssm.scan_fwd(u, dl, B, C, A, return_last_state=False)
    assert hl is None
    ref = oracle.scan(inp.u, inp.delta, inp.B, inp.C, inp.A)
    check("y", host(y), ref["y"], ref["y_mag"], TOL["f32"])


def test_tiny_workload():
    inp = workloads.config_inputs("tiny_f32")
    y, hl = run_batch(inp, "f32")
    ref = oracle_batch(inp)
    check("y", y, ref["y"], ref["y_mag"], TOL["f32"])
    check("h_last", hl, ref["h_last"], ref["h_mag"], TOL["f32"])


def test_batch_f32_workload():
    inp = workloads.config_inputs("batch_f32")
    y, hl = run_batch(inp, "f32")
    ch = np.arange(0, inp.u.shape[1], 7)                # every 7th channel, both batch rows
    ref = oracle_batch(inp, channels=ch)
    check("y", y[:, ch], ref["y"], ref["y_mag"], TOL["f32"])
    check("h_last", hl[:, ch], ref["h_last"], ref["h_mag"], TOL["f32"])


def _varlen_run(inp, dtype, pitch, gate=True, h0=None, y_dtype=None):
    T = inp.meta["total"]
    u, dl = dev(inp.u, dtype, pitch=pitch), dev(inp.delta, dtype, pitch=pitch)
    z = dev(inp.z, dtype, pitch=pitch) if gate else None
    B, C = dev(inp.B, dtype, pitch=pitch), dev(inp.C, dtype, pitch=pitch)
    A, D, bias = (torch.from_numpy(x).cuda() for x in (inp.A, inp.Dskip, inp.bias))
    cu = torch.from_numpy(inp.cu_seqlens).cuda()
    h0t = torch.from_numpy(h0).cuda() if h0 is not None else None
    y, hl = ssm.scan_fwd_varlen(u, dl, B, C, A, cu, D, bias, z, h0t, total=T, y_dtype=y_dtype)
    torch.cuda.synchronize()
    return host(y, T), host(hl)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("lengths,pitch_mult", [
    ([5, 1, 17, 0, 300, 9, 64, 1000], 8),    # empty and length-1 sequences, unaligned starts
    ([257, 255, 512, 3], 1),                 # unpadded rows: T odd -> element-wise staging
    ([4096, 256, 1024], 8),
])
def test_varlen_small_full(lengths, pitch_mult, dtype):
    D, N = 24, 16
    inp = workloads.varlen_inputs(lengths, D, N, dtype, seed=len(lengths) + sum(lengths))
    T = inp.meta["total"]
    y, hl = _varlen_run(inp, dtype, round_up(T, pitch_mult))
    ref = oracle.scan_varlen(inp.u, inp.delta, inp.B, inp.C, inp.A, inp.cu_seqlens, inp.Dskip, inp.bias, inp.z,
                             nthreads=NTHREADS)
    check("y", y, ref["y"], ref["y_mag"], TOL[dtype], dtype)
    check("h_last", hl, ref["h_last"], ref["h_mag"], TOL[dtype])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_varlen_many_sequences(dtype):
    """More packed sequences than the kernel ranks by length (64): CTAs take them in order."""
    rng = np.random.default_rng(77)
    lengths = [int(x) for x in rng.integers(0, 60, size=150)]
    lengths[3] = 0
    lengths[100] = 200
    D, N = 24, 16
    inp = workloads.varlen_inputs(lengths, D, N, dtype, seed=78)
    T = inp.meta["total"]
    y, hl = _varlen_run(inp, dtype, round_up(T, 8))
    ref = oracle.scan_varlen(inp.u, inp.delta, inp.B, inp.C, inp.A, inp.cu_seqlens, inp.Dskip, inp.bias, inp.z,
                             nthreads=NTHREADS)
    check("y", y, ref["y"], ref["y_mag"], TOL[dtype], dtype)
    check("h_last", hl, ref["h_last"], ref["h_mag"], TOL[dtype])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_varlen_dstate_256(dtype):
    lengths = [100, 0, 37, 300, 1]
    D, N = 20, 256
    inp = workloads.varlen_inputs(lengths, D, N, dtype, seed=256)
    T = inp.meta["total"]
    y, hl = _varlen_run(inp, dtype, round_up(T, 8))
    ref = oracle.scan_varlen(inp.u, inp.delta, inp.B, inp.C, inp.A, inp.cu_seqlens, inp.Dskip, inp.bias, inp.z,
                             nthreads=NTHREADS)
    check("y", y, ref["y"], ref["y_mag"], TOL[dtype], dtype)
    check("h_last", hl, ref["h_last"], ref["h_mag"], TOL[dtype])


def test_varlen_with_initial_states():
    lengths = [100, 0, 37, 400]
    D, N = 16, 16
    inp = workloads.varlen_inputs(lengths, D, N, "f32", seed=3)
    h0 = np.random.default_rng(1).standard_normal((len(lengths), D, N)).astype(np.float32)
    y, hl = _varlen_run(inp, "f32", round_up(inp.meta["total"], 4), h0=h0)
    cu = inp.cu_seqlens
    for s in range(len(lengths)):
        sl = slice(cu[s], cu[s + 1])
        ref = oracle.scan(inp.u[None, :, sl], inp.delta[None, :, sl], inp.B[None, :, sl], inp.C[None, :, sl],
                          inp.A, inp.Dskip, inp.bias, inp.z[None, :, sl], h0[s][None])
        check(f"y[{s}]", y[:, sl], ref["y"][0], ref["y_mag"][0], TOL["f32"])
        check(f"h[{s}]", hl[s], ref["h_last"][0], ref["h_mag"][0], TOL["f32"])


def test_varlen_workload_sampled():
    inp = workloads.config_inputs("varlen_bf16")
    T = inp.meta["total"]
    y, hl = _varlen_run(inp, "bf16", round_up(T, 8))
    ch = np.arange(3, inp.u.shape[0], 29)
    ref = oracle.scan_varlen(inp.u[ch], inp.delta[ch], inp.B, inp.C, inp.A[ch], inp.cu_seqlens, inp.Dskip[ch],
                             inp.bias[ch], inp.z[ch], nthreads=NTHREADS)
    check("y", y[ch], ref["y"], ref["y_mag"], TOL["bf16"], "bf16")
    check("h_last", hl[:, ch], ref["h_last"], ref["h_mag"], TOL["bf16"])
    assert np.all(np.isfinite(y))


@pytest.mark.parametrize("name,stride", [("long_bf16", 331), ("long_n128_bf16", 127)])
def test_long_workloads_sampled(name, stride):
    inp = workloads.config_inputs(name)
    y, hl = run_batch(inp, "bf16")
    ch = np.arange(5, inp.u.shape[1], stride)
    ref = oracle_batch(inp, channels=ch)
    check("y", y[:, ch], ref["y"], ref["y_mag"], TOL["bf16"], "bf16")
    check("h_last", hl[:, ch], ref["h_last"], ref["h_mag"], TOL["bf16"])
    assert np.all(np.isfinite(y))


def test_large_step_does_not_overflow():
    # delta + bias = 40 on every step: Delta ~ 40, exp(Delta A) underflows to 0, no inf/nan
    inp = workloads.batch_inputs(1, 8, 16, 300, "f32", seed=4)
    inp.delta[:] = 40.0
    inp.bias[:] = 0.0
    y, hl = run_batch(inp, "f32")
    ref = oracle_batch(inp)
    assert np.all(np.isfinite(y)) and np.all(np.isfinite(hl))
    check("y", y, ref["y"], ref["y_mag"], TOL["f32"])


@pytest.mark.parametrize("shape", [(1, 16, 16, 256), (2, 40, 16, 1000), (3, 9, 16, 777), (1, 10, 128, 200)])
def test_bf16_inputs_float32_output_strict(shape):
    """bf16 inputs with a float32 y: the 3e-3 gate with no output-rounding allowance."""
    b, D, N, L = shape
    inp = workloads.batch_inputs(b, D, N, L, "bf16", seed=200 + L)
    y, hl = run_batch(inp, "bf16", y_dtype=torch.float32)
    ref = oracle_batch(inp)
    check("y", y, ref["y"], ref["y_mag"], TOL["bf16"], "f32")
    check("h_last", hl, ref["h_last"], ref["h_mag"], TOL["bf16"])


def test_varlen_workload_float32_output_strict():
    inp = workloads.config_inputs("varlen_bf16")
    T = inp.meta["total"]
    y, hl = _varlen_run(inp, "bf16", round_up(T, 8), y_dtype=torch.float32)
    ch = np.arange(11, inp.u.shape[0], 97)
    ref = oracle.scan_varlen(inp.u[ch], inp.delta[ch], inp.B, inp.C, inp.A[ch], inp.cu_seqlens, inp.Dskip[ch],
                             inp.bias[ch], inp.z[ch], nthreads=NTHREADS)
    check("y", y[ch], ref["y"], ref["y_mag"], TOL["bf16"], "f32")


def test_persistent_paths_and_workspace():
    """Aligned fixed-length batches run on the persistent ticketed grid (state handed between
    units through the workspace); narrow problems split the states over two warps."""
    import ctypes
    lib = ssm.load()
    # more chains than CTA slots split into several units handed on through the workspace
    # (3 x 1000 and 3 x 1100 channels); fewer chains run as one unit each
    for (b, D, L, seed, dt) in [(1, 8, 4096, 21, "bf16"), (3, 40, 2304, 22, "bf16"), (2, 2048 + 8, 512, 23, "bf16"),
                                (3, 1000, 2304, 27, "bf16"), (1, 8, 4100, 25, "f32"), (3, 1100, 1540, 26, "f32")]:
        inp = workloads.batch_inputs(b, D, 16, L, dt, seed=seed)
        y, hl = run_batch(inp, dt, y_dtype=torch.float32)
        ch = np.arange(0, D, max(1, D // 24))
        ref = oracle_batch(inp, channels=ch)
        check("y", y[:, ch], ref["y"], ref["y_mag"], TOL[dt], "f32")
        check("h_last", hl[:, ch], ref["h_last"], ref["h_mag"], TOL[dt])
    # the workspace size is reported and enforced
    inp = workloads.batch_inputs(1, 8, 16, 256, "bf16", seed=24)
    u, dl, z, B, C = (dev(x, "bf16") for x in (inp.u, inp.delta, inp.z, inp.B, inp.C))
    A = torch.from_numpy(inp.A).cuda()
    y = torch.empty_like(u)
    p = ssm.scan_params(u, dl, B, C, A, z=z, y=y)
    need = lib.ssm_scan_workspace_size(ctypes.byref(p), 0)
    assert need > 0
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.ssm_scan_fwd(ctypes.byref(p), None, 0, stream) == 6                    # SSM_ERR_WORKSPACE
    small = torch.empty(need - 16, dtype=torch.uint8, device="cuda")
    assert lib.ssm_scan_fwd(ctypes.byref(p), ctypes.c_void_p(small.data_ptr()), need - 16, stream) == 6
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    for _ in range(2):                                                                # reuse of a workspace
        assert lib.ssm_scan_fwd(ctypes.byref(p), ctypes.c_void_p(ws.data_ptr()), need, stream) == 0
    torch.cuda.synchronize()
    ref = oracle.scan(inp.u, inp.delta, inp.B, inp.C, inp.A, z=inp.z)
    check("y", host(y), ref["y"], ref["y_mag"], TOL["bf16"], "bf16")
    assert ssm.device_status() == 0


def test_handoff_wait_is_bounded_and_reported():
    """The wait for the state handed on between the units of a chain is bounded: with the test
    hook no unit of the first chunk group runs, the later units give up waiting, the kernel
    records SSM_ERR_TIMEOUT, and the next call on the same context is correct."""
    inp = workloads.batch_inputs(1, 8, 16, 1024, "bf16", seed=31)   # 2 chains of 4 chunks
    ssm.load().ssm_test_drop_first_handoff()
    run_batch(inp, "bf16")                      # outputs unusable
    assert ssm.device_status() == 5             # SSM_ERR_TIMEOUT, read and cleared
    assert ssm.device_status() == 0
    y, hl = run_batch(inp, "bf16")
    ref = oracle_batch(inp)
    check("y", y, ref["y"], ref["y_mag"], TOL["bf16"], "bf16")
    check("h_last", hl, ref["h_last"], ref["h_mag"], TOL["bf16"])
    assert ssm.device_status() == 0


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape,G", [
    ((2, 64, 16, 512), 2),      # persistent tiles, one group per 32 channels
    ((1, 24, 16, 1000), 3),     # narrow tile, 8 channels per group (tiles end at group edges)
    ((1, 40, 128, 200), 4),     # N=128
    ((3, 18, 16, 777), 3),      # element-wise staging, 6 channels per group
])
def test_channel_groups(shape, G, dtype):
    """Channel groups: channel d reads B, C of group d // (D / G)."""
    b, D, N, L = shape
    inp = workloads.batch_inputs(b, D, N, L, dtype, seed=300 + G + L)
    rng = np.random.default_rng(301)
    rnd = lambda: workloads.round_to_bf16(rng.standard_normal((b, G, N, L)).astype(np.float32))  # noqa: E731
    B4, C4 = (rnd(), rnd()) if dtype == "bf16" else tuple(rng.standard_normal((2, b, G, N, L)).astype(np.float32))
    u, dl, z = (dev(x, dtype) for x in (inp.u, inp.delta, inp.z))
    A, Dk, bias = (torch.from_numpy(x).cuda() for x in (inp.A, inp.Dskip, inp.bias))
    y, hl = ssm.scan_fwd(u, dl, dev(B4, dtype), dev(C4, dtype), A, Dk, bias, z)
    torch.cuda.synchronize()
    ref = oracle.scan(inp.u, inp.delta, B4, C4, inp.A, inp.Dskip, inp.bias, inp.z, nthreads=NTHREADS)
    check("y", host(y), ref["y"], ref["y_mag"], TOL[dtype], dtype)
    check("h_last", host(hl), ref["h_last"], ref["h_mag"], TOL[dtype])


def test_channel_groups_varlen():
    lengths = [300, 0, 77, 1000]
    D, N, G = 48, 16, 4
    inp = workloads.varlen_inputs(lengths, D, N, "bf16", seed=302)
    T = inp.meta["total"]
    rng = np.random.default_rng(303)
    B3, C3 = (workloads.round_to_bf16(rng.standard_normal((G, N, T)).astype(np.float32)) for _ in range(2))
    pitch = round_up(T, 8)
    u, dl, z = (dev(x, "bf16", pitch=pitch) for x in (inp.u, inp.delta, inp.z))
    A, Dk, bias = (torch.from_numpy(x).cuda() for x in (inp.A, inp.Dskip, inp.bias))
    y, hl = ssm.scan_fwd_varlen(u, dl, dev(B3, "bf16", pitch=pitch), dev(C3, "bf16", pitch=pitch), A,
                                torch.from_numpy(inp.cu_seqlens).cuda(), Dk, bias, z, total=T)
    torch.cuda.synchronize()
    ref = oracle.scan_varlen(inp.u, inp.delta, B3, C3, inp.A, inp.cu_seqlens, inp.Dskip, inp.bias, inp.z,
                             nthreads=NTHREADS)
    check("y", host(y, T), ref["y"], ref["y_mag"], TOL["bf16"], "bf16")
    check("h_last", host(hl), ref["h_last"], ref["h_mag"], TOL["bf16"])
