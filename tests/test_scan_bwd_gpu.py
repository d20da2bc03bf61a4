"""GPU parity of the backward kernel (ssm_scan_bwd, through the C ABI) against the fp64 oracle's
reverse-mode derivative (oracle.scan_bwd, pinned by central differences of the forward oracle).

Error metric.  Gradients are sums with cancellation (over states, channels or time) and the
oracle gives no magnitude bound for them, so each gradient is compared row by row along its
last axis: max_t |g - g_ref| / max_t |g_ref| for every row (a row of zeros must come out
zero).  Gates: 1e-4 for float32 inputs, 3e-3 for bf16 inputs; a bf16 gradient output is
allowed its own half-ulp rounding, 2^-8 |g_ref|, on top.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle  # noqa: E402
import selective_state_space_15_b200 as ssm  # noqa: E402
import workloads  # noqa: E402
from helpers import TOL, dev, host  # noqa: E402

NTHREADS = oracle.default_threads()
NAMES = ("du", "ddelta", "dz", "dB", "dC", "dA", "dDskip", "dbias", "dh0")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ssm.load()


def row_error(x, ref, rounding=0.0):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if not np.all(np.isfinite(x)):
        return float("inf")
    x2, r2 = x.reshape(-1, x.shape[-1]), ref.reshape(-1, ref.shape[-1])
    diff = np.maximum(np.abs(x2 - r2) - rounding * np.abs(r2), 0.0)
    scale = np.abs(r2).max(axis=1, keepdims=True)
    with np.errstate(divide="ignore", invalid="ignore"):
        e = np.where(scale > 0, diff / np.where(scale > 0, scale, 1.0), np.where(diff > 0, np.inf, 0.0))
    return float(e.max()) if e.size else 0.0


def check_grads(got, ref, tol, grad_dtype, names=NAMES):
    for name in names:
        if ref.get(name) is None or got.get(name) is None:
            continue
        per_step = name in ("du", "ddelta", "dz")
        rounding = 2.0 ** -8 if (per_step and grad_dtype == "bf16") else 0.0
        e = row_error(got[name], ref[name], rounding)
        assert e <= tol, f"{name}: row-normwise error {e:.3e} > {tol:.1e}"


def run_bwd(inp, dtype, dy, grad_dtype=None, h0=None, dh_last=None, gate=True, to_host=True, zoh=False):
    u, dl = dev(inp.u, dtype), dev(inp.delta, dtype)
    z = dev(inp.z, dtype) if gate else None
    B, C = dev(inp.B, dtype), dev(inp.C, dtype)
    A, D, bias = (torch.from_numpy(x).cuda() for x in (inp.A, inp.Dskip, inp.bias))
    gdt = grad_dtype or dtype
    dyt = dev(dy, gdt)
    h0t = torch.from_numpy(h0).cuda() if h0 is not None else None
    dht = torch.from_numpy(dh_last).cuda() if dh_last is not None else None
    out = ssm.scan_bwd(u, dl, B, C, A, dyt, D, bias, z, h0t, dht,
                       grad_dtype=torch.float32 if gdt == "f32" else None, zoh=zoh)
    torch.cuda.synchronize()
    if not to_host:
        return out
    return {k: (host(v) if v is not None else None) for k, v in out.items()}


def oracle_bwd(inp, dy, h0=None, dh_last=None, gate=True, channels=None, zoh=False):
    sl = slice(None) if channels is None else channels
    r = oracle.scan_bwd(inp.u[:, sl], inp.delta[:, sl], inp.B, inp.C, inp.A[sl], dy[:, sl], inp.Dskip[sl],
                        inp.bias[sl], inp.z[:, sl] if gate else None, None if h0 is None else h0[:, sl],
                        None if dh_last is None else dh_last[:, sl], nthreads=NTHREADS, zoh=zoh)
    return r


def draw_dy(shape, dtype, seed):
    x = np.random.default_rng(seed).standard_normal(shape).astype(np.float32)
    return workloads.round_to_bf16(x) if dtype == "bf16" else x


@pytest.mark.parametrize("zoh", [False, True], ids=["euler", "zoh"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [
    (1, 16, 16, 256),      # the tiny workload's shape
    (2, 40, 16, 104),      # a ragged tile (40 = 32 + 8), a partial chunk and block
    (3, 33, 16, 8),        # one block
    (1, 64, 16, 1000),
])
def test_bwd_small_full(shape, dtype, zoh):
    b, D, N, L = shape
    inp = workloads.batch_inputs(b, D, N, L, dtype, seed=800 + L + D, h0=True)
    dy = draw_dy((b, D, L), dtype, 801 + L)
    dh_last = np.random.default_rng(802).standard_normal((b, D, N)).astype(np.float32)
    got = run_bwd(inp, dtype, dy, h0=inp.h0, dh_last=dh_last, zoh=zoh)
    ref = oracle_bwd(inp, dy, h0=inp.h0, dh_last=dh_last, zoh=zoh)
    check_grads(got, ref, TOL[dtype], dtype)


def test_bwd_zoh_with_zero_and_positive_decays():
    """Zero-order hold where A = 0 for some states (c = Delta, dc/dA = Delta^2 / 2 from the
    series) and small |Delta A| everywhere else in a channel (the series side of both
    coefficients), next to the usual decays."""
    b, D, N, L = 1, 24, 16, 200
    inp = workloads.batch_inputs(b, D, N, L, "f32", seed=870, h0=True)
    A = inp.A.copy()
    A[0:8, 0:4] = 0.0
    A[8:16] *= 1e-3
    inp.A = A
    dy = draw_dy((b, D, L), "f32", 871)
    got = run_bwd(inp, "f32", dy, h0=inp.h0, zoh=True)
    ref = oracle_bwd(inp, dy, h0=inp.h0, zoh=True)
    check_grads(got, ref, TOL["f32"], "f32")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_bwd_no_gate_no_initial_state(dtype):
    b, D, N, L = 2, 48, 16, 304
    inp = workloads.batch_inputs(b, D, N, L, dtype, seed=810, gate=False)
    dy = draw_dy((b, D, L), dtype, 811)
    got = run_bwd(inp, dtype, dy, gate=False)
    ref = oracle_bwd(inp, dy, gate=False)
    check_grads(got, ref, TOL[dtype], dtype)


def test_bwd_bf16_inputs_float32_gradients_strict():
    """bf16 inputs with float32 dy and gradients: the 3e-3 gate with no rounding allowance."""
    b, D, N, L = 2, 40, 16, 520
    inp = workloads.batch_inputs(b, D, N, L, "bf16", seed=820)
    dy = draw_dy((b, D, L), "f32", 821)
    got = run_bwd(inp, "bf16", dy, grad_dtype="f32")
    ref = oracle_bwd(inp, dy)
    check_grads(got, ref, TOL["bf16"], "f32")


@pytest.mark.parametrize("zoh", [False, True], ids=["euler", "zoh"])
def test_bwd_batch_f32_workload(zoh):
    """The float32 batch workload (batch 2, D=1536, N=16, L=2048), every gradient in full."""
    inp = workloads.config_inputs("batch_f32")
    b, D, L = inp.u.shape
    dy = draw_dy((b, D, L), "f32", 830)
    got = run_bwd(inp, "f32", dy, zoh=zoh)
    ref = oracle_bwd(inp, dy, zoh=zoh)
    check_grads(got, ref, TOL["f32"], "f32")


@pytest.mark.parametrize("zoh", [False, True], ids=["euler", "zoh"])
def test_bwd_long_workload_sampled(zoh):
    """The long bf16 workload (1 x 2560 channels x 131072 steps) with dy nonzero on sampled
    channels only: the gradients then come from those channels alone (the others carry no
    adjoint), so the oracle run on the sample gives every gradient exactly -- dB and dC, which
    sum over channels, included.  The other channels' per-step gradients must be zero."""
    inp = workloads.config_inputs("long_bf16")
    b, D, L = inp.u.shape
    ch = np.arange(9, D, 523) if not zoh else np.arange(301, D, 611)
    dy = np.zeros((b, D, L), dtype=np.float32)
    dy[:, ch] = draw_dy((b, len(ch), L), "bf16", 840)
    got = run_bwd(inp, "bf16", dy, to_host=False, zoh=zoh)
    ref = oracle_bwd(inp, dy, channels=ch, zoh=zoh)
    idx = torch.from_numpy(ch).cuda()
    sub = {k: host(v.index_select(1, idx) if k in ("du", "ddelta", "dz", "dh0") else
                   v.index_select(0, idx) if k in ("dA", "dDskip", "dbias") else v)
           for k, v in got.items() if v is not None}
    check_grads(sub, ref, TOL["bf16"], "bf16")
    others = torch.from_numpy(np.setdiff1d(np.arange(D), ch)[::97]).cuda()
    for k in ("du", "ddelta", "dz"):
        assert not torch.any(got[k].index_select(1, others)), k


def test_bwd_rejections_and_workspace():
    lib = ssm.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    inp = workloads.batch_inputs(1, 32, 16, 64, "bf16", seed=850)
    u, dl, z, B, C = (dev(x, "bf16") for x in (inp.u, inp.delta, inp.z, inp.B, inp.C))
    A = torch.from_numpy(inp.A).cuda()
    p = ssm.scan_params(u, dl, B, C, A, z=z)
    need = lib.ssm_scan_bwd_workspace_size(ctypes.byref(p))
    assert need > 0
    g = ssm.ScanGrads()
    dy = torch.zeros_like(u)
    outs = [torch.empty_like(u) for _ in range(3)]
    dB, dC = torch.empty(1, 16, 64, device="cuda"), torch.empty(1, 16, 64, device="cuda")
    dA = torch.empty(32, 16, device="cuda")
    g.dy, g.du, g.ddelta, g.dz = dy.data_ptr(), outs[0].data_ptr(), outs[1].data_ptr(), outs[2].data_ptr()
    g.dB, g.dC, g.dA = dB.data_ptr(), dC.data_ptr(), dA.data_ptr()
    assert lib.ssm_scan_bwd(ctypes.byref(p), ctypes.byref(g), None, 0, stream) == 6          # SSM_ERR_WORKSPACE
    g2 = ssm.ScanGrads()
    g2.dy = dy.data_ptr()
    assert lib.ssm_scan_bwd(ctypes.byref(p), ctypes.byref(g2), None, 0, stream) == 1         # outputs missing
    pz = ssm.scan_params(u, dl, B, C, A, z=z, zoh=True)
    assert lib.ssm_scan_bwd(ctypes.byref(pz), ctypes.byref(g), None, 0, stream) == 6         # zero-order hold: supported
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    assert lib.ssm_scan_bwd(ctypes.byref(p), ctypes.byref(g), ctypes.c_void_p(ws.data_ptr()), need, stream) == 0
    torch.cuda.synchronize()
    assert ssm.device_status() == 0


def test_bwd_padded_rows_ragged_length_through_the_abi():
    """Rows padded to a 16-byte stride (304) around a length that is not a multiple of 4 (301):
    the per-step gradients keep u's strides and must leave the padding alone, and dB, dC
    ([b, N, L] contiguous: 1204-byte rows) take the scalar-atomic path of the channel sums."""
    b, D, N, L, P = 2, 40, 16, 301, 304
    inp = workloads.batch_inputs(b, D, N, L, "f32", seed=860, h0=True)
    dy_h = draw_dy((b, D, L), "f32", 861)
    view = lambda x: dev(x, "f32", pitch=P)[..., :L]  # noqa: E731  (NaN in the padding)
    u, dl, z, B, C, dy = (view(x) for x in (inp.u, inp.delta, inp.z, inp.B, inp.C, dy_h))
    A, Dk, bias, h0 = (torch.from_numpy(x).cuda() for x in (inp.A, inp.Dskip, inp.bias, inp.h0))
    outs = {k: torch.full((b, D, P), float("nan"), device="cuda")[..., :L] for k in ("du", "ddelta", "dz")}
    dB, dC = torch.empty(b, N, L, device="cuda"), torch.empty(b, N, L, device="cuda")
    dA, dD, db = torch.empty(D, N, device="cuda"), torch.empty(D, device="cuda"), torch.empty(D, device="cuda")
    dh0 = torch.empty(b, D, N, device="cuda")
    p = ssm.scan_params(u, dl, B, C, A, Dk, bias, z, h0)
    lib = ssm.load()
    need = lib.ssm_scan_bwd_workspace_size(ctypes.byref(p))
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    g = ssm.ScanGrads()
    g.dy, g.du, g.ddelta, g.dz = dy.data_ptr(), outs["du"].data_ptr(), outs["ddelta"].data_ptr(), outs["dz"].data_ptr()
    g.dB, g.dC, g.dA, g.dDskip, g.ddelta_bias, g.dh0 = (t.data_ptr() for t in (dB, dC, dA, dD, db, dh0))
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.ssm_scan_bwd(ctypes.byref(p), ctypes.byref(g), ctypes.c_void_p(ws.data_ptr()), need, stream) == 0
    torch.cuda.synchronize()
    assert ssm.device_status() == 0
    got = {"du": host(outs["du"]), "ddelta": host(outs["ddelta"]), "dz": host(outs["dz"]), "dB": host(dB),
           "dC": host(dC), "dA": host(dA), "dDskip": host(dD), "dbias": host(db), "dh0": host(dh0)}
    ref = oracle_bwd(inp, dy_h, h0=inp.h0)
    check_grads(got, ref, TOL["f32"], "f32")
    for k in ("du", "ddelta", "dz"):
        pad = outs[k].as_strided((b, D, P - L), (D * P, P, 1), storage_offset=L)
        assert torch.isnan(pad).all(), f"{k}: the kernel wrote into the row padding"
