"""GPU parity of the zero-order-hold discretisation against the fp64 oracle.

Bbar = (Delta A)^-1 (exp(Delta A) - I) Delta B ("企业官网建设流程全解析" page, discosf.com, §1.2),
chosen per call with ``zoh=True``.  The inputs add, to the usual workload distributions, state
columns with A = 0 (the coefficient is Delta), channels with a large step (|Delta A| up to
~40, where exp(Delta A) - 1 is about -1) and the small |Delta A| of the configs (the series
branch of the kernels).  Error metric and gates as in test_scan_gpu.py.
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


def _widen_range(inp):
    """A = 0 in some states, very negative A in others, larger steps on some channels."""
    A = inp.A.copy()
    A[::3, 0] = 0.0
    A[1::3, -1] = -40.0
    inp.A = A
    inp.bias = (inp.bias + np.where(np.arange(inp.bias.shape[0]) % 4 == 0, 3.0, 0.0)).astype(np.float32)
    return inp


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [
    (1, 16, 16, 256),      # narrow persistent tile
    (2, 40, 16, 1000),     # narrow, several units and a ragged chunk
    (3, 9, 16, 777),       # rows not 16-byte aligned: element-wise staging
    (1, 24, 32, 512),
    (1, 12, 64, 304),
    (1, 10, 128, 200),     # N=128 (narrow 16-warp tile for bf16)
    (1, 9, 256, 160),      # N=256
])
def test_zoh_batch_matches_oracle(shape, dtype):
    b, D, N, L = shape
    inp = _widen_range(workloads.batch_inputs(b, D, N, L, dtype, seed=300 + L, h0=True))
    u, dl, z, B, C = (dev(x, dtype) for x in (inp.u, inp.delta, inp.z, inp.B, inp.C))
    A, Dk, bias, h0 = (torch.from_numpy(x).cuda() for x in (inp.A, inp.Dskip, inp.bias, inp.h0))
    y, hl = ssm.scan_fwd(u, dl, B, C, A, Dk, bias, z, h0, zoh=True)
    torch.cuda.synchronize()
    assert ssm.device_status() == 0
    ref = oracle.scan(inp.u, inp.delta, inp.B, inp.C, inp.A, inp.Dskip, inp.bias, inp.z, inp.h0,
                      nthreads=NTHREADS, zoh=True)
    check("y", host(y), ref["y"], ref["y_mag"], TOL[dtype], dtype)
    check("h_last", host(hl), ref["h_last"], ref["h_mag"], TOL[dtype])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_zoh_wide_batch_sampled(dtype):
    """batch * dim >= 8192: the wide 32-channel tile on the persistent grid."""
    b, D, N, L = 1, 8192 + 64, 16, 200
    inp = _widen_range(workloads.batch_inputs(b, D, N, L, dtype, seed=310))
    u, dl, z, B, C = (dev(x, dtype) for x in (inp.u, inp.delta, inp.z, inp.B, inp.C))
    A, Dk, bias = (torch.from_numpy(x).cuda() for x in (inp.A, inp.Dskip, inp.bias))
    y, hl = ssm.scan_fwd(u, dl, B, C, A, Dk, bias, z, zoh=True)
    torch.cuda.synchronize()
    ch = np.arange(0, D, 97)
    ref = oracle.scan(inp.u[:, ch], inp.delta[:, ch], inp.B, inp.C, inp.A[ch], inp.Dskip[ch], inp.bias[ch],
                      inp.z[:, ch], nthreads=NTHREADS, zoh=True)
    check("y", host(y)[:, ch], ref["y"], ref["y_mag"], TOL[dtype], dtype)
    check("h_last", host(hl)[:, ch], ref["h_last"], ref["h_mag"], TOL[dtype])


@pytest.mark.parametrize("dtype,pitch_mult", [("f32", 4), ("bf16", 8), ("bf16", 1)])
def test_zoh_varlen_matches_oracle(dtype, pitch_mult):
    lengths = [300, 0, 37, 1000, 64, 5]
    D, N = 40, 16
    inp = _widen_range(workloads.varlen_inputs(lengths, D, N, dtype, seed=320 + pitch_mult))
    T = inp.meta["total"]
    pitch = round_up(T, pitch_mult)
    u, dl, z = (dev(x, dtype, pitch=pitch) for x in (inp.u, inp.delta, inp.z))
    B, C = dev(inp.B, dtype, pitch=pitch), dev(inp.C, dtype, pitch=pitch)
    A, Dk, bias = (torch.from_numpy(x).cuda() for x in (inp.A, inp.Dskip, inp.bias))
    cu = torch.from_numpy(inp.cu_seqlens).cuda()
    y, hl = ssm.scan_fwd_varlen(u, dl, B, C, A, cu, Dk, bias, z, total=T, zoh=True)
    torch.cuda.synchronize()
    ref = oracle.scan_varlen(inp.u, inp.delta, inp.B, inp.C, inp.A, inp.cu_seqlens, inp.Dskip, inp.bias, inp.z,
                             nthreads=NTHREADS, zoh=True)
    check("y", host(y, T), ref["y"], ref["y_mag"], TOL[dtype], dtype)
    check("h_last", host(hl), ref["h_last"], ref["h_mag"], TOL[dtype])


@pytest.mark.parametrize("dtype,N", [("bf16", 16), ("f32", 16), ("bf16", 8), ("f32", 64)])
def test_zoh_decode_matches_oracle(dtype, N):
    S, D, R = 12, 72, 5
    rng = np.random.default_rng(330 + N)
    _, Dsk, bias0 = workloads.channel_params(rng, D, N)
    A = -rng.uniform(0.0, 2.0, size=(D, N)).astype(np.float32)
    A[::3, 0] = 0.0
    A[1::3, -1] = -40.0
    bias = (bias0 + np.where(np.arange(D) % 4 == 0, 3.0, 0.0)).astype(np.float32)
    pool0 = rng.standard_normal((S, D, N)).astype(np.float32)
    slots = rng.permutation(S)[:R].astype(np.int32)
    tok = {k: rng.standard_normal(shape).astype(np.float32)
           for k, shape in (("u", (R, D)), ("delta", (R, D)), ("z", (R, D)), ("B", (R, N)), ("C", (R, N)))}
    if dtype == "bf16":
        tok = {k: workloads.round_to_bf16(v) for k, v in tok.items()}
    pool_t = torch.from_numpy(pool0).cuda()
    At, Dt, bt = (torch.from_numpy(x).cuda() for x in (A, Dsk, bias))
    y = ssm.state_update(pool_t, torch.from_numpy(slots).cuda(), dev(tok["u"], dtype), dev(tok["delta"], dtype),
                         dev(tok["B"], dtype), dev(tok["C"], dtype), At, Dt, bt, dev(tok["z"], dtype), zoh=True)
    torch.cuda.synchronize()
    assert ssm.device_status() == 0
    pool = pool0.astype(np.float64)
    pool_mag = np.abs(pool)
    ref = oracle.state_update(pool, slots, tok["u"], tok["delta"], tok["B"], tok["C"], A, Dsk, bias, tok["z"],
                              pool_mag=pool_mag, zoh=True)
    check("y", host(y), ref["y"], ref["y_mag"], TOL[dtype], dtype)
    check("pool", host(pool_t)[slots], pool[slots], pool_mag[slots], TOL[dtype])
    others = np.setdiff1d(np.arange(S), slots)
    assert np.array_equal(pool_t.cpu().numpy()[others], pool0[others])
