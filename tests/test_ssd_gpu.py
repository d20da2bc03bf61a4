"""GPU parity of the SSD (Mamba-2 chunked) kernel, ssm_ssd_fwd, against the fp64 sequential-scan
oracle.

With a scalar A per head and Delta shared by the head's channels, the SSD recurrence is the
selective scan with A[d][n] = A[h] for the channels d = h P + p of head h, Delta given directly
and no skip term or gate.  The scan oracle takes Delta through softplus(delta + bias), so it is
fed delta = log(expm1(Delta)) (softplus of which returns Delta to fp64 rounding) and no bias;
it also returns the magnitude bounds used by the error metric (max |x - x_oracle| / m).  The
kernel rounds the operands it computes (M, V, C', H) to float16 (11 significant bits) and sums
in float32, so its error is a few times 2^-11 of the magnitude bound: the bf16 gate (3e-3)
applies, and the bf16 output y gets its half-ulp allowance on top.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle  # noqa: E402
import selective_state_space_15_b200 as ssm  # noqa: E402
import workloads  # noqa: E402
from helpers import TOL, check, host  # noqa: E402

NTHREADS = oracle.default_threads()


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ssm.load()


def run_ssd(inp):
    bf = lambda a: torch.from_numpy(a).cuda().to(torch.bfloat16)  # noqa: E731
    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    h0 = f32(inp.h0) if inp.h0 is not None else None
    y, hl = ssm.ssd_fwd(bf(inp.x), f32(inp.dt), f32(inp.A), bf(inp.B), bf(inp.C), h0)
    torch.cuda.synchronize()
    return host(y), host(hl)


def oracle_ssd(inp, heads=None):
    """The scan oracle on the channels of the given heads (all by default)."""
    b, H, P, L = inp.x.shape
    N = inp.B.shape[1]
    heads = np.arange(H) if heads is None else np.asarray(heads)
    u = inp.x[:, heads].reshape(b, len(heads) * P, L)
    dt = np.repeat(inp.dt[:, heads].astype(np.float64), P, axis=1)          # [b, D, L]
    delta = np.log(np.expm1(dt))                                             # softplus^-1
    A = np.repeat(inp.A[heads].astype(np.float64), P)[:, None] * np.ones((1, N))
    h0 = None if inp.h0 is None else inp.h0[:, heads].reshape(b, len(heads) * P, N)
    r = oracle.scan(u, delta, inp.B, inp.C, A, None, None, None, h0, nthreads=NTHREADS)
    sh = (b, len(heads), P)
    return (r["y"].reshape(sh + (L,)), r["y_mag"].reshape(sh + (L,)), r["h_last"].reshape(sh + (N,)),
            r["h_mag"].reshape(sh + (N,)))


@pytest.mark.parametrize("shape,h0", [
    ((1, 1, 64, 128, 128), False),    # one chunk, one CTA
    ((1, 2, 64, 128, 256), True),     # two chunks: the state carried between them, an initial state
    ((2, 3, 64, 128, 1000), True),    # a ragged last chunk (1000 = 7 x 128 + 104)
    ((1, 2, 64, 128, 8), False),      # a single 8-step stretch
])
def test_ssd_small_full(shape, h0):
    b, H, P, N, L = shape
    inp = workloads.ssd_inputs(b, H, P, N, L, seed=900 + L + H, h0=h0)
    y, hl = run_ssd(inp)
    ry, my, rh, mh = oracle_ssd(inp)
    check("y", y, ry, my, TOL["bf16"], "bf16")
    check("h_last", hl, rh, mh, TOL["bf16"])


def test_ssd_bench_shape_sampled():
    """The SSD bench shape (4 sequences x 32 heads x 64 channels, N = 128, L = 4096), heads sampled."""
    inp = workloads.ssd_inputs(4, 32, 64, 128, 4096, seed=910)
    y, hl = run_ssd(inp)
    heads = np.array([0, 13, 31])
    ry, my, rh, mh = oracle_ssd(inp, heads)
    check("y", y[:, heads], ry, my, TOL["bf16"], "bf16")
    check("h_last", hl[:, heads], rh, mh, TOL["bf16"])
    assert np.all(np.isfinite(y))


def test_ssd_host_rejections():
    import ctypes
    lib = ssm.load()
    p = ssm.SsdParams()
    p.batch, p.nheads, p.headdim, p.dstate, p.seqlen = 1, 1, 64, 128, 128
    assert lib.ssm_ssd_fwd(ctypes.byref(p), None) == 1                   # no tensors
    fake = 0x10000
    p.x = p.dt = p.A = p.B = p.C = p.y = fake
    p.headdim = 32
    assert lib.ssm_ssd_fwd(ctypes.byref(p), None) == 2                   # head dim 64 only
    p.headdim, p.seqlen = 64, 100
    assert lib.ssm_ssd_fwd(ctypes.byref(p), None) == 2                   # seqlen a multiple of 8


@pytest.mark.parametrize("shape,h0", [
    ((1, 2, 64, 128, 384), True),     # three chunks, initial state
    ((2, 3, 64, 128, 200), False),    # ragged last chunk
])
def test_ssd_against_the_chunked_ssd_oracle(shape, h0):
    """The kernel against oracle/ssd.py's fp64 chunked form (itself pinned against the scan
    oracle on the CPU), with the same 128-step chunking: y within the bf16 budget of the
    oracle's own output scale per head, h_last likewise."""
    from oracle.ssd import ssd_chunked
    b, H, P, N, L = shape
    inp = workloads.ssd_inputs(b, H, P, N, L, seed=930 + L + H, h0=h0)
    y, hl = run_ssd(inp)
    for s in range(b):
        ry, rh = ssd_chunked(inp.x[s], inp.dt[s], inp.A, inp.B[s], inp.C[s], 128,
                             None if inp.h0 is None else inp.h0[s])
        for h in range(H):
            ey = np.max(np.abs(y[s, h] - ry[h])) / np.max(np.abs(ry[h]))
            eh = np.max(np.abs(hl[s, h] - rh[h])) / np.max(np.abs(rh[h]))
            assert ey <= TOL["bf16"] + 2.0 ** -8 and eh <= TOL["bf16"], (s, h, ey, eh)
