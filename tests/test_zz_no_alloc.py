"""GPU test of ssm_scan_fwd_noalloc, the scan entry point that allocates nothing.

Callers such as an inference-engine plugin (whose enqueue step must not allocate) or a
serving loop that bans cudaMalloc after start-up (cudaMalloc can synchronise the device)
cannot hand the scan a freshly allocated workspace.  ssm_scan_fwd_noalloc uses a static
scratch array inside the library instead.  This file checks, through the C ABI, that two
calls in a row give the same outputs as ssm_scan_fwd with a caller-provided workspace.
It is collected last so that a run stopping at the first failure has run everything else.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import selective_state_space_15_b200 as ssm  # noqa: E402
import workloads  # noqa: E402
from helpers import TOL, check, dev, host  # noqa: E402


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = ssm.load()
    # a fixed-length batch that runs on the persistent path, so the scratch is really used
    inp = workloads.batch_inputs(2, 40, 16, 2048, "bf16", seed=41)
    u, dl, z, B, C = (dev(x, "bf16") for x in (inp.u, inp.delta, inp.z, inp.B, inp.C))
    A, D, bias = (torch.from_numpy(x).cuda() for x in (inp.A, inp.Dskip, inp.bias))
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    y_ref, h_ref = ssm.scan_fwd(u, dl, B, C, A, D, bias, z)          # caller-provided workspace
    torch.cuda.synchronize()
    p_ref = ssm.scan_params(u, dl, B, C, A, D, bias, z, None, y_ref, h_ref)
    need = lib.ssm_scan_workspace_size(ctypes.byref(p_ref), 0)
    assert 0 < need <= ssm.NOALLOC_SCRATCH_BYTES

    ref = oracle.scan(inp.u, inp.delta, inp.B, inp.C, inp.A, inp.Dskip, inp.bias, inp.z)
    for call in range(2):
        y = torch.full_like(u, float("nan"))
        h = torch.full_like(h_ref, float("nan"))
        p = ssm.scan_params(u, dl, B, C, A, D, bias, z, None, y, h)
        assert lib.ssm_scan_fwd_noalloc(ctypes.byref(p), stream) == 0
        torch.cuda.synchronize()
        check(f"y vs ssm_scan_fwd (call {call})", host(y), host(y_ref), ref["y_mag"], TOL["bf16"])
        check(f"h_last vs ssm_scan_fwd (call {call})", host(h), host(h_ref), ref["h_mag"], TOL["bf16"])
        check(f"y vs oracle (call {call})", host(y), ref["y"], ref["y_mag"], TOL["bf16"], "bf16")
    assert ssm.device_status() == 0


@pytest.mark.gpu
def test_noalloc_hands_state_between_units_through_the_scratch():
    """A single long sequence of 2560 channels runs on the chunked kernel's narrow tile: 640
    chains, more than the CTA slots, so every chain is split into units that hand their state
    on through the flags and carries in the static scratch (not only its ticket).  Two calls in
    a row match ssm_scan_fwd with a caller workspace, and sampled channels match the oracle."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = ssm.load()
    inp = workloads.batch_inputs(1, 2560, 16, 8192, "bf16", seed=42)
    u, dl, z, B, C = (dev(x, "bf16") for x in (inp.u, inp.delta, inp.z, inp.B, inp.C))
    A, D, bias = (torch.from_numpy(x).cuda() for x in (inp.A, inp.Dskip, inp.bias))
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    y_ref, h_ref = ssm.scan_fwd(u, dl, B, C, A, D, bias, z, algorithm="chunked")
    torch.cuda.synchronize()
    p_ref = ssm.scan_params(u, dl, B, C, A, D, bias, z, None, y_ref, h_ref, algorithm="chunked")
    need = lib.ssm_scan_workspace_size(ctypes.byref(p_ref), 0)
    assert 640 * 4 < need <= ssm.NOALLOC_SCRATCH_BYTES     # flags and carries, not only the ticket
    ch = np.arange(3, 2560, 157)
    ref = oracle.scan(inp.u[:, ch], inp.delta[:, ch], inp.B, inp.C, inp.A[ch], inp.Dskip[ch], inp.bias[ch],
                      inp.z[:, ch], nthreads=oracle.default_threads())
    for call in range(2):
        y = torch.full_like(u, float("nan"))
        h = torch.full_like(h_ref, float("nan"))
        p = ssm.scan_params(u, dl, B, C, A, D, bias, z, None, y, h, algorithm="chunked")
        assert lib.ssm_scan_fwd_noalloc(ctypes.byref(p), stream) == 0
        torch.cuda.synchronize()
        assert torch.equal(y, y_ref) and torch.equal(h, h_ref), f"call {call}"
        check(f"y vs oracle (call {call})", host(y)[:, ch], ref["y"], ref["y_mag"], TOL["bf16"], "bf16")
        check(f"h_last vs oracle (call {call})", host(h)[:, ch], ref["h_last"], ref["h_mag"], TOL["bf16"])
    assert ssm.device_status() == 0
