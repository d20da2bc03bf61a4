"""GPU parity of the packed prefill into a state pool (ssm_scan_fwd_varlen_pool) against the
fp64 oracle: prompts fed in two pieces through the pool, then a decode step on the same pool.

Error metric as in test_scan_gpu.py: max |x - x_oracle| / m with the oracle's magnitude bound
m; gates 1e-4 (float32 inputs) and 3e-3 (bf16 inputs, plus a bf16 output's own rounding).
Slots that no sequence names must come back bitwise unchanged.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle  # noqa: E402
import selective_state_space_15_b200 as ssm  # noqa: E402
import workloads  # noqa: E402
from helpers import TOL, check, dev, host, round_up  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ssm.load()


def _pieces(cu, cuts):
    """Column indices and offsets of two packed batches: the first cuts[i] steps of every
    sequence, and the rest."""
    first, rest = [], []
    for i in range(len(cu) - 1):
        lo, hi = int(cu[i]), int(cu[i + 1])
        first.append(np.arange(lo, lo + cuts[i]))
        rest.append(np.arange(lo + cuts[i], hi))
    out = []
    for parts in (first, rest):
        idx = np.concatenate(parts).astype(np.int64)
        cu2 = np.concatenate([[0], np.cumsum([len(p) for p in parts])]).astype(np.int32)
        out.append((idx, cu2))
    return out


def _prefill(inp, idx, cu, pool_t, slots_t, dtype, pitch_mult):
    T = len(idx)
    pitch = round_up(max(T, 1), pitch_mult)
    cols = lambda a: np.ascontiguousarray(a[:, idx])  # noqa: E731
    u, dl, z = (dev(cols(x), dtype, pitch=pitch) for x in (inp.u, inp.delta, inp.z))
    B, C = dev(cols(inp.B), dtype, pitch=pitch), dev(cols(inp.C), dtype, pitch=pitch)
    A, D, bias = (torch.from_numpy(x).cuda() for x in (inp.A, inp.Dskip, inp.bias))
    y = ssm.scan_fwd_varlen_pool(u, dl, B, C, A, torch.from_numpy(cu).cuda(), pool_t, slots_t, D, bias, z, total=T)
    torch.cuda.synchronize()
    return host(y, T)


@pytest.mark.parametrize("dtype,pitch_mult", [("f32", 4), ("bf16", 8), ("bf16", 1)])
def test_two_piece_prefill_matches_one_shot_oracle(dtype, pitch_mult):
    lengths = [300, 0, 37, 1000, 64, 5]
    cuts = [128, 0, 36, 333, 64, 0]           # aligned, unaligned, whole-sequence and empty pieces
    D, N, S = 40, 16, 9
    inp = workloads.varlen_inputs(lengths, D, N, dtype, seed=71 + pitch_mult)
    rng = np.random.default_rng(72)
    pool0 = rng.standard_normal((S, D, N)).astype(np.float32)
    slots = np.array([7, 2, 0, 5, 3, 8], dtype=np.int32)
    pool_t = torch.from_numpy(pool0).cuda()
    slots_t = torch.from_numpy(slots).cuda()
    y = np.zeros(inp.u.shape)
    for idx, cu in _pieces(inp.cu_seqlens, cuts):
        y[:, idx] = _prefill(inp, idx, cu, pool_t, slots_t, dtype, pitch_mult)
    assert ssm.device_status() == 0
    pool = pool0.astype(np.float64)
    pool_mag = np.abs(pool)
    ref = oracle.scan_varlen_pool(inp.u, inp.delta, inp.B, inp.C, inp.A, inp.cu_seqlens, pool, slots, inp.Dskip,
                                  inp.bias, inp.z, pool_mag=pool_mag)
    check("y", y, ref["y"], ref["y_mag"], TOL[dtype], dtype)
    got = host(pool_t)
    check("pool", got[slots], pool[slots], pool_mag[slots], TOL[dtype])
    others = np.setdiff1d(np.arange(S), slots)
    assert np.array_equal(pool_t.cpu().numpy()[others], pool0[others])      # bitwise unchanged


def test_prefill_then_decode_on_the_same_pool():
    lengths = [250, 97]
    D, N, S = 24, 16, 4
    inp = workloads.varlen_inputs(lengths, D, N, "bf16", seed=73)
    slots = np.array([3, 1], dtype=np.int32)
    pool_t = torch.zeros((S, D, N), dtype=torch.float32, device="cuda")
    slots_t = torch.from_numpy(slots).cuda()
    T = inp.meta["total"]
    _prefill(inp, np.arange(T), inp.cu_seqlens, pool_t, slots_t, "bf16", 8)
    pool = np.zeros((S, D, N))
    pool_mag = np.zeros_like(pool)
    oracle.scan_varlen_pool(inp.u, inp.delta, inp.B, inp.C, inp.A, inp.cu_seqlens, pool, slots, inp.Dskip,
                            inp.bias, inp.z, pool_mag=pool_mag)
    # one decode token per request on the prefilled states
    rng = np.random.default_rng(74)
    tok = {k: workloads.round_to_bf16(rng.standard_normal(shape).astype(np.float32))
           for k, shape in (("u", (2, D)), ("delta", (2, D)), ("z", (2, D)), ("B", (2, N)), ("C", (2, N)))}
    bf = lambda a: torch.from_numpy(a).cuda().to(torch.bfloat16)  # noqa: E731
    A, Dk, bias = (torch.from_numpy(x).cuda() for x in (inp.A, inp.Dskip, inp.bias))
    y = ssm.state_update(pool_t, slots_t, bf(tok["u"]), bf(tok["delta"]), bf(tok["B"]), bf(tok["C"]), A, Dk, bias,
                         bf(tok["z"]))
    torch.cuda.synchronize()
    ref = oracle.state_update(pool, slots, tok["u"], tok["delta"], tok["B"], tok["C"], inp.A, inp.Dskip, inp.bias,
                              tok["z"], pool_mag=pool_mag)
    check("decode y", host(y), ref["y"], ref["y_mag"], TOL["bf16"], "bf16")
    check("pool", host(pool_t)[slots], pool[slots], pool_mag[slots], TOL["bf16"])
    assert ssm.device_status() == 0


def test_bad_slot_starts_from_zero_and_leaves_the_pool():
    lengths = [64, 80]
    D, N, S = 16, 16, 3
    inp = workloads.varlen_inputs(lengths, D, N, "f32", seed=75)
    pool0 = np.full((S, D, N), 0.5, dtype=np.float32)
    slots = np.array([5, 1], dtype=np.int32)             # 5 is out of range
    pool_t = torch.from_numpy(pool0).cuda()
    T = inp.meta["total"]
    y = _prefill(inp, np.arange(T), inp.cu_seqlens, pool_t, torch.from_numpy(slots).cuda(), "f32", 4)
    assert ssm.device_status() == 4                      # SSM_ERR_BAD_SLOT, read and cleared
    assert ssm.device_status() == 0
    pool = pool0.astype(np.float64)
    pool_mag = np.abs(pool)
    ref = oracle.scan_varlen_pool(inp.u, inp.delta, inp.B, inp.C, inp.A, inp.cu_seqlens, pool, slots, inp.Dskip,
                                  inp.bias, inp.z, pool_mag=pool_mag)
    check("y", y, ref["y"], ref["y_mag"], TOL["f32"])
    got = pool_t.cpu().numpy()
    assert np.array_equal(got[0], pool0[0]) and np.array_equal(got[2], pool0[2])
    check("pool[1]", got[1].astype(np.float64), pool[1], pool_mag[1], TOL["f32"])
