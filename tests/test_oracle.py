"""Pins for the fp64 oracle, independent of the oracle's own code (CPU only).

Each check compares the oracle with something the pages or plain mathematics fix, chosen so
that a plausible slip (a dropped term, a sign, h_{t-1} instead of h_t, B and C swapped, A
transposed, a wrong reset) fails at least one of them:
  * a hand-derived worked example (tests/golden/worked_example.json);
  * a 50-digit decimal brute force of the unrolled sum (oracle/brute.py);
  * the time-invariant case equals a causal convolution (discosf.com §1.1: "train with the
    convolution, infer with the recurrence"; kj168168.com §三.3 kernel of decaying powers);
  * A = 0 reduces the state to a cumulative sum;
  * chunk transfer operators compose to the sequential result (ufo.work §3.1);
  * varlen equals independent scans; L decode steps equal one scan (ufo.work §4.1, §4.2);
  * extreme step sizes (ufo.work §6 pitfall 1: Δ large must not overflow).
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle import brute
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_example.json")


def _rand_problem(rng, b, D, N, L, gate=True, h0=True, A_range=(0.2, 3.0)):
    u = rng.standard_normal((b, D, L))
    delta = rng.standard_normal((b, D, L))
    z = rng.standard_normal((b, D, L)) if gate else None
    B = rng.standard_normal((b, N, L))
    C = rng.standard_normal((b, N, L))
    A = -rng.uniform(*A_range, size=(D, N))
    Dskip = rng.standard_normal(D)
    bias = rng.uniform(-3.0, 1.0, size=D)
    h = rng.standard_normal((b, D, N)) if h0 else None
    return dict(u=u, delta=delta, z=z, B=B, C=C, A=A, Dskip=Dskip, bias=bias, h0=h)


def test_golden_worked_example():
    g = json.load(open(GOLDEN))
    c = g["common"]
    ln2 = math.log(2.0)
    shape = (1, 1, 4)
    for case in g["cases"]:
        u = np.array(c["u"]).reshape(shape)
        z = None if case["z"] is None else np.array(case["z"]).reshape(shape)
        h0 = None if case["h0"] is None else np.array(case["h0"]).reshape(1, 1, 2)
        out = oracle.scan(u, np.array(c["delta"]).reshape(shape), np.array(c["B"])[None],
                          np.array(c["C"])[None], np.array(c["A"]), Dskip=np.array(c["Dskip"]),
                          bias=np.array(c["bias"]), z=z, h0=h0)
        y_exp = np.array([a * ln2 + k for a, k in case["y"]])
        if "silu" in case:
            y_exp = y_exp * np.array(case["silu"])
        h_exp = np.array([a * ln2 + k for a, k in case["h_last"]])
        np.testing.assert_allclose(out["y"].ravel(), y_exp, rtol=1e-14, atol=1e-15, err_msg=case["name"])
        np.testing.assert_allclose(out["h_last"].ravel(), h_exp, rtol=1e-14, atol=1e-15, err_msg=case["name"])
        assert np.all(out["y_mag"] >= np.abs(out["y"]) * (1 - 1e-15))


@pytest.mark.parametrize("shape,gate,h0,seed", [
    ((1, 1, 1, 1), False, False, 0),
    ((1, 2, 3, 7), True, True, 1),
    ((2, 2, 4, 12), True, False, 2),
    ((1, 2, 4, 10), False, True, 3),
])
def test_brute_force_tiny(shape, gate, h0, seed):
    b, D, N, L = shape
    p = _rand_problem(np.random.default_rng(seed), b, D, N, L, gate, h0)
    out = oracle.scan(**p)
    y_ref, h_ref = brute.scan(p["u"], p["delta"], p["B"], p["C"], p["A"], p["Dskip"], p["bias"], p["z"], p["h0"])
    assert oracle.scaled_error(out["y"], y_ref, out["y_mag"]) < 1e-13
    assert oracle.scaled_error(out["h_last"], h_ref, out["h_mag"]) < 1e-13


def test_brute_force_catches_swapped_B_C():
    # B and C play different roles; swapping them must change the result well beyond rounding.
    p = _rand_problem(np.random.default_rng(11), 1, 2, 3, 6)
    out = oracle.scan(**p)
    y_swapped, _ = brute.scan(p["u"], p["delta"], p["C"], p["B"], p["A"], p["Dskip"], p["bias"], p["z"], p["h0"])
    assert oracle.scaled_error(out["y"], y_swapped, out["y_mag"]) > 1e-3


def _delta_for_steps(steps, bias):
    """δ such that softplus(δ + bias) = steps exactly in real arithmetic (inverse softplus)."""
    return np.log(np.expm1(steps)) - bias


def test_time_invariant_equals_causal_convolution():
    rng = np.random.default_rng(5)
    D, N, L = 3, 5, 64
    steps = np.array([0.01, 0.2, 1.3])               # constant Δ per channel
    bias = rng.uniform(-2, 0, size=D)
    delta = np.repeat(_delta_for_steps(steps, bias)[:, None], L, axis=1)[None]
    beta = rng.standard_normal(N)
    gamma = rng.standard_normal(N)
    B = np.repeat(beta[:, None], L, axis=1)[None]
    C = np.repeat(gamma[:, None], L, axis=1)[None]
    A = -rng.uniform(0.1, 2.0, size=(D, N))
    Dskip = rng.standard_normal(D)
    u = rng.standard_normal((1, D, L))
    out = oracle.scan(u, delta, B, C, A, Dskip=Dskip, bias=bias)
    j = np.arange(L)
    for d in range(D):
        # K_j = sum_n C_n exp(j Δ A_n) Δ B_n, then y = K * u + D u (causal convolution).
        K = (gamma[None, :] * np.exp(j[:, None] * steps[d] * A[d][None, :]) * steps[d] * beta[None, :]).sum(1)
        y_conv = np.convolve(u[0, d], K)[:L] + Dskip[d] * u[0, d]
        err = np.max(np.abs(out["y"][0, d] - y_conv) / out["y_mag"][0, d])
        assert err < 1e-12, (d, err)


def test_A_zero_is_cumulative_sum():
    rng = np.random.default_rng(6)
    D, N, L = 2, 4, 50
    bias = np.zeros(D)
    delta = np.zeros((1, D, L))                      # Δ = softplus(0) = ln 2
    u = rng.standard_normal((1, D, L))
    B = rng.standard_normal((1, N, L))
    C = rng.standard_normal((1, N, L))
    Dskip = rng.standard_normal(D)
    out = oracle.scan(u, delta, B, C, np.zeros((D, N)), Dskip=Dskip, bias=bias)
    for d in range(D):
        h = np.cumsum(math.log(2.0) * B[0] * u[0, d][None, :], axis=1)   # [N, L]
        y = (C[0] * h).sum(0) + Dskip[d] * u[0, d]
        np.testing.assert_allclose(out["y"][0, d], y, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(out["h_last"][0, d], h[:, -1], rtol=1e-12, atol=1e-12)


def test_chunk_operators_compose_to_sequential():
    """h_end = Abar_chunk h_start + Bbar_chunk, composed over any chunking, equals the full scan."""
    rng = np.random.default_rng(7)
    D, N, L = 2, 3, 97
    bias = rng.uniform(-3, 0, size=D)
    steps = rng.uniform(1e-3, 0.5, size=(D, L))
    delta = _delta_for_steps(steps, bias[:, None])[None]
    u = rng.standard_normal((1, D, L))
    B = rng.standard_normal((1, N, L))
    C = rng.standard_normal((1, N, L))
    A = -rng.uniform(0.1, 3.0, size=(D, N))
    h0 = rng.standard_normal((1, D, N))
    full = oracle.scan(u, delta, B, C, A, bias=bias, h0=h0)
    for cuts in ([0, L], [0, 1, L], [0, 40, 41, 90, L], list(range(0, L, 8)) + [L], list(range(L + 1))):
        h = h0[0].copy()
        ys = []
        for s, e in zip(cuts[:-1], cuts[1:]):
            sl = slice(s, e)
            # transfer operator of the chunk: Abar = exp(A * sum Δ), Bbar = scan from zero
            zero = oracle.scan(u[..., sl], delta[..., sl], B[..., sl], C[..., sl], A, bias=bias)
            Abar = np.exp(A * steps[:, sl].sum(1)[:, None])
            h_next = Abar * h + zero["h_last"][0]
            # chained run with the carried state reproduces the chunk's outputs
            chained = oracle.scan(u[..., sl], delta[..., sl], B[..., sl], C[..., sl], A, bias=bias, h0=h[None])
            ys.append(chained["y"][0])
            np.testing.assert_allclose(chained["h_last"][0], h_next, rtol=1e-12, atol=1e-13)
            h = chained["h_last"][0]
        np.testing.assert_allclose(h, full["h_last"][0], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(np.concatenate(ys, axis=1), full["y"][0], rtol=1e-12, atol=1e-13)


def test_varlen_equals_independent_scans():
    rng = np.random.default_rng(8)
    D, N = 3, 4
    lens = [5, 1, 17, 9]
    T = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)])
    p = dict(u=rng.standard_normal((D, T)), delta=rng.standard_normal((D, T)),
             z=rng.standard_normal((D, T)), B=rng.standard_normal((N, T)), C=rng.standard_normal((N, T)))
    A = -rng.uniform(0.1, 2, size=(D, N))
    Dskip = rng.standard_normal(D)
    bias = rng.uniform(-3, 0, size=D)
    out = oracle.scan_varlen(p["u"], p["delta"], p["B"], p["C"], A, cu, Dskip=Dskip, bias=bias, z=p["z"])
    for s in range(len(lens)):
        sl = slice(cu[s], cu[s + 1])
        one = oracle.scan(p["u"][None, :, sl], p["delta"][None, :, sl], p["B"][None, :, sl],
                          p["C"][None, :, sl], A, Dskip=Dskip, bias=bias, z=p["z"][None, :, sl])
        np.testing.assert_array_equal(out["y"][:, sl], one["y"][0])
        np.testing.assert_array_equal(out["h_last"][s], one["h_last"][0])


def test_varlen_resets_state_at_boundaries():
    # Two sequences: the second must not see the first's state; compare with a zero prefix.
    rng = np.random.default_rng(9)
    D, N, T1, T2 = 2, 3, 6, 5
    u = rng.standard_normal((D, T1 + T2))
    delta = rng.standard_normal((D, T1 + T2))
    B = rng.standard_normal((N, T1 + T2))
    C = rng.standard_normal((N, T1 + T2))
    A = -np.ones((D, N)) * 0.01                       # slow decay: leakage would be visible
    out = oracle.scan_varlen(u, delta, B, C, A, [0, T1, T1 + T2])
    u2 = u.copy()
    u2[:, :T1] = 0.0                                  # zero input before the boundary = zero state
    ref = oracle.scan(u2[None], delta[None], B[None], C[None], A)
    np.testing.assert_allclose(out["y"][:, T1:], ref["y"][0, :, T1:], rtol=1e-13, atol=1e-15)


def test_decode_steps_equal_scan():
    rng = np.random.default_rng(10)
    S, D, N, L = 5, 3, 4, 9
    slots = np.array([3, 0])
    R = len(slots)
    pool = rng.standard_normal((S, D, N))
    pool_before = pool.copy()
    A = -rng.uniform(0.1, 2, size=(D, N))
    Dskip = rng.standard_normal(D)
    bias = rng.uniform(-3, 0, size=D)
    u = rng.standard_normal((L, R, D))
    delta = rng.standard_normal((L, R, D))
    z = rng.standard_normal((L, R, D))
    B = rng.standard_normal((L, R, N))
    C = rng.standard_normal((L, R, N))
    ys = []
    for t in range(L):
        ys.append(oracle.state_update(pool, slots, u[t], delta[t], B[t], C[t], A, Dskip, bias, z[t])["y"])
    ys = np.stack(ys)                                 # [L, R, D]
    for r, s in enumerate(slots):
        ref = oracle.scan(u[:, r].T[None], delta[:, r].T[None], B[:, r].T[None], C[:, r].T[None], A,
                          Dskip=Dskip, bias=bias, z=z[:, r].T[None], h0=pool_before[s][None])
        np.testing.assert_allclose(ys[:, r].T, ref["y"][0], rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(pool[s], ref["h_last"][0], rtol=1e-13, atol=1e-14)
    untouched = [s for s in range(S) if s not in slots]
    np.testing.assert_array_equal(pool[untouched], pool_before[untouched])


def test_extreme_steps():
    rng = np.random.default_rng(12)
    D, N, L = 2, 3, 5
    u = rng.standard_normal((1, D, L))
    B = rng.standard_normal((1, N, L))
    C = rng.standard_normal((1, N, L))
    A = -np.ones((D, N))
    h0 = rng.standard_normal((1, D, N))
    # Δ ≈ 30: abar = e^-30 wipes the previous state, h_t ≈ Δ B_t u_t, no overflow
    big = oracle.scan(u, np.full((1, D, L), 30.0), B, C, A, h0=h0)
    assert np.all(np.isfinite(big["y"]))
    np.testing.assert_allclose(big["h_last"][0], 30.0 * B[0, :, -1][None, :] * u[0, :, -1][:, None],
                               rtol=1e-11, atol=1e-10)
    # Δ ≈ e^-50: abar ≈ 1 and the input term vanishes, so the state stays h0
    tiny = oracle.scan(u, np.full((1, D, L), -50.0), B, C, A, h0=h0)
    np.testing.assert_allclose(tiny["h_last"], h0, rtol=1e-15, atol=1e-20)
    np.testing.assert_allclose(tiny["y"][0], np.einsum("nl,dn->dl", C[0], h0[0]), rtol=1e-12, atol=1e-14)


def test_softplus_of_generated_bias_recovers_step():
    """The workload recipe sets bias = log(expm1(dt)); the oracle's Δ = softplus(bias) must
    satisfy the defining identity e^Δ - 1 = e^bias."""
    rng = np.random.default_rng(3)
    _, _, bias = workloads.channel_params(rng, 64, 1)
    bias = bias.astype(np.float64)
    D = bias.shape[0]
    one = np.ones((1, D, 1))
    out = oracle.scan(one, np.zeros((1, D, 1)), np.ones((1, 1, 1)), np.ones((1, 1, 1)),
                      np.zeros((D, 1)), bias=bias)              # y = h = Δ · 1 · 1
    dt = out["y"][0, :, 0]
    np.testing.assert_allclose(np.expm1(dt), np.exp(bias), rtol=1e-13)
    assert dt.min() > 0.9e-3 and dt.max() < 1.1e-1


def test_scaled_error_semantics():
    ref = np.array([1.0, -2.0, 0.0])
    mag = np.array([2.0, 4.0, 0.0])
    assert oracle.scaled_error(ref, ref, mag) == 0.0
    assert oracle.scaled_error(np.array([1.5, -2.0, 0.0]), ref, mag) == pytest.approx(0.25)
    assert oracle.scaled_error(np.array([1.0, -2.0, 1e-30]), ref, mag) == float("inf")
    assert oracle.scaled_error(np.array([np.nan, -2.0, 0.0]), ref, mag) == float("inf")


def test_workload_generator_is_deterministic_and_bf16_exact():
    a = workloads.batch_inputs(1, 4, 16, 64, "bf16", seed=3)
    b = workloads.batch_inputs(1, 4, 16, 64, "bf16", seed=3)
    np.testing.assert_array_equal(a.u, b.u)
    bits = a.u.view(np.uint32)
    assert np.all((bits & 0xFFFF) == 0)               # representable in bf16
    # ties round to even: 1 + 2^-8 (exactly halfway between two bf16 values) rounds down to 1
    x = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8], dtype=np.float32)
    np.testing.assert_array_equal(workloads.round_to_bf16(x), np.array([1.0, 1.0 + 2.0 ** -6], dtype=np.float32))


def _split_packed(inp, cuts):
    """Two packed batches holding the first and the rest of each sequence (cut i in sequence i)."""
    cu = inp.cu_seqlens
    first, rest = [], []
    for i in range(len(cu) - 1):
        lo, hi = int(cu[i]), int(cu[i + 1])
        first.append(np.arange(lo, lo + cuts[i]))
        rest.append(np.arange(lo + cuts[i], hi))

    def pack(parts):
        idx = np.concatenate(parts) if parts else np.zeros(0, dtype=np.int64)
        cu2 = np.concatenate([[0], np.cumsum([len(p) for p in parts])]).astype(np.int32)
        return idx, cu2
    return pack(first), pack(rest)


def test_pool_prefill_from_zero_is_the_varlen_scan():
    """A pool of zeros: the prefill is the packed scan, and the slots receive its final states."""
    inp = workloads.varlen_inputs([37, 0, 120, 64], 6, 8, "f32", seed=41)
    slots = np.array([3, 0, 1, 4], dtype=np.int32)
    pool = np.zeros((5, 6, 8))
    got = oracle.scan_varlen_pool(inp.u, inp.delta, inp.B, inp.C, inp.A, inp.cu_seqlens, pool, slots,
                                  inp.Dskip, inp.bias, inp.z)
    ref = oracle.scan_varlen(inp.u, inp.delta, inp.B, inp.C, inp.A, inp.cu_seqlens, inp.Dskip, inp.bias, inp.z)
    assert np.allclose(got["y"], ref["y"], rtol=0, atol=1e-13)
    for i, s in enumerate(slots):
        if i == 1:
            assert np.all(pool[s] == 0.0)                   # empty sequence: the slot is untouched
        else:
            assert np.allclose(pool[s], ref["h_last"][i], rtol=0, atol=1e-13)
    assert np.all(pool[2] == 0.0)                           # slot used by nobody


def test_pool_prefill_in_two_pieces_equals_one_call():
    """Chunked prefill: feeding every prompt in two pieces through the pool gives the same
    outputs, final states and magnitude bounds as one call (the state is carried exactly)."""
    rng = np.random.default_rng(42)
    lens = [37, 5, 120, 64]
    inp = workloads.varlen_inputs(lens, 6, 8, "f32", seed=42)
    slots = np.array([2, 0, 4, 1], dtype=np.int32)
    pool0 = rng.standard_normal((5, 6, 8))
    mag0 = np.abs(pool0) * 1.5                              # a bound looser than |pool|
    pool_a, mag_a = pool0.copy(), mag0.copy()
    one = oracle.scan_varlen_pool(inp.u, inp.delta, inp.B, inp.C, inp.A, inp.cu_seqlens, pool_a, slots,
                                  inp.Dskip, inp.bias, inp.z, pool_mag=mag_a)
    (i1, cu1), (i2, cu2) = _split_packed(inp, [10, 0, 77, 64])
    pool_b, mag_b = pool0.copy(), mag0.copy()
    y = np.zeros_like(one["y"])
    y_mag = np.zeros_like(one["y_mag"])
    for idx, cu in ((i1, cu1), (i2, cu2)):
        r = oracle.scan_varlen_pool(inp.u[:, idx], inp.delta[:, idx], inp.B[:, idx], inp.C[:, idx], inp.A, cu,
                                    pool_b, slots, inp.Dskip, inp.bias, inp.z[:, idx], pool_mag=mag_b)
        y[:, idx] = r["y"]
        y_mag[:, idx] = r["y_mag"]
    assert np.allclose(y, one["y"], rtol=1e-12, atol=1e-13)
    assert np.allclose(pool_b, pool_a, rtol=1e-12, atol=1e-13)
    assert np.allclose(y_mag, one["y_mag"], rtol=1e-12, atol=1e-13)
    assert np.allclose(mag_b, mag_a, rtol=1e-12, atol=1e-13)
    assert np.all(np.abs(one["y"]) <= one["y_mag"] * (1 + 1e-12))


def test_pool_prefill_bad_slot_starts_from_zero_and_writes_nothing():
    inp = workloads.varlen_inputs([20, 30], 4, 8, "f32", seed=43)
    pool = np.ones((3, 4, 8))
    before = pool.copy()
    got = oracle.scan_varlen_pool(inp.u, inp.delta, inp.B, inp.C, inp.A, inp.cu_seqlens, pool,
                                  np.array([7, 1], dtype=np.int32), inp.Dskip, inp.bias, inp.z)
    ref = oracle.scan_varlen(inp.u, inp.delta, inp.B, inp.C, inp.A, inp.cu_seqlens, inp.Dskip, inp.bias, inp.z)
    assert np.allclose(got["y"][:, :20], ref["y"][:, :20], rtol=0, atol=1e-13)   # from zero
    assert np.array_equal(pool[0], before[0]) and np.array_equal(pool[2], before[2])
    assert not np.array_equal(pool[1], before[1])


def test_grouped_scan_with_equal_groups_is_the_plain_scan():
    """Channel groups that all carry the same B and C reduce to the ungrouped scan."""
    inp = workloads.batch_inputs(2, 12, 8, 40, "f32", seed=51)
    B4 = np.repeat(inp.B[:, None], 3, axis=1)
    C4 = np.repeat(inp.C[:, None], 3, axis=1)
    g = oracle.scan(inp.u, inp.delta, B4, C4, inp.A, inp.Dskip, inp.bias, inp.z)
    r = oracle.scan(inp.u, inp.delta, inp.B, inp.C, inp.A, inp.Dskip, inp.bias, inp.z)
    for k in ("y", "h_last", "y_mag", "h_mag"):
        np.testing.assert_array_equal(g[k], r[k])


def test_grouped_scan_reads_each_groups_own_b_and_c():
    """Swapping the B/C of two groups equals swapping which channels sit in which group."""
    rng = np.random.default_rng(52)
    bsz, D, N, L, G = 1, 8, 4, 30, 2
    u, dl, z = (rng.standard_normal((bsz, D, L)) for _ in range(3))
    B, C = rng.standard_normal((bsz, G, N, L)), rng.standard_normal((bsz, G, N, L))
    A = -rng.uniform(0.1, 2, size=(D, N))
    Dk, bias = rng.standard_normal(D), rng.uniform(-3, 0, size=D)
    out = oracle.scan(u, dl, B, C, A, Dk, bias, z)
    perm = np.r_[D // 2:D, 0:D // 2]                     # group 1's channels first
    sw = oracle.scan(u[:, perm], dl[:, perm], B[:, ::-1], C[:, ::-1], A[perm], Dk[perm], bias[perm], z[:, perm])
    np.testing.assert_array_equal(sw["y"][:, perm.argsort()], out["y"])
    np.testing.assert_array_equal(sw["h_last"][:, perm.argsort()], out["h_last"])
    # and group 0 really uses B[:, 0]: a plain scan of its channels with B[:, 0]
    one = oracle.scan(u[:, :4], dl[:, :4], B[:, 0], C[:, 0], A[:4], Dk[:4], bias[:4], z[:, :4])
    np.testing.assert_array_equal(out["y"][:, :4], one["y"])


def test_grouped_varlen_matches_grouped_fixed_length_per_sequence():
    inp = workloads.varlen_inputs([23, 40], 6, 4, "f32", seed=53)
    rng = np.random.default_rng(54)
    T = inp.meta["total"]
    B3, C3 = rng.standard_normal((3, 4, T)), rng.standard_normal((3, 4, T))
    v = oracle.scan_varlen(inp.u, inp.delta, B3, C3, inp.A, inp.cu_seqlens, inp.Dskip, inp.bias, inp.z)
    cu = inp.cu_seqlens
    for s in range(2):
        sl = slice(cu[s], cu[s + 1])
        f = oracle.scan(inp.u[None, :, sl], inp.delta[None, :, sl], B3[None, :, :, sl], C3[None, :, :, sl], inp.A,
                        inp.Dskip, inp.bias, inp.z[None, :, sl])
        np.testing.assert_array_equal(v["y"][:, sl], f["y"][0])
        np.testing.assert_array_equal(v["h_last"][s], f["h_last"][0])


# ---- zero-order hold (discosf.com §1.2: Bbar = (Δ A)^-1 (exp(Δ A) - I) Δ B) ----

def _zoh_exact_reference(p):
    """The continuous system h' = A h + B u with u and B held over each step of length Δ, solved
    exactly per (channel, state) by the matrix exponential of the augmented system
    [[A, B u], [0, 0]] Δ (scipy's Padé expm; independent of the oracle's closed form)."""
    from scipy.linalg import expm
    b, D, L = p["u"].shape
    N = p["A"].shape[1]
    h = p["h0"].copy() if p["h0"] is not None else np.zeros((b, D, N))
    y = np.zeros((b, D, L))
    for bb in range(b):
        for d in range(D):
            for t in range(L):
                dt = np.logaddexp(0.0, p["delta"][bb, d, t] + p["bias"][d])
                acc = 0.0
                for n in range(N):
                    M = np.array([[p["A"][d, n], p["B"][bb, n, t] * p["u"][bb, d, t]], [0.0, 0.0]]) * dt
                    h[bb, d, n] = (expm(M) @ np.array([h[bb, d, n], 1.0]))[0]
                    acc += p["C"][bb, n, t] * h[bb, d, n]
                yt = acc + p["Dskip"][d] * p["u"][bb, d, t]
                if p["z"] is not None:
                    zz = p["z"][bb, d, t]
                    yt *= zz / (1.0 + np.exp(-zz))
                y[bb, d, t] = yt
    return y, h


@pytest.mark.parametrize("seed,A_range", [(90, (0.2, 3.0)), (91, (1e-4, 0.05)), (92, (2.0, 40.0))])
def test_zoh_step_is_the_exact_ode_solution(seed, A_range):
    rng = np.random.default_rng(seed)
    p = _rand_problem(rng, 2, 3, 4, 7, A_range=A_range)
    out = oracle.scan(p["u"], p["delta"], p["B"], p["C"], p["A"], p["Dskip"], p["bias"], p["z"], p["h0"], zoh=True)
    y_ref, h_ref = _zoh_exact_reference(p)
    np.testing.assert_allclose(out["y"], y_ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(out["h_last"], h_ref, rtol=1e-11, atol=1e-12)
    # and it is not the Euler input matrix
    eul = oracle.scan(p["u"], p["delta"], p["B"], p["C"], p["A"], p["Dskip"], p["bias"], p["z"], p["h0"])
    assert np.abs(eul["h_last"] - h_ref).max() > 1e-6


def test_zoh_with_A_zero_is_euler():
    rng = np.random.default_rng(93)
    p = _rand_problem(rng, 1, 3, 4, 9)
    p["A"][:] = 0.0
    a = oracle.scan(p["u"], p["delta"], p["B"], p["C"], p["A"], p["Dskip"], p["bias"], p["z"], p["h0"], zoh=True)
    e = oracle.scan(p["u"], p["delta"], p["B"], p["C"], p["A"], p["Dskip"], p["bias"], p["z"], p["h0"])
    assert np.array_equal(a["y"], e["y"]) and np.array_equal(a["h_last"], e["h_last"])


def test_zoh_varlen_and_decode_agree_with_the_fixed_length_scan():
    rng = np.random.default_rng(94)
    D, N = 3, 4
    lengths = [5, 0, 3, 8]
    T = sum(lengths)
    cu = np.concatenate([[0], np.cumsum(lengths)])
    p = _rand_problem(rng, 1, D, N, T, h0=False)
    v = oracle.scan_varlen(p["u"][0], p["delta"][0], p["B"][0], p["C"][0], p["A"], cu, p["Dskip"], p["bias"],
                           p["z"][0], zoh=True)
    pool = np.zeros((len(lengths), D, N))
    for i, (lo, hi) in enumerate(zip(cu[:-1], cu[1:])):
        sl = slice(lo, hi)
        r = oracle.scan(p["u"][:, :, sl], p["delta"][:, :, sl], p["B"][:, :, sl], p["C"][:, :, sl], p["A"],
                        p["Dskip"], p["bias"], p["z"][:, :, sl], zoh=True)
        np.testing.assert_allclose(v["y"][:, sl], r["y"][0], rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(v["h_last"][i], r["h_last"][0], rtol=1e-13, atol=1e-14)
        # the same sequence token by token through the decode step
        for t in range(lo, hi):
            dec = oracle.state_update(pool, [i], p["u"][0, :, t][None], p["delta"][0, :, t][None],
                                      p["B"][0, :, t][None], p["C"][0, :, t][None], p["A"], p["Dskip"], p["bias"],
                                      p["z"][0, :, t][None], zoh=True)
            np.testing.assert_allclose(dec["y"][0], v["y"][:, t], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(pool[i], v["h_last"][i], rtol=1e-12, atol=1e-13)


# ---- backward: the reverse-mode derivative of the scan (ufo.work §2.2 discusses how training
# ---- keeps or recomputes the states; the values follow from the forward definition) ----

_GRAD_OF = {"u": "du", "delta": "ddelta", "z": "dz", "B": "dB", "C": "dC", "A": "dA", "Dskip": "dDskip",
            "bias": "dbias", "h0": "dh0"}


@pytest.mark.parametrize("zoh", [False, True])
@pytest.mark.parametrize("gate,h0,A_range,seed", [(True, True, (0.2, 3.0), 400), (False, False, (1e-4, 0.05), 401),
                                                  (True, False, (2.0, 40.0), 402)])
def test_backward_matches_central_differences(zoh, gate, h0, A_range, seed):
    """<grad, V> equals the central difference of L = <dy, y> + <dh_last, h_last> along V, for a
    random direction V of every input (fp64, step 1e-6)."""
    rng = np.random.default_rng(seed + 10 * zoh)
    p = _rand_problem(rng, 2, 3, 4, 9, gate=gate, h0=h0, A_range=A_range)
    p["A"][0, 1] = 0.0                              # the A = 0 limit of the zero-order hold
    if p["h0"] is None:
        p["h0"] = np.zeros((2, 3, 4))
    dy = rng.standard_normal(p["u"].shape)
    dhl = rng.standard_normal((2, 3, 4))
    g = oracle.scan_bwd(p["u"], p["delta"], p["B"], p["C"], p["A"], dy, p["Dskip"], p["bias"], p["z"], p["h0"],
                        dhl, zoh=zoh)

    def loss(q):
        r = oracle.scan(q["u"], q["delta"], q["B"], q["C"], q["A"], q["Dskip"], q["bias"], q["z"], q["h0"], zoh=zoh)
        return float((r["y"] * dy).sum() + (r["h_last"] * dhl).sum())

    eps = 1e-6
    for name, gname in _GRAD_OF.items():
        if p[name] is None:
            assert g[gname] is None
            continue
        V = rng.standard_normal(p[name].shape)
        plus, minus = dict(p), dict(p)
        plus[name] = p[name] + eps * V
        minus[name] = p[name] - eps * V
        fd = (loss(plus) - loss(minus)) / (2 * eps)
        an = float((g[gname] * V).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


def test_backward_of_the_cumulative_sum_case():
    """A = 0, Euler, no gate, no skip: h_t = sum_{s<=t} Delta_s B_s u_s and y_t = C_t . h_t, so
    dC_t = sum_d dy_t h_t and dB_s = sum_d Delta_s u_s sum_{t>=s} dy_t C_t (reverse cumsum)."""
    rng = np.random.default_rng(403)
    b, D, N, L = 2, 3, 4, 11
    p = _rand_problem(rng, b, D, N, L, gate=False, h0=False)
    p["A"][:] = 0.0
    dy = rng.standard_normal((b, D, L))
    g = oracle.scan_bwd(p["u"], p["delta"], p["B"], p["C"], p["A"], dy, None, p["bias"])
    dt = np.logaddexp(0.0, p["delta"] + p["bias"][None, :, None])            # [b, D, L]
    h = np.cumsum(dt[:, :, None, :] * p["B"][:, None] * p["u"][:, :, None, :], axis=-1)   # [b, D, N, L]
    dC = np.einsum("bdt,bdnt->bnt", dy, h)
    rc = np.flip(np.cumsum(np.flip(dy[:, :, None, :] * p["C"][:, None], -1), -1), -1)       # sum_{t>=s}
    dB = np.einsum("bds,bdns->bns", dt * p["u"], rc)
    np.testing.assert_allclose(g["dC"], dC, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g["dB"], dB, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g["dDskip"], np.einsum("bdt,bdt->d", dy, p["u"]), rtol=1e-12, atol=1e-12)


def test_backward_is_independent_of_the_thread_count():
    rng = np.random.default_rng(404)
    p = _rand_problem(rng, 3, 5, 4, 13)
    dy = rng.standard_normal(p["u"].shape)
    args = (p["u"], p["delta"], p["B"], p["C"], p["A"], dy, p["Dskip"], p["bias"], p["z"], p["h0"])
    g1 = oracle.scan_bwd(*args, nthreads=1)
    g4 = oracle.scan_bwd(*args, nthreads=4)
    for k in g1:
        np.testing.assert_allclose(g4[k], g1[k], rtol=1e-13, atol=1e-13, err_msg=k)


# ---- the chunked SSD form (ufo.work second article §1.1, §2.2), scalar A per head ----

@pytest.mark.parametrize("chunk", [1, 5, 16, 64])
def test_ssd_chunked_form_equals_the_sequential_scan(chunk):
    from oracle import ssd
    rng = np.random.default_rng(500 + chunk)
    H, P, N, L = 3, 4, 8, 37
    x = rng.standard_normal((H, P, L))
    dt = np.exp(rng.uniform(np.log(1e-3), np.log(0.5), size=(H, L)))
    A = -rng.uniform(0.5, 8.0, size=H)
    B = rng.standard_normal((N, L))
    C = rng.standard_normal((N, L))
    h0 = rng.standard_normal((H, P, N))
    y, hl = ssd.ssd_chunked(x, dt, A, B, C, chunk, h0)
    # the same problem as a scan over H*P channels: every channel of head h has A[d, :] = A_h
    # and delta with softplus(delta) = dt (no bias, skip or gate)
    D = H * P
    delta = np.repeat(np.log(np.expm1(dt)), P, axis=0)[None]            # [1, D, L]
    ref = oracle.scan(x.reshape(1, D, L), delta, B[None], C[None], np.repeat(A, P)[:, None] * np.ones((D, N)),
                      h0=h0.reshape(1, D, N))
    np.testing.assert_allclose(y.reshape(D, L), ref["y"][0], rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(hl.reshape(D, N), ref["h_last"][0], rtol=1e-10, atol=1e-11)


@pytest.mark.parametrize("chunk,zoh", [(1, False), (4, False), (64, False), (3, True)])
def test_chunk_checkpointed_backward_equals_the_unchunked_one(chunk, zoh):
    """ufo.work §2.2 / its second article §3.1: keeping only chunk-boundary states and
    recomputing the inside of each chunk during the backward gives the same gradients."""
    from oracle import bwd_chunked
    rng = np.random.default_rng(600 + chunk)
    p = _rand_problem(rng, 2, 3, 4, 11)
    dy = rng.standard_normal(p["u"].shape)
    dhl = rng.standard_normal((2, 3, 4))
    args = (p["u"], p["delta"], p["B"], p["C"], p["A"], dy, p["Dskip"], p["bias"], p["z"], p["h0"], dhl)
    ref = oracle.scan_bwd(*args, zoh=zoh)
    got = bwd_chunked.scan_bwd_chunked(*args, chunk=chunk, zoh=zoh)
    for k in ref:
        np.testing.assert_allclose(got[k], ref[k], rtol=1e-11, atol=1e-12, err_msg=k)
