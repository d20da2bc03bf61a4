"""GPU parity of the decode step (ssm_state_update) against the fp64 oracle."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle  # noqa: E402
import selective_state_space_15_b200 as ssm  # noqa: E402
import workloads  # noqa: E402
from helpers import TOL, check, dev, host  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ssm.load()


def _step(prob, pool_t, slots_t, step, A, D, bias):
    x = workloads.decode_step_inputs(prob, step)
    u, dl, z = (dev(x[k], prob.dtype) for k in ("u", "delta", "z"))
    B, C = dev(x["B"], prob.dtype), dev(x["C"], prob.dtype)
    y = ssm.state_update(pool_t, slots_t, u, dl, B, C, A, D, bias, z)
    return x, y


@pytest.mark.parametrize("dtype,N", [("bf16", 16), ("f32", 16), ("bf16", 64), ("f32", 128), ("f32", 4), ("bf16", 8),
                                     ("f32", 12), ("bf16", 24), ("bf16", 48), ("bf16", 256), ("f32", 200)])
def test_decode_small_matches_oracle_and_leaves_other_slots(dtype, N):
    prob = workloads.decode_problem(num_slots=37, dim=48, dstate=N, R=11, dtype=dtype, seed=5)
    pool_t = torch.from_numpy(prob.pool0).cuda()
    slots_t = torch.from_numpy(prob.slot_ids).cuda()
    A, D, bias = (torch.from_numpy(x).cuda() for x in (prob.A, prob.Dskip, prob.bias))
    pool = prob.pool0.astype(np.float64)
    pool_mag = np.abs(pool)
    for step in range(6):
        x, y = _step(prob, pool_t, slots_t, step, A, D, bias)
        ref = oracle.state_update(pool, prob.slot_ids, x["u"], x["delta"], x["B"], x["C"], prob.A, prob.Dskip,
                                  prob.bias, x["z"], pool_mag=pool_mag)
        check(f"y step {step}", host(y), ref["y"], ref["y_mag"], TOL[dtype], dtype)
    got = host(pool_t)
    check("pool", got[prob.slot_ids], pool[prob.slot_ids], pool_mag[prob.slot_ids], TOL[dtype])
    others = np.setdiff1d(np.arange(37), prob.slot_ids)
    assert np.array_equal(pool_t.cpu().numpy()[others], prob.pool0[others])   # bitwise unchanged


def test_decode_workload_first_steps_full_width():
    prob = workloads.config_inputs("decode_bf16")
    pool_t = torch.from_numpy(prob.pool0).cuda()
    slots_t = torch.from_numpy(prob.slot_ids).cuda()
    A, D, bias = (torch.from_numpy(x).cuda() for x in (prob.A, prob.Dskip, prob.bias))
    sub = prob.pool0[prob.slot_ids].astype(np.float64)        # oracle tracks only the active slots
    mag = np.abs(sub)
    ids = np.arange(prob.R)
    for step in range(3):
        x, y = _step(prob, pool_t, slots_t, step, A, D, bias)
        ref = oracle.state_update(sub, ids, x["u"], x["delta"], x["B"], x["C"], prob.A, prob.Dskip, prob.bias,
                                  x["z"], pool_mag=mag)
        check(f"y step {step}", host(y), ref["y"], ref["y_mag"], TOL["bf16"], "bf16")
    check("pool", host(pool_t)[prob.slot_ids], sub, mag, TOL["bf16"])
    others = np.setdiff1d(np.arange(prob.pool0.shape[0]), prob.slot_ids)
    assert np.array_equal(pool_t.cpu().numpy()[others], prob.pool0[others])


def test_decode_workload_1000_steps_channel_subset():
    """1000 steps of the full-width decode; the oracle follows every 64th channel."""
    prob = workloads.config_inputs("decode_bf16")
    pool_t = torch.from_numpy(prob.pool0).cuda()
    slots_t = torch.from_numpy(prob.slot_ids).cuda()
    A, D, bias = (torch.from_numpy(x).cuda() for x in (prob.A, prob.Dskip, prob.bias))
    ch = np.arange(0, prob.dim, 64)
    sub = np.ascontiguousarray(prob.pool0[prob.slot_ids][:, ch], dtype=np.float64)
    mag = np.abs(sub)
    ids = np.arange(prob.R)
    worst = 0.0
    for step in range(1000):
        x, y = _step(prob, pool_t, slots_t, step, A, D, bias)
        ref = oracle.state_update(sub, ids, x["u"][:, ch], x["delta"][:, ch], x["B"], x["C"], prob.A[ch],
                                  prob.Dskip[ch], prob.bias[ch], x["z"][:, ch], pool_mag=mag)
        if step % 50 == 0 or step == 999:
            worst = max(worst, check(f"y step {step}", host(y)[:, ch], ref["y"], ref["y_mag"], TOL["bf16"], "bf16"))
    check("pool after 1000 steps", host(pool_t)[prob.slot_ids][:, ch], sub, mag, TOL["bf16"])


def test_bad_slot_is_skipped_and_reported():
    prob = workloads.decode_problem(num_slots=8, dim=16, dstate=16, R=3, dtype="f32", seed=6)
    pool_t = torch.from_numpy(prob.pool0).cuda()
    before = pool_t.clone()
    slots = torch.tensor([2, 8, -1], dtype=torch.int32, device="cuda")    # 8 and -1 are out of range
    A, D, bias = (torch.from_numpy(x).cuda() for x in (prob.A, prob.Dskip, prob.bias))
    ssm.device_status()                                                     # clear
    x = workloads.decode_step_inputs(prob, 0)
    y = torch.full((3, 16), 123.0, device="cuda")
    ssm.state_update(pool_t, slots, dev(x["u"]), dev(x["delta"]), dev(x["B"]), dev(x["C"]), A, D, bias,
                     dev(x["z"]), y=y)
    assert ssm.device_status() == 4                                         # SSM_ERR_BAD_SLOT
    assert ssm.device_status() == 0                                         # read clears it
    assert torch.all(y[1:] == 123.0)                                        # skipped rows untouched
    changed = (pool_t != before).any(dim=(1, 2)).cpu().numpy()
    assert changed.tolist() == [False, False, True, False, False, False, False, False]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decode_many_requests_per_block_with_bad_slots(dtype):
    """More requests than resident blocks per channel group (every block walks several
    requests through its staging ring), a ragged last channel group (300 = 256 + 44) and bad
    slot ids spread over the requests: good rows match the oracle, bad rows are skipped."""
    prob = workloads.decode_problem(num_slots=800, dim=300, dstate=16, R=700, dtype=dtype, seed=9)
    slots = prob.slot_ids.copy()
    bad = np.arange(5, 700, 97)
    slots[bad] = np.where(bad % 2 == 0, -1, 800 + bad)
    pool_t = torch.from_numpy(prob.pool0).cuda()
    slots_t = torch.from_numpy(slots).cuda()
    A, D, bias = (torch.from_numpy(x).cuda() for x in (prob.A, prob.Dskip, prob.bias))
    good = np.setdiff1d(np.arange(700), bad)
    pool = prob.pool0.astype(np.float64)
    pool_mag = np.abs(pool)
    ssm.device_status()
    for step in range(3):
        x = workloads.decode_step_inputs(prob, step)
        u, dl, z = (dev(x[k], dtype) for k in ("u", "delta", "z"))
        B, C = dev(x["B"], dtype), dev(x["C"], dtype)
        y = torch.full(u.shape, 7.0, device="cuda", dtype=u.dtype)
        ssm.state_update(pool_t, slots_t, u, dl, B, C, A, D, bias, z, y=y)
        assert ssm.device_status() == 4                                     # SSM_ERR_BAD_SLOT
        ref = oracle.state_update(pool, slots[good], x["u"][good], x["delta"][good], x["B"][good], x["C"][good],
                                  prob.A, prob.Dskip, prob.bias, x["z"][good], pool_mag=pool_mag)
        check(f"y step {step}", host(y)[good], ref["y"], ref["y_mag"], TOL[dtype], dtype)
        assert torch.all(y[torch.from_numpy(bad).cuda()] == 7.0)
    got = host(pool_t)
    check("pool", got[slots[good]], pool[slots[good]], pool_mag[slots[good]], TOL[dtype])
    others = np.setdiff1d(np.arange(800), slots[good])
    assert np.array_equal(pool_t.cpu().numpy()[others], prob.pool0[others])
