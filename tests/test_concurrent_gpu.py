"""Concurrent first calls from several host threads.

The library keeps per-(kernel, device) launch facts (the dynamic shared-memory attribute and
the occupancy behind the persistent grids) in a table filled on first use under a lock.  This
test starts a fresh process (so every table entry is filled during the test), releases 16
threads at once -- two per entry point and shape, each on its own stream, so that the same
kernel's entry is also raced -- and then checks every result against the same call made again
on one thread once the table is warm: forward outputs and per-step gradients are reproducible
bit for bit (each chain's arithmetic is fixed), and the device status word must stay clean.
Parity with the oracle is the business of the other GPU tests.
"""
import os
import subprocess
import sys

import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import threading
import numpy as np
import torch
import selective_state_space_15_b200 as ssm
import workloads

def up(x, dt):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda().to(dt)

def scan_job(b, D, N, L, dtype, algorithm, seed):
    inp = workloads.batch_inputs(b, D, N, L, "bf16" if dtype == torch.bfloat16 else "f32", seed=seed)
    t = [up(x, dtype) for x in (inp.u, inp.delta, inp.B, inp.C, inp.z)]
    A, Dd, bias = (up(x, torch.float32) for x in (inp.A, inp.Dskip, inp.bias))
    def run(stream):
        y, hl = ssm.scan_fwd(t[0], t[1], t[2], t[3], A, Dd, bias, t[4], stream=stream, algorithm=algorithm)
        return [y, hl]
    return run

def varlen_job(seed):
    inp = workloads.varlen_inputs([300, 77, 1024, 5], 96, 16, "bf16", seed=seed)
    t = [up(x, torch.bfloat16) for x in (inp.u, inp.delta, inp.B, inp.C, inp.z)]
    A, Dd, bias = (up(x, torch.float32) for x in (inp.A, inp.Dskip, inp.bias))
    cu = torch.from_numpy(inp.cu_seqlens).cuda()
    def run(stream):
        y, hl = ssm.scan_fwd_varlen(t[0], t[1], t[2], t[3], A, cu, Dd, bias, t[4], stream=stream)
        return [y, hl]
    return run

def decode_job(seed):
    prob = workloads.decode_problem(64, 320, 16, 24, "bf16", seed=seed)
    x = workloads.decode_step_inputs(prob, 0)
    t = {k: up(v, torch.bfloat16) for k, v in x.items()}
    A, Dd, bias = (up(v, torch.float32) for v in (prob.A, prob.Dskip, prob.bias))
    slots = torch.from_numpy(prob.slot_ids).cuda()
    pool0 = up(prob.pool0, torch.float32)
    def run(stream):
        pool = pool0.clone()
        y = ssm.state_update(pool, slots, t["u"], t["delta"], t["B"], t["C"], A, Dd, bias, t["z"], stream=stream)
        return [y, pool]
    return run

def ssd_job(seed):
    s = workloads.ssd_inputs(1, 2, 64, 128, 256, seed=seed)
    x, B, C = (up(v, torch.bfloat16) for v in (s.x, s.B, s.C))
    dt, A = up(s.dt, torch.float32), up(s.A, torch.float32)
    def run(stream):
        y, hl = ssm.ssd_fwd(x, dt, A, B, C, stream=stream)
        return [y, hl]
    return run

def bwd_job(seed):
    inp = workloads.batch_inputs(1, 40, 16, 264, "f32", seed=seed)
    t = [up(x, torch.float32) for x in (inp.u, inp.delta, inp.B, inp.C, inp.z)]
    A, Dd, bias = (up(x, torch.float32) for x in (inp.A, inp.Dskip, inp.bias))
    dy = up(np.random.default_rng(seed).standard_normal(inp.u.shape), torch.float32)
    def run(stream):
        g = ssm.scan_bwd(t[0], t[1], t[2], t[3], A, dy, Dd, bias, t[4], stream=stream)
        return [g["du"], g["ddelta"], g["dz"]]
    return run

jobs = [
    scan_job(2, 40, 16, 1000, torch.float32, "auto", 1),
    scan_job(1, 64, 32, 515, torch.bfloat16, "auto", 2),
    scan_job(1, 10, 128, 200, torch.bfloat16, "auto", 3),
    scan_job(2, 64, 16, 512, torch.bfloat16, "sequential", 4),
    varlen_job(5),
    decode_job(6),
    ssd_job(7),
    bwd_job(8),
]
jobs = jobs + jobs            # two threads per job: the same table entry is raced as well
streams = [torch.cuda.Stream() for _ in jobs]
torch.cuda.synchronize()
start = threading.Barrier(len(jobs))
results, errors = [None] * len(jobs), []

def worker(i):
    try:
        start.wait()
        with torch.cuda.stream(streams[i]):
            out = jobs[i](streams[i])
        streams[i].synchronize()
        results[i] = [o.detach().clone() for o in out]
    except Exception as e:  # reported below
        errors.append(f"job {i}: {e!r}")

threads = [threading.Thread(target=worker, args=(i,)) for i in range(len(jobs))]
for th in threads:
    th.start()
for th in threads:
    th.join()
torch.cuda.synchronize()
assert not errors, errors
status = ssm.device_status()
assert status == 0, f"device status {status}"
for i, job in enumerate(jobs):
    again = job(None)
    torch.cuda.synchronize()
    for a, b in zip(results[i], again):
        assert torch.equal(a, b), f"job {i}: concurrent result differs from the serial one"
print("ALL-OK", len(jobs))
"""


def test_concurrent_first_calls_from_many_threads():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    env = dict(os.environ)
    env["PYTHONPATH"] = ROOT + os.pathsep + env.get("PYTHONPATH", "")
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "ALL-OK 16" in r.stdout
