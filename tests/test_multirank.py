"""The multi-rank host logic of bench.py on CPU: two processes joined by a gloo process group.

`bench.py --gpus N` runs one rank per GPU; every rank scans its own packed batch (no
collective on the data path), and the job's figures are the slowest rank's time and the sum
of all ranks' tokens.  These tests run that logic with world_size 2 on the host: the
reduction, the per-rank batches, and the reference arm that only rank 0 runs.
"""
import os
import socket
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    import bench
    import workloads
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # job figures: max of the per-rank times, sum of the per-rank tokens
        ms, tok = bench.reduce_over_ranks(dist, 1.5 + rank, 1000.0 * (rank + 1), torch.device("cpu"))
        # each rank draws its own packed batch
        c = workloads.CONFIGS[bench.WORKLOAD]
        lens = workloads.varlen_lengths(c["nseq"], c["len_lo"], c["len_hi"], bench.rank_seed(rank))
        gathered = [None] * world
        dist.all_gather_object(gathered, [int(x) for x in lens])

        # the reference arm: ranks other than 0 leave at once, without work
        class Args:
            steps, warmup, gpus = 1, 3, world
        ref_rc = bench.run_reference(Args(), rank, world) if rank != 0 else 0
        dist.barrier()
        out[rank] = (ms, tok, gathered, ref_rc)
    finally:
        dist.destroy_process_group()


def test_two_ranks_reduce_and_shard():
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert sorted(res) == [0, 1]
    for rank in range(world):
        ms, tok, gathered, ref_rc = res[rank]
        assert ms == 2.5                        # the slowest rank's time
        assert tok == 3000.0                    # all ranks' tokens
        assert gathered[0] != gathered[1]       # distinct batches per rank
        assert ref_rc == 0
    assert res[0][2] == res[1][2]               # both ranks saw the same set of batches


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_over_ranks(None, 3.0, 7, torch.device("cpu")) == (3.0, 7)
    assert bench.rank_seed(0) != bench.rank_seed(1)
