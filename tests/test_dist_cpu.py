"""The multi-rank plumbing of bench.py on CPU: two gloo ranks, as torchrun
would start them (RANK / WORLD_SIZE / LOCAL_RANK, rendezvous on 127.0.0.1).

The ranks run independent replicas of the workload (weak scaling: no
collective on the data path). They meet only to take the slowest rank's step
time and the sum of their bytes. Only rank 0 runs the CPU reference arm.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    try:
        os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                          MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        sys.path.insert(0, ROOT)
        import bench
        d = bench.Dist()
        d.init("gloo")
        ms = d.max(10.0 + 5.0 * rank)            # per-rank step times 10 and 15 ms
        total = d.sum(1.0e9 * (rank + 1))        # per-rank bytes 1 GB and 2 GB
        d.barrier()

        class Args:
            workload = "single_head_d128_b3"
            warmup = 0
            steps = 1

        # the reference arm: rank 0 alone; the other ranks return without work
        ref = bench.run_reference(Args, d) if rank != 0 else "skipped on rank 0 here"
        q.put((rank, ms, total, bench.whole_job_gbs(total, ms), ref))
        d.close()
    except Exception as e:   # report instead of hanging the parent
        q.put((rank, "error", repr(e), None, None))


def test_two_gloo_ranks_take_max_time_and_summed_bytes():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in procs:
        r = q.get(timeout=120)
        res[r[0]] = r
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in (0, 1):
        _, ms, total, gbs, ref = res[rank]
        assert ms == 15.0, res[rank]
        assert total == 3.0e9
        assert gbs == pytest.approx(3.0e9 / 0.015 / 1e9)
    assert res[1][4] is None          # rank 1 does no reference work
