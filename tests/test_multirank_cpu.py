"""The multi-GPU (replica) bookkeeping of bench.py, as world-size-2 gloo ranks on CPU.

A decode step has no cross-GPU exchange, so N GPUs run N independent replicas:
each rank draws its own seeded batch, the job's time is the slowest rank's and
its value counts every rank's bytes.  Nothing here needs a GPU.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import dsgen


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        r, lr, wsz = bench.rank_env()
        base = dsgen.workload("tiny-B1-H4-T1K")
        w = bench.replica_workload(base, r)
        # each rank's own (fake) device time: rank 1 is the slow one
        my_ms = 10.0 + 5.0 * r
        slowest = bench.max_over_ranks(my_ms, wsz, "cpu")
        val = bench.job_gbs(w.sparse_step_bytes(), wsz, slowest)
        q, _, _ = dsgen.qkv(w, want=("Q",))
        out[rank] = (r, lr, wsz, w.seed, slowest, val, int(q.sum()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_replicas_two_gloo_ranks():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    r0, r1 = out[0], out[1]
    assert (r0[0], r0[2], r1[0], r1[2]) == (0, 2, 1, 2)
    # distinct seeds, distinct inputs
    assert r0[3] != r1[3] and r0[6] != r1[6]
    # both ranks agree on the slowest rank's time and the job value
    assert r0[4] == r1[4] == 15.0
    w = dsgen.workload("tiny-B1-H4-T1K")
    assert r0[5] == pytest.approx(2 * w.sparse_step_bytes() / 15e-3 / 1e9)
    assert r0[5] == r1[5]


def test_single_rank_is_the_identity():
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5
    assert bench.replica_workload(dsgen.workload("tiny-B1-H4-T1K"), 0).seed == \
        dsgen.workload("tiny-B1-H4-T1K").seed
    assert bench.job_gbs(1_000_000_000, 1, 1000.0) == pytest.approx(1.0)
