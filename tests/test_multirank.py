"""The N > 1 path of bench.py on CPU: two gloo ranks on 127.0.0.1.

The path shards without any exchange (replicas only): every rank runs its own
batch of the workload from its own seed, and the reported time is the max
over ranks.  These tests check that host logic with world size 2.
"""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from hybrid_ssm_sliding_b200.workloads import WORKLOADS, make_prefill_inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                           timeout=__import__("datetime").timedelta(seconds=60))
    try:
        # each rank times a different number; every rank must see the max
        my_ms = 10.0 + 5.0 * rank
        ms = bench.max_over_ranks(my_ms, torch.device("cpu"))
        # each rank's inputs come from its own seed
        wl = bench.rank_workload(WORKLOADS["tiny"], rank)
        inp = make_prefill_inputs(wl, device="cpu")
        xs = [torch.zeros_like(inp["x"]) for _ in range(world)]
        dist.all_gather(xs, inp["x"])
        same = bool(torch.equal(xs[0], xs[1]))
        rate = bench.whole_job_rate(wl.batch * wl.seqlen, world, ms)
        out[rank] = (ms, wl.seed, same, rate)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_time_is_max_and_batches_differ():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    (ms0, seed0, same0, rate0), (ms1, seed1, same1, rate1) = out[0], out[1]
    assert ms0 == ms1 == 15.0              # the max over ranks, on every rank
    assert seed0 != seed1                   # each rank its own batch
    assert not same0 and not same1          # ... so the inputs differ
    wl = WORKLOADS["tiny"]
    assert rate0 == rate1 == pytest.approx(2 * wl.batch * wl.seqlen / 0.015)


def test_single_process_reduction_is_identity():
    assert bench.max_over_ranks(3.5, torch.device("cpu")) == 3.5
    assert bench.whole_job_rate(100, 1, 10.0) == pytest.approx(1e4)
