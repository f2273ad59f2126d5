"""Multi-rank host logic of bench.py on CPU: two gloo ranks on 127.0.0.1.

Each GPU of a data-parallel run serves its own batch with its own copy of the
weights; the only cross-rank steps are the barriers around the timed region
and the max of the per-rank device times.  These tests run that logic with
world size 2 and no GPU.
"""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    from mixture_experts_layer_counts_b200.inputs import WORKLOADS

    r, w, local = bench.dist_setup(world)
    try:
        assert (r, w, local) == (rank, world, rank)
        assert torch.distributed.get_backend() == "gloo"
        # max over ranks reaches every rank
        m = bench.max_over_ranks(10.0 + 5.0 * rank, w)
        bench.barrier(w)
        # rank batches: different hidden states, identical weights
        inp = bench.rank_inputs(WORKLOADS["tiny"], "cpu", r, w)
        sums = torch.tensor([inp["hidden"].float().sum().item(), inp["w13"].float().sum().item(),
                             inp["router_w"].float().sum().item()], dtype=torch.float64)
        gathered = [torch.zeros_like(sums) for _ in range(w)]
        torch.distributed.all_gather(gathered, sums)
        out[rank] = (m, [g.tolist() for g in gathered])
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    assert sorted(out.keys()) == [0, 1]
    for rank in range(world):
        m, gathered = out[rank]
        assert m == 15.0                       # max of 10 and 15 on both ranks
        (h0, w0, r0), (h1, w1, r1) = gathered
        assert h0 != h1                        # each rank has its own batch
        assert w0 == w1 and r0 == r1           # and the same experts and router


def test_whole_job_value_and_single_rank_paths():
    sys.path.insert(0, ROOT)
    import bench

    # tokens of all ranks over the slowest rank's time
    assert bench.whole_job_tokens_per_s(4, 16, 100, 2000.0) == pytest.approx(3200.0)
    # world size 1: no process group, values pass through
    assert bench.max_over_ranks(3.5, 1) == 3.5
    bench.barrier(1)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    sys.path.insert(0, ROOT)
    import argparse

    import bench
    from mixture_experts_layer_counts_b200.inputs import WORKLOADS

    args = argparse.Namespace(steps=1, warmup=0, workload="tiny")
    bench.run_reference(args, dict(WORKLOADS["tiny"]), rank=1, world=2)
    assert capsys.readouterr().out == ""       # other ranks exit without work
