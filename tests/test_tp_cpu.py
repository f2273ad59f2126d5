"""Tensor parallelism over I, host side, with two gloo ranks on CPU.

Each rank slices the experts' weights with the library's shard helper, runs
the fp64 oracle on its slice (the oracle's unrounded output is exactly the
rank's partial sum), the partials are all-gathered over the process group and
added in rank order.  The result must equal the unsharded layer up to fp64
rounding, and each rank's bf16 intermediate must be exactly the matching
columns of the unsharded intermediate (h of a column depends only on that
column's gate and up rows).
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer_inputs():
    from mixture_experts_layer_counts_b200.inputs import make_inputs

    wl = dict(T=6, H=256, E=8, top_k=3, I=512, dtype="bf16", zipf=True, seed=5)
    return wl, make_inputs(wl, "cpu")


def _oracle(inp, w13, w2, k):
    from mixture_experts_layer_counts_b200.inputs import host_bits
    from oracle import moe_forward_ref

    bias = None if inp["router_bias"] is None else inp["router_bias"].numpy()
    return moe_forward_ref(host_bits(inp["hidden"]), host_bits(inp["router_w"]), bias, host_bits(w13),
                           host_bits(w2), k, keep_intermediate=True)


def _worker(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    from mixture_experts_layer_counts_b200.tp import shard_bounds, shard_expert_weights

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        wl, inp = _layer_inputs()
        w13_s, w2_s = shard_expert_weights(inp["w13"], inp["w2"], rank, world)
        res = _oracle(inp, w13_s, w2_s, wl["top_k"])
        part = torch.from_numpy(res["out"])                      # fp64 [T, H]: this rank's partial
        gathered = torch.empty((world,) + tuple(part.shape), dtype=part.dtype)
        dist.all_gather(list(gathered.unbind(0)), part)          # rank order
        total = gathered[0].clone()
        for g in range(1, world):
            total += gathered[g]
        lo, hi = shard_bounds(wl["I"], rank, world)
        out[rank] = (total.numpy(), res["inter"], lo, hi, res["ids"])
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_tp_partials_sum_to_the_unsharded_layer(world):
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
    sys.path.insert(0, ROOT)
    wl, inp = _layer_inputs()
    full = _oracle(inp, inp["w13"], inp["w2"], wl["top_k"])
    for rank in range(world):
        total, inter, lo, hi, ids = out[rank]
        assert np.array_equal(ids, full["ids"])                 # identical routing on every rank
        assert np.array_equal(inter, full["inter"][:, lo:hi])   # the same bf16 intermediate columns
        np.testing.assert_allclose(total, full["out"], rtol=1e-12, atol=1e-12 * np.abs(full["out"]).max())
        assert np.array_equal(total, out[0][0])                 # every rank holds the same sum


def test_shard_bounds_and_layout():
    from mixture_experts_layer_counts_b200.tp import shard_bounds, shard_expert_weights

    assert shard_bounds(1024, 1, 4) == (256, 512)
    with pytest.raises(ValueError):
        shard_bounds(384, 0, 2)            # 192 is not a multiple of 128
    w13 = torch.arange(2 * 512 * 2, dtype=torch.float32).reshape(2, 2 * 256, 2)
    w2 = torch.arange(2 * 2 * 256, dtype=torch.float32).reshape(2, 2, 256)
    a, b = shard_expert_weights(w13, w2, 1, 2)
    assert a.shape == (2, 256, 2) and b.shape == (2, 2, 128)
    assert torch.equal(a[:, :128], w13[:, 128:256]) and torch.equal(a[:, 128:], w13[:, 384:512])
    assert torch.equal(b, w2[:, :, 128:256]) and a.is_contiguous() and b.is_contiguous()
