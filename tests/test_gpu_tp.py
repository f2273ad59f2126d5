"""Tensor parallelism over I on one GPU: the ranks' shares run one after the
other (no rank waits on another), then the rank-order sum.

moe_forward_partial on each slice must match the oracle run on that slice
(fp32 partial against the fp64 partial), and moe_sum_partials over the
slices must meet the layer's bf16 bound against the unsharded oracle.
"""
import numpy as np
import pytest
import torch

from helpers import assert_output_close, oracle_of
from mixture_experts_layer_counts_b200 import layer
from mixture_experts_layer_counts_b200.inputs import WORKLOADS, make_inputs
from mixture_experts_layer_counts_b200.tp import shard_expert_weights

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world", [2, 4, 8])
def test_tp_shares_sum_to_the_layer(cuda_ok, world):
    inp = make_inputs(WORKLOADS["decode"], "cuda")          # I = 1024: slices of 512, 256, 128
    k = inp["top_k"]
    parts = []
    for g in range(world):
        w13_s, w2_s = shard_expert_weights(inp["w13"], inp["w2"], g, world)
        parts.append(layer.moe_forward_partial(inp["hidden"], inp["router_w"], inp["router_bias"], w13_s,
                                               w2_s, k))
        if g == world - 1:       # one slice against the oracle on that slice
            ref_g = oracle_of(dict(inp, w13=w13_s, w2=w2_s, I=w13_s.shape[1] // 2))
            p = parts[-1].cpu().numpy().astype(np.float64)
            scale = np.sqrt(np.mean(ref_g["out"] ** 2))
            assert np.abs(p - ref_g["out"]).max() <= 2e-2 * scale
    stacked = torch.stack(parts)
    out = layer.sum_partials(stacked)
    torch.cuda.synchronize()
    # the rank-order sum, recomputed on the host in fp32 and rounded once
    host = stacked.cpu()
    acc = host[0].clone()
    for g in range(1, world):
        acc += host[g]
    assert torch.equal(out.cpu(), acc.to(torch.bfloat16))
    ref = oracle_of(inp)
    assert_output_close(out, ref, fp8=False)
