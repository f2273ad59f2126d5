"""Failure detection without a GPU fault.

A debug switch makes the first gate/up GEMM CTA arm one pipeline stage and
issue no copy for it, so nothing will ever complete that stage: the MMA
issuer's bounded wait runs out after the requested limit, the kernel records
MOE_ERR_DEVICE_TIMEOUT in the workspace status word, drains what it issued,
frees its tensor memory and returns.  The host reads the status; the context
stays usable and the next call on the same workspace is correct.
"""
import pytest
import torch

from helpers import assert_output_close, custom_inputs, oracle_of
from mixture_experts_layer_counts_b200 import layer

pytestmark = pytest.mark.gpu


def _call(inp, ws, **kw):
    out = layer.moe_forward(inp["hidden"], inp["router_w"], inp["router_bias"], inp["w13"], inp["w2"],
                            inp["top_k"], workspace=ws, **kw)
    torch.cuda.synchronize()
    return out


def test_bounded_wait_reports_timeout_and_recovers(cuda_ok):
    T, H, E, I, k = 16, 512, 8, 256, 2
    inp = custom_inputs(T, H, E, I, k, seed=21)
    ws = layer.make_workspace(T, H, E, I, k, 0)
    assert layer.get_status(ws)[0] == 0
    _call(inp, ws, inject_stall=1, wait_timeout_us=50_000)
    code, info = layer.get_status(ws)
    assert code == 5, f"expected MOE_ERR_DEVICE_TIMEOUT, got {code} (info {info})"
    assert layer.get_status(ws)[0] == 0            # cleared once read
    out = _call(inp, ws)                            # same workspace, no injection
    assert layer.get_status(ws)[0] == 0
    fresh = _call(inp, layer.make_workspace(T, H, E, I, k, 0))
    assert torch.equal(out.view(torch.int16), fresh.view(torch.int16))   # as if nothing had failed
    ref = oracle_of(inp)
    assert_output_close(out, ref, fp8=False)        # the stated bf16 bound
