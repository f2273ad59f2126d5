"""moe_route_static: the router for callers that cannot allocate device memory.

Some callers receive their input and output buffers from a host program but
have no way to allocate scratch of their own (a plug-in inside a runtime that
owns all device memory, a hot loop that must not allocate).  For them the
library keeps the router's scratch in a fixed 8 MiB device array.  These tests
call that entry point through the C ABI and check that it returns the same
routing as moe_route (which uses a caller-provided workspace), on two calls in
a row with different inputs, so stale contents of the shared array would show.

This file is collected last on purpose: the static array is shared by every
call in the process, and the test must pass both alone and after all others.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from helpers import WEIGHT_ATOL
from mixture_experts_layer_counts_b200 import _lib, layer
from mixture_experts_layer_counts_b200.inputs import WORKLOADS, make_hidden, make_router, zipf_bias


def _route_static(hidden, router_w, bias, k):
    T, H = hidden.shape
    E = router_w.shape[0]
    ids = torch.full((T, k), -1, dtype=torch.int32, device=hidden.device)
    w = torch.full((T, k), -1.0, dtype=torch.float32, device=hidden.device)
    p = lambda t: None if t is None else C.c_void_p(t.data_ptr())
    rc = _lib.lib().moe_route_static(p(hidden), p(router_w), p(bias), T, H, E, k, p(ids), p(w),
                                     C.c_void_p(torch.cuda.current_stream().cuda_stream))
    _lib.check(rc, "moe_route_static")
    return ids, w


def _cases():
    out = []
    for name in ("decode", "decode-fp8", "decode-zipf"):
        wl = WORKLOADS[name]
        out.append((make_hidden(wl, "cuda"), make_router(wl, "cuda"),
                    zipf_bias(wl["E"]).cuda() if wl["zipf"] else None, wl["top_k"]))
    # duplicated router rows: exact ties exercise the fp64 / exact fallback scratch
    g = torch.Generator(device="cuda").manual_seed(7)
    x = torch.randn(24, 256, generator=g, device="cuda").to(torch.bfloat16)
    wr = (torch.randn(40, 256, generator=g, device="cuda") * 0.1).to(torch.bfloat16)
    wr[7] = wr[3]
    wr[21] = wr[30]
    out.append((x, wr.contiguous(), None, 6))
    return out


@pytest.mark.gpu
def test_route_static_matches_route(cuda_ok):
    cases = _cases()
    for round_ in range(2):                      # two calls in a row per input, inputs alternate
        for hidden, router_w, bias, k in cases:
            ids_s, w_s = _route_static(hidden, router_w, bias, k)
            ids_r, w_r = layer.moe_route(hidden, router_w, bias, k)
            torch.cuda.synchronize()
            assert torch.equal(ids_s, ids_r), f"routing differs (round {round_})"
            assert float((w_s - w_r).abs().max()) <= WEIGHT_ATOL
            assert np.allclose(w_s.sum(1).cpu().numpy(), 1.0, atol=1e-5)


def test_route_static_rejects_oversized_shapes():
    L = _lib.lib()
    # 4096 x 1024 logits plus fallback scratch need ~80 MiB: rejected before anything runs
    rc = L.moe_route_static(C.c_void_p(16), C.c_void_p(16), None, 4096, 256, 1024, 8,
                            C.c_void_p(16), C.c_void_p(16), None)
    assert rc == 8
    assert L.moe_status_string(8) == b"shape exceeds the fixed static scratch"
