"""moe_route_static: the router for callers that cannot allocate device memory.

Some callers receive their input and output buffers from a host program but
have no way to allocate scratch of their own (a plug-in inside a runtime that
owns all device memory, a hot loop that must not allocate).  For them the
library keeps the router's scratch in a fixed 8 MiB device array.  These tests
call that entry point through the C ABI and check that it returns the same
routing as moe_route (which uses a caller-provided workspace) and as the fp64
oracle, on two calls in a row with different inputs, so stale contents of the
shared array would show; one case sits exactly at the array's capacity.

This file is collected last on purpose: the static array is shared by every
call in the process, and the test must pass both alone and after all others.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from helpers import WEIGHT_ATOL
from mixture_experts_layer_counts_b200 import _lib, layer
from mixture_experts_layer_counts_b200.inputs import WORKLOADS, host_bits, make_hidden, make_router, zipf_bias
from oracle import bf16_bits_to_f64, route_ref

STATIC_BYTES = 8 << 20


def static_bytes(T, E):
    """Bytes of the static scratch the router needs: header, logits, norms,
    per-token amax and fallback candidates, each region 1024-byte aligned."""
    up = lambda v: (v + 1023) // 1024 * 1024
    return sum(up(b) for b in (256, T * E * 4, T * 4, E * 4, T * 4, T * E * 16))


def capacity_T(E):
    T = 1
    while static_bytes(T + 1, E) <= STATIC_BYTES:
        T += 1
    return T


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
    refs = []
    for hidden, router_w, bias, k in cases:
        rids, rw, _, _ = route_ref(bf16_bits_to_f64(host_bits(hidden)), bf16_bits_to_f64(host_bits(router_w)),
                                   None if bias is None else bias.cpu().numpy(), k)
        refs.append((rids, rw))
    for round_ in range(2):                      # two calls in a row per input, inputs alternate
        for (hidden, router_w, bias, k), (rids, rw) in zip(cases, refs):
            ids_s, w_s = _route_static(hidden, router_w, bias, k)
            ids_r, w_r = layer.moe_route(hidden, router_w, bias, k)
            torch.cuda.synchronize()
            assert np.array_equal(ids_s.cpu().numpy(), rids), f"routing differs from the oracle (round {round_})"
            assert np.abs(w_s.cpu().numpy() - rw).max() <= WEIGHT_ATOL
            assert torch.equal(ids_s, ids_r), f"routing differs from moe_route (round {round_})"
            assert float((w_s - w_r).abs().max()) <= WEIGHT_ATOL
            assert np.allclose(w_s.sum(1).cpu().numpy(), 1.0, atol=1e-5)


@pytest.mark.gpu
def test_route_static_at_capacity(cuda_ok):
    E, H, k = 128, 256, 8
    T = capacity_T(E)
    assert static_bytes(T, E) <= STATIC_BYTES < static_bytes(T + 1, E)
    g = torch.Generator(device="cuda").manual_seed(3)
    x = torch.randn(T + 1, H, generator=g, device="cuda").to(torch.bfloat16)
    wr = (torch.randn(E, H, generator=g, device="cuda") * 0.1).to(torch.bfloat16)
    # one token more than fits: refused before anything runs
    ids = torch.empty((T + 1, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T + 1, k), dtype=torch.float32, device="cuda")
    rc = _lib.lib().moe_route_static(C.c_void_p(x.data_ptr()), C.c_void_p(wr.data_ptr()), None, T + 1, H, E, k,
                                     C.c_void_p(ids.data_ptr()), C.c_void_p(w.data_ptr()),
                                     C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 8
    # exactly at capacity: the oracle's routing
    xs = x[:T].contiguous()
    ids_s, w_s = _route_static(xs, wr, None, k)
    torch.cuda.synchronize()
    rids, rw, _, _ = route_ref(bf16_bits_to_f64(host_bits(xs)), bf16_bits_to_f64(host_bits(wr)), None, k)
    assert np.array_equal(ids_s.cpu().numpy(), rids)
    assert np.abs(w_s.cpu().numpy() - rw).max() <= WEIGHT_ATOL


def test_route_static_rejects_oversized_shapes():
    L = _lib.lib()
    # 4096 x 1024 logits plus fallback scratch need ~80 MiB: rejected before anything runs
    rc = L.moe_route_static(C.c_void_p(16), C.c_void_p(16), None, 4096, 256, 1024, 8,
                            C.c_void_p(16), C.c_void_p(16), None)
    assert rc == 8
    assert L.moe_status_string(8) == b"shape exceeds the fixed static scratch"


def test_route_static_rejects_misaligned_bias():
    L = _lib.lib()
    # the bias is read as fp32: an address that is not 4-byte aligned is refused
    rc = L.moe_route_static(C.c_void_p(16), C.c_void_p(16), C.c_void_p(18), 4, 256, 8, 2,
                            C.c_void_p(16), C.c_void_p(16), None)
    assert rc == 7
