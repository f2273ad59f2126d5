"""Python entry points of the fused MoE layer (thin wrappers over the C ABI).

PyTorch supplies device memory and the current CUDA stream; every step of the
layer runs in ``libmoe.so``.  Tensors must be CUDA, contiguous, and of the
storage dtypes the C ABI expects (bf16, uint8 E4M3 codes, fp32 scales).
"""
from __future__ import annotations

import ctypes as C

import torch

from . import _lib
from ._lib import MOE_DTYPE_BF16, MOE_DTYPE_FP8_E4M3, DebugOut, check

N_STAGE_EVENTS = 8
STAGES = ("start", "router", "align", "gather", "w13", "requant", "w2", "combine")


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return C.c_void_p(s.cuda_stream)


def _need(t, dtype, name, device=True):
    if t is None:
        raise ValueError(f"{name} is required")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise TypeError(f"{name}: dtype {t.dtype}")
    if device and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def dtype_code(w13: torch.Tensor) -> int:
    if w13.dtype == torch.bfloat16:
        return MOE_DTYPE_BF16
    if w13.dtype in (torch.uint8, torch.float8_e4m3fn):
        return MOE_DTYPE_FP8_E4M3
    raise TypeError(f"unsupported weight dtype {w13.dtype}")


def workspace_size(T, H, E, I, top_k, dtype) -> int:
    return int(_lib.lib().moe_workspace_size(T, H, E, I, top_k, dtype))


def make_workspace(T, H, E, I, top_k, dtype, device="cuda") -> torch.Tensor:
    n = workspace_size(T, H, E, I, top_k, dtype)
    if n == 0:
        raise ValueError("unsupported shape")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    check(_lib.lib().moe_workspace_init(_ptr(ws), n, _stream()), "moe_workspace_init")
    return ws


def moe_forward(hidden, router_w, router_bias, w13, w2, top_k, w13_scale=None, w2_scale=None,
                out=None, workspace=None, debug: dict | None = None, stream=None,
                force_orient: int = 0, stage_events=None, wait_timeout_us: int = 0,
                inject_stall: int = 0, batch_invariant: bool = False) -> torch.Tensor:
    """out[T, H] bf16 of the fused MoE layer (see include/moe.h).

    ``debug``: optional dict; keys filled on return (device tensors):
    topk_ids, topk_w, counts, offsets, perm, inv_perm, inter, act_scales and,
    on the FP8 path, hidden_q (the E4M3 codes of hidden / s1).
    ``stage_events``: optional list of 8 torch.cuda.Event recorded at the
    stage boundaries on the launch stream.
    ``batch_invariant``: call moe_forward_batch_invariant (bf16 only): each
    token's output row is independent of the rest of the batch.
    """
    _need(hidden, torch.bfloat16, "hidden")
    _need(router_w, torch.bfloat16, "router_w")
    _need(w13, (torch.bfloat16, torch.uint8, torch.float8_e4m3fn), "w13")
    _need(w2, (torch.bfloat16, torch.uint8, torch.float8_e4m3fn), "w2")
    T, H = hidden.shape
    E = router_w.shape[0]
    I = w13.shape[1] // 2
    dt = dtype_code(w13)
    if router_bias is not None:
        _need(router_bias, torch.float32, "router_bias")
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=hidden.device)
    if workspace is None:
        workspace = make_workspace(T, H, E, I, top_k, dt, hidden.device)
    dbg_p = None
    keep = []
    if debug is not None or force_orient or stage_events is not None or wait_timeout_us or inject_stall:
        dbg = DebugOut()
        dbg.force_orient = int(force_orient)
        dbg.wait_timeout_us = int(wait_timeout_us)
        dbg.inject_stall = int(inject_stall)
        if debug is not None:
            A = T * top_k
            dev = hidden.device
            debug["topk_ids"] = torch.empty((T, top_k), dtype=torch.int32, device=dev)
            debug["topk_w"] = torch.empty((T, top_k), dtype=torch.float32, device=dev)
            debug["counts"] = torch.empty(E, dtype=torch.int32, device=dev)
            debug["offsets"] = torch.empty(E + 1, dtype=torch.int32, device=dev)
            debug["perm"] = torch.empty(A, dtype=torch.int32, device=dev)
            debug["inv_perm"] = torch.empty(A, dtype=torch.int32, device=dev)
            debug["inter"] = torch.empty((A, I), dtype=torch.bfloat16 if dt == MOE_DTYPE_BF16 else torch.uint8,
                                         device=dev)
            debug["act_scales"] = torch.zeros(2, dtype=torch.float32, device=dev)
            names = ["topk_ids", "topk_w", "counts", "offsets", "perm", "inv_perm", "inter", "act_scales"]
            if dt == MOE_DTYPE_FP8_E4M3:
                debug["hidden_q"] = torch.empty((T, H), dtype=torch.uint8, device=dev)
                names.append("hidden_q")
            for k in names:
                setattr(dbg, k, debug[k].data_ptr())
        if stage_events is not None:
            arr = (C.c_void_p * N_STAGE_EVENTS)(
                *[C.c_void_p(None if ev is None else ev.cuda_event) for ev in stage_events])
            keep.append(arr)
            dbg.stage_events = C.cast(arr, C.c_void_p)
        dbg_p = C.pointer(dbg)
        keep.append(dbg)
    if batch_invariant:
        if dt != MOE_DTYPE_BF16 or w13_scale is not None or w2_scale is not None:
            raise TypeError("the batch-invariant layer is bf16 only")
        rc = _lib.lib().moe_forward_batch_invariant(
            _ptr(hidden), _ptr(router_w), _ptr(router_bias), _ptr(w13), _ptr(w2), T, H, E, I, top_k,
            _ptr(out), _ptr(workspace), workspace.numel(), dbg_p, _stream(stream))
        check(rc, "moe_forward_batch_invariant")
        return out
    rc = _lib.lib().moe_forward(
        _ptr(hidden), _ptr(router_w), _ptr(router_bias), _ptr(w13), _ptr(w2), _ptr(w13_scale),
        _ptr(w2_scale), T, H, E, I, top_k, dt, _ptr(out), _ptr(workspace), workspace.numel(),
        dbg_p, _stream(stream))
    check(rc, "moe_forward")
    return out


def moe_forward_hostio(hidden_host, router_w, router_bias, w13, w2, top_k, out_host,
                       workspace, w13_scale=None, w2_scale=None, stream=None) -> None:
    """Layer call with pinned host activations in and out (copies enqueued too)."""
    _need(hidden_host, torch.bfloat16, "hidden_host", device=False)
    _need(out_host, torch.bfloat16, "out_host", device=False)
    T, H = hidden_host.shape
    E = router_w.shape[0]
    I = w13.shape[1] // 2
    rc = _lib.lib().moe_forward_hostio(
        _ptr(hidden_host), _ptr(router_w), _ptr(router_bias), _ptr(w13), _ptr(w2),
        _ptr(w13_scale), _ptr(w2_scale), T, H, E, I, top_k, dtype_code(w13), _ptr(out_host),
        _ptr(workspace), workspace.numel(), _stream(stream))
    check(rc, "moe_forward_hostio")


def moe_route(hidden, router_w, router_bias, top_k, workspace=None, stream=None):
    """(topk_ids [T, k] int32, topk_w [T, k] fp32) on the device."""
    _need(hidden, torch.bfloat16, "hidden")
    _need(router_w, torch.bfloat16, "router_w")
    T, H = hidden.shape
    E = router_w.shape[0]
    if workspace is None:
        workspace = make_workspace(T, H, E, 128, top_k, MOE_DTYPE_BF16, hidden.device)
    ids = torch.empty((T, top_k), dtype=torch.int32, device=hidden.device)
    w = torch.empty((T, top_k), dtype=torch.float32, device=hidden.device)
    check(_lib.lib().moe_route(_ptr(hidden), _ptr(router_w), _ptr(router_bias), T, H, E, top_k,
                               _ptr(ids), _ptr(w), _ptr(workspace), workspace.numel(),
                               _stream(stream)), "moe_route")
    return ids, w


def moe_align(topk_ids, E, workspace=None, stream=None):
    """(counts [E], offsets [E+1], perm [A], inv_perm [A]) int32 on the device."""
    _need(topk_ids, torch.int32, "topk_ids")
    T, k = topk_ids.shape
    dev = topk_ids.device
    if workspace is None:
        workspace = make_workspace(T, 128, E, 128, k, MOE_DTYPE_BF16, dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(T * k, dtype=torch.int32, device=dev)
    inv = torch.empty(T * k, dtype=torch.int32, device=dev)
    check(_lib.lib().moe_align(_ptr(topk_ids), T, E, k, _ptr(counts), _ptr(offsets), _ptr(perm),
                               _ptr(inv), _ptr(workspace), workspace.numel(), _stream(stream)),
          "moe_align")
    return counts, offsets, perm, inv


def get_status(workspace, stream=None):
    """(status code, info) recorded on the device since the last call; clears it."""
    info = C.c_uint32(0)
    code = _lib.lib().moe_get_status(_ptr(workspace), _stream(stream), C.byref(info))
    return int(code), int(info.value)


def moe_forward_partial(hidden, router_w, router_bias, w13_shard, w2_shard, top_k, w13_scale=None,
                        w2_scale=None, out=None, workspace=None, stream=None) -> torch.Tensor:
    """One tensor-parallel rank's share of the layer: fp32 [T, H], unrounded
    (see moe_forward_partial in include/moe.h).  w13_shard [E, 2 I_g, H] holds
    the rank's gate rows then its up rows, w2_shard [E, H, I_g] the matching
    down-projection columns (shard_expert_weights builds both)."""
    _need(hidden, torch.bfloat16, "hidden")
    _need(router_w, torch.bfloat16, "router_w")
    _need(w13_shard, (torch.bfloat16, torch.uint8, torch.float8_e4m3fn), "w13_shard")
    _need(w2_shard, (torch.bfloat16, torch.uint8, torch.float8_e4m3fn), "w2_shard")
    T, H = hidden.shape
    E = router_w.shape[0]
    I_g = w13_shard.shape[1] // 2
    dt = dtype_code(w13_shard)
    if out is None:
        out = torch.empty((T, H), dtype=torch.float32, device=hidden.device)
    _need(out, torch.float32, "out")
    if workspace is None:
        workspace = make_workspace(T, H, E, I_g, top_k, dt, hidden.device)
    rc = _lib.lib().moe_forward_partial(
        _ptr(hidden), _ptr(router_w), _ptr(router_bias), _ptr(w13_shard), _ptr(w2_shard), _ptr(w13_scale),
        _ptr(w2_scale), T, H, E, I_g, top_k, dt, _ptr(out), _ptr(workspace), workspace.numel(), _stream(stream))
    check(rc, "moe_forward_partial")
    return out


def sum_partials(partials, out=None, stream=None) -> torch.Tensor:
    """bf16 [T, H] = sum over ranks g = 0, 1, ... of partials[g] (fp32 [G, T, H]),
    added in rank order and rounded once."""
    _need(partials, torch.float32, "partials")
    G, T, H = partials.shape
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=partials.device)
    check(_lib.lib().moe_sum_partials(_ptr(partials), G, T, H, _ptr(out), _stream(stream)), "moe_sum_partials")
    return out


def inv_rope_fp8_quant(x, positions, cos_tab, sin_tab, codes=None, scales=None, stream=None):
    """(codes [T, nH, D] uint8 E4M3, scales [T, nH] fp32) of the fused inverse
    RoPE + per-head FP8 quantisation (see include/moe.h).  x [T, nH, D] bf16,
    positions [T] int32, cos_tab / sin_tab [max_pos, D/2] fp32."""
    _need(x, torch.bfloat16, "x")
    _need(positions, torch.int32, "positions")
    _need(cos_tab, torch.float32, "cos_tab")
    _need(sin_tab, torch.float32, "sin_tab")
    T, nH, D = x.shape
    if codes is None:
        codes = torch.empty((T, nH, D), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((T, nH), dtype=torch.float32, device=x.device)
    check(_lib.lib().moe_inv_rope_fp8_quant(_ptr(x), _ptr(positions), _ptr(cos_tab), _ptr(sin_tab), T, nH, D,
                                            cos_tab.shape[0], _ptr(codes), _ptr(scales), _stream(stream)),
          "moe_inv_rope_fp8_quant")
    return codes, scales
