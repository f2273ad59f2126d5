"""Seeded synthetic inputs for the fused MoE layer.

This module is shared by the tests, the benchmark and the oracle side of the
parity tests.  It holds none of the layer's arithmetic: only random draws,
storage conversions done by torch's own casts (float32 -> bfloat16, and
float32 -> float8_e4m3fn for the pre-quantised FP8 weights), and the Zipf
router bias vector.  It imports nothing else from this package.

Workloads (the five layer shapes the library is measured on):

=================  ====  ====  ===  =  ====  =====  ======  ====
name                 T     H    E   k    I   dtype  router  seed
=================  ====  ====  ===  =  ====  =====  ======  ====
tiny                 4   256    8   2   512  bf16   plain     0
decode              16  2048   64   8  1024  bf16   plain     1
decode-zipf         32  4096  128   8  1536  bf16   zipf      2
decode-fp8          64  7168  256   8  2048  fp8    plain     3
prefill-zipf      4096  4096  128   8  1536  bf16   zipf      4
=================  ====  ====  ===  =  ====  =====  ======  ====

Distributions: hidden ~ N(0, 1); router_w ~ N(0, 0.1); expert weights
~ N(0, 0.02) (before quantisation on the FP8 workload); all drawn in fp32 and
rounded to bf16 by torch's RNE cast.  FP8 weights: one fp32 scale per expert
matrix, s = amax|W| / 448, codes = E4M3(W / s).  The Zipf(s=1.1) skew is a
router bias b[e] = -1.1 * ln(e + 1): the log of the unnormalised Zipf pmf
with expert 0 the most popular (the normaliser cancels in the softmax).
"""
from __future__ import annotations

import math

import numpy as np
import torch

WORKLOADS = {
    "tiny": dict(T=4, H=256, E=8, top_k=2, I=512, dtype="bf16", zipf=False, seed=0),
    "decode": dict(T=16, H=2048, E=64, top_k=8, I=1024, dtype="bf16", zipf=False, seed=1),
    "decode-zipf": dict(T=32, H=4096, E=128, top_k=8, I=1536, dtype="bf16", zipf=True, seed=2),
    "decode-fp8": dict(T=64, H=7168, E=256, top_k=8, I=2048, dtype="fp8", zipf=False, seed=3),
    "prefill-zipf": dict(T=4096, H=4096, E=128, top_k=8, I=1536, dtype="bf16", zipf=True, seed=4),
}

_HIDDEN, _ROUTER, _W13, _W2 = 1, 2, 3, 4


def describe(wl: dict) -> str:
    return (f"T={wl['T']} H={wl['H']} E={wl['E']} top_k={wl['top_k']} I={wl['I']} "
            f"{wl['dtype']}{' zipf' if wl['zipf'] else ''}")


def _gen(device, seed: int, tensor_id: int, sub: int = 0) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1_000_003 + tensor_id * 100_003 + sub)
    return g


def _randn(shape, std, device, seed, tensor_id, sub=0):
    g = _gen(device, seed, tensor_id, sub)
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std


def zipf_bias(E: int, s: float = 1.1) -> torch.Tensor:
    return torch.tensor([-s * math.log(e + 1.0) for e in range(E)], dtype=torch.float32)


def make_hidden(wl: dict, device="cpu", seed=None, T=None) -> torch.Tensor:
    seed = wl["seed"] if seed is None else seed
    T = wl["T"] if T is None else T
    return _randn((T, wl["H"]), 1.0, device, seed, _HIDDEN).to(torch.bfloat16)


def make_router(wl: dict, device="cpu", seed=None) -> torch.Tensor:
    seed = wl["seed"] if seed is None else seed
    return _randn((wl["E"], wl["H"]), 0.1, device, seed, _ROUTER).to(torch.bfloat16)


def make_inputs(wl: dict, device="cpu", seed: int | None = None, T: int | None = None) -> dict:
    """All tensors of one layer call, on ``device``.

    Weights are drawn one expert matrix at a time (each from its own seeded
    generator), so memory stays bounded and a single expert can be redrawn.
    """
    seed = wl["seed"] if seed is None else seed
    H, E, I = wl["H"], wl["E"], wl["I"]
    fp8 = wl["dtype"] == "fp8"
    out = dict(T=wl["T"] if T is None else T, H=H, E=E, I=I, top_k=wl["top_k"], dtype=wl["dtype"])
    out["hidden"] = make_hidden(wl, device, seed, out["T"])
    out["router_w"] = make_router(wl, device, seed)
    out["router_bias"] = zipf_bias(E).to(device) if wl["zipf"] else None
    store = torch.uint8 if fp8 else torch.bfloat16
    w13 = torch.empty((E, 2 * I, H), dtype=store, device=device)
    w2 = torch.empty((E, H, I), dtype=store, device=device)
    s13 = torch.ones(E, dtype=torch.float32, device=device)
    s2 = torch.ones(E, dtype=torch.float32, device=device)
    for e in range(E):
        for dst, sc, tid, shape in ((w13, s13, _W13, (2 * I, H)), (w2, s2, _W2, (H, I))):
            w = _randn(shape, 0.02, device, seed, tid, e)
            if fp8:
                s = w.abs().max() / 448.0
                dst[e] = (w / s).to(torch.float8_e4m3fn).view(torch.uint8)
                sc[e] = s
            else:
                dst[e] = w.to(torch.bfloat16)
            del w
    out["w13"], out["w2"] = w13, w2
    out["w13_scale"] = s13 if fp8 else None
    out["w2_scale"] = s2 if fp8 else None
    return out


# --------------------------------------------------- host views for checks --
def host_bits(t: torch.Tensor) -> np.ndarray:
    """Raw storage of a bf16 (-> uint16) or uint8 tensor as a host numpy array."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.uint8:
        return t.numpy()
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    raise TypeError(f"no raw view for {t.dtype}")


class ExpertView:
    """Per-expert lazy host copy of a [E, rows, cols] weight tensor."""

    def __init__(self, t: torch.Tensor):
        self.t = t

    def __len__(self):
        return self.t.shape[0]

    def __getitem__(self, e: int) -> np.ndarray:
        return host_bits(self.t[e])
