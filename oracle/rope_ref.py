"""Oracle of the fused inverse-RoPE + per-head FP8 quantisation kernel.

TEST INFRASTRUCTURE ONLY.  This module is imported, called or executed only
by ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline legs of
``bench.py``; the CUDA library never uses it and shares no code with it.

What it computes.  The pages name the kernel (a fused RoPE + FP8 quantisation
kernel, per head, whose token count must not be a compile-time
specialisation: "AWS details MoE kernel fixes for SageMaker, upstreams them
to vLLM", third fix; "Fused MoE on Hopper, bit-exact vLLM across processes,
and linear attention on TPUs", TL;DR) but give no formula.  The readings
taken:

  Q0  input x [T, nH, D] bf16 (a head vector that carries the rotary
      position embedding), positions pos [T] int32, and the rotary table the
      serving engine keeps in fp32: cos_tab, sin_tab [max_pos, D/2].
  Q1  rotation pairs: element i is paired with element i + D/2 (the split
      into halves), angle index i; the inverse rotation turns each pair by
      minus the angle:
          y[i]       = x[i] * c + x[i + D/2] * s
          y[i + D/2] = x[i + D/2] * c - x[i] * s
      with c = cos_tab[pos[t], i], s = sin_tab[pos[t], i].
  Q2  arithmetic in fp32 as the kernel performs it: each product rounded to
      fp32, then the sum (or difference) rounded to fp32 (no fused
      multiply-add), so the integer codes below are decided in the same
      precision on both sides.
  Q3  per-head quantisation: one scale per (token, head),
      scale = fp32(amax_d |y|) / 448 (one fp32 division; amax 0 gives 1),
      code = E4M3(fp32(y / scale)), round-to-nearest-even, saturating to
      +-448 (the E4M3 convention of the layer's FP8 path).
  Q4  a position outside [0, max_pos) has no table row: its head vectors
      get code 0 and scale 0.

Pins live in ``tests/test_oracle_rope.py``: the identity rotation, the
quarter turn (an exact permutation with a sign), undoing a forward rotation
written independently in fp64, norm preservation, a hand-computed golden
case and the E4M3 cast of torch.
"""
from __future__ import annotations

import numpy as np

from .formats import E4M3_MAX, e4m3_value_to_code, round_to_e4m3_satfinite


def inv_rope_ref(x: np.ndarray, pos: np.ndarray, cos_tab: np.ndarray, sin_tab: np.ndarray) -> np.ndarray:
    """Q1-Q2: the inversely rotated head vectors, fp32 [T, nH, D].

    ``x`` holds the decoded bf16 values (any float array), ``pos`` [T],
    ``cos_tab`` / ``sin_tab`` [max_pos, D/2] fp32.  Rows whose position is
    out of range come back as zeros (Q4)."""
    x = np.asarray(x, dtype=np.float32)
    T, nH, D = x.shape
    half = D // 2
    cos_tab = np.asarray(cos_tab, dtype=np.float32)
    sin_tab = np.asarray(sin_tab, dtype=np.float32)
    y = np.zeros((T, nH, D), dtype=np.float32)
    for t in range(T):
        p = int(pos[t])
        if not 0 <= p < cos_tab.shape[0]:
            continue
        c = cos_tab[p][None, :]            # [1, D/2], broadcast over heads
        s = sin_tab[p][None, :]
        a = x[t, :, :half]
        b = x[t, :, half:]
        # numpy float32 arithmetic: every product and every sum rounded to fp32
        y[t, :, :half] = (a * c) + (b * s)
        y[t, :, half:] = (b * c) - (a * s)
    return y


def per_head_fp8_ref(y: np.ndarray, valid: np.ndarray):
    """Q3-Q4: (codes uint8 [T, nH, D], scales fp32 [T, nH]) of fp32 vectors."""
    y = np.asarray(y, dtype=np.float32)
    amax = np.abs(y).max(axis=2)                              # fp32, exact
    scale = np.where(amax == 0, np.float32(1.0), amax / np.float32(E4M3_MAX)).astype(np.float32)
    q = (y / scale[:, :, None]).astype(np.float32)           # one fp32 division per element
    codes = e4m3_value_to_code(round_to_e4m3_satfinite(q.astype(np.float64)))
    codes = np.where(valid[:, None, None], codes, np.uint8(0)).astype(np.uint8)
    scale = np.where(valid[:, None], scale, np.float32(0.0)).astype(np.float32)
    return codes, scale


def inv_rope_fp8_ref(x, pos, cos_tab, sin_tab):
    """The whole kernel (Q0-Q4): (codes [T, nH, D] uint8, scales [T, nH] fp32)."""
    pos = np.asarray(pos)
    valid = (pos >= 0) & (pos < np.asarray(cos_tab).shape[0])
    return per_head_fp8_ref(inv_rope_ref(x, pos, cos_tab, sin_tab), valid)
