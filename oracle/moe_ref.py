"""fp64 CPU oracle of the fused Mixture-of-Experts layer at decode time.

TEST INFRASTRUCTURE ONLY.  This package is imported, called or executed only
by ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py``.  The product path (the CUDA
library and its Python binding) never touches it and shares no code with it.

What the layer computes.  The pages describe fused MoE only in words: one
batched GPU operation that does the routing of tokens, the movement of their
data and the experts' arithmetic ("AWS describes a fused MoE optimization for
the NVIDIA Hopper architecture", body), with the scaling, the matrix products
and the aggregation of expert outputs done in one pass ("AWS details MoE
kernel fixes...", body paragraph on the Triton backend).  The step-by-step
definition followed here is the plain gated-MLP MoE layer:

  R0  decode the given bf16 / E4M3 bytes exactly; dequantised weight =
      code value * per-expert fp32 scale.
  R1  router logits l[t,e] = sum_h x[t,h] * Wr[e,h] (+ bias[e]), defined on
      the exact real numbers.  fp64 BLAS is used with a rigorous error bound;
      any token whose top-(k+1) ordering is not certified by that bound is
      recomputed with exact integer arithmetic.
  R2  top-k: the k largest logits, in descending order, exact ties broken
      toward the lower expert index.
  R3  weights: softmax over all E logits, then the k selected probabilities
      renormalised to sum to one.
  R4  align: counts[e], offsets = exclusive prefix sum, perm = flat indices
      f = t*k + j sorted stably by expert (ascending f inside an expert),
      inv_perm[perm[p]] = p.
  R5  (FP8 only) per-tensor activation quantisation: s1 = fp32(amax|x|)/448
      in fp32, x_q = E4M3(fp32(x / s1)) with RNE and saturation; x_hat =
      x_q * s1.  amax == 0 gives s1 = 1.
  R6  per assignment (t, j, e): g = W1[e] x_hat_t, u = W3[e] x_hat_t (W1 = rows
      [0, I) of w13[e], W3 = rows [I, 2I)), h = g*u / (1 + exp(-g)); rounded
      once to bf16 (bf16 path) or quantised per tensor to E4M3 with
      s2 = fp32(amax|h|)/448 (FP8 path).
  R7  y = W2[e] h_hat; out_t = sum_j w[t,j] * y[t,j] in slot order j = 0..k-1,
      returned unrounded in fp64.

Parity pins for every function live in ``tests/test_oracle_*.py``: brute
force on tiny inputs, invariants, closed forms and library routines for the
number formats.  No function in this module is "parity unpinned".
"""
from __future__ import annotations

import math

import numpy as np

from .formats import (
    E4M3_MAX,
    bf16_bits_to_f64,
    e4m3_code_to_f64,
    e4m3_value_to_code,
    round_to_bf16,
    round_to_e4m3_satfinite,
)

U64 = 2.0 ** -53          # unit roundoff of binary64
EXACT_SCALE = 300         # every bf16*bf16 product is a multiple of 2^-266,
                          # every fp32 bias a multiple of 2^-149


# ------------------------------------------------------------------- R0 -----
def decode_weight(raw: np.ndarray, scale: float | None) -> np.ndarray:
    """Exact fp64 value of one expert matrix (R0).

    ``raw`` is uint16 (bf16 bit patterns) or uint8 (E4M3 codes, then ``scale``
    is the matrix's fp32 scale).  code * scale is exact in fp64 (4 + 24
    significant bits).
    """
    if raw.dtype == np.uint16:
        return bf16_bits_to_f64(raw)
    if raw.dtype == np.uint8:
        return e4m3_code_to_f64(raw) * float(np.float32(scale))
    raise TypeError(f"unsupported weight storage {raw.dtype}")


# ------------------------------------------------------------- R1 - R3 ------
def router_logits(x: np.ndarray, wr: np.ndarray, bias: np.ndarray | None):
    """fp64 logits and a rigorous per-logit bound on their rounding error (R1).

    Products of two bf16 values are exact in fp64, so the only error is the
    summation: for any summation order |fl(sum) - sum| <= gamma_n * sum|terms|
    with gamma_n = n*u/(1-n*u).  Adding the fp32 bias costs one more rounding.
    """
    L = x @ wr.T
    S = np.abs(x) @ np.abs(wr).T
    n = x.shape[1] + 2
    gamma = n * U64 / (1.0 - n * U64)
    if bias is not None:
        L = L + np.asarray(bias, dtype=np.float32).astype(np.float64)[None, :]
    R = gamma * S * (1.0 + 1e-6) + 4.0 * U64 * np.abs(L)
    return L, R


def exact_logit_scaled(xrow: np.ndarray, wrow: np.ndarray, b: float | None) -> int:
    """Exact value of one logit times 2^EXACT_SCALE, as a Python integer."""
    acc = 0
    one = 1 << EXACT_SCALE
    prods = xrow * wrow                         # exact: bf16 * bf16 in fp64
    for p in prods[prods != 0.0]:
        num, den = float(p).as_integer_ratio()  # den is a power of two
        acc += num * (one // den)
    if b is not None and b != 0.0:
        num, den = float(np.float32(b)).as_integer_ratio()
        acc += num * (one // den)
    return acc


def topk_exact_order(values_by_expert: dict, k: int) -> list:
    """Order experts by (value descending, index ascending) and take k (R2)."""
    keys = sorted(values_by_expert, key=lambda e: (-values_by_expert[e], e))
    return keys[:k]


def route_ref(x: np.ndarray, wr: np.ndarray, bias: np.ndarray | None, k: int):
    """Router (R1-R3): returns ids [T,k] int32, weights [T,k] fp64, logits.

    Selection is on the exact logits; a token whose fp64 ordering of its
    top k+1 entries is not separated by twice the error bound is re-ranked
    exactly.  Weights come from the fp64 logits.
    """
    T, E = x.shape[0], wr.shape[0]
    if not 1 <= k <= E:
        raise ValueError("top_k must lie in [1, E]")
    L, R = router_logits(x, wr, bias)
    ids = np.zeros((T, k), dtype=np.int32)
    n_exact = 0
    for t in range(T):
        row = L[t]
        r = float(R[t].max())
        order = sorted(range(E), key=lambda e: (-row[e], e))
        top = [row[e] for e in order[: min(k + 1, E)]]
        certified = all(top[i] - top[i + 1] > 2.0 * r for i in range(len(top) - 1))
        if certified:
            ids[t] = order[:k]
            continue
        n_exact += 1
        kth = row[order[k - 1]]
        cand = [e for e in range(E) if row[e] + 2.0 * r >= kth]
        b = None if bias is None else bias
        exact = {e: exact_logit_scaled(x[t], wr[e], None if b is None else float(b[e]))
                 for e in cand}
        ids[t] = topk_exact_order(exact, k)
    # R3: softmax over all experts, then renormalise the selected entries.
    m = L.max(axis=1, keepdims=True)
    p = np.exp(L - m)
    p = p / p.sum(axis=1, keepdims=True)
    sel = np.take_along_axis(p, ids.astype(np.int64), axis=1)
    w = sel / sel.sum(axis=1, keepdims=True)
    return ids, w, L, n_exact


# ------------------------------------------------------------------ R4 ------
def align_ref(ids: np.ndarray, E: int):
    """Group the T*k assignments by expert (R4).

    counts[e] = number of (t, j) with ids[t, j] == e; offsets = exclusive
    prefix sum (length E+1); perm[p] = flat index t*k+j of the p-th assignment
    in expert-major order, ascending flat index inside an expert; inv_perm is
    its inverse.
    """
    flat = ids.reshape(-1).astype(np.int64)
    counts = np.bincount(flat, minlength=E).astype(np.int32)
    offsets = np.zeros(E + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    perm = np.argsort(flat, kind="stable").astype(np.int32)
    inv_perm = np.empty_like(perm)
    inv_perm[perm] = np.arange(flat.size, dtype=np.int32)
    return counts, offsets, perm, inv_perm


# ------------------------------------------------------------------ R5 ------
def act_quant_ref(x: np.ndarray):
    """Per-tensor dynamic E4M3 quantisation of the bf16 activations (R5).

    s1 = fp32(amax|x|) / 448 as one fp32 division; x_q = E4M3 RNE-satfinite of
    the fp32 quotient x / s1.  Returns (s1 as np.float32, codes uint8, x_hat).
    """
    amax = np.float32(np.abs(x).max()) if x.size else np.float32(0.0)
    s1 = np.float32(1.0) if amax == 0 else np.float32(amax / np.float32(E4M3_MAX))
    q = (x.astype(np.float32) / s1).astype(np.float64)    # IEEE fp32 division
    xq = round_to_e4m3_satfinite(q)
    return s1, e4m3_value_to_code(xq), xq * np.float64(s1)


# ------------------------------------------------------------------ R6 ------
def silu_mul(g: np.ndarray, u: np.ndarray) -> np.ndarray:
    """SiLU(gate) * up = g * u / (1 + exp(-g)), in fp64 (R6)."""
    with np.errstate(over="ignore"):
        return g * u / (1.0 + np.exp(-g))


# -------------------------------------------------------------- R0 - R7 -----
def moe_forward_ref(hidden_bits, router_w_bits, router_bias, w13, w2, top_k,
                    dtype="bf16", w13_scale=None, w2_scale=None, tokens=None,
                    keep_intermediate=False):
    """Whole layer (R0-R7).

    ``w13[e]`` / ``w2[e]`` may be numpy arrays or any object indexable by
    expert (a lazy accessor), holding bf16 bit patterns (uint16) or E4M3 codes
    (uint8).  ``tokens``: optional subset of token indices whose outputs are
    wanted (bf16 path computes only their assignments; the FP8 path still
    needs every assignment's intermediate for the per-tensor scale s2, and
    then restricts the down projection).

    Returns a dict with ids, weights, logits, counts, offsets, perm, inv_perm,
    s1/s2/xq (FP8), out [T,H] fp64 (rows outside ``tokens`` are NaN) and,
    when asked, the rounded intermediate in perm order.
    """
    fp8 = dtype == "fp8"
    x = bf16_bits_to_f64(hidden_bits)
    wr = bf16_bits_to_f64(router_w_bits)
    T, H = x.shape
    E = wr.shape[0]
    k = top_k
    ids, wts, L, n_exact = route_ref(x, wr, router_bias, k)
    counts, offsets, perm, inv_perm = align_ref(ids, E)
    res = dict(ids=ids, weights=wts, logits=L, n_exact=n_exact, counts=counts,
               offsets=offsets, perm=perm, inv_perm=inv_perm)
    if fp8:
        s1, xq_codes, xhat = act_quant_ref(x)
        res.update(s1=s1, xq=xq_codes)
    else:
        xhat = x

    want = np.ones(T, dtype=bool) if tokens is None else np.isin(np.arange(T), tokens)
    A = T * k
    need_row = want[perm // k]                 # perm position -> wanted?
    if fp8:
        need_row[:] = True                     # s2 needs every intermediate row

    # R6: gate/up projections and SiLU(g)*u per expert, rows in perm order.
    h = {}
    amax_h = 0.0
    I = None
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        rows = [p for p in range(lo, hi) if need_row[p]]
        if not rows:
            continue
        W = decode_weight(np.asarray(w13[e]), None if w13_scale is None else w13_scale[e])
        I = W.shape[0] // 2
        toks = perm[rows] // k
        Xe = xhat[toks]
        g = Xe @ W[:I].T
        u = Xe @ W[I:].T
        he = silu_mul(g, u)
        for r, p in enumerate(rows):
            h[p] = he[r]
        if he.size:
            amax_h = max(amax_h, float(np.abs(he).max()))
    if fp8:
        a32 = np.float32(amax_h)
        s2 = np.float32(1.0) if a32 == 0 else np.float32(a32 / np.float32(E4M3_MAX))
        res["s2"] = s2
        hhat = {p: round_to_e4m3_satfinite(v / np.float64(s2)) * np.float64(s2) for p, v in h.items()}
    else:
        hhat = {p: round_to_bf16(v) for p, v in h.items()}
    if keep_intermediate and I is not None:
        inter = np.full((A, I), np.nan)
        for p, v in hhat.items():
            inter[p] = v
        res["inter"] = inter

    # R7: down projection, then router-weighted sum over slots j = 0..k-1.
    y = {}
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        rows = [p for p in range(lo, hi) if want[perm[p] // k]]
        if not rows:
            continue
        W2 = decode_weight(np.asarray(w2[e]), None if w2_scale is None else w2_scale[e])
        He = np.stack([hhat[p] for p in rows])
        Ye = He @ W2.T
        for r, p in enumerate(rows):
            y[int(perm[p])] = Ye[r]
    out = np.full((T, H), np.nan)
    for t in np.nonzero(want)[0]:
        acc = np.zeros(H)
        for j in range(k):
            acc = acc + wts[t, j] * y[t * k + j]
        out[t] = acc
    res["out"] = out
    return res


def bf16_tolerance_violation(gpu: np.ndarray, ref: np.ndarray, extra=None) -> float:
    """Largest ratio |gpu - ref| / (2e-2 |ref| + 2e-3 rms(ref) + extra) (R8).

    A value <= 1 passes the bf16 acceptance bound; rms is over all compared
    elements.  ``extra`` (same shape, default 0) widens the bound where an
    intermediate value's bf16 rounding has two correct results (its exact
    value sits closer to a rounding midpoint than fp32 arithmetic resolves).
    """
    ref = np.asarray(ref, dtype=np.float64)
    gpu = np.asarray(gpu, dtype=np.float64)
    rms = math.sqrt(float(np.mean(ref * ref))) if ref.size else 0.0
    bound = 2e-2 * np.abs(ref) + 2e-3 * rms
    if extra is not None:
        bound = bound + np.asarray(extra, dtype=np.float64)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.abs(gpu - ref) / bound
    ratio = np.where(bound == 0, np.where(gpu == ref, 0.0, np.inf), ratio)
    return float(ratio.max()) if ratio.size else 0.0


def rel_l2(gpu: np.ndarray, ref: np.ndarray) -> float:
    """Relative L2 error ||gpu - ref|| / ||ref|| (FP8 acceptance, R8)."""
    ref = np.asarray(ref, dtype=np.float64)
    d = np.asarray(gpu, dtype=np.float64) - ref
    nr = float(np.sqrt(np.sum(ref * ref)))
    return float(np.sqrt(np.sum(d * d))) / nr if nr > 0 else float(np.sqrt(np.sum(d * d)))
