"""Pins of the oracle's whole-layer path (R5-R8) on CPU.

Each test fixes the result by something other than the oracle itself: pure
Python loops written from the layer's definition, the dense-MLP and one-hot
special cases, closed forms of SiLU, linearity, and torch's FP8 cast.
"""
import math

import numpy as np
import pytest
import torch
from scipy.special import expit

from mixture_experts_layer_counts_b200.inputs import WORKLOADS, host_bits, make_inputs
from oracle import (
    act_quant_ref,
    bf16_bits_to_f64,
    bf16_tolerance_violation,
    e4m3_code_to_f64,
    moe_forward_ref,
    rel_l2,
    round_to_bf16,
    silu_mul,
)


def to_bits(a):
    t = torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def naive_layer(x, wr, w13, w2, k, bias=None):
    """Pure-Python loops: route, then per token per slot the gated MLP.

    Uses scipy's expit for the sigmoid and explicit loops for every sum.
    """
    T, H = len(x), len(x[0])
    E, I = len(w13), len(w13[0]) // 2
    out = []
    for t in range(T):
        logits = []
        for e in range(E):
            s = 0.0
            for h in range(H):
                s += x[t][h] * wr[e][h]
            logits.append(s + (0.0 if bias is None else float(bias[e])))
        order = sorted(range(E), key=lambda e: (-logits[e], e))[:k]
        mx = max(logits)
        den = sum(math.exp(v - mx) for v in logits)
        probs = [math.exp(logits[e] - mx) / den for e in order]
        z = sum(probs)
        acc = [0.0] * H
        for j, e in enumerate(order):
            hvec = []
            for i in range(I):
                g = sum(w13[e][i][h] * x[t][h] for h in range(H))
                u = sum(w13[e][I + i][h] * x[t][h] for h in range(H))
                hvec.append(float(round_to_bf16(np.array(g * expit(g) * u))))
            for o in range(H):
                y = sum(w2[e][o][i] * hvec[i] for i in range(I))
                acc[o] += probs[j] / z * y
        out.append(acc)
    return np.array(out)


@pytest.mark.parametrize("seed,k,bias", [(0, 2, False), (1, 3, True), (2, 1, False)])
def test_oracle_equals_naive_loops(seed, k, bias):
    rng = np.random.default_rng(seed)
    T, H, E, I = 3, 8, 4, 4
    xb = to_bits(rng.standard_normal((T, H)))
    wrb = to_bits(rng.standard_normal((E, H)) * 0.5)
    w13b = to_bits(rng.standard_normal((E, 2 * I, H)) * 0.3)
    w2b = to_bits(rng.standard_normal((E, H, I)) * 0.3)
    bvec = rng.standard_normal(E).astype(np.float32) if bias else None
    res = moe_forward_ref(xb, wrb, bvec, w13b, w2b, k)
    f = bf16_bits_to_f64
    ref = naive_layer(f(xb).tolist(), f(wrb).tolist(), f(w13b).tolist(), f(w2b).tolist(), k, bvec)
    assert np.allclose(res["out"], ref, rtol=1e-11, atol=1e-13)


def dense_gated_mlp(x, W13, W2):
    I = W13.shape[0] // 2
    out = np.zeros((x.shape[0], W2.shape[0]))
    for t in range(x.shape[0]):
        g = np.array([np.dot(W13[i], x[t]) for i in range(I)])
        u = np.array([np.dot(W13[I + i], x[t]) for i in range(I)])
        hv = round_to_bf16(g * expit(g) * u)
        out[t] = np.array([np.dot(W2[o], hv) for o in range(W2.shape[0])])
    return out


def test_topk_all_identical_experts_is_dense_mlp():
    rng = np.random.default_rng(7)
    T, H, E, I = 5, 16, 6, 8
    xb = to_bits(rng.standard_normal((T, H)))
    wrb = to_bits(rng.standard_normal((E, H)))
    one13 = to_bits(rng.standard_normal((2 * I, H)) * 0.2)
    one2 = to_bits(rng.standard_normal((H, I)) * 0.2)
    w13b = np.stack([one13] * E)
    w2b = np.stack([one2] * E)
    res = moe_forward_ref(xb, wrb, None, w13b, w2b, E)
    assert np.allclose(res["weights"].sum(axis=1), 1.0, rtol=0, atol=1e-14)
    ref = dense_gated_mlp(bf16_bits_to_f64(xb), bf16_bits_to_f64(one13), bf16_bits_to_f64(one2))
    assert np.allclose(res["out"], ref, rtol=1e-12, atol=1e-14)


def test_one_hot_routing_is_single_expert_mlp():
    rng = np.random.default_rng(8)
    T, H, E, I = 6, 16, 5, 8
    target = np.array([3, 0, 4, 4, 1, 2])
    x = rng.standard_normal((T, H))
    x[:, :E] = 0.0
    for t in range(T):
        x[t, target[t]] = 64.0              # router column e reads x[:, e]
    wr = np.zeros((E, H))
    for e in range(E):
        wr[e, e] = 1.0
    xb, wrb = to_bits(x), to_bits(wr)
    w13b = to_bits(rng.standard_normal((E, 2 * I, H)) * 0.2)
    w2b = to_bits(rng.standard_normal((E, H, I)) * 0.2)
    res = moe_forward_ref(xb, wrb, None, w13b, w2b, 1)
    assert np.array_equal(res["ids"][:, 0], target)
    xf = bf16_bits_to_f64(xb)
    for t in range(T):
        e = target[t]
        ref = dense_gated_mlp(xf[t:t + 1], bf16_bits_to_f64(w13b[e]), bf16_bits_to_f64(w2b[e]))
        assert np.allclose(res["out"][t], ref[0], rtol=1e-12, atol=1e-14)


def test_silu_closed_forms():
    c = np.array([-30.0, -3.0, -1.0, -0.5, 0.0, 0.5, 1.0, 3.0, 30.0])
    one = np.ones_like(c)
    s = silu_mul(c, one)
    assert s[4] == 0.0
    assert np.allclose(s - silu_mul(-c, one), c, rtol=1e-15, atol=1e-15)   # silu(c)-silu(-c)=c
    assert np.allclose(s, c * expit(c), rtol=1e-15, atol=0)
    assert np.allclose(silu_mul(c, 3 * one), 3 * s, rtol=1e-15, atol=0)


def test_down_projection_is_linear():
    rng = np.random.default_rng(9)
    T, H, E, I, k = 4, 16, 4, 8, 2
    xb = to_bits(rng.standard_normal((T, H)))
    wrb = to_bits(rng.standard_normal((E, H)))
    w13b = to_bits(rng.standard_normal((E, 2 * I, H)) * 0.2)
    w2 = bf16_bits_to_f64(to_bits(rng.standard_normal((E, H, I)) * 0.2))
    a = moe_forward_ref(xb, wrb, None, w13b, to_bits(w2), k)["out"]
    b = moe_forward_ref(xb, wrb, None, w13b, to_bits(2 * w2), k)["out"]
    assert np.array_equal(2 * a, b)


def test_act_quant_matches_torch_cast():
    rng = np.random.default_rng(10)
    x = bf16_bits_to_f64(to_bits(rng.standard_normal((8, 64)) * 3))
    s1, codes, xhat = act_quant_ref(x)
    assert s1 == np.float32(np.float32(np.abs(x).max()) / np.float32(448.0))
    q = torch.tensor(x.astype(np.float32)) / torch.tensor(float(s1), dtype=torch.float32)
    ref = q.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes, ref)
    assert np.abs(e4m3_code_to_f64(codes)).max() == 448.0
    s0, c0, _ = act_quant_ref(np.zeros((2, 4)))
    assert s0 == np.float32(1.0) and np.all(c0 == 0)


def test_fp8_weight_decode_matches_torch():
    wl = dict(WORKLOADS["tiny"], dtype="fp8")
    inp = make_inputs(wl, "cpu")
    e = 3
    ours = e4m3_code_to_f64(host_bits(inp["w13"][e])) * float(inp["w13_scale"][e])
    ref = (inp["w13"][e].view(torch.float8_e4m3fn).to(torch.float64) * float(inp["w13_scale"][e])).numpy()
    assert np.array_equal(ours, ref)


def test_fp8_layer_close_to_bf16_layer():
    """The FP8 path differs from the bf16 path by E4M3 quantisation noise only.

    Three mantissa bits give a few percent of relative noise per quantised
    tensor (activations, weights, intermediate); this is a sanity bound, not
    the FP8 acceptance test (which compares two FP8 computations).
    """
    wl = dict(WORKLOADS["tiny"], dtype="fp8")
    inp = make_inputs(wl, "cpu")
    args = (host_bits(inp["hidden"]), host_bits(inp["router_w"]), None)
    q = moe_forward_ref(*args, host_bits(inp["w13"]), host_bits(inp["w2"]), wl["top_k"], "fp8",
                        inp["w13_scale"].numpy(), inp["w2_scale"].numpy())
    # the same weights, dequantised and rounded to bf16, through the bf16 path
    d13 = [to_bits(e4m3_code_to_f64(host_bits(inp["w13"][e])) * float(inp["w13_scale"][e]))
           for e in range(wl["E"])]
    d2 = [to_bits(e4m3_code_to_f64(host_bits(inp["w2"][e])) * float(inp["w2_scale"][e]))
          for e in range(wl["E"])]
    b = moe_forward_ref(*args, d13, d2, wl["top_k"], "bf16")
    assert np.array_equal(q["ids"], b["ids"])
    assert 1e-3 < rel_l2(q["out"], b["out"]) < 0.1


def test_token_subset_matches_full():
    inp = make_inputs(WORKLOADS["tiny"], "cpu")
    args = (host_bits(inp["hidden"]), host_bits(inp["router_w"]), None,
            host_bits(inp["w13"]), host_bits(inp["w2"]), 2)
    full = moe_forward_ref(*args)["out"]
    sub = moe_forward_ref(*args, tokens=[1, 3])["out"]
    assert np.array_equal(sub[[1, 3]], full[[1, 3]]) and np.all(np.isnan(sub[[0, 2]]))


def test_tolerance_helpers():
    ref = np.array([1.0, -2.0, 0.0, 4.0])
    assert bf16_tolerance_violation(ref, ref) == 0.0
    rms = math.sqrt(np.mean(ref ** 2))
    edge = ref + 2e-2 * np.abs(ref) + 2e-3 * rms
    assert bf16_tolerance_violation(edge, ref) == pytest.approx(1.0)
    assert rel_l2(ref * 1.01, ref) == pytest.approx(0.01)
