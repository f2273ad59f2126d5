"""Pin of the oracle's FP8 intermediate branch by a closed-form case (CPU).

tests/golden/fp8_intermediate_closed_form.txt fixes, by hand, the activation
scale s1, the intermediate scale s2, the E4M3 codes of the activations and of
the intermediate, and the layer output of a one-slot layer whose gate
pre-activation is 21 everywhere (SiLU(21) is 21 up to 7.6e-10), so that
h = 31.5 * U * (1 - d) sits just below E4M3 grid points after the division by
s2.  The case tells apart a per-token intermediate scale, truncation instead
of round-to-nearest, an amax without the absolute value and s1 used in place
of s2; the last test plants one of those mistakes in the oracle and checks
that the pin catches it.
"""
import os

import numpy as np
import torch

import oracle.moe_ref as moe_ref
from oracle import e4m3_code_to_f64, moe_forward_ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "fp8_intermediate_closed_form.txt")
H, E, I = 8, 2, 4


def golden():
    d = {}
    for ln in open(GOLDEN):
        ln = ln.split("#", 1)[0].strip()
        if ln:
            name, vals = (s.strip() for s in ln.split(";"))
            d[name] = np.array([float(v) for v in vals.split()])
    return d


def bf16_bits(a):
    t = torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def e4m3_codes(a):
    t = torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


def golden_inputs(g):
    x = np.zeros((2, H))
    x[0, 0] = x[1, 1] = 672.0
    x[:, 2] = 1.5
    wr = np.zeros((E, H))
    wr[0, 0] = wr[1, 1] = 1.0
    w13 = np.zeros((E, 2 * I, H))
    w13[:, :I, 2] = 14.0
    w13[0, I:, 2] = g["U0"]
    w13[1, I:, 2] = g["U1"]
    w2 = np.zeros((E, H, I))
    for i in range(I):
        w2[:, 4 + i, i] = 1.0
    codes13, codes2 = e4m3_codes(w13), e4m3_codes(w2)
    # every weight is an exact E4M3 value (the casts above change nothing)
    assert np.array_equal(e4m3_code_to_f64(codes13), w13)
    assert np.array_equal(e4m3_code_to_f64(codes2), w2)
    return bf16_bits(x), bf16_bits(wr), codes13, codes2, np.ones(E, np.float32), np.ones(E, np.float32)


def run_golden():
    g = golden()
    xb, wrb, c13, c2, s13, s2 = golden_inputs(g)
    return g, moe_forward_ref(xb, wrb, None, c13, c2, 1, "fp8", s13, s2, keep_intermediate=True)


def test_fp8_scales_codes_and_output_closed_form():
    g, res = run_golden()
    assert list(res["ids"][:, 0]) == [0, 1] and np.array_equal(res["weights"], np.ones((2, 1)))
    assert res["s1"] == np.float32(g["s1"][0])
    assert res["s2"] == np.float32(g["s2"][0])
    assert np.array_equal(e4m3_code_to_f64(res["xq"]), np.stack([g["xq0"], g["xq1"]]))
    # intermediate in perm order (token 0 -> row 0, token 1 -> row 1), dequantised
    s2 = float(g["s2"][0])
    assert np.array_equal(res["inter"], np.stack([g["codes0"], g["codes1"]]) * s2)
    assert np.array_equal(res["out"], np.stack([g["out0"], g["out1"]]))


def test_fp8_golden_codes_are_grid_points():
    # the expected codes are E4M3 values (the E4M3 cast leaves them unchanged)
    g = golden()
    for name in ("codes0", "codes1", "xq0", "xq1"):
        assert np.array_equal(e4m3_code_to_f64(e4m3_codes(g[name])), g[name])


def test_fp8_golden_catches_truncation(monkeypatch):
    # plant a mistake in the oracle: E4M3 encoding by truncation toward zero
    rne = moe_ref.round_to_e4m3_satfinite

    def trunc_e4m3(v):
        v = np.asarray(v, dtype=np.float64)
        r = rne(v)
        step_down = np.where(np.abs(r) > np.abs(v), np.sign(v), 0.0)
        grid = e4m3_code_to_f64(np.arange(256, dtype=np.uint8))
        grid = np.sort(np.unique(np.abs(grid[np.isfinite(grid)])))
        out = r.copy()
        for idx in zip(*np.nonzero(step_down)):
            a = abs(v[idx])
            out[idx] = np.sign(v[idx]) * grid[grid <= a].max()
        return out

    monkeypatch.setattr(moe_ref, "round_to_e4m3_satfinite", trunc_e4m3)
    g, res = run_golden()
    s2 = float(g["s2"][0])
    assert not np.array_equal(res["inter"], np.stack([g["codes0"], g["codes1"]]) * s2)
