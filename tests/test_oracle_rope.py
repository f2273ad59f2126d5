"""Pins of the inverse-RoPE + per-head FP8 oracle (CPU).

Each test fixes the result by something other than the oracle: the identity
and quarter-turn rotations (exact), undoing a forward rotation written here
in fp64, the rotation's norm preservation, a hand-computed golden head and
torch's E4M3 cast for the quantisation.  The last test plants the forward
sign in the oracle and checks that the golden case catches it.
"""
import os

import numpy as np
import torch

import oracle.rope_ref as rope_ref
from oracle import e4m3_code_to_f64
from oracle.rope_ref import inv_rope_fp8_ref, inv_rope_ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "inv_rope_fp8_closed_form.txt")


def golden():
    d = {}
    for ln in open(GOLDEN):
        ln = ln.split("#", 1)[0].strip()
        if ln:
            name, vals = (s.strip() for s in ln.split(";"))
            d[name] = np.array([float(v) for v in vals.split()])
    return d


def bf16(a):
    return torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).float().numpy()


def torch_per_head_codes(y):
    """Per-head E4M3 codes by torch's cast: scale = amax / 448 in fp32."""
    t = torch.tensor(y, dtype=torch.float32)
    amax = t.abs().amax(dim=-1, keepdim=True)
    scale = torch.where(amax == 0, torch.ones_like(amax), amax / 448.0)
    return (t / scale).to(torch.float8_e4m3fn).view(torch.uint8).numpy(), scale[..., 0].numpy()


def tables(max_pos, half, base=10000.0):
    inv = base ** (-np.arange(half) * 2.0 / (2 * half))
    ang = np.arange(max_pos)[:, None] * inv[None, :]
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32), ang


def test_golden_head():
    g = golden()
    x = g["x"].reshape(1, 1, 4)
    ct, st = g["cos"].reshape(1, 2), g["sin"].reshape(1, 2)
    y = inv_rope_ref(x, np.array([0]), ct, st)
    assert np.array_equal(y[0, 0], g["y"])
    codes, scale = inv_rope_fp8_ref(x, np.array([0]), ct, st)
    assert np.array_equal(e4m3_code_to_f64(codes[0, 0]), g["codes"])
    assert scale[0, 0] == np.float32(g["scale"][0])


def test_identity_rotation_is_plain_per_head_quant():
    rng = np.random.default_rng(1)
    x = bf16(rng.standard_normal((5, 3, 64)))
    ct = np.ones((8, 32), np.float32)
    st = np.zeros((8, 32), np.float32)
    pos = np.array([0, 3, 7, 1, 2])
    y = inv_rope_ref(x, pos, ct, st)
    assert np.array_equal(y, x)
    codes, scale = inv_rope_fp8_ref(x, pos, ct, st)
    tc, ts = torch_per_head_codes(x)
    assert np.array_equal(codes, tc) and np.array_equal(scale, ts)


def test_quarter_turn_is_an_exact_permutation():
    rng = np.random.default_rng(2)
    x = bf16(rng.standard_normal((4, 2, 16)))
    ct = np.zeros((1, 8), np.float32)
    st = np.ones((1, 8), np.float32)
    y = inv_rope_ref(x, np.zeros(4, int), ct, st)
    assert np.array_equal(y[..., :8], x[..., 8:])
    assert np.array_equal(y[..., 8:], -x[..., :8])


def test_undoes_a_forward_rotation():
    rng = np.random.default_rng(3)
    T, nH, D = 6, 4, 128
    half = D // 2
    ct, st, ang = tables(64, half)
    pos = rng.integers(0, 64, T)
    x = rng.standard_normal((T, nH, D))
    # forward rotation in fp64 from the angles themselves
    c, s = np.cos(ang[pos])[:, None, :], np.sin(ang[pos])[:, None, :]
    fwd = np.concatenate([x[..., :half] * c - x[..., half:] * s, x[..., half:] * c + x[..., :half] * s], -1)
    y = inv_rope_ref(fwd.astype(np.float32), pos, ct, st).astype(np.float64)
    assert np.abs(y - x).max() <= 1e-5 * np.abs(x).max()
    # a rotation keeps every pair's length
    n_in = fwd[..., :half] ** 2 + fwd[..., half:] ** 2
    n_out = y[..., :half] ** 2 + y[..., half:] ** 2
    assert np.allclose(n_in, n_out, rtol=1e-5)


def test_quantisation_matches_torch_cast_and_out_of_range_rows():
    rng = np.random.default_rng(4)
    T, nH, D = 7, 3, 64
    ct, st, _ = tables(16, D // 2)
    pos = np.array([0, 15, 16, -1, 5, 5, 9])           # 16 and -1 have no table row
    x = bf16(rng.standard_normal((T, nH, D)) * 3)
    codes, scale = inv_rope_fp8_ref(x, pos, ct, st)
    y = inv_rope_ref(x, pos, ct, st)
    tc, ts = torch_per_head_codes(y)
    ok = (pos >= 0) & (pos < 16)
    assert np.array_equal(codes[ok], tc[ok]) and np.array_equal(scale[ok], ts[ok])
    assert not codes[~ok].any() and not scale[~ok].any()
    # the largest element of every head maps to +-448
    assert np.all(np.abs(e4m3_code_to_f64(codes[ok])).max(axis=-1) == 448.0)


def test_golden_catches_the_forward_sign(monkeypatch):
    g = golden()
    orig = rope_ref.inv_rope_ref

    def forward(x, pos, c, s):          # planted mistake: rotate by plus the angle
        return orig(x, pos, c, -np.asarray(s, np.float32))

    monkeypatch.setattr(rope_ref, "inv_rope_ref", forward)
    codes, _ = rope_ref.inv_rope_fp8_ref(g["x"].reshape(1, 1, 4), np.array([0]), g["cos"].reshape(1, 2),
                                         g["sin"].reshape(1, 2))
    assert not np.array_equal(e4m3_code_to_f64(codes[0, 0]), g["codes"])
