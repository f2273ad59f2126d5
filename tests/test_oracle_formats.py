"""Pins of the oracle's number formats against torch's own casts (CPU)."""
import numpy as np
import pytest
import torch

from oracle import (
    E4M3_MAX,
    bf16_bits_to_f64,
    e4m3_code_to_f64,
    e4m3_value_to_code,
    round_to_bf16,
    round_to_e4m3_satfinite,
)


def test_e4m3_decode_all_codes_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = e4m3_code_to_f64(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    fin = ~np.isnan(ref)
    assert np.array_equal(ours[fin], ref[fin])
    assert ours[0x7E] == E4M3_MAX and np.isnan(ours[0x7F]) and np.isnan(ours[0xFF])
    assert ours[1] == 2.0 ** -9           # smallest subnormal


def test_e4m3_code_roundtrip():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = e4m3_code_to_f64(codes)
    back = e4m3_value_to_code(vals)
    # +0 and -0 both decode to zero; signbit keeps them apart
    assert np.array_equal(back, codes)


def test_e4m3_rne_matches_torch_inside_range():
    rng = np.random.default_rng(0)
    grid = np.concatenate([
        np.linspace(-463.9, 463.9, 200001),
        rng.standard_normal(100000) * 10,
        rng.standard_normal(100000) * 1e-2,
        (e4m3_code_to_f64(np.arange(0, 0x7E, dtype=np.uint8)) +
         e4m3_code_to_f64(np.arange(1, 0x7F, dtype=np.uint8))) / 2,   # exact midpoints
    ]).astype(np.float32)
    ours = round_to_e4m3_satfinite(grid.astype(np.float64))
    ref = torch.from_numpy(grid).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_saturates_beyond_range():
    x = np.array([464.0, 480.0, 1e6, -470.0, np.inf, -np.inf])
    assert np.array_equal(round_to_e4m3_satfinite(x),
                          np.array([448, 448, 448, -448, 448, -448], dtype=np.float64))
    assert np.isnan(round_to_e4m3_satfinite(np.array([np.nan])))[0]


def test_bf16_decode_all_patterns_matches_torch():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = bf16_bits_to_f64(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    fin = ~np.isnan(ref)
    assert np.array_equal(ours[fin], ref[fin])


def test_bf16_rne_matches_torch():
    rng = np.random.default_rng(1)
    base = bf16_bits_to_f64(np.arange(0, 0x7F7F, 7, dtype=np.uint32).astype(np.uint16))
    nxt = bf16_bits_to_f64(np.arange(1, 0x7F80, 7, dtype=np.uint32).astype(np.uint16))
    x = np.concatenate([
        rng.standard_normal(200000),
        rng.standard_normal(50000) * 1e-38,           # subnormal range
        (base + nxt) / 2,                              # exact ties
        -(base + nxt) / 2,
        np.array([3.3895313892515355e38, 3.4e38]),     # at / past the overflow midpoint
    ]).astype(np.float32)
    ours = round_to_bf16(x.astype(np.float64))
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(ours, ref)


@pytest.mark.parametrize("v", [1.0, -2.5, 0.0078125, 448.0, 2.0 ** -9])
def test_e4m3_value_code_value(v):
    assert e4m3_code_to_f64(e4m3_value_to_code(np.array([v])))[0] == v
