"""Number formats used by the oracle, written from their definitions.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module;
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may use the oracle package.

Formats:

* bfloat16 -- the upper half of an IEEE-754 binary32: 1 sign bit, 8 exponent
  bits (bias 127), 7 fraction bits.  Rounding from a wider value is
  round-to-nearest, ties-to-even (RNE), with overflow to +-inf.
* E4M3FN -- the OCP 8-bit floating point format (OCP "8-bit Floating Point
  Specification (OFP8)", E4M3 variant): 1 sign bit, 4 exponent bits (bias 7),
  3 mantissa bits, no infinities, NaN only at S.1111.111, largest finite 448.
  Encoding here is RNE followed by saturation to +-448 ("satfinite"), the
  convention the fused-MoE FP8 path uses for both activations and the
  intermediate (the pages only say the FP8 models use one scale per tensor;
  they do not spell out the rounding, so RNE + saturation is the reading
  taken).

Every function works element-wise on numpy arrays and is vectorised only with
plain numpy primitives (frexp, rint, where), so each line can be checked
against the definitions above.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


# ---------------------------------------------------------------- bfloat16 --
def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Decode raw bfloat16 bit patterns (uint16) to exact float64 values.

    Field decode: sign = bit 15, exponent field = bits 14..7, fraction = bits
    6..0.  exponent 0 is the subnormal range (fraction * 2^-133), 255 is
    inf/NaN, otherwise (128 + fraction) * 2^(exponent - 134).
    """
    b = np.asarray(bits).astype(np.uint32)
    sign = np.where((b >> 15) & 1, -1.0, 1.0)
    ef = ((b >> 7) & 0xFF).astype(np.int64)
    frac = (b & 0x7F).astype(np.float64)
    normal = np.ldexp(128.0 + frac, (ef - 134).astype(np.int32))
    sub = np.ldexp(frac, -133)
    val = np.where(ef == 0, sub, normal)
    special = np.where(frac == 0, np.inf, np.nan)
    val = np.where(ef == 255, special, val)
    return sign * val


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 value (RNE), as float64.

    The quantum (spacing) of bfloat16 at a value whose leading bit has
    exponent p is 2^(p-7) for normal values (p >= -126) and 2^-133 below.
    Values whose magnitude rounds to 2^128 or beyond overflow to inf.
    """
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)                       # |x| = f * 2^e, f in [0.5, 1)
    p = e.astype(np.int64) - 1               # exponent of the leading bit
    qexp = np.where(p < -126, -133, p - 7)
    q = np.ldexp(np.ones_like(x), qexp.astype(np.int32))
    r = np.rint(x / q) * q                   # np.rint: ties to even
    r = np.where(np.abs(r) >= 2.0 ** 128, np.copysign(np.inf, x), r)
    r = np.where(x == 0, x, r)               # keep signed zero
    r = np.where(np.isfinite(x), r, x)
    return r


# ------------------------------------------------------------------ E4M3FN --
def e4m3_code_to_f64(codes: np.ndarray) -> np.ndarray:
    """Decode OCP E4M3FN codes (uint8) to exact float64 values.

    sign = bit 7, exponent field = bits 6..3 (bias 7), mantissa = bits 2..0.
    exponent 0: subnormal, value m * 2^-9.  Otherwise (8 + m) * 2^(e - 10).
    The pattern S.1111.111 is NaN; there is no infinity.
    """
    c = np.asarray(codes).astype(np.uint32)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    ef = ((c >> 3) & 0xF).astype(np.int64)
    m = (c & 0x7).astype(np.float64)
    normal = np.ldexp(8.0 + m, (ef - 10).astype(np.int32))
    sub = np.ldexp(m, -9)
    val = np.where(ef == 0, sub, normal)
    val = np.where((ef == 15) & (m == 7), np.nan, val)
    return sign * val


def round_to_e4m3_satfinite(x: np.ndarray) -> np.ndarray:
    """Round float64 values to E4M3FN with RNE, then saturate to +-448.

    Quantum at leading-bit exponent p: 2^(p-3) for p >= -6 (normals),
    2^-9 in the subnormal range.  NaN stays NaN.
    """
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)
    p = e.astype(np.int64) - 1
    qexp = np.where(p < -6, -9, p - 3)
    q = np.ldexp(np.ones_like(x), qexp.astype(np.int32))
    with np.errstate(invalid="ignore"):
        r = np.rint(x / q) * q
    r = np.clip(r, -E4M3_MAX, E4M3_MAX)
    r = np.where(x == 0, x, r)
    r = np.where(np.isnan(x), np.nan, r)
    r = np.where(np.isinf(x), np.copysign(E4M3_MAX, x), r)
    return r


def e4m3_value_to_code(v: np.ndarray) -> np.ndarray:
    """Encode float64 values that are exactly representable in E4M3FN."""
    v = np.asarray(v, dtype=np.float64)
    sign = (np.signbit(v)).astype(np.uint32) << 7
    a = np.abs(v)
    _, e = np.frexp(np.where(a == 0, 1.0, a))
    p = e.astype(np.int64) - 1
    is_sub = a < 2.0 ** -6
    ef = np.where(is_sub, 0, p + 7)
    mant = np.where(is_sub, a / 2.0 ** -9, a / np.ldexp(1.0, (p - 3).astype(np.int32)) - 8.0)
    code = sign | (ef.astype(np.uint32) << 3) | mant.astype(np.uint32)
    code = np.where(np.isnan(v), 0x7F, code)
    return code.astype(np.uint8)
