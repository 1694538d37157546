"""Bit-level number codecs used by the oracle (test infrastructure only).

bfloat16: the upper 16 bits of an IEEE-754 binary32 (1 sign, 8 exponent,
7 fraction bits).  Decoding is exact; encoding rounds to nearest, ties to even.

E4M3: the OCP 8-bit floating point format "E4M3" (1 sign bit, 4 exponent bits
with bias 7, 3 fraction bits).  It has no infinities; S.1111.111 is NaN; the
largest finite magnitude is 1.75 * 2**8 = 448, which is the static factor the
Sage formula multiplies probabilities by ("P = softmax_row(S), quantized to
E4M3 as 448 * p", "FlashInfer PrimTS, Sage Attention 도입으로 8비트 양자화 및
성능 최적화 달성", section "코드 분석" item 1, README "Sage attention").
Exponent field 0 encodes subnormals m/8 * 2**-6, down to 2**-9.

All functions are vectorised over NumPy arrays and compute in float64, where
every value of both formats, and every midpoint between neighbours, is exact.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
E4M3_MIN_SUBNORMAL = 2.0 ** -9
E4M3_MIN_NORMAL = 2.0 ** -6


def bf16_bits_to_f64(bits) -> np.ndarray:
    """Decode raw bfloat16 bit patterns (uint16) to float64, exactly."""
    b = np.asarray(bits).astype(np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def f64_to_bf16_bits(x) -> np.ndarray:
    """Round float64 values to bfloat16 (nearest, ties to even); return uint16 bits.

    A single rounding from float64 (no intermediate float32).  NaN maps to the
    quiet NaN 0x7FC0; overflow rounds to +-inf as in IEEE-754.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros(x.shape, dtype=np.uint16)
    sign = np.signbit(x)
    a = np.abs(x)
    nan = np.isnan(x)
    # bfloat16: 8 significant bits, exponent range like binary32 (min normal 2**-126,
    # subnormal quantum 2**-133, max finite (2 - 2**-7) * 2**127).
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        _, e = np.frexp(a)                    # a = f * 2**e, f in [0.5, 1)
        e = e.astype(np.int64) - 1           # floor(log2 a) for a > 0
        e = np.maximum(e, -126)              # subnormal binade shares the quantum
        q = np.ldexp(1.0, (e - 7).astype(np.int64))
        n = np.rint(a / q)                   # exact scaling by a power of two; RNE
        v = n * q
    maxf = (2.0 - 2.0 ** -7) * 2.0 ** 127
    inf = ~nan & (v > maxf)
    v = np.where(inf | nan, 0.0, v)
    f32 = v.astype(np.float32)               # exact: v has at most 8 significant bits
    bits = (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    bits = np.where(inf, np.uint16(0x7F80), bits)
    bits = np.where(nan, np.uint16(0x7FC0), bits)
    bits = np.where(sign & ~nan, bits | np.uint16(0x8000), bits)
    out[...] = bits
    return out


def bf16_half_ulp(x) -> np.ndarray:
    """Half the bfloat16 spacing at |x|: the largest error of rounding x to bfloat16."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    with np.errstate(divide="ignore"):
        _, e = np.frexp(a)
    e = np.maximum(e.astype(np.int64) - 1, -126)
    return np.ldexp(1.0, (e - 8).astype(np.int64))


def e4m3_to_f64(codes) -> np.ndarray:
    """Decode E4M3 bytes (uint8) to float64, exactly; 0x7F / 0xFF decode to NaN."""
    c = np.asarray(codes).astype(np.uint8).astype(np.int64)
    s = np.where((c >> 7) & 1, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    normal = np.ldexp(1.0 + m / 8.0, (e - 7))
    sub = np.ldexp(m / 8.0, -6)
    v = np.where(e == 0, sub, normal)
    v = np.where((e == 15) & (m == 7), np.nan, v)
    return s * v


def f64_to_e4m3(x) -> np.ndarray:
    """Round float64 values to E4M3: nearest, ties to even, saturating to +-448.

    Magnitudes at or above 448 become 448 ("satfinite"); values below half the
    smallest subnormal (2**-10) become signed zero; NaN becomes 0x7F.
    """
    x = np.asarray(x, dtype=np.float64)
    sign = np.signbit(x)
    a = np.abs(x)
    nan = np.isnan(x)
    a = np.where(nan, 0.0, np.minimum(a, E4M3_MAX))
    with np.errstate(divide="ignore"):
        _, e = np.frexp(a)
    e = e.astype(np.int64) - 1                     # floor(log2 a)
    e = np.clip(e, -6, 8)                          # below 2**-6 the quantum stays 2**-9
    q = np.ldexp(1.0, e - 3)
    n = np.rint(a / q)                             # RNE on the scaled significand
    v = n * q                                      # <= 448 because a <= 448
    # encode v (exactly representable) into the code
    _, ev = np.frexp(v)
    ev = ev.astype(np.int64) - 1
    is_sub = v < E4M3_MIN_NORMAL
    mant_sub = np.rint(v / E4M3_MIN_SUBNORMAL).astype(np.int64)          # 0..7 (8 -> min normal)
    exp_field = np.where(is_sub, 0, ev + 7)
    mant_norm = np.rint((v / np.ldexp(1.0, ev) - 1.0) * 8.0).astype(np.int64)
    mant = np.where(is_sub, mant_sub, mant_norm)
    # a subnormal that rounded up to 2**-6 has mant_sub == 8: that is exponent 1, mantissa 0
    carry = is_sub & (mant_sub == 8)
    exp_field = np.where(carry, 1, exp_field)
    mant = np.where(carry, 0, mant)
    code = (exp_field << 3) | mant
    code = np.where(sign, code | 0x80, code)
    code = np.where(nan, 0x7F, code)
    return code.astype(np.uint8)
