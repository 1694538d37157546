"""Pins for the oracle's bfloat16 and E4M3 codecs.

The codecs are written from the format definitions; here they are checked
exhaustively against torch's CPU casts (an independent library routine) and
against closed-form properties of the formats.
"""
import numpy as np
import torch

from oracle import codecs


def test_bf16_decode_exhaustive_matches_torch():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = codecs.bf16_bits_to_f64(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


def test_bf16_encode_matches_torch_rne():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(200_000).astype(np.float32),
        (rng.standard_normal(50_000) * 1e-38).astype(np.float32),    # subnormal range
        (rng.standard_normal(50_000) * 1e30).astype(np.float32),
    ])
    # every midpoint between two neighbouring bf16 values in [1, 4): ties go to even
    grid = np.arange(0x3F80, 0x4080, dtype=np.uint32)
    mids = ((grid << 16) | 0x8000).view(np.float32)
    x = np.concatenate([x, mids, -mids])
    ours = codecs.f64_to_bf16_bits(x.astype(np.float64))
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_bf16_half_ulp():
    assert codecs.bf16_half_ulp(1.0) == 2.0 ** -8
    assert codecs.bf16_half_ulp(3.99) == 2.0 ** -7
    assert codecs.bf16_half_ulp(4.0) == 2.0 ** -6
    assert codecs.bf16_half_ulp(-0.75) == 2.0 ** -9


def test_e4m3_decode_all_codes_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = codecs.e4m3_to_f64(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert nan.sum() == 2 and nan[0x7F] and nan[0xFF]
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


def test_e4m3_format_constants():
    v = codecs.e4m3_to_f64(np.arange(256, dtype=np.uint8))
    finite = v[np.isfinite(v)]
    assert finite.max() == 448.0 == codecs.E4M3_MAX
    assert codecs.e4m3_to_f64(np.uint8(0x7E)) == 448.0
    assert np.min(finite[finite > 0]) == 2.0 ** -9
    assert codecs.e4m3_to_f64(np.uint8(0x08)) == 2.0 ** -6     # smallest normal


def test_e4m3_encode_roundtrip_and_midpoints_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    vals = codecs.e4m3_to_f64(codes)
    fin = np.isfinite(vals)
    # exact values encode to themselves (both zeros keep their sign)
    assert np.array_equal(codecs.f64_to_e4m3(vals[fin]), codes[fin])
    # all midpoints between neighbouring positive values, and random values
    pos = np.unique(vals[fin & (vals >= 0)])
    mids = (pos[1:] + pos[:-1]) / 2
    rng = np.random.default_rng(1)
    rnd = np.concatenate([rng.uniform(0, 463.9, 100_000), np.exp(rng.uniform(-14, 6, 100_000))])
    x = np.concatenate([mids, -mids, rnd, -rnd]).astype(np.float32)
    x = x[np.abs(x) < 464.0]            # torch's cast does not saturate beyond the last midpoint
    ours = codecs.f64_to_e4m3(x.astype(np.float64))
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_saturates_and_flushes():
    assert codecs.f64_to_e4m3(1e9) == 0x7E
    assert codecs.f64_to_e4m3(-1e9) == 0xFE
    assert codecs.f64_to_e4m3(470.0) == 0x7E
    assert codecs.f64_to_e4m3(2.0 ** -11) == 0x00          # below half the smallest subnormal
    assert codecs.f64_to_e4m3(2.0 ** -10) == 0x00          # exactly half: tie to even (zero)
    assert codecs.f64_to_e4m3(1.5 * 2.0 ** -10) == 0x01    # above half: smallest subnormal
    assert codecs.f64_to_e4m3(np.nan) == 0x7F
    # 448 * p for p = 1 is the largest finite code, as the Sage formula's static factor implies
    assert codecs.f64_to_e4m3(448.0 * 1.0) == 0x7E
