"""Pins of the FP8-KV decode oracle (oracle.attention.decode_fp8).

An FP8 cache of codes whose dequantised values are exact in bf16 must give exactly
the bf16 decode of those values (itself pinned against torch SDPA and plain loops);
the result must agree with torch SDPA on the dequantised tensors; trading a power of
two between the codes and k_scale changes nothing; v_scale scales O linearly.
"""
import math

import numpy as np
import torch

from oracle import attention as oa
from oracle.codecs import e4m3_to_f64, f64_to_bf16_bits, f64_to_e4m3


def _case(rng, lens, hq, hkv, d, P, spare=2):
    need = [(L + P - 1) // P for L in lens]
    num_pages = sum(need) + spare
    perm = rng.permutation(num_pages)
    table = np.zeros((len(lens), max(1, max(need))), dtype=np.int64)
    off = 0
    for r, n in enumerate(need):
        table[r, :n] = perm[off:off + n]
        off += n
    S = num_pages * P
    k8 = f64_to_e4m3(16 * rng.standard_normal((S, hkv, d)))
    v8 = f64_to_e4m3(16 * rng.standard_normal((S, hkv, d)))
    q = f64_to_bf16_bits(rng.standard_normal((len(lens), hq, d)))
    return q, k8, v8, table


def test_fp8_decode_equals_bf16_decode_of_the_dequantised_cache():
    rng = np.random.default_rng(31)
    lens, hq, hkv, d, P = [200, 1, 77], 8, 2, 32, 16
    q, k8, v8, table = _case(rng, lens, hq, hkv, d, P)
    ks, vs = 1 / 16, 1 / 8          # powers of two: every dequantised value is exact in bf16
    kb = f64_to_bf16_bits(ks * e4m3_to_f64(k8))
    vb = f64_to_bf16_bits(vs * e4m3_to_f64(v8))
    o8, l8 = oa.decode_fp8(q, k8, v8, ks, vs, table, lens, P, 1 / math.sqrt(d))
    ob, lb = oa.decode(q, kb, vb, table, lens, P, 1 / math.sqrt(d))
    assert np.array_equal(o8, ob) and np.array_equal(l8, lb)


def test_fp8_decode_matches_torch_sdpa_on_dequantised_tensors():
    rng = np.random.default_rng(32)
    lens, hq, hkv, d, P = [130, 64], 4, 1, 64, 64
    q, k8, v8, table = _case(rng, lens, hq, hkv, d, P)
    ks, vs = 0.0371, 0.0193        # arbitrary scales
    o, _ = oa.decode_fp8(q, k8, v8, ks, vs, table, lens, P, 0.125)
    from oracle.codecs import bf16_bits_to_f64
    for r, L in enumerate(lens):
        slots = oa.gather_slots(table, L, P, r)
        K = torch.from_numpy(ks * e4m3_to_f64(k8[slots])).permute(1, 0, 2)
        V = torch.from_numpy(vs * e4m3_to_f64(v8[slots])).permute(1, 0, 2)
        Q = torch.from_numpy(bf16_bits_to_f64(q[r]))[:, None, :]
        ref = torch.nn.functional.scaled_dot_product_attention(Q, K.repeat_interleave(hq, 0),
                                                               V.repeat_interleave(hq, 0), scale=0.125)
        assert np.allclose(o[r], ref[:, 0, :].numpy(), atol=1e-12, rtol=0)


def test_fp8_scales_trade_with_the_codes_and_scale_v_linearly():
    rng = np.random.default_rng(33)
    lens, hq, hkv, d, P = [90, 33], 4, 2, 16, 1
    q, _, v8, table = _case(rng, lens, hq, hkv, d, P)
    S = v8.shape[0]
    # codes with exponent field >= 2 halve exactly (no subnormal step)
    k_val = (np.sign(rng.standard_normal((S, hkv, d))) * 2.0 ** rng.integers(-4, 6, (S, hkv, d))
             * (1 + rng.integers(0, 8, (S, hkv, d)) / 8))
    k8 = f64_to_e4m3(k_val)
    k8_half = f64_to_e4m3(e4m3_to_f64(k8) / 2)
    assert np.array_equal(e4m3_to_f64(k8_half) * 2, e4m3_to_f64(k8))
    o1, l1 = oa.decode_fp8(q, k8, v8, 0.05, 0.3, table, lens, P, 0.25)
    o2, l2 = oa.decode_fp8(q, k8_half, v8, 0.1, 0.3, table, lens, P, 0.25)
    o3, _ = oa.decode_fp8(q, k8, v8, 0.05, 0.6, table, lens, P, 0.25)
    assert np.allclose(o1, o2, atol=1e-13, rtol=0) and np.allclose(l1, l2, atol=1e-13, rtol=0)
    assert np.allclose(o3, 2 * o1, atol=1e-13, rtol=0)
