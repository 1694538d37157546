"""Pins for the oracle's 8-bit Sage decode.

Closed forms derived by hand from the pages' formula (equal scores, a single
key, a two-key case whose E4M3 step is visible), the reduction to plain
softmax attention when the quantisation step is switched off, and invariants
(v_mean shifts O exactly, sfV scales O - v_mean, shuffling pages together
with their K scales is invisible).
"""
import math

import numpy as np
import pytest

from oracle import attention as oa
from oracle import sage
from oracle.codecs import e4m3_to_f64, f64_to_e4m3


def _case(rng, lens, hq, hkv, d, P=64, spare=2):
    need = [(L + P - 1) // P for L in lens]
    pages = sum(need) + spare
    perm = rng.permutation(pages)
    table = np.zeros((len(lens), max(1, max(need))), dtype=np.int64)
    off = 0
    for r, n in enumerate(need):
        table[r, :n] = perm[off:off + n]
        off += n
    S = pages * P
    q8 = rng.integers(-127, 128, (len(lens), hq, d)).astype(np.int8)
    k8 = rng.integers(-127, 128, (S, hkv, d)).astype(np.int8)
    v8 = f64_to_e4m3(16 * rng.standard_normal((S, hkv, d)))
    sf_q = np.exp(-4 + 0.5 * rng.standard_normal((len(lens), hq))).astype(np.float32)
    sf_k = np.exp(-4 + 0.5 * rng.standard_normal((S // 64, hkv))).astype(np.float32)
    sf_v = np.exp(-4 + 0.5 * rng.standard_normal((hkv, d))).astype(np.float32)
    v_mean = (0.1 * rng.standard_normal((hkv, d))).astype(np.float32)
    return q8, sf_q, k8, v8, sf_k, sf_v, v_mean, table


def test_equal_scores_give_scaled_mean_of_v8_plus_v_mean():
    rng = np.random.default_rng(20)
    d = 16
    k8 = rng.integers(-127, 128, (9, d)).astype(np.int8)
    v8 = f64_to_e4m3(16 * rng.standard_normal((9, d)))
    sf_v = rng.uniform(0.5, 2, d)
    vm = rng.standard_normal(d)
    o = sage.sage_row(np.zeros(d, np.int8), k8, v8, 0.3, np.full(9, 0.2, np.float32), sf_v, vm)
    # S = 0 everywhere: p = 1, P8 = 448, l = 9, so O = sfV * mean(V8) + v_mean
    assert np.allclose(o, sf_v * e4m3_to_f64(v8).mean(axis=0) + vm, atol=1e-13, rtol=0)


def test_single_key_returns_sf_v_times_v8_plus_v_mean():
    rng = np.random.default_rng(21)
    d = 8
    v8 = f64_to_e4m3(16 * rng.standard_normal((1, d)))
    sf_v = rng.uniform(0.5, 2, d)
    vm = rng.standard_normal(d)
    q8 = rng.integers(-127, 128, d).astype(np.int8)
    k8 = rng.integers(-127, 128, (1, d)).astype(np.int8)
    o = sage.sage_row(q8, k8, v8, 0.01, np.array([0.02], np.float32), sf_v, vm)
    assert np.allclose(o, sf_v * e4m3_to_f64(v8[0]) + vm, atol=1e-13, rtol=0)


def test_two_key_closed_form_shows_the_e4m3_step_and_unquantised_l():
    # dot = [64, 0], sfQ = 1, sfK = 1/64 (exact in fp32): S = [1, 0], m = 1,
    # p = [1, e^-1]; 448 p = [448, 164.8...] -> E4M3 [448, 160] (spacing 16 in [128, 256));
    # l = 1 + e^-1 is the unquantised sum.
    d = 4
    q8 = np.array([1, 0, 0, 0], np.int8)
    k8 = np.array([[64, 0, 0, 0], [0, 5, 0, 0]], np.int8)
    v8 = f64_to_e4m3(np.array([[1.0, 2.0, -3.0, 0.5], [4.0, -1.0, 0.25, 8.0]]))
    sf_v = np.array([1.0, 0.5, 2.0, 1.0])
    vm = np.array([0.0, 1.0, 0.0, -1.0])
    o = sage.sage_row(q8, k8, v8, 1.0, np.array([1 / 64, 1 / 64], np.float32), sf_v, vm)
    V = e4m3_to_f64(v8)
    expect = sf_v * (448 * V[0] + 160 * V[1]) / (448 * (1 + math.exp(-1))) + vm
    assert np.allclose(o, expect, atol=1e-13, rtol=0)


def test_without_quantisation_and_with_unit_scales_it_is_softmax_attention():
    rng = np.random.default_rng(22)
    lens = [70, 130, 1]
    hq, hkv, d = 4, 2, 32
    q8, _, k8, v8, _, _, _, table = _case(rng, lens, hq, hkv, d)
    B, S = len(lens), k8.shape[0]
    ones_q = np.ones((B, hq), np.float32)
    ones_k = np.ones((S // 64, hkv), np.float32)
    ones_v = np.ones((hkv, d), np.float32)
    # scale the integer dot so that softmax is not degenerate: sfQ = 1/2048 exactly
    sfq = ones_q / 2048
    o = sage.sage_decode(q8, sfq, k8, v8, ones_k, ones_v, None, table, lens, 64, quantize_p=False)
    for r, L in enumerate(lens):
        slots = oa.gather_slots(table, L, 64, r)
        for h in range(hq):
            ref, _ = oa.softmax_attend(q8[r, h][None, :].astype(np.float64),
                                       k8[slots, h // 2].astype(np.float64),
                                       e4m3_to_f64(v8[slots, h // 2]), 1 / 2048)
            assert np.allclose(o[r, h], ref[0], atol=1e-12, rtol=1e-12)


def test_v_mean_shift_and_sf_v_scaling():
    rng = np.random.default_rng(23)
    lens = [200, 64]
    q8, sf_q, k8, v8, sf_k, sf_v, vm, table = _case(rng, lens, 4, 2, 16)
    o0 = sage.sage_decode(q8, sf_q, k8, v8, sf_k, sf_v, None, table, lens, 64)
    o1 = sage.sage_decode(q8, sf_q, k8, v8, sf_k, sf_v, vm, table, lens, 64)
    G = 2
    for h in range(4):
        assert np.allclose(o1[:, h] - o0[:, h], vm[h // G][None, :], atol=1e-13, rtol=0)
    o2 = sage.sage_decode(q8, sf_q, k8, v8, sf_k, 2 * sf_v, vm, table, lens, 64)
    for h in range(4):
        assert np.allclose(o2[:, h] - vm[h // G], 2 * (o1[:, h] - vm[h // G]), atol=1e-13, rtol=0)


def test_page_shuffle_with_scales_is_invisible_and_empty_row_is_v_mean():
    rng = np.random.default_rng(24)
    lens = [129, 0, 300]
    q8, sf_q, k8, v8, sf_k, sf_v, vm, table = _case(rng, lens, 8, 4, 16)
    o1 = sage.sage_decode(q8, sf_q, k8, v8, sf_k, sf_v, vm, table, lens, 64)
    pages = k8.shape[0] // 64
    perm = rng.permutation(pages)
    inv = np.argsort(perm)
    idx = (perm[:, None] * 64 + np.arange(64)[None, :]).reshape(-1)
    o2 = sage.sage_decode(q8, sf_q, k8[idx], v8[idx], sf_k[perm], sf_v, vm, inv[table], lens, 64)
    assert np.array_equal(o1, o2)
    for h in range(8):
        assert np.array_equal(o1[1, h], vm[h // 2].astype(np.float64))


def test_top_key_quantises_to_448():
    rng = np.random.default_rng(25)
    d = 32
    q8 = rng.integers(-127, 128, d).astype(np.int8)
    k8 = rng.integers(-127, 128, (40, d)).astype(np.int8)
    sfk = np.exp(-4 + 0.5 * rng.standard_normal(40)).astype(np.float32)
    S = sage.sage_scores_f32(q8, k8, np.float32(0.02), sfk)
    p = np.exp(S.astype(np.float64) - S.max())
    codes = f64_to_e4m3(448 * p)
    assert codes[np.argmax(S)] == 0x7E
    assert e4m3_to_f64(codes).max() == 448.0


def test_scores_use_the_exact_integer_dot():
    # 127 * 127 * 128 = 2064512 < 2**24: the dot is exact, and so is its float32 value
    q8 = np.full(128, 127, np.int8)
    k8 = np.full((1, 128), 127, np.int8)
    S = sage.sage_scores_f32(q8, k8, np.float32(1.0), np.array([1.0], np.float32))
    assert S[0] == 2064512.0
    q8n = np.full(128, -127, np.int8)
    S = sage.sage_scores_f32(q8n, k8, np.float32(0.5), np.array([0.25], np.float32))
    assert S[0] == -2064512.0 / 8


def test_kv_store_sage_rows_and_block_scales():
    rng = np.random.default_rng(15)
    k8 = rng.integers(-127, 128, (256, 2, 4)).astype(np.int8)
    v8 = rng.integers(0, 256, (256, 2, 4)).astype(np.uint8)
    sf = rng.random((4, 2)).astype(np.float32)
    kn = rng.integers(-127, 128, (4, 2, 4)).astype(np.int8)
    vn = rng.integers(0, 256, (4, 2, 4)).astype(np.uint8)
    sfn = np.array([[9, 8], [7, 6], [5, 4], [3, 2]], dtype=np.float32)
    # slot 128 opens block 2, slot 70 is inside block 1, 256 is outside the pool, 0 opens block 0
    k2, v2, sf2 = sage.kv_store_sage(k8, v8, sf, [128, 70, 256, 0], kn, vn, sfn)
    assert np.array_equal(k2[128], kn[0]) and np.array_equal(v2[70], vn[1]) and np.array_equal(k2[0], kn[3])
    assert sf2[2].tolist() == [9, 8] and sf2[0].tolist() == [3, 2]
    assert np.array_equal(sf2[1], sf[1]) and np.array_equal(sf2[3], sf[3])      # mid-block token, outside slot
    untouched = [s for s in range(256) if s not in (128, 70, 0)]
    assert np.array_equal(k2[untouched], k8[untouched]) and np.array_equal(v2[untouched], v8[untouched])
    k3, v3, sf3 = sage.kv_store_sage(k8, v8, sf, [64], kn[:1], vn[:1], None)      # no scales given
    assert np.array_equal(sf3, sf) and np.array_equal(k3[64], kn[0])


def _sage_case(rng, lens, hq, hkv, spare=2):
    P = 64
    need = [(L + P - 1) // P for L in lens]
    num_pages = sum(need) + spare
    perm = rng.permutation(num_pages)
    table = np.zeros((len(lens), max(1, max(need))), dtype=np.int64)
    off = 0
    for r, n in enumerate(need):
        table[r, :n] = perm[off:off + n]
        off += n
    S = num_pages * P
    q8 = rng.integers(-127, 128, (len(lens), hq, 128)).astype(np.int8)
    k8 = rng.integers(-127, 128, (S, hkv, 128)).astype(np.int8)
    v8 = f64_to_e4m3(16 * rng.standard_normal((S, hkv, 128)))
    sfq = np.exp(-4 + 0.5 * rng.standard_normal((len(lens), hq))).astype(np.float32)
    sfk = np.exp(-4 + 0.5 * rng.standard_normal((num_pages, hkv))).astype(np.float32)
    sfv = np.exp(-4 + 0.5 * rng.standard_normal((hkv, 128))).astype(np.float32)
    vm = 0.1 * rng.standard_normal((hkv, 128))
    return q8, k8, v8, sfq, sfk, sfv, vm, table


def test_block_sparse_equals_dense_on_the_compacted_cache():
    # selecting blocks = a dense call over a page table holding only the selected pages
    rng = np.random.default_rng(41)
    lens, hq, hkv = [300, 64, 130, 1], 8, 2
    q8, k8, v8, sfq, sfk, sfv, vm, table = _sage_case(rng, lens, hq, hkv)
    mask = np.array([[1, 0, 1, 1, 0], [1, 0, 0, 0, 0], [0, 1, 1, 0, 0], [1, 0, 0, 0, 0]])
    sparse = sage.sage_decode(q8, sfq, k8, v8, sfk, sfv, vm, table, lens, 64, block_mask=mask)
    for r, L in enumerate(lens):
        nb = -(-L // 64)
        keep = [b for b in range(nb) if mask[r][b]]
        sub_table = np.array([[table[r][b] for b in keep] or [0]])
        # keys of a kept block: all 64, or the tail for the last block
        sub_len = sum(min(64, L - 64 * b) for b in keep)
        # (only the request's last block can be partial, so it is also last in the compacted row)
        dense = sage.sage_decode(q8[r:r + 1], sfq[r:r + 1], k8, v8, sfk, sfv, vm, sub_table, [sub_len], 64)
        assert np.array_equal(sparse[r], dense[0])


def test_block_sparse_all_ones_is_dense_and_none_selected_is_v_mean():
    rng = np.random.default_rng(42)
    lens, hq, hkv = [200, 70], 4, 1
    q8, k8, v8, sfq, sfk, sfv, vm, table = _sage_case(rng, lens, hq, hkv)
    dense = sage.sage_decode(q8, sfq, k8, v8, sfk, sfv, vm, table, lens, 64)
    ones = sage.sage_decode(q8, sfq, k8, v8, sfk, sfv, vm, table, lens, 64, block_mask=np.ones((2, 4), int))
    assert np.array_equal(dense, ones)
    none = sage.sage_decode(q8, sfq, k8, v8, sfk, sfv, vm, table, lens, 64, block_mask=np.zeros((2, 4), int))
    assert np.array_equal(none, np.repeat(vm[None, :, :], 2, 0).repeat(hq // hkv, 1))


def test_sage_extend_rows_equal_decodes_of_their_visible_prefix():
    rng = np.random.default_rng(43)
    lens_new, prefix, hq, hkv = [3, 1, 2], [130, 0, 64], 4, 2
    lens = [p + n for p, n in zip(prefix, lens_new)]
    _, k8, v8, _, sfk, sfv, vm, table = _sage_case(rng, lens, hq, hkv)
    T = sum(lens_new)
    q8 = rng.integers(-127, 128, (T, hq, 128)).astype(np.int8)
    sfq = np.exp(-4 + 0.5 * rng.standard_normal((T, hq))).astype(np.float32)
    cu = np.concatenate([[0], np.cumsum(lens_new)])
    o = sage.sage_extend(q8, sfq, cu, k8, v8, sfk, sfv, vm, table, lens, 64)
    for r in range(len(lens)):
        for i in range(lens_new[r]):
            row = cu[r] + i
            d = sage.sage_decode(q8[row:row + 1], sfq[row:row + 1], k8, v8, sfk, sfv, vm, table[r:r + 1],
                                 [prefix[r] + i + 1], 64)
            # the extend takes a request's rows as one block: the same terms, summed in another order
            assert np.allclose(o[row], d[0], rtol=1e-12, atol=1e-15)


def test_sage_extend_ignores_keys_after_the_row():
    rng = np.random.default_rng(44)
    lens_new, prefix, hq, hkv = [5], [60], 2, 1
    lens = [65]
    _, k8, v8, _, sfk, sfv, vm, table = _sage_case(rng, lens, hq, hkv)
    q8 = rng.integers(-127, 128, (5, hq, 128)).astype(np.int8)
    sfq = np.exp(-4 + 0.5 * rng.standard_normal((5, hq))).astype(np.float32)
    cu = np.array([0, 5])
    o1 = sage.sage_extend(q8, sfq, cu, k8, v8, sfk, sfv, vm, table, lens, 64)
    k8b, v8b = k8.copy(), v8.copy()
    last = table[0][1] * 64 + 0                      # key 64 (the last) lives in the second page
    k8b[last] = 5
    v8b[last] = 0x38
    o2 = sage.sage_extend(q8, sfq, cu, k8b, v8b, sfk, sfv, vm, table, lens, 64)
    assert np.array_equal(o1[:4], o2[:4]) and not np.array_equal(o1[4], o2[4])


def test_float32_scores_move_the_sage_decode_workload_by_rounding_only():
    """The one place the oracle takes the kernel's precision (S and its row max in float32,
    then the E4M3 code of 448 p decided from them) changes the Sage decode workload's
    outputs by far less than the 3e-2 bar: S formed entirely in float64 gives the same
    result to within 1e-3 of each row's largest element."""
    import workloads as wl
    spec = wl.SPECS["sage_decode"]
    batch = wl.make_batch(spec)
    lay = wl.make_sage_layer(spec, batch, 0)
    args = [getattr(lay, k).numpy() for k in ("q8", "sf_q", "k8", "v8", "sf_k", "sf_v", "v_mean")]
    table, lens = batch.page_table.numpy(), batch.seq_lens.numpy()
    o32 = sage.sage_decode(*args, table, lens, 64)
    o64 = sage.sage_decode(*args, table, lens, 64, score_f64=True)
    num = np.max(np.abs(o32 - o64), axis=-1)
    den = np.maximum(np.max(np.abs(o64), axis=-1), 1e-6)
    assert np.max(num / den) <= 1e-3
