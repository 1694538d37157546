"""Pins for the oracle's slot gather, DECODE, EXTEND and LSE merge.

Each pin ties the oracle to something other than itself: closed forms
(a single key returns V, equal scores return the mean of V), invariants
(adding a constant row to V, shuffling the physical slots, causal
independence from future keys), a plain-loop materialised N x N computation,
and library routines (torch's fp64 scaled_dot_product_attention, scipy's
logsumexp).
"""
import math

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

from oracle import attention as oa
from oracle.codecs import bf16_bits_to_f64, f64_to_bf16_bits


def _bf16(rng, *shape, scale=1.0):
    return f64_to_bf16_bits(rng.standard_normal(shape) * scale)


def _paged_case(rng, lens, hq, hkv, d, page_size, spare=3):
    """Random pools and a scattered page table for the given lengths (bf16 bits)."""
    need = [(L + page_size - 1) // page_size for L in lens]
    num_pages = sum(need) + spare
    perm = rng.permutation(num_pages)
    pitch = max(1, max(need))
    table = np.zeros((len(lens), pitch), dtype=np.int64)
    off = 0
    for r, n in enumerate(need):
        table[r, :n] = perm[off:off + n]
        off += n
    slots = num_pages * page_size
    k = _bf16(rng, slots, hkv, d)
    v = _bf16(rng, slots, hkv, d)
    return k, v, table


def test_gather_slots_closed_form():
    table = np.array([[5, 2, 9], [1, 0, 0]])
    assert list(oa.gather_slots(table, 7, 3, 0)) == [15, 16, 17, 6, 7, 8, 27]
    assert list(oa.gather_slots(table, 2, 3, 1)) == [3, 4]
    # page size 1: the table is req_to_token itself
    assert list(oa.gather_slots(np.array([[4, 8, 1]]), 3, 1, 0)) == [4, 8, 1]
    assert len(oa.gather_slots(table, 0, 3, 0)) == 0


def test_single_key_returns_v():
    rng = np.random.default_rng(2)
    k, v, table = _paged_case(rng, [1], 4, 2, 16, 1)
    q = _bf16(rng, 1, 4, 16)
    o, lse = oa.decode(q, k, v, table, [1], 1, 0.3)
    slot = table[0, 0]
    for h in range(4):
        assert np.array_equal(o[0, h], bf16_bits_to_f64(v[slot, h // 2]))
        s = 0.3 * bf16_bits_to_f64(q[0, h]) @ bf16_bits_to_f64(k[slot, h // 2])
        assert lse[0, h] == pytest.approx(s, abs=1e-12)


def test_equal_scores_return_mean_of_v():
    rng = np.random.default_rng(3)
    lens = [37, 5]
    k, v, table = _paged_case(rng, lens, 4, 4, 32, 4)
    q = np.zeros((2, 4, 32), dtype=np.uint16)                 # q = 0: every score is 0
    o, lse = oa.decode(q, k, v, table, lens, 4, 1.0)
    for r, L in enumerate(lens):
        slots = oa.gather_slots(table, L, 4, r)
        for h in range(4):
            mean = bf16_bits_to_f64(v[slots, h]).mean(axis=0)
            assert np.allclose(o[r, h], mean, atol=1e-13, rtol=0)
            assert lse[r, h] == pytest.approx(math.log(L), abs=1e-13)


def test_constant_shift_of_v_shifts_output():
    rng = np.random.default_rng(4)
    q = rng.standard_normal((5, 16))
    k = rng.standard_normal((23, 16))
    v = rng.standard_normal((23, 16))
    c = rng.standard_normal(16)
    o1, l1 = oa.softmax_attend(q, k, v, 0.25)
    o2, l2 = oa.softmax_attend(q, k, v + c, 0.25)
    assert np.allclose(o2, o1 + c, atol=1e-13, rtol=0)
    assert np.array_equal(l1, l2)


def test_shuffling_physical_slots_is_invisible():
    rng = np.random.default_rng(5)
    lens = [50, 17, 64]
    for P in (1, 16):
        k, v, table = _paged_case(rng, lens, 8, 2, 32, P)
        q = _bf16(rng, 3, 8, 32)
        o1, l1 = oa.decode(q, k, v, table, lens, P, 0.2)
        num_pages = k.shape[0] // P
        perm = rng.permutation(num_pages)               # new page i holds old page perm[i]
        inv = np.argsort(perm)
        idx = (perm[:, None] * P + np.arange(P)[None, :]).reshape(-1)
        k2, v2 = k[idx], v[idx]
        t2 = inv[table]
        o2, l2 = oa.decode(q, k2, v2, t2, lens, P, 0.2)
        assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_decode_matches_plain_loop_materialised_reference():
    rng = np.random.default_rng(6)
    lens = [9, 3]
    hq, hkv, d = 4, 2, 8
    k, v, table = _paged_case(rng, lens, hq, hkv, d, 2)
    q = _bf16(rng, 2, hq, d)
    o, lse = oa.decode(q, k, v, table, lens, 2, 0.7)
    for r, L in enumerate(lens):
        slots = oa.gather_slots(table, L, 2, r)
        for h in range(hq):
            kk = bf16_bits_to_f64(k[slots, h // 2]).tolist()
            vv = bf16_bits_to_f64(v[slots, h // 2]).tolist()
            qq = [bf16_bits_to_f64(q[r, h]).tolist()]
            O, LSE = oa.materialised_reference(qq, kk, vv, 0.7)
            assert np.allclose(o[r, h], O[0], atol=1e-12, rtol=0)
            assert lse[r, h] == pytest.approx(LSE[0], abs=1e-12)


def test_decode_matches_torch_sdpa_and_scipy_logsumexp():
    rng = np.random.default_rng(7)
    lens = [300, 1, 129]
    hq, hkv, d = 8, 2, 64
    k, v, table = _paged_case(rng, lens, hq, hkv, d, 1)
    q = _bf16(rng, 3, hq, d)
    scale = 1 / math.sqrt(d)
    o, lse = oa.decode(q, k, v, table, lens, 1, scale)
    for r, L in enumerate(lens):
        slots = oa.gather_slots(table, L, 1, r)
        K = torch.from_numpy(bf16_bits_to_f64(k[slots])).permute(1, 0, 2)        # [Hkv, L, D]
        V = torch.from_numpy(bf16_bits_to_f64(v[slots])).permute(1, 0, 2)
        Q = torch.from_numpy(bf16_bits_to_f64(q[r]))[:, None, :]                  # [Hq, 1, D]
        ref = torch.nn.functional.scaled_dot_product_attention(
            Q, K.repeat_interleave(hq // hkv, 0), V.repeat_interleave(hq // hkv, 0), scale=scale)
        assert np.allclose(o[r], ref[:, 0, :].numpy(), atol=1e-12, rtol=0)
        for h in range(hq):
            s = scale * (K[h // (hq // hkv)].numpy() @ Q[h, 0].numpy())
            assert lse[r, h] == pytest.approx(logsumexp(s), abs=1e-12)


def test_empty_sequence_gives_zero_and_minus_inf():
    rng = np.random.default_rng(8)
    k, v, table = _paged_case(rng, [4, 0], 2, 1, 8, 1)
    q = _bf16(rng, 2, 2, 8)
    o, lse = oa.decode(q, k, v, table, [4, 0], 1, 1.0)
    assert np.all(o[1] == 0) and np.all(np.isneginf(lse[1]))
    assert np.all(np.isfinite(o[0]))


def _extend_case(rng, prefix, new, hq, hkv, d, P):
    lens = [p + n for p, n in zip(prefix, new)]
    k, v, table = _paged_case(rng, lens, hq, hkv, d, P)
    cu = np.concatenate([[0], np.cumsum(new)]).astype(np.int64)
    q = _bf16(rng, int(cu[-1]), hq, d)
    return q, cu, k, v, table, lens


def test_extend_matches_plain_loop_causal_reference():
    rng = np.random.default_rng(9)
    prefix, new = [5, 0], [4, 6]
    hq, hkv, d, P = 2, 1, 8, 4
    q, cu, k, v, table, lens = _extend_case(rng, prefix, new, hq, hkv, d, P)
    o, lse = oa.extend(q, cu, k, v, table, lens, P, 0.5)
    for r in range(2):
        slots = oa.gather_slots(table, lens[r], P, r)
        for h in range(hq):
            kk = bf16_bits_to_f64(k[slots, 0]).tolist()
            vv = bf16_bits_to_f64(v[slots, 0]).tolist()
            qq = bf16_bits_to_f64(q[cu[r]:cu[r + 1], h]).tolist()
            O, LSE = oa.materialised_reference(qq, kk, vv, 0.5, causal_offset=prefix[r])
            assert np.allclose(o[cu[r]:cu[r + 1], h], np.array(O), atol=1e-12, rtol=0)
            assert np.allclose(lse[cu[r]:cu[r + 1], h], np.array(LSE), atol=1e-12, rtol=0)


def test_extend_without_prefix_matches_torch_causal_sdpa():
    rng = np.random.default_rng(10)
    n, hq, hkv, d = 70, 4, 2, 32
    q, cu, k, v, table, lens = _extend_case(rng, [0], [n], hq, hkv, d, 8)
    o, _ = oa.extend(q, cu, k, v, table, lens, 8, 1 / math.sqrt(d))
    slots = oa.gather_slots(table, n, 8, 0)
    K = torch.from_numpy(bf16_bits_to_f64(k[slots])).permute(1, 0, 2).repeat_interleave(2, 0)
    V = torch.from_numpy(bf16_bits_to_f64(v[slots])).permute(1, 0, 2).repeat_interleave(2, 0)
    Q = torch.from_numpy(bf16_bits_to_f64(q)).permute(1, 0, 2)
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, is_causal=True, scale=1 / math.sqrt(d))
    assert np.allclose(o, ref.permute(1, 0, 2).numpy(), atol=1e-12, rtol=0)


def test_extend_single_new_token_equals_decode():
    rng = np.random.default_rng(11)
    prefix = [40, 0, 7]
    q, cu, k, v, table, lens = _extend_case(rng, prefix, [1, 1, 1], 8, 4, 16, 4)
    oe, le = oa.extend(q, cu, k, v, table, lens, 4, 0.3)
    od, ld = oa.decode(q, k, v, table, lens, 4, 0.3)
    assert np.allclose(oe, od, atol=1e-14, rtol=0)
    assert np.allclose(le, ld, atol=1e-14, rtol=0)


def test_extend_is_independent_of_future_keys():
    rng = np.random.default_rng(12)
    q, cu, k, v, table, lens = _extend_case(rng, [6], [5], 2, 2, 8, 1)
    o1, _ = oa.extend(q, cu, k, v, table, lens, 1, 0.5)
    slots = oa.gather_slots(table, lens[0], 1, 0)
    k2, v2 = k.copy(), v.copy()
    last = slots[-1]                                     # key 10, visible only to the last query
    k2[last] = _bf16(rng, *k2[last].shape, scale=5.0)
    v2[last] = _bf16(rng, *v2[last].shape, scale=5.0)
    o2, _ = oa.extend(q, cu, k2, v2, table, lens, 1, 0.5)
    assert np.array_equal(o1[:4], o2[:4])
    assert not np.allclose(o1[4], o2[4])


def test_merge_of_any_split_equals_unsplit():
    rng = np.random.default_rng(13)
    q = rng.standard_normal((3, 16))
    k = rng.standard_normal((50, 16)) * 3
    v = rng.standard_normal((50, 16))
    full_o, full_l = oa.softmax_attend(q, k, v, 0.4)
    for cuts in ([0, 50], [0, 1, 50], [0, 10, 11, 30, 50], [0, 25, 25, 50]):
        os_, ls_ = [], []
        for a, b in zip(cuts[:-1], cuts[1:]):
            o, l = oa.softmax_attend(q, k[a:b], v[a:b], 0.4)
            os_.append(o)
            ls_.append(l)
        mo, ml = oa.merge_partials(np.stack(os_), np.stack(ls_))
        assert np.allclose(mo, full_o, atol=1e-13, rtol=0)
        assert np.allclose(ml, full_l, atol=1e-13, rtol=0)
    eo, el = oa.merge_partials(np.zeros((2, 3, 16)), np.full((2, 3), -np.inf))
    assert np.all(eo == 0) and np.all(np.isneginf(el))


def test_materialised_memory_figure_from_the_page():
    import json
    import os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "fa_memory_example.json")))
    per_head = oa.materialised_score_bytes(g["seq_len"], g["elem_bytes"])
    assert per_head == g["bytes_per_head"]
    assert per_head / 2 ** 20 == g["approx_mib_per_head"]
    total = oa.materialised_score_bytes(g["seq_len"], g["elem_bytes"], g["batch"], g["heads"])
    assert total / 2 ** 30 == g["approx_gib_total"]


def test_kv_store_closed_form():
    rng = np.random.default_rng(14)
    k = _bf16(rng, 10, 2, 4)
    v = _bf16(rng, 10, 2, 4)
    kn = _bf16(rng, 3, 2, 4)
    vn = _bf16(rng, 3, 2, 4)
    k2, v2 = oa.kv_store(k, v, [7, 2, 99], kn, vn)          # slot 99 is outside the pool: skipped
    assert np.array_equal(k2[7], kn[0]) and np.array_equal(v2[2], vn[1])
    untouched = [s for s in range(10) if s not in (7, 2)]
    assert np.array_equal(k2[untouched], k[untouched]) and np.array_equal(v2[untouched], v[untouched])
    assert np.array_equal(k[7], k[7])                        # inputs are not modified in place
