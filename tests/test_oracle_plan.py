"""Pins for the oracle's integer plan.

Hand-derived golden cases (tests/golden/plan_cases.json) and invariants that
any correct split-KV plan has: the splits of a request cover [0, L) exactly
once, in order, on tile boundaries; the flat partitions give no slot more than
its share of units; EXTEND items run longest first; the item count stays within
the host-side bound used to size the grid; and the plan depends only on the
lengths.
"""
import json
import os

import numpy as np
import pytest

from oracle import plan as op

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "plan_cases.json")))


@pytest.mark.parametrize("case", GOLDEN["cases"], ids=[c["name"] for c in GOLDEN["cases"]])
def test_hand_derived_plans(case):
    got = op.plan(case["mode"], case["seq_lens"], case.get("cu_seqlens_q"), hkv=case["hkv"],
                  page_size=case["page_size"], num_sms=case["num_sms"],
                  max_q_tokens=(case.get("cu_seqlens_q") or [0])[-1], block_mask=case.get("block_mask"))
    e = case["expect"]
    assert got["tile"] == e["tile"]
    assert got["chunk_tiles"] == e["chunk_tiles"]
    assert got["req_splits"] == e["req_splits"]
    assert got["req_base"] == e["req_base"]
    assert [list(x) for x in got["items"]] == e["items"]
    if "slot_first" in e:
        assert got["slot_first"] == e["slot_first"]
    for k in ("sel_base", "sel_block"):
        if k in e:
            assert got[k] == e[k]


def _check_flat_invariants(pl, lens, U, C, unit_keys_of):
    """Every request covered exactly once, in order, by U-aligned pieces; execution order is
    generation order; each slot holds at most `per` units and the slots hold all of them."""
    per = pl["chunk_tiles"]
    sf = pl["slot_first"]
    assert len(sf) == C + 1 and sf == sorted(sf) and sf[-1] == pl["num_items"]
    by_req = {}
    for i, (r, s, a, b) in enumerate(pl["items"]):
        by_req.setdefault(r, []).append((s, a, b))
        assert a % U == 0 and (a < b or lens[r] == 0)
        assert i == pl["req_base"][r] + s
    for r, L in enumerate(lens):
        parts = by_req[r]
        assert [s for s, _, _ in parts] == list(range(pl["req_splits"][r]))
        assert parts[0][1] == 0 and parts[-1][2] == L
        assert all(b0 == a1 for (_, _, b0), (_, a1, _) in zip(parts, parts[1:]))
    units = 0
    for c in range(C):
        u = sum(unit_keys_of(a, b) for (_, _, a, b) in pl["items"][sf[c]:sf[c + 1]])
        assert u <= per
        units += u
    assert units == sum(-(-L // U) for L in lens)
    assert pl["req_base"][-1] == pl["num_items"]


def _check_decode_invariants(lens, hkv, P, num_sms):
    pl = op.plan(op.MODE_DECODE, lens, hkv=hkv, page_size=P, num_sms=num_sms)
    T = pl["tile"]
    assert T == max(64, P)
    C = op.flat_slots(hkv, num_sms)
    assert pl["num_items"] <= op.max_items(op.MODE_DECODE, len(lens), hkv, num_sms) == C + len(lens)
    _check_flat_invariants(pl, lens, T, C, lambda a, b: -(-(b - a) // T))
    return pl


def test_decode_invariants_random():
    rng = np.random.default_rng(30)
    for _ in range(300):
        B = int(rng.integers(1, 70))
        lens = [int(x) for x in rng.integers(0, 20000, B)]
        if rng.random() < 0.3:
            lens[int(rng.integers(0, B))] = 0
        hkv = int(rng.choice([1, 2, 4, 8]))
        P = int(rng.choice([1, 16, 64, 128, 256]))
        _check_decode_invariants(lens, hkv, P, int(rng.integers(1, 200)))


def test_decode_plan_at_the_workload_shapes():
    # Llama-3-8B decode shape and the 128k long-context shape on 148 SMs
    rng = np.random.default_rng(31)
    lens = [int(x) for x in rng.integers(512, 8193, 64)]
    _check_decode_invariants(lens, 8, 1, 148)
    pl = op.plan(op.MODE_DECODE, [131072] * 8, hkv=8, page_size=64, num_sms=148)
    # one item covers all 8 KV heads: C = 148 * 2 = 296 slots; 8 * 2048 tiles,
    # per = ceil(16384 / 296) = 56 tiles; request r holds global tiles [2048 r, 2048 (r+1))
    assert op.flat_slots(8, 148) == 296 and pl["chunk_tiles"] == 56
    # request 0: slots 0..36 (2048 = 36 * 56 + 32): 37 pieces; request 1 starts at tile 2048 =
    # 36 * 56 + 32, so its first piece is the 24 tiles left of slot 36
    assert pl["req_splits"][0] == 37 and pl["items"][0] == (0, 0, 0, 56 * 64)
    assert pl["items"][37] == (1, 0, 0, 24 * 64)
    assert pl["num_items"] <= op.max_items(op.MODE_DECODE, 8, 8, 148) == 304
    # 16 KV heads: two CTAs per item, so half the slots
    assert op.decode_head_groups(16) == 2 and op.decode_head_groups(12) == 3 and op.decode_head_groups(8) == 1
    assert op.flat_slots(16, 148) == 148


def test_plan_is_a_function_of_lengths_only():
    rng = np.random.default_rng(32)
    lens = [int(x) for x in rng.integers(1, 5000, 17)]
    a = op.plan(op.MODE_DECODE, lens, hkv=4, page_size=16, num_sms=148)
    b = op.plan(op.MODE_DECODE, np.array(lens), hkv=4, page_size=16, num_sms=148)
    assert a == b


def test_extend_invariants_random():
    rng = np.random.default_rng(33)
    for _ in range(200):
        B = int(rng.integers(1, 12))
        new = rng.integers(0, 700, B)
        pre = rng.integers(0, 3000, B)
        cu = np.concatenate([[0], np.cumsum(new)]).tolist()
        lens = (new + pre).tolist()
        pl = op.plan(op.MODE_EXTEND, lens, cu, hkv=8, page_size=16, num_sms=148, max_q_tokens=cu[-1])
        assert pl["num_items"] <= op.max_items(op.MODE_EXTEND, B, 8, 148, cu[-1])
        seen = {}
        for (r, t, q0, q1) in pl["items"]:
            seen.setdefault(r, []).append((t, q0, q1))
        for r in range(B):
            parts = sorted(seen.get(r, []))
            assert sum(q1 - q0 for _, q0, q1 in parts) == new[r]
            for (t, q0, q1) in parts:
                assert q0 == 128 * t and 0 < q1 - q0 <= 128
        keys = [-(-(lens[r] - new[r] + q1) // 128) for (r, t, q0, q1) in pl["items"]]
        assert keys == sorted(keys, reverse=True)


def test_rejects_negative_lengths():
    with pytest.raises(ValueError):
        op.plan(op.MODE_DECODE, [5, -1], hkv=1, page_size=1, num_sms=1)
    with pytest.raises(ValueError):
        op.plan(op.MODE_EXTEND, [5], [0, 6], hkv=1, page_size=1, num_sms=1)


def test_sage_flat_partition_invariants_random():
    rng = np.random.default_rng(7)
    for _ in range(200):
        B = int(rng.integers(1, 40))
        lens = [int(x) for x in rng.integers(0, 5000, B)]
        if rng.random() < 0.2:
            lens[int(rng.integers(0, B))] = 0
        hkv = int(rng.choice([1, 2, 8, 16]))
        num_sms = int(rng.integers(1, 200))
        pl = op.plan(op.MODE_SAGE_DECODE, lens, hkv=hkv, page_size=64, num_sms=num_sms)
        C = op.flat_slots(hkv, num_sms)
        assert pl["num_items"] <= op.max_items(op.MODE_SAGE_DECODE, B, hkv, num_sms)
        _check_flat_invariants(pl, lens, 32, C, lambda a, b: -(-(b - a) // 32))


def test_sage_sparse_units_cover_exactly_the_selected_keys():
    rng = np.random.default_rng(8)
    for _ in range(150):
        B = int(rng.integers(1, 20))
        lens = [int(x) for x in rng.integers(0, 3000, B)]
        nbm = max(1, max(-(-L // 64) for L in lens))
        mask = (rng.random((B, nbm)) < rng.choice([0.0, 0.1, 0.5, 1.0])).astype(int)
        hkv, num_sms = int(rng.choice([1, 2, 8])), int(rng.integers(1, 100))
        pl = op.plan(op.MODE_SAGE_SPARSE, lens, hkv=hkv, page_size=64, num_sms=num_sms, block_mask=mask)
        sb, blk = pl["sel_base"], pl["sel_block"]
        per = pl["chunk_tiles"]
        C = op.flat_slots(hkv, num_sms)
        assert pl["num_items"] <= op.max_items(op.MODE_SAGE_SPARSE, B, hkv, num_sms)
        for r, L in enumerate(lens):
            want = [j for j in range(L) if mask[r][j // 64]]
            got = []
            for (rr, s, u0, u1) in pl["items"]:
                if rr != r:
                    continue
                for u in range(u0, u1):
                    k0 = 64 * blk[sb[r] + u // 2] + 32 * (u % 2)
                    got += list(range(k0, min(k0 + 32, L)))
            assert got == want
            assert blk[sb[r]:sb[r + 1]] == sorted(b for b in range(-(-L // 64)) if mask[r][b])
        for c in range(C):
            assert sum(u1 - u0 for (_, _, u0, u1) in pl["items"][pl["slot_first"][c]:pl["slot_first"][c + 1]]) <= per
