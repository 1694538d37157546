"""GPU parity of the plan, the slot/page gather and the bf16 split-KV decode, through the C ABI.

Plan and gather are compared bit for bit with the oracle; decode outputs
within the bf16 tolerance (max |err| <= 1e-2 beyond the output's own bf16
rounding, mean |err| <= 1e-3), LSEs within 4e-3, on the seeded workloads,
scaled-down versions of them that still span many tiles and ragged tails, the
full-size shapes (sampled), and the edge cases.
"""
import math
import os

import numpy as np
import pytest
import torch

import paged_kv_flashattention_split_b200 as pa
import workloads as wl
from oracle import attention as oa
from oracle import plan as op
from tests.helpers import LSE_ABS, alloc_ws, assert_bf16_close, bits16, read_plan

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    if not os.path.exists(pa.LIB_PATH):
        from paged_kv_flashattention_split_b200 import build
        build.build()
    pa.lib()


def num_sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def decode_params(spec, batch, plan_sms=0):
    return pa.make_params(pa.PA_MODE_DECODE, spec.batch, spec.hq, spec.hkv, spec.head_dim, spec.page_size,
                          max_kv_len=batch.page_table.shape[1] * spec.page_size, num_sms=plan_sms)


def run_decode(spec, batch, q, k, v, plan_sms=0, ws=None, plan=True):
    params = decode_params(spec, batch, plan_sms)
    if ws is None:
        ws = alloc_ws(params)
    if plan:
        pa.attn_plan(params, batch.seq_lens, None, ws)
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[0], q.shape[1], dtype=torch.float32, device=DEV)
    pa.attn_decode_paged(params, ws, q, k, v, batch.page_table, spec.sm_scale, out, lse)
    torch.cuda.synchronize()
    assert pa.pa_read_device_error(ws) == pa.PA_OK
    return out, lse, ws, params


def oracle_decode(spec, batch, q, k, v):
    return oa.decode(bits16(q), bits16(k), bits16(v), batch.page_table.cpu().numpy(),
                     batch.seq_lens.cpu().numpy(), spec.page_size, spec.sm_scale)


def check_lse(lse_gpu, lse_ref):
    g = lse_gpu.cpu().numpy().astype(np.float64)
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(g), fin)
    assert np.max(np.abs(g[fin] - lse_ref[fin]), initial=0.0) <= LSE_ABS


def device_case(spec, seed_shift=0, layer=0):
    batch = wl.make_batch(spec, DEV, seed=None if not seed_shift else 1000 + spec.cfg + seed_shift)
    k, v = wl.make_bf16_pools(spec, batch, layer, DEV)
    q = wl.make_bf16_queries(spec, spec.batch, layer, DEV)
    return batch, q, k, v


# ---------------------------------------------------------------- plan

def _gpu_plan(mode, lens, cu=None, hq=8, hkv=2, page_size=1, max_kv_len=None, max_q=0, plan_sms=0):
    B = len(lens)
    max_kv_len = max(lens + [1]) if max_kv_len is None else max_kv_len
    params = pa.make_params(mode, B, hq, hkv, 128, page_size, max_kv_len=max_kv_len, max_q_tokens=max_q,
                            num_sms=plan_sms, sage_k_block=64 if mode == 2 else 0)
    ws = alloc_ws(params)
    sl = torch.tensor(lens, dtype=torch.int32, device=DEV)
    cut = None if cu is None else torch.tensor(cu, dtype=torch.int32, device=DEV)
    pa.attn_plan(params, sl, cut, ws)
    torch.cuda.synchronize()
    return read_plan(ws, mode, B, hq), ws


def _oracle_plan(mode, lens, cu=None, hkv=2, page_size=1, max_q=0, plan_sms=0):
    return op.plan(mode, lens, cu, hkv=hkv, page_size=page_size, num_sms=plan_sms or num_sms(), max_q_tokens=max_q)


def _assert_same_plan(g, o):
    assert g["magic"] == 0x4C504150 and g["error_word"] == 0
    assert g["num_items"] == o["num_items"]
    assert g["tile"] == o["tile"] and g["chunk_tiles"] == o["chunk_tiles"]
    assert g["req_splits"] == o["req_splits"]
    assert g["req_base"] == o["req_base"]
    assert g["items"] == [tuple(x) for x in o["items"]]
    if "slot_first" in o:
        assert g["slot_first"] == o["slot_first"]


def test_decode_plan_bit_exact():
    rng = np.random.default_rng(100)
    # (lengths, Hkv, page size, plan SMs: 0 = the device's count)
    cases = [([300, 17, 0, 129, 64], 2, 1, 1), ([131072] * 8, 8, 64, 0), ([1], 1, 1, 0), ([0, 0], 4, 16, 0),
             ([200, 0, 300], 8, 1, 2)]
    for _ in range(25):
        B = int(rng.integers(1, 80))
        lens = [int(x) for x in rng.integers(0, 9000, B)]
        cases.append((lens, int(rng.choice([1, 2, 4, 8])), int(rng.choice([1, 2, 16, 64, 128, 256])),
                      int(rng.choice([0, 1, 3, 17]))))
    cases.append(([int(x) for x in rng.integers(1, 300, 4096)], 8, 1, 0))   # large batch
    for lens, hkv, P, sms in cases:
        g, _ = _gpu_plan(0, lens, hq=hkv * 2, hkv=hkv, page_size=P, plan_sms=sms)
        _assert_same_plan(g, _oracle_plan(0, lens, hkv=hkv, page_size=P, plan_sms=sms))


def test_extend_and_sage_plans_bit_exact():
    rng = np.random.default_rng(101)
    for _ in range(15):
        B = int(rng.integers(1, 12))
        new = rng.integers(0, 2100, B)
        pre = rng.integers(0, 4097, B)
        cu = np.concatenate([[0], np.cumsum(new)]).astype(int).tolist()
        lens = (new + pre).astype(int).tolist()
        g, _ = _gpu_plan(1, lens, cu, hq=32, hkv=8, page_size=16, max_q=cu[-1])
        _assert_same_plan(g, _oracle_plan(1, lens, cu, hkv=8, page_size=16, max_q=cu[-1]))
        lens_s = [int(x) for x in rng.integers(0, 4097, int(rng.integers(1, 40)))]
        g, _ = _gpu_plan(2, lens_s, hq=32, hkv=8, page_size=64, max_kv_len=4096)
        _assert_same_plan(g, _oracle_plan(2, lens_s, hkv=8, page_size=64))


def test_plan_identical_on_recompute_and_untouched_by_layer_calls():
    spec = wl.SPECS["decode_llama3_8b"].scaled(batch=16, pool_slots=150_000)
    batch, q, k, v = device_case(spec)
    params = decode_params(spec, batch)
    ws = alloc_ws(params)
    pa.attn_plan(params, batch.seq_lens, None, ws)
    first = read_plan(ws, 0, 16, 32)
    pa.attn_plan(params, batch.seq_lens, None, ws)
    assert read_plan(ws, 0, 16, 32) == first
    for layer in range(2):
        k, v = wl.make_bf16_pools(spec, batch, layer, DEV)
        out = torch.empty_like(q)
        pa.attn_decode_paged(params, ws, q, k, v, batch.page_table, spec.sm_scale, out)
    torch.cuda.synchronize()
    assert read_plan(ws, 0, 16, 32) == first


def test_plan_flags_out_of_range_lengths():
    g, ws = _gpu_plan(0, [10, 5000], max_kv_len=100)
    assert g["req_len"] == [10, 100]
    assert pa.pa_read_device_error(ws) == pa.PA_ERR_DEVICE_INDEX
    assert pa.pa_read_device_error(ws) == pa.PA_OK          # reading clears the word


# ---------------------------------------------------------------- gather

@pytest.mark.parametrize("P", [1, 16, 64])
def test_gather_bit_exact(P):
    spec = wl.Spec("gather", 9, "decode", batch=5, len_lo=1, len_hi=700, hq=8, hkv=4, page_size=P,
                   pool_slots=6000, spare_pages=0.2)
    batch = wl.make_batch(spec, DEV)
    k, _ = wl.make_bf16_pools(spec, batch, 0, DEV)
    table = batch.page_table.cpu().numpy()
    kh = bits16(k)
    for r in range(spec.batch):
        L = int(batch.seq_lens[r])
        for h in (0, 3):
            slots = torch.empty(L, dtype=torch.int32, device=DEV)
            rows = torch.empty(L, 128, dtype=torch.bfloat16, device=DEV)
            pa.attn_debug_gather(batch.seq_lens, r, h, spec.hkv, P, L, k, batch.page_table, slots, rows)
            torch.cuda.synchronize()
            ref = oa.gather_slots(table, L, P, r)
            assert np.array_equal(slots.cpu().numpy(), ref)
            assert np.array_equal(bits16(rows), kh[ref, h, :])


def test_out_of_range_page_is_skipped_and_reported():
    spec = wl.SPECS["decode_tiny"]
    batch, q, k, v = device_case(spec)
    params = decode_params(spec, batch)
    ws = alloc_ws(params)
    bad = batch.page_table.clone()
    bad[1, 3] = 10 ** 8                                   # slot far beyond the pool
    pa.attn_plan(params, batch.seq_lens, None, ws)
    out = torch.empty_like(q)
    pa.attn_decode_paged(params, ws, q, k, v, bad, spec.sm_scale, out)
    assert pa.pa_read_device_error(ws) == pa.PA_ERR_DEVICE_INDEX
    assert torch.isfinite(out.float()).all()


def test_wrong_architecture_is_rejected(monkeypatch):
    spec = wl.SPECS["decode_tiny"]
    batch, q, k, v = device_case(spec)
    params = decode_params(spec, batch)
    ws = alloc_ws(params)
    monkeypatch.setenv("PAGEDATTN_TEST_FORCE_ARCH", "90")
    assert pa.attn_plan(params, batch.seq_lens, None, ws, raise_on_error=False) == pa.PA_ERR_ARCH
    monkeypatch.delenv("PAGEDATTN_TEST_FORCE_ARCH")
    assert pa.attn_plan(params, batch.seq_lens, None, ws, raise_on_error=False) == pa.PA_OK


# ---------------------------------------------------------------- decode parity

def test_decode_tiny_config():
    spec = wl.SPECS["decode_tiny"]
    batch, q, k, v = device_case(spec)
    out, lse, _, _ = run_decode(spec, batch, q, k, v)
    ref, ref_lse = oracle_decode(spec, batch, q, k, v)
    assert_bf16_close(out, ref, "decode_tiny")
    check_lse(lse, ref_lse)


@pytest.mark.parametrize("plan_sms", [0, 1, 7])
def test_decode_llama3_8b_shape_scaled(plan_sms):
    # plan_sms = 1 gives two slots, so each CTA walks many items of several requests
    spec = wl.SPECS["decode_llama3_8b"].scaled(batch=12, pool_slots=120_000)
    batch, q, k, v = device_case(spec)
    out, lse, _, _ = run_decode(spec, batch, q, k, v, plan_sms=plan_sms)
    ref, ref_lse = oracle_decode(spec, batch, q, k, v)
    assert_bf16_close(out, ref, f"decode_8b plan_sms={plan_sms}")
    check_lse(lse, ref_lse)


def test_decode_long_context_peaked_scaled():
    spec = wl.SPECS["decode_long_llama3_70b"].scaled(batch=2, len_lo=20000, len_hi=33000, layers=1, distinct_pools=0)
    batch, q, k, v = device_case(spec)
    out, lse, _, _ = run_decode(spec, batch, q, k, v)
    ref, ref_lse = oracle_decode(spec, batch, q, k, v)
    assert_bf16_close(out, ref, "decode_long")
    check_lse(lse, ref_lse)


@pytest.mark.parametrize("G,P,lo,hi", [(1, 1, 1, 200), (2, 2, 60, 70), (4, 8, 1, 129), (8, 128, 100, 3000),
                                       (8, 256, 255, 1025), (4, 64, 64, 64)])
def test_decode_head_groups_page_sizes_and_ragged_tails(G, P, lo, hi):
    spec = wl.Spec("edge", 11, "decode", batch=7, len_lo=lo, len_hi=hi, hq=2 * G, hkv=2, page_size=P,
                   pool_slots=8000, spare_pages=0.1)
    batch, q, k, v = device_case(spec)
    out, lse, _, _ = run_decode(spec, batch, q, k, v)
    ref, ref_lse = oracle_decode(spec, batch, q, k, v)
    assert_bf16_close(out, ref, f"G={G} P={P}")
    check_lse(lse, ref_lse)


def test_decode_empty_and_single_key_requests():
    spec = wl.Spec("empty", 12, "decode", batch=3, len_lo=1, len_hi=1, hq=8, hkv=2, page_size=1, pool_slots=64)
    batch, q, k, v = device_case(spec)
    batch.seq_lens[:] = torch.tensor([0, 1, 0], dtype=torch.int32)
    out, lse, _, _ = run_decode(spec, batch, q, k, v)
    assert torch.all(out[0] == 0) and torch.all(out[2] == 0)
    assert torch.isneginf(lse[0]).all() and torch.isneginf(lse[2]).all()
    slot = int(batch.page_table[1, 0])
    expect = v[slot].repeat_interleave(spec.hq // spec.hkv, dim=0)      # one key: O = V exactly
    assert torch.equal(out[1].view(torch.int16), expect.view(torch.int16))


def test_decode_shuffle_invariance_and_aliased_pages():
    spec = wl.SPECS["decode_llama3_8b"].scaled(batch=4, pool_slots=40_000, len_hi=3000)
    batch, q, k, v = device_case(spec)
    out1, lse1, _, _ = run_decode(spec, batch, q, k, v)
    perm = torch.randperm(k.shape[0], generator=torch.Generator().manual_seed(5)).to(DEV)
    inv = torch.argsort(perm)
    t2 = inv[batch.page_table.long()].to(torch.int32)
    b2 = wl.Batch(batch.seq_lens, t2, batch.num_slots, batch.used_slot_mask)
    out2, lse2, _, _ = run_decode(spec, b2, q, k[perm].contiguous(), v[perm].contiguous())
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    assert torch.equal(lse1, lse2)
    # two requests sharing all their pages (prefix sharing) and the same query give identical rows
    t3 = batch.page_table.clone()
    t3[1] = t3[0]
    sl3 = batch.seq_lens.clone()
    sl3[1] = sl3[0]
    q3 = q.clone()
    q3[1] = q3[0]
    out3, _, _, _ = run_decode(spec, wl.Batch(sl3, t3, batch.num_slots, batch.used_slot_mask), q3, k, v)
    assert torch.equal(out3[0].view(torch.int16), out3[1].view(torch.int16))


@pytest.mark.parametrize("layer", [0, 31])
def test_decode_full_size_llama3_8b(layer):
    """Every output element and LSE of the first and the last layer of the Llama-3-8B decode
    workload (each layer has its own pool)."""
    spec = wl.SPECS["decode_llama3_8b"]
    batch, q, k, v = device_case(spec, layer=layer)
    out, lse, _, _ = run_decode(spec, batch, q, k, v)
    ref, ref_lse = oracle_decode(spec, batch, q, k, v)
    assert_bf16_close(out, ref, f"decode_8b_full layer {layer}")
    check_lse(lse, ref_lse)


@pytest.mark.parametrize("layer", [0, 79])
def test_decode_full_size_long_context(layer):
    """Every output element and LSE of the first and the last layer of the 128k-key decode
    workload, all 64 (request, KV head) pairs.  The 80 layers rotate over 8 pools, so the
    last layer reads pool 7 with its own queries, as in the bench."""
    spec = wl.SPECS["decode_long_llama3_70b"]
    batch = wl.make_batch(spec, DEV)
    k, v = wl.make_bf16_pools(spec, batch, layer % spec.distinct_pools, DEV)
    q = wl.make_bf16_queries(spec, spec.batch, layer, DEV)
    out, lse, _, _ = run_decode(spec, batch, q, k, v)
    qh, kh, vh = bits16(q), bits16(k), bits16(v)
    del k, v
    table, lens = batch.page_table.cpu().numpy(), batch.seq_lens.cpu().numpy()
    ref = np.zeros(qh.shape)
    ref_lse = np.zeros(qh.shape[:2])
    for r in range(spec.batch):                   # one request at a time keeps the host memory bounded
        ref[r:r + 1], ref_lse[r:r + 1] = oa.decode(qh[r:r + 1], kh, vh, table[r:r + 1], lens[r:r + 1],
                                                   spec.page_size, spec.sm_scale)
    assert_bf16_close(out, ref, f"decode_long_full layer {layer}")
    check_lse(lse, ref_lse)
