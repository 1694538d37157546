"""GPU tests of the KV-cache stores (bf16 and 8-bit Sage) and of a CUDA-graph-captured decode step.

The store is compared bit for bit with the oracle's scatter; a decode step that
stores the new token's K/V and then attends (the order of a forward pass) matches
the oracle; and the whole step (store, plan, per-layer decode) captured once in a
CUDA graph and replayed with new inputs gives the same bits as eager calls.
"""
import os

import numpy as np
import pytest
import torch

import paged_kv_flashattention_split_b200 as pa
import workloads as wl
from oracle import attention as oa
from tests.helpers import alloc_ws, assert_bf16_close, bits16

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    if not os.path.exists(pa.LIB_PATH):
        from paged_kv_flashattention_split_b200 import build
        build.build()
    pa.lib()


def test_store_is_bit_exact_and_flags_bad_slots():
    g = torch.Generator(device=DEV).manual_seed(5)
    k = torch.randn(5000, 8, 128, device=DEV, generator=g).to(torch.bfloat16)
    v = torch.randn(5000, 8, 128, device=DEV, generator=g).to(torch.bfloat16)
    kn = torch.randn(300, 8, 128, device=DEV, generator=g).to(torch.bfloat16)
    vn = torch.randn(300, 8, 128, device=DEV, generator=g).to(torch.bfloat16)
    loc = torch.randperm(5000, device=DEV, generator=g)[:300].to(torch.int32)
    loc[17] = 5000                                            # outside the pool: skipped and flagged
    ref_k, ref_v = oa.kv_store(bits16(k), bits16(v), loc.cpu().numpy(), bits16(kn), bits16(vn))
    params = pa.make_params(pa.PA_MODE_DECODE, 1, 8, 8, 128, 1, max_kv_len=1, num_sms=0)
    ws = alloc_ws(params)
    pa.attn_kv_store(kn, vn, loc, k, v, ws=ws)
    torch.cuda.synchronize()
    assert np.array_equal(bits16(k), ref_k) and np.array_equal(bits16(v), ref_v)
    assert pa.pa_read_device_error(ws) == pa.PA_ERR_DEVICE_INDEX


def _decode_step_case():
    spec = wl.SPECS["decode_llama3_8b"].scaled(batch=8, pool_slots=60_000, len_hi=3000, layers=2)
    batch = wl.make_batch(spec, DEV)
    pools = [wl.make_bf16_pools(spec, batch, l, DEV) for l in range(spec.layers)]
    # the decode token of every request goes to a fresh (unused, NaN-filled) slot, appended to its row
    unused = torch.nonzero(~batch.used_slot_mask).flatten()[: spec.batch].to(torch.int32)
    table = torch.zeros(spec.batch, batch.page_table.shape[1] + 1, dtype=torch.int32, device=DEV)
    table[:, :-1] = batch.page_table
    lens = batch.seq_lens.clone()
    for r in range(spec.batch):
        table[r, int(lens[r])] = unused[r]
    lens += 1
    return spec, wl.Batch(lens, table, batch.num_slots, batch.used_slot_mask), pools, unused


def test_store_then_decode_matches_the_oracle():
    spec, batch, pools, loc = _decode_step_case()
    g = torch.Generator(device=DEV).manual_seed(9)
    q = torch.randn(spec.batch, spec.hq, 128, device=DEV, generator=g).to(torch.bfloat16)
    kn = torch.randn(spec.batch, spec.hkv, 128, device=DEV, generator=g).to(torch.bfloat16)
    vn = torch.randn(spec.batch, spec.hkv, 128, device=DEV, generator=g).to(torch.bfloat16)
    k, v = pools[0]
    ref_k, ref_v = oa.kv_store(bits16(k), bits16(v), loc.cpu().numpy(), bits16(kn), bits16(vn))
    params = pa.make_params(pa.PA_MODE_DECODE, spec.batch, spec.hq, spec.hkv, 128, 1,
                            max_kv_len=batch.page_table.shape[1])
    ws = alloc_ws(params)
    pa.attn_kv_store(kn, vn, loc, k, v)
    pa.attn_plan(params, batch.seq_lens, None, ws)
    out = torch.empty_like(q)
    pa.attn_decode_paged(params, ws, q, k, v, batch.page_table, spec.sm_scale, out)
    torch.cuda.synchronize()
    ref, _ = oa.decode(bits16(q), ref_k, ref_v, batch.page_table.cpu().numpy(), batch.seq_lens.cpu().numpy(), 1,
                       spec.sm_scale)
    assert_bf16_close(out, ref, "store + decode")


def test_decode_step_captured_in_a_cuda_graph_replays_bit_exactly():
    spec, batch, pools, loc = _decode_step_case()
    params = pa.make_params(pa.PA_MODE_DECODE, spec.batch, spec.hq, spec.hkv, 128, 1,
                            max_kv_len=batch.page_table.shape[1])
    ws = alloc_ws(params)
    shape_q, shape_kv = (spec.batch, spec.hq, 128), (spec.batch, spec.hkv, 128)
    q = torch.zeros(spec.layers, *shape_q, dtype=torch.bfloat16, device=DEV)
    kn = torch.zeros(spec.layers, *shape_kv, dtype=torch.bfloat16, device=DEV)
    vn = torch.zeros_like(kn)
    out = torch.zeros_like(q)

    def step():
        pa.attn_plan(params, batch.seq_lens, None, ws)
        for l in range(spec.layers):
            k, v = pools[l]
            pa.attn_kv_store(kn[l], vn[l], loc, k, v)
            pa.attn_decode_paged(params, ws, q[l], k, v, batch.page_table, spec.sm_scale, out[l])

    def fill(seed):
        g = torch.Generator(device=DEV).manual_seed(seed)
        q.copy_(torch.randn(q.shape, device=DEV, generator=g).to(torch.bfloat16))
        kn.copy_(torch.randn(kn.shape, device=DEV, generator=g).to(torch.bfloat16))
        vn.copy_(torch.randn(vn.shape, device=DEV, generator=g).to(torch.bfloat16))

    fill(1)
    step()                                     # eager warm-up (sets kernel attributes before capture)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            step()
    torch.cuda.synchronize()
    for seed in (2, 3):
        fill(seed)
        step()
        torch.cuda.synchronize()
        eager = out.clone()
        out.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), eager.view(torch.int16))
    del graph


def test_sage_store_is_bit_exact_with_block_scales():
    from oracle import sage as osg
    g = torch.Generator(device=DEV).manual_seed(6)
    S, H = 64 * 80, 8
    k8 = torch.randint(-127, 128, (S, H, 128), device=DEV, generator=g, dtype=torch.int32).to(torch.int8)
    v8 = torch.randint(0, 256, (S, H, 128), device=DEV, generator=g, dtype=torch.int32).to(torch.uint8)
    sf = torch.rand(S // 64, H, device=DEV, generator=g)
    n = 200
    kn = torch.randint(-127, 128, (n, H, 128), device=DEV, generator=g, dtype=torch.int32).to(torch.int8)
    vn = torch.randint(0, 256, (n, H, 128), device=DEV, generator=g, dtype=torch.int32).to(torch.uint8)
    sfn = torch.rand(n, H, device=DEV, generator=g) + 1.0
    loc = torch.randperm(S, device=DEV, generator=g)[:n].to(torch.int32)
    loc[:10] = torch.arange(10, device=DEV, dtype=torch.int32) * 64       # tokens that open blocks 0..9
    loc[50] = -3                                                          # outside the pool: skipped, flagged
    ref = osg.kv_store_sage(k8.cpu().numpy(), v8.cpu().numpy(), sf.cpu().numpy(), loc.cpu().numpy(),
                            kn.cpu().numpy(), vn.cpu().numpy(), sfn.cpu().numpy())
    params = pa.make_params(pa.PA_MODE_DECODE, 1, 8, 8, 128, 1, max_kv_len=1, num_sms=0)
    ws = alloc_ws(params)
    pa.attn_kv_store_sage(kn, vn, sfn, loc, k8, v8, sf, ws=ws)
    torch.cuda.synchronize()
    assert np.array_equal(k8.cpu().numpy(), ref[0]) and np.array_equal(v8.cpu().numpy(), ref[1])
    assert np.array_equal(sf.cpu().numpy(), ref[2])
    assert pa.pa_read_device_error(ws) == pa.PA_ERR_DEVICE_INDEX


def test_sage_store_then_decode_matches_the_oracle():
    from oracle import sage as osg
    spec = wl.SPECS["sage_decode"].scaled(batch=6, len_lo=100, len_hi=1500)
    batch = wl.make_batch(spec, DEV)
    lay = wl.make_sage_layer(spec, batch, 0, DEV)
    # every request's decode token goes to the first slot of a spare (unused) page, appended
    pages_used = set(int(x) for x in batch.page_table.flatten().tolist())
    spare = [p for p in range(batch.num_slots // 64) if p not in pages_used][: spec.batch]
    assert len(spare) == spec.batch
    table = torch.zeros(spec.batch, batch.page_table.shape[1] + 1, dtype=torch.int32, device=DEV)
    table[:, :-1] = batch.page_table
    lens = batch.seq_lens.clone()
    loc = torch.empty(spec.batch, dtype=torch.int32, device=DEV)
    for r in range(spec.batch):
        L = int(lens[r])
        if L % 64 == 0:                          # the next position starts a new page
            table[r, L // 64] = spare[r]
            loc[r] = spare[r] * 64
        else:                                    # the next position is inside the last page
            loc[r] = int(table[r, L // 64]) * 64 + L % 64
    lens += 1
    g = torch.Generator(device=DEV).manual_seed(12)
    kn = torch.randint(-127, 128, (spec.batch, spec.hkv, 128), device=DEV, generator=g, dtype=torch.int32).to(torch.int8)
    vn = (16 * torch.randn(spec.batch, spec.hkv, 128, device=DEV, generator=g)).to(torch.float8_e4m3fn).view(torch.uint8)
    sfn = torch.exp(-4 + 0.5 * torch.randn(spec.batch, spec.hkv, device=DEV, generator=g))
    k8, v8, sfk = osg.kv_store_sage(lay.k8.cpu().numpy(), lay.v8.cpu().numpy(), lay.sf_k.cpu().numpy(),
                                    loc.cpu().numpy(), kn.cpu().numpy(), vn.cpu().numpy(), sfn.cpu().numpy())
    pa.attn_kv_store_sage(kn, vn, sfn, loc, lay.k8, lay.v8, lay.sf_k)
    b2 = wl.Batch(lens, table, batch.num_slots, batch.used_slot_mask)
    params = pa.make_params(pa.PA_MODE_SAGE_DECODE, spec.batch, spec.hq, spec.hkv, 128, 64,
                            max_kv_len=table.shape[1] * 64, sage_k_block=64)
    ws = alloc_ws(params)
    pa.attn_plan(params, lens, None, ws)
    out = torch.empty(spec.batch, spec.hq, 128, dtype=torch.bfloat16, device=DEV)
    pa.attn_decode_paged_sage(params, ws, lay.q8, lay.sf_q, lay.k8, lay.v8, lay.sf_k, lay.sf_v, lay.v_mean,
                              table, out)
    torch.cuda.synchronize()
    assert pa.pa_read_device_error(ws) == pa.PA_OK
    ref = osg.sage_decode(lay.q8.cpu().numpy(), lay.sf_q.cpu().numpy(), k8, v8, sfk, lay.sf_v.cpu().numpy(),
                          lay.v_mean.cpu().numpy(), table.cpu().numpy(), lens.cpu().numpy(), 64)
    from tests.helpers import SAGE_REL, sage_row_rel_error
    assert sage_row_rel_error(out, ref) <= SAGE_REL


def test_graph_captured_at_one_batch_size_serves_new_lengths_at_that_size():
    """A captured plan + decode step serves one batch size: its launch geometry depends only on
    the plan parameters (batch, heads, max_kv_len), never on device data, so after the caller
    writes new sequence lengths and page-table rows into the same device buffers (same B, lengths
    within max_kv_len) a replay re-plans from them and matches the oracle on the new lengths."""
    spec = wl.SPECS["decode_llama3_8b"].scaled(batch=8, pool_slots=60_000, len_lo=100, len_hi=3000)
    batch = wl.make_batch(spec, DEV)
    k, v = wl.make_bf16_pools(spec, batch, 0, DEV)
    q = wl.make_bf16_queries(spec, spec.batch, 0, DEV)
    max_len = batch.page_table.shape[1]
    params = pa.make_params(pa.PA_MODE_DECODE, spec.batch, spec.hq, spec.hkv, 128, 1, max_kv_len=max_len)
    ws = alloc_ws(params)
    lens, table = batch.seq_lens.clone(), batch.page_table.clone()
    out = torch.zeros_like(q)

    def step():
        pa.attn_plan(params, lens, None, ws)
        pa.attn_decode_paged(params, ws, q, k, v, table, spec.sm_scale, out)

    step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            step()
    torch.cuda.synchronize()
    g = torch.Generator().manual_seed(77)
    for trial in range(3):
        # new lengths for the same requests (shorter prefixes of their rows, one request empty on
        # the last trial): the table rows still hold the same slots, so every length stays valid
        new = torch.randint(0, 1 << 30, (spec.batch,), generator=g) % (batch.seq_lens.cpu() + 1)
        if trial == 2:
            new[3] = 0
        lens.copy_(new.to(torch.int32))
        # and a reversed row order, so the table contents change too
        perm = torch.arange(spec.batch - 1, -1, -1)
        table.copy_(batch.page_table[perm.to(DEV)])
        lens.copy_(new[perm].to(torch.int32))
        out.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        assert pa.pa_read_device_error(ws) == pa.PA_OK
        ref, _ = oa.decode(bits16(q), bits16(k), bits16(v), table.cpu().numpy(), lens.cpu().numpy(), 1,
                           spec.sm_scale)
        assert_bf16_close(out, ref, f"graph replay with new lengths, trial {trial}")
    del graph
