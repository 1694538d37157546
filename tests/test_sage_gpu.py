"""GPU parity of the 8-bit Sage decode against the quantisation-emulating oracle.

The bar: max over output rows (r, h) of ||O_gpu - O_ref||_inf / max(||O_ref||_inf, 1e-6)
<= 3e-2, on the full Sage workload, scaled variants across head-group sizes and
KV-head counts, ragged and empty rows, rows split into many key ranges (the
row max is exchanged between the splits), one split per row, and without
v_mean.
"""
import os

import numpy as np
import pytest
import torch

import paged_kv_flashattention_split_b200 as pa
import workloads as wl
from oracle import sage as osg
from tests.helpers import SAGE_REL, alloc_ws, bits16, sage_row_rel_error

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    if not os.path.exists(pa.LIB_PATH):
        from paged_kv_flashattention_split_b200 import build
        build.build()
    pa.lib()


def sage_params(spec, batch, num_sms=0):
    return pa.make_params(pa.PA_MODE_SAGE_DECODE, spec.batch, spec.hq, spec.hkv, 128, 64,
                          max_kv_len=batch.page_table.shape[1] * 64, sage_k_block=64, num_sms=num_sms)


def run_sage(spec, batch, lay, use_v_mean=True, num_sms=0):
    params = sage_params(spec, batch, num_sms)
    ws = alloc_ws(params)
    pa.attn_plan(params, batch.seq_lens, None, ws)
    out = torch.full((spec.batch, spec.hq, 128), float("nan"), dtype=torch.bfloat16, device=DEV)
    pa.attn_decode_paged_sage(params, ws, lay.q8, lay.sf_q, lay.k8, lay.v8, lay.sf_k, lay.sf_v,
                              lay.v_mean if use_v_mean else None, batch.page_table, out)
    torch.cuda.synchronize()
    assert pa.pa_read_device_error(ws) == pa.PA_OK
    return out


def oracle_sage(spec, batch, lay, use_v_mean=True):
    return osg.sage_decode(lay.q8.cpu().numpy(), lay.sf_q.cpu().numpy(), lay.k8.cpu().numpy(),
                           lay.v8.cpu().numpy(), lay.sf_k.cpu().numpy(), lay.sf_v.cpu().numpy(),
                           lay.v_mean.cpu().numpy() if use_v_mean else None,
                           batch.page_table.cpu().numpy(), batch.seq_lens.cpu().numpy(), 64)


@pytest.mark.parametrize("layer", [0, 31])
def test_sage_full_workload(layer):
    """Every output row of the first and the last layer of the Sage decode workload."""
    spec = wl.SPECS["sage_decode"]
    batch = wl.make_batch(spec, DEV)
    lay = wl.make_sage_layer(spec, batch, layer, DEV)
    out = run_sage(spec, batch, lay)
    ref = oracle_sage(spec, batch, lay)
    err = sage_row_rel_error(out, ref)
    assert err <= SAGE_REL, err


@pytest.mark.parametrize("G,lo,hi", [(1, 1, 63), (2, 64, 64), (4, 65, 700), (8, 1000, 5000)])
def test_sage_head_groups_and_ragged_lengths(G, lo, hi):
    spec = wl.Spec("sage_edge", 21, "sage", batch=6, len_lo=lo, len_hi=hi, hq=2 * G, hkv=2, page_size=64,
                   spare_pages=0.2)
    batch = wl.make_batch(spec, DEV)
    lay = wl.make_sage_layer(spec, batch, 0, DEV)
    out = run_sage(spec, batch, lay)
    ref = oracle_sage(spec, batch, lay)
    assert sage_row_rel_error(out, ref) <= SAGE_REL


@pytest.mark.parametrize("hq,hkv", [(8, 1), (16, 4), (64, 8), (32, 16)])
def test_sage_kv_head_counts(hq, hkv):
    spec = wl.Spec("sage_heads", 22, "sage", batch=3, len_lo=1, len_hi=900, hq=hq, hkv=hkv, page_size=64,
                   spare_pages=0.2)
    batch = wl.make_batch(spec, DEV)
    lay = wl.make_sage_layer(spec, batch, 0, DEV)
    out = run_sage(spec, batch, lay)
    assert sage_row_rel_error(out, oracle_sage(spec, batch, lay)) <= SAGE_REL


def test_sage_long_rows_split_many_ways():
    # rows far longer than one CTA's share: each is split into many key ranges whose maxima
    # are combined before any probability is quantised, and whose sums are merged
    spec = wl.Spec("sage_long", 23, "sage", batch=3, len_lo=20000, len_hi=40000, hq=32, hkv=8, page_size=64,
                   spare_pages=0.05)
    batch = wl.make_batch(spec, DEV)
    lay = wl.make_sage_layer(spec, batch, 0, DEV)
    params = sage_params(spec, batch)
    ws = alloc_ws(params)
    pa.attn_plan(params, batch.seq_lens, None, ws)
    from tests.helpers import read_plan
    assert min(read_plan(ws, 2, spec.batch, spec.hq)["req_splits"]) > 50
    out = run_sage(spec, batch, lay)
    assert sage_row_rel_error(out, oracle_sage(spec, batch, lay)) <= SAGE_REL


def test_sage_few_slots_match_many():
    # a plan for one SM (two CTA slots: long pieces) and the device's full plan give the same
    # quantised probabilities, so both meet the bar
    spec = wl.SPECS["sage_decode"].scaled(batch=6, len_lo=2000, len_hi=4000)
    batch = wl.make_batch(spec, DEV)
    lay = wl.make_sage_layer(spec, batch, 0, DEV)
    ref = oracle_sage(spec, batch, lay)
    few = run_sage(spec, batch, lay, num_sms=1)
    many = run_sage(spec, batch, lay)
    assert sage_row_rel_error(few, ref) <= SAGE_REL
    assert sage_row_rel_error(many, ref) <= SAGE_REL


def test_sage_without_v_mean_and_with_an_empty_row():
    spec = wl.SPECS["sage_decode"].scaled(batch=5, len_lo=100, len_hi=1500)
    batch = wl.make_batch(spec, DEV)
    lay = wl.make_sage_layer(spec, batch, 0, DEV)
    out = run_sage(spec, batch, lay, use_v_mean=False)
    ref = oracle_sage(spec, batch, lay, use_v_mean=False)
    assert sage_row_rel_error(out, ref) <= SAGE_REL
    # an empty request returns v_mean exactly (rounded to bf16)
    batch.seq_lens[2] = 0
    out = run_sage(spec, batch, lay)
    vm = lay.v_mean.to(torch.bfloat16).repeat_interleave(spec.hq // spec.hkv, dim=0)
    assert torch.equal(out[2].view(torch.int16), vm.view(torch.int16))


def test_sage_shuffled_pages_with_their_scales_give_identical_output():
    spec = wl.SPECS["sage_decode"].scaled(batch=4, len_lo=500, len_hi=2000)
    batch = wl.make_batch(spec, DEV)
    lay = wl.make_sage_layer(spec, batch, 0, DEV)
    out1 = run_sage(spec, batch, lay)
    pages = lay.k8.shape[0] // 64
    perm = torch.randperm(pages, generator=torch.Generator().manual_seed(3)).to(DEV)
    inv = torch.argsort(perm)
    idx = (perm[:, None] * 64 + torch.arange(64, device=DEV)[None, :]).reshape(-1)
    lay2 = wl.SageLayer(lay.q8, lay.sf_q, lay.k8[idx].contiguous(), lay.v8[idx].contiguous(),
                        lay.sf_k[perm].contiguous(), lay.sf_v, lay.v_mean)
    b2 = wl.Batch(batch.seq_lens, inv[batch.page_table.long()].to(torch.int32), batch.num_slots,
                  batch.used_slot_mask)
    out2 = run_sage(spec, b2, lay2)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


def test_sage_requires_sm100(monkeypatch):
    spec = wl.SPECS["sage_decode"].scaled(batch=2, len_lo=64, len_hi=128)
    batch = wl.make_batch(spec, DEV)
    params = sage_params(spec, batch)
    ws = alloc_ws(params)
    monkeypatch.setenv("PAGEDATTN_TEST_FORCE_ARCH", "90")
    assert pa.attn_plan(params, batch.seq_lens, None, ws, raise_on_error=False) == pa.PA_ERR_ARCH
