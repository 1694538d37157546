"""GPU tests of the block-sparse Sage decode (attn_plan_sage_sparse + attn_decode_paged_sage).

The sparse plan is bit-exact against the oracle's; the output meets the Sage bar (max
row-normwise relative error 3e-2) against the oracle restricted to the selected blocks, at
density 0.125 on the full sparse workload and on small ragged cases; an all-ones mask gives
exactly the dense kernels' bits; an all-zeros mask gives v_mean.
"""
import os

import numpy as np
import pytest
import torch

import paged_kv_flashattention_split_b200 as pa
import workloads as wl
from oracle import plan as op
from oracle import sage as osg
from tests.helpers import SAGE_REL, alloc_ws, read_plan, sage_row_rel_error

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    if not os.path.exists(pa.LIB_PATH):
        from paged_kv_flashattention_split_b200 import build
        build.build()
    pa.lib()


def params_for(spec, batch, mode):
    return pa.make_params(mode, spec.batch, spec.hq, spec.hkv, 128, 64, max_kv_len=batch.page_table.shape[1] * 64,
                          sage_k_block=64)


def run(spec, batch, lay, mask=None):
    mode = pa.PA_MODE_SAGE_DECODE if mask is None else pa.PA_MODE_SAGE_SPARSE
    params = params_for(spec, batch, mode)
    ws = alloc_ws(params)
    if mask is None:
        pa.attn_plan(params, batch.seq_lens, None, ws)
    else:
        pa.attn_plan_sage_sparse(params, batch.seq_lens, mask, ws)
    out = torch.full((spec.batch, spec.hq, 128), float("nan"), dtype=torch.bfloat16, device=DEV)
    pa.attn_decode_paged_sage(params, ws, lay.q8, lay.sf_q, lay.k8, lay.v8, lay.sf_k, lay.sf_v, lay.v_mean,
                              batch.page_table, out)
    torch.cuda.synchronize()
    assert pa.pa_read_device_error(ws) == pa.PA_OK
    return out, ws, params


def oracle(spec, batch, lay, mask):
    return osg.sage_decode(lay.q8.cpu().numpy(), lay.sf_q.cpu().numpy(), lay.k8.cpu().numpy(), lay.v8.cpu().numpy(),
                           lay.sf_k.cpu().numpy(), lay.sf_v.cpu().numpy(), lay.v_mean.cpu().numpy(),
                           batch.page_table.cpu().numpy(), batch.seq_lens.cpu().numpy(), 64,
                           block_mask=None if mask is None else mask.cpu().numpy())


def test_sparse_plan_bit_exact():
    rng = np.random.default_rng(71)
    # (batch, longest length): rows within one 512-block mask step, and rows of 2-3 steps with
    # more requests than the plan has warps
    shapes = [(int(rng.integers(1, 40)), int(rng.integers(1, 9000))) for _ in range(12)] + [(50, 70000), (7, 40000)]
    for B, len_hi in shapes:
        spec = wl.Spec("sp_plan", 71, "sage", batch=B, len_lo=0, len_hi=len_hi, hq=32,
                       hkv=int(rng.choice([2, 8, 16])), page_size=64, spare_pages=0.1,
                       density=float(rng.choice([0.0, 0.1, 0.5, 1.0])))
        spec = spec.scaled(hq=spec.hkv * 2)
        batch = wl.make_batch(spec, DEV, seed=int(rng.integers(1 << 30)))
        mask = wl.make_block_mask(spec, batch, DEV, seed=int(rng.integers(1 << 30)))
        params = params_for(spec, batch, pa.PA_MODE_SAGE_SPARSE)
        ws = alloc_ws(params)
        pa.attn_plan_sage_sparse(params, batch.seq_lens, mask, ws)
        torch.cuda.synchronize()
        g = read_plan(ws, 3, B, spec.hq, max_kv_len=params.max_kv_len)
        o = op.plan(op.MODE_SAGE_SPARSE, batch.seq_lens.cpu().tolist(), hkv=spec.hkv, page_size=64,
                    num_sms=g["num_sms"],
                    block_mask=mask.cpu().numpy())
        assert g["error_word"] == 0
        assert g["items"] == [tuple(x) for x in o["items"]]
        assert g["slot_first"] == o["slot_first"] and g["sel_base"] == o["sel_base"]
        assert g["req_splits"] == o["req_splits"] and g["req_base"] == o["req_base"]
        raw = ws.cpu().numpy().view(np.uint8)
        from tests.helpers import ws_offsets
        off = ws_offsets(3, B, spec.hq, g["max_items"], hkv=spec.hkv, slots=g["slots"],
                         max_kv_len=params.max_kv_len)["sel_block"]
        nsel = o["sel_base"][-1]
        assert raw[off:off + 4 * nsel].view(np.int32).tolist() == o["sel_block"]


@pytest.mark.parametrize("layer", [0, 31])
def test_sparse_full_workload_density_0125(layer):
    """Every output row of the first and the last layer (32 layers rotate over 8 pools, so
    the last layer reads pool 7, as in the bench)."""
    spec = wl.SPECS["sage_sparse_decode"]
    batch = wl.make_batch(spec, DEV)
    lay = wl.make_sage_layer(spec, batch, layer % spec.distinct_pools, DEV)
    mask = wl.make_block_mask(spec, batch, DEV)
    out, _, _ = run(spec, batch, lay, mask)
    assert sage_row_rel_error(out, oracle(spec, batch, lay, mask)) <= SAGE_REL


@pytest.mark.parametrize("hq,hkv,lo,hi,density", [(8, 2, 1, 700, 0.3), (16, 4, 60, 70, 0.5), (64, 8, 100, 4000, 0.1),
                                                  (32, 16, 1, 2000, 0.125)])
def test_sparse_small_cases(hq, hkv, lo, hi, density):
    spec = wl.Spec("sp_small", 72, "sage", batch=6, len_lo=lo, len_hi=hi, hq=hq, hkv=hkv, page_size=64,
                   spare_pages=0.2, density=density)
    batch = wl.make_batch(spec, DEV)
    lay = wl.make_sage_layer(spec, batch, 0, DEV)
    mask = wl.make_block_mask(spec, batch, DEV)
    out, _, _ = run(spec, batch, lay, mask)
    assert sage_row_rel_error(out, oracle(spec, batch, lay, mask)) <= SAGE_REL


def test_all_ones_mask_is_bit_identical_to_dense_and_all_zeros_is_v_mean():
    spec = wl.SPECS["sage_decode"].scaled(batch=8, len_lo=100, len_hi=3000)
    batch = wl.make_batch(spec, DEV)
    lay = wl.make_sage_layer(spec, batch, 0, DEV)
    dense, _, _ = run(spec, batch, lay)
    ones, _, _ = run(spec, batch, lay, torch.ones_like(batch.page_table, dtype=torch.uint8))
    assert torch.equal(dense.view(torch.int16), ones.view(torch.int16))
    zeros, _, _ = run(spec, batch, lay, torch.zeros_like(batch.page_table, dtype=torch.uint8))
    vm = lay.v_mean.to(torch.bfloat16).repeat_interleave(spec.hq // spec.hkv, dim=0)
    assert torch.equal(zeros.view(torch.int16), vm[None].expand_as(zeros).contiguous().view(torch.int16))
