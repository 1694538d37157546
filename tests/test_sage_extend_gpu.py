"""GPU parity of the 8-bit Sage EXTEND (tcgen05, two passes) against the oracle.

The bar is the Sage decode's: max over output rows (token, head) of
||O_gpu - O_ref||_inf / max(||O_ref||_inf, 1e-6) <= 3e-2; on small cases that span several
query and key tiles with ragged tails, head groups 1-8, no prefix, one new token per
request (which equals the Sage decode of the same row), without v_mean, and on the full
Sage extend workload (every head of the first and last layer).
"""
import os

import numpy as np
import pytest
import torch

import paged_kv_flashattention_split_b200 as pa
import workloads as wl
from oracle import sage as osg
from tests.helpers import SAGE_REL, alloc_ws, sage_row_rel_error

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    if not os.path.exists(pa.LIB_PATH):
        from paged_kv_flashattention_split_b200 import build
        build.build()
    pa.lib()


def case(spec, layer=0):
    batch = wl.make_batch(spec, DEV)
    T = int(batch.cu_seqlens_q[-1])
    lay = wl.make_sage_layer(spec, batch, layer, DEV, q_rows=T)
    return batch, lay, T


def run(spec, batch, lay, T, use_v_mean=True):
    params = pa.make_params(pa.PA_MODE_EXTEND, spec.batch, spec.hq, spec.hkv, 128, 64,
                            max_kv_len=batch.page_table.shape[1] * 64, max_q_tokens=T)
    ws = alloc_ws(params)
    pa.attn_plan(params, batch.seq_lens, batch.cu_seqlens_q, ws)
    out = torch.full((T, spec.hq, 128), float("nan"), dtype=torch.bfloat16, device=DEV)
    pa.attn_extend_paged_sage(params, ws, lay.q8, lay.sf_q, lay.k8, lay.v8, lay.sf_k, lay.sf_v,
                              lay.v_mean if use_v_mean else None, batch.page_table, out)
    torch.cuda.synchronize()
    assert pa.pa_read_device_error(ws) == pa.PA_OK
    return out


def oracle(spec, batch, lay, use_v_mean=True):
    cu = batch.cu_seqlens_q.cpu().numpy()
    table, lens = batch.page_table.cpu().numpy(), batch.seq_lens.cpu().numpy()
    q8, sfq = lay.q8.cpu().numpy(), lay.sf_q.cpu().numpy()
    k8, v8, sfk = lay.k8.cpu().numpy(), lay.v8.cpu().numpy(), lay.sf_k.cpu().numpy()
    sfv, vm = lay.sf_v.cpu().numpy(), lay.v_mean.cpu().numpy() if use_v_mean else None
    return osg.sage_extend(q8, sfq, cu, k8, v8, sfk, sfv, vm, table, lens, 64)


def small(**kw):
    base = dict(name="sage_ext_small", cfg=81, mode="extend", batch=3, len_lo=0, len_hi=300, hq=4, hkv=2,
                page_size=64, spare_pages=0.2, new_lo=1, new_hi=200)
    base.update(kw)
    return wl.Spec(**base)


def test_sage_extend_small_first():
    spec = small()
    batch, lay, T = case(spec)
    out = run(spec, batch, lay, T)
    assert sage_row_rel_error(out, oracle(spec, batch, lay)) <= SAGE_REL


@pytest.mark.parametrize("G,lo,hi,nlo,nhi", [
    (1, 0, 0, 1, 260),          # no prefix, MHA
    (2, 127, 129, 128, 128),    # one full query tile, prefix around a key-tile boundary
    (4, 300, 900, 1, 300),
    (8, 50, 700, 200, 400),
])
def test_sage_extend_groups_and_ragged_tiles(G, lo, hi, nlo, nhi):
    spec = small(hq=2 * G, hkv=2, len_lo=lo, len_hi=hi, new_lo=nlo, new_hi=nhi, batch=4)
    batch, lay, T = case(spec)
    out = run(spec, batch, lay, T)
    assert sage_row_rel_error(out, oracle(spec, batch, lay)) <= SAGE_REL


def test_sage_extend_one_new_token_matches_sage_decode_and_no_v_mean():
    spec = small(batch=5, len_lo=50, len_hi=1500, new_lo=1, new_hi=1, hq=8, hkv=2)
    batch, lay, T = case(spec)
    out = run(spec, batch, lay, T, use_v_mean=False)
    ref = osg.sage_decode(lay.q8.cpu().numpy(), lay.sf_q.cpu().numpy(), lay.k8.cpu().numpy(), lay.v8.cpu().numpy(),
                          lay.sf_k.cpu().numpy(), lay.sf_v.cpu().numpy(), None, batch.page_table.cpu().numpy(),
                          batch.seq_lens.cpu().numpy(), 64)
    assert sage_row_rel_error(out, ref) <= SAGE_REL


@pytest.mark.parametrize("layer", [0, 31])
def test_sage_extend_full_workload(layer):
    """Every output row, all 32 query heads, of the first and the last layer of the Sage extend
    workload (the oracle's heads spread over a process pool)."""
    from tests import oracle_jobs
    spec = wl.SPECS["sage_extend_prefix"]
    batch, lay, T = case(spec, layer)
    out = run(spec, batch, lay, T)
    h = {k: getattr(lay, k).cpu().numpy() for k in ("q8", "sf_q", "k8", "v8", "sf_k", "sf_v", "v_mean")}
    ref = oracle_jobs.sage_extend_all_heads(h["q8"], h["sf_q"], batch.cu_seqlens_q.cpu().numpy(), h["k8"], h["v8"],
                                            h["sf_k"], h["sf_v"], h["v_mean"], batch.page_table.cpu().numpy(),
                                            batch.seq_lens.cpu().numpy())
    assert sage_row_rel_error(out, ref) <= SAGE_REL
