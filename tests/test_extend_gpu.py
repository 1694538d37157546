"""GPU parity of the causal paged EXTEND (tcgen05 / TMEM kernel) against the fp64 oracle.

Bar: max |err| <= 1e-2 beyond the bf16 output rounding, mean |err| <= 1e-3, LSE
within 4e-3; on small cases that span several query and key tiles with ragged
tails, all page sizes and head groupings, peaked scores (the rescale path), the
full extend workload (sampled heads), and the degenerate cases (one new token,
no prefix).
"""
import os

import numpy as np
import pytest
import torch

import paged_kv_flashattention_split_b200 as pa
import workloads as wl
from oracle import attention as oa
from oracle.codecs import bf16_bits_to_f64
from tests.helpers import LSE_ABS, alloc_ws, assert_bf16_close, bits16

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    if not os.path.exists(pa.LIB_PATH):
        from paged_kv_flashattention_split_b200 import build
        build.build()
    pa.lib()


def extend_case(spec, layer=0, peaked=False):
    batch = wl.make_batch(spec, DEV)
    if peaked:
        spec = spec.scaled(peaked_frac=0.02, peaked_scale=8.0)
    k, v = wl.make_bf16_pools(spec, batch, layer, DEV)
    total = int(batch.cu_seqlens_q[-1])
    q = wl.make_bf16_queries(spec, total, layer, DEV)
    return batch, q, k, v


def run_extend(spec, batch, q, k, v):
    total = q.shape[0]
    params = pa.make_params(pa.PA_MODE_EXTEND, spec.batch, spec.hq, spec.hkv, 128, spec.page_size,
                            max_kv_len=batch.page_table.shape[1] * spec.page_size, max_q_tokens=total)
    ws = alloc_ws(params)
    pa.attn_plan(params, batch.seq_lens, batch.cu_seqlens_q, ws)
    out = torch.full_like(q, float("nan"))
    lse = torch.full(q.shape[:2], float("nan"), dtype=torch.float32, device=DEV)
    pa.attn_extend_paged(params, ws, q, k, v, batch.page_table, spec.sm_scale, out, lse)
    torch.cuda.synchronize()
    st = pa.pa_read_device_error(ws)
    assert st == pa.PA_OK, pa.status_string(st)
    return out, lse


def oracle_extend(spec, batch, q, k, v):
    return oa.extend(bits16(q), batch.cu_seqlens_q.cpu().numpy(), bits16(k), bits16(v), batch.page_table.cpu().numpy(),
                     batch.seq_lens.cpu().numpy(), spec.page_size, spec.sm_scale)


def check_lse(lse_gpu, ref):
    g = lse_gpu.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(g))
    assert np.max(np.abs(g - ref)) <= LSE_ABS


def small_spec(**kw):
    base = dict(name="extend_small", cfg=31, mode="extend", batch=3, len_lo=0, len_hi=400, hq=4, hkv=2,
                page_size=16, spare_pages=0.2, new_lo=1, new_hi=300)
    base.update(kw)
    return wl.Spec(**base)


def test_extend_small_first():
    spec = small_spec()
    batch, q, k, v = extend_case(spec)
    out, lse = run_extend(spec, batch, q, k, v)
    ref, ref_lse = oracle_extend(spec, batch, q, k, v)
    assert_bf16_close(out, ref, "extend_small")
    check_lse(lse, ref_lse)


@pytest.mark.parametrize("P,G,lo,hi,nlo,nhi", [
    (8, 1, 0, 0, 1, 260),          # no prefix, MHA, page size 8
    (16, 4, 127, 129, 128, 128),   # one full query tile, prefix around a key-tile boundary
    (64, 8, 1000, 3000, 1, 1),     # single new token per request (decode through extend)
    (128, 2, 0, 700, 200, 600),
    (256, 4, 300, 900, 1, 400),
    (1, 1, 0, 500, 1, 300),        # page size 1: the table is req_to_token (slot-by-slot gathers)
    (1, 4, 100, 700, 100, 400),
    (2, 8, 0, 300, 50, 200),
    (4, 4, 60, 70, 120, 140),      # a CTA pair whose second K half is empty on the last tile
    (2, 2, 10, 900, 1, 260),
    (4, 1, 129, 129, 127, 127),
])
def test_extend_page_sizes_groups_and_ragged_tiles(P, G, lo, hi, nlo, nhi):
    spec = small_spec(page_size=P, hq=2 * G, hkv=2, len_lo=lo, len_hi=hi, new_lo=nlo, new_hi=nhi, batch=4)
    batch, q, k, v = extend_case(spec)
    out, lse = run_extend(spec, batch, q, k, v)
    ref, ref_lse = oracle_extend(spec, batch, q, k, v)
    assert_bf16_close(out, ref, f"extend P={P} G={G}")
    check_lse(lse, ref_lse)


def test_extend_peaked_scores_take_the_rescale_path():
    spec = small_spec(batch=2, len_lo=2000, len_hi=3000, new_lo=100, new_hi=300, hq=8, hkv=2)
    batch, q, k, v = extend_case(spec, peaked=True)
    out, lse = run_extend(spec, batch, q, k, v)
    ref, ref_lse = oracle_extend(spec, batch, q, k, v)
    assert_bf16_close(out, ref, "extend peaked")
    check_lse(lse, ref_lse)


def test_extend_with_one_new_token_equals_decode():
    spec = small_spec(batch=5, len_lo=50, len_hi=2000, new_lo=1, new_hi=1, hq=8, hkv=2, page_size=16)
    batch, q, k, v = extend_case(spec)
    out, lse = run_extend(spec, batch, q, k, v)
    dparams = pa.make_params(pa.PA_MODE_DECODE, spec.batch, spec.hq, spec.hkv, 128, 16,
                             max_kv_len=batch.page_table.shape[1] * 16)
    ws = alloc_ws(dparams)
    pa.attn_plan(dparams, batch.seq_lens, None, ws)
    dout = torch.empty_like(q)
    pa.attn_decode_paged(dparams, ws, q, k, v, batch.page_table, spec.sm_scale, dout)
    torch.cuda.synchronize()
    assert_bf16_close(out, bf16_bits_to_f64(bits16(dout)), "extend n=1 vs decode")


@pytest.mark.parametrize("layer", [0, 31])
def test_extend_full_workload(layer):
    """Every output element and LSE, all 32 query heads, of the first and the last layer of the
    extend workload (the oracle's heads spread over a process pool)."""
    from tests import oracle_jobs
    spec = wl.SPECS["extend_prefix"]
    batch, q, k, v = extend_case(spec, layer=layer)
    out, lse = run_extend(spec, batch, q, k, v)
    ref, ref_lse = oracle_jobs.extend_all_heads(bits16(q), batch.cu_seqlens_q.cpu().numpy(), bits16(k), bits16(v),
                                                batch.page_table.cpu().numpy(), batch.seq_lens.cpu().numpy(),
                                                spec.page_size, spec.sm_scale)
    assert_bf16_close(out, ref, f"extend full layer {layer}")
    check_lse(lse, ref_lse)


def test_extend_page_size_one_at_the_extend_workload_lengths():
    """The extend workload's lengths and heads over a slot-granular cache (page size 1, the
    table being req_to_token itself), on a sample of query heads of every KV head."""
    spec = wl.SPECS["extend_prefix"].scaled(page_size=1, spare_pages=0.0, pool_slots=0, layers=1)
    batch, q, k, v = extend_case(spec)
    out, lse = run_extend(spec, batch, q, k, v)
    heads = [0, 5, 10, 15, 16, 21, 26, 31]                      # two of each KV head's four query heads
    G = spec.hq // spec.hkv
    qb = bits16(q)[:, heads]
    kv = sorted({h // G for h in heads})
    kb, vb = bits16(k)[:, kv], bits16(v)[:, kv]
    # the oracle over the sampled heads: query head i of the sample reads sampled KV head kv.index(h // G)
    qs = np.stack([qb[:, i] for i in range(len(heads))], axis=1)
    ref = np.zeros(qs.shape)
    ref_lse = np.zeros(qs.shape[:2])
    for i, h in enumerate(heads):
        hk = kv.index(h // G)
        o, l = oa.extend(qs[:, i:i + 1], batch.cu_seqlens_q.cpu().numpy(), kb[:, hk:hk + 1], vb[:, hk:hk + 1],
                         batch.page_table.cpu().numpy(), batch.seq_lens.cpu().numpy(), 1, spec.sm_scale)
        ref[:, i], ref_lse[:, i] = o[:, 0], l[:, 0]
    assert_bf16_close(out[:, heads], ref, "extend P=1 at the extend workload lengths")
    check_lse(lse[:, heads], ref_lse)
