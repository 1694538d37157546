"""GPU parity of the FP8-KV decode (attn_decode_paged_fp8) against the fp64 oracle.

The bar is the bf16 decode's: max |err| <= 1e-2 beyond the bf16 output rounding, mean
|err| <= 1e-3, LSE within 4e-3, on the full FP8 workload and on small cases across page
sizes, head groupings, KV-head counts, ragged and empty rows and peaked scores.
"""
import os

import numpy as np
import pytest
import torch

import paged_kv_flashattention_split_b200 as pa
import workloads as wl
from oracle import attention as oa
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


def run_fp8(spec, batch, q, k8, v8, ks=wl.FP8_SCALE, vs=wl.FP8_SCALE):
    P = spec.page_size
    params = pa.make_params(pa.PA_MODE_DECODE, spec.batch, spec.hq, spec.hkv, 128, P,
                            max_kv_len=batch.page_table.shape[1] * P)
    ws = alloc_ws(params)
    pa.attn_plan(params, batch.seq_lens, None, ws)
    out = torch.full_like(q, float("nan"))
    lse = torch.full(q.shape[:2], float("nan"), dtype=torch.float32, device=DEV)
    pa.attn_decode_paged_fp8(params, ws, q, k8, v8, ks, vs, batch.page_table, spec.sm_scale, out, lse)
    torch.cuda.synchronize()
    assert pa.pa_read_device_error(ws) == pa.PA_OK
    return out, lse


def oracle_fp8(spec, batch, q, k8, v8, ks=wl.FP8_SCALE, vs=wl.FP8_SCALE):
    return oa.decode_fp8(bits16(q), k8.cpu().numpy(), v8.cpu().numpy(), ks, vs, batch.page_table.cpu().numpy(),
                         batch.seq_lens.cpu().numpy(), spec.page_size, spec.sm_scale)


def case(spec, peaked=False, layer=0):
    batch = wl.make_batch(spec, DEV)
    k8, v8 = wl.make_fp8_pools(spec, batch, layer, DEV)
    if peaked:   # 2% of the (slot, head) K rows scaled by 8 (still within E4M3's range: clamp)
        g = torch.Generator(device=DEV).manual_seed(44)
        sel = torch.rand(k8.shape[:2], generator=g, device=DEV) < 0.02
        kf = k8.view(torch.float8_e4m3fn).float()
        kf = torch.where(sel[..., None], (kf * 8).clamp(-448, 448), kf)
        k8 = torch.where(sel[..., None], kf.to(torch.float8_e4m3fn).view(torch.uint8), k8)
    q = wl.make_bf16_queries(spec, spec.batch, layer, DEV)
    return batch, q, k8, v8


def check(spec, batch, q, k8, v8, what, **kw):
    out, lse = run_fp8(spec, batch, q, k8, v8, **kw)
    ref, ref_lse = oracle_fp8(spec, batch, q, k8, v8, **kw)
    assert_bf16_close(out, ref, what)
    g = lse.cpu().numpy().astype(np.float64)
    fin = np.isfinite(ref_lse)
    assert np.all(np.isneginf(g[~fin])) and np.max(np.abs(g[fin] - ref_lse[fin]), initial=0.0) <= LSE_ABS


@pytest.mark.parametrize("layer", [0, 31])
def test_fp8_decode_full_workload(layer):
    """Every output element of the first and the last layer of the FP8-KV decode workload."""
    spec = wl.SPECS["decode_fp8_llama3_8b"]
    batch, q, k8, v8 = case(spec, layer=layer)
    check(spec, batch, q, k8, v8, "fp8 full")


@pytest.mark.parametrize("P,hq,hkv,lo,hi", [
    (1, 8, 2, 1, 300), (16, 32, 8, 17, 2000), (64, 16, 16, 63, 65), (256, 8, 1, 200, 900), (2, 4, 4, 0, 40),
])
def test_fp8_decode_page_sizes_and_head_layouts(P, hq, hkv, lo, hi):
    spec = wl.Spec("fp8_small", 61, "fp8", batch=5, len_lo=lo, len_hi=hi, hq=hq, hkv=hkv, page_size=P,
                   pool_slots=4096 if P == 1 else 0, spare_pages=0.2)
    batch, q, k8, v8 = case(spec)
    check(spec, batch, q, k8, v8, f"fp8 P={P} hq={hq} hkv={hkv}")


def test_fp8_decode_peaked_scores_and_other_scales():
    spec = wl.Spec("fp8_peaked", 62, "fp8", batch=4, len_lo=3000, len_hi=6000, hq=32, hkv=8, page_size=16,
                   spare_pages=0.1)
    batch, q, k8, v8 = case(spec, peaked=True)
    check(spec, batch, q, k8, v8, "fp8 peaked", ks=0.05, vs=0.031)


def test_fp8_decode_with_an_empty_row():
    spec = wl.Spec("fp8_empty", 63, "fp8", batch=3, len_lo=10, len_hi=500, hq=8, hkv=2, page_size=16,
                   spare_pages=0.3)
    batch, q, k8, v8 = case(spec)
    batch.seq_lens[1] = 0
    out, lse = run_fp8(spec, batch, q, k8, v8)
    assert torch.all(out[1].float() == 0) and torch.all(torch.isneginf(lse[1]))
    ref, _ = oracle_fp8(spec, batch, q, k8, v8)
    assert_bf16_close(out, ref, "fp8 empty row")
