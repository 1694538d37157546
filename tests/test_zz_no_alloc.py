"""GPU test of attn_decode_paged_noalloc, the decode entry point that allocates nothing.

Some callers cannot give the library a workspace: a host framework that owns
all device memory and exposes no allocator, a plugin that must not touch its
host process's memory pool, or a call site where allocating would synchronise
the device.  For them the library keeps the plan and the split partials in a
fixed 16 MiB device array.  This file checks, through the C ABI, that the
no-allocation call decodes exactly like attn_decode_paged with a caller
workspace, and within the bf16 bar of the fp64 oracle, on two calls in a row
(the second finds the first one's leftovers in the shared array); that repeated
calls leave the device's free memory and torch's reserved memory unchanged;
that an out-of-range page id is reported by pa_noalloc_read_device_error; and
that a plan too large for the array is refused.

It is named to be collected last, so that a run stopping at the first failure
has run every other test before it; it also passes alone in a fresh process.
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


def _params(spec, batch):
    return pa.make_params(pa.PA_MODE_DECODE, spec.batch, spec.hq, spec.hkv, spec.head_dim, spec.page_size,
                          max_kv_len=batch.page_table.shape[1] * spec.page_size)


def test_noalloc_matches_the_workspace_entry_point_on_consecutive_calls():
    cases = []
    spec = wl.SPECS["decode_llama3_8b"].scaled(batch=16, pool_slots=150_000)
    batch = wl.make_batch(spec, DEV)
    cases += [(spec, batch, 0), (spec, batch, 1)]
    spec2 = wl.SPECS["decode_tiny"]                      # a different batch and head layout on the third call
    cases += [(spec2, wl.make_batch(spec2, DEV), 0)]
    for spec, batch, layer in cases:
        params = _params(spec, batch)
        assert pa.pa_plan_workspace_size(params) <= 16 << 20
        k, v = wl.make_bf16_pools(spec, batch, layer, DEV)
        q = wl.make_bf16_queries(spec, spec.batch, layer, DEV)
        ws = alloc_ws(params)
        ref = torch.empty_like(q)
        ref_lse = torch.empty(q.shape[:2], dtype=torch.float32, device=DEV)
        pa.attn_plan(params, batch.seq_lens, None, ws)
        pa.attn_decode_paged(params, ws, q, k, v, batch.page_table, spec.sm_scale, ref, ref_lse)
        out = torch.full_like(q, float("nan"))
        lse = torch.full(q.shape[:2], float("nan"), dtype=torch.float32, device=DEV)
        pa.attn_decode_paged_noalloc(params, batch.seq_lens, q, k, v, batch.page_table, spec.sm_scale, out, lse)
        torch.cuda.synchronize()
        assert pa.pa_noalloc_read_device_error() == pa.PA_OK
        assert_bf16_close(out, bf16_bits_to_f64(bits16(ref)), f"noalloc layer {layer}")
        assert np.max(np.abs(lse.cpu().numpy() - ref_lse.cpu().numpy())) <= LSE_ABS
        o_ref, l_ref = oa.decode(bits16(q), bits16(k), bits16(v), batch.page_table.cpu().numpy(),
                                 batch.seq_lens.cpu().numpy(), spec.page_size, spec.sm_scale)
        assert_bf16_close(out, o_ref, f"noalloc vs oracle, layer {layer}")
        assert np.max(np.abs(lse.cpu().numpy() - l_ref)) <= LSE_ABS


def test_noalloc_calls_leave_device_memory_unchanged_and_report_bad_page_ids():
    spec = wl.SPECS["decode_tiny"]
    batch = wl.make_batch(spec, DEV)
    params = _params(spec, batch)
    k, v = wl.make_bf16_pools(spec, batch, 0, DEV)
    q = wl.make_bf16_queries(spec, spec.batch, 0, DEV)
    out = torch.empty_like(q)
    pa.attn_decode_paged_noalloc(params, batch.seq_lens, q, k, v, batch.page_table, spec.sm_scale, out)
    torch.cuda.synchronize()
    free0, reserved0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_reserved()
    for _ in range(5):
        pa.attn_decode_paged_noalloc(params, batch.seq_lens, q, k, v, batch.page_table, spec.sm_scale, out)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0 and torch.cuda.memory_reserved() == reserved0
    assert pa.pa_noalloc_read_device_error() == pa.PA_OK
    # one page id past the pool: the kernels skip that key (it reads as zero) and record the error
    bad = batch.page_table.clone()
    bad[1, 0] = batch.num_slots + 5
    pa.attn_decode_paged_noalloc(params, batch.seq_lens, q, k, v, bad, spec.sm_scale, out)
    assert pa.pa_noalloc_read_device_error() == pa.PA_ERR_DEVICE_INDEX
    assert pa.pa_noalloc_read_device_error() == pa.PA_OK        # reading clears the word


def test_noalloc_refuses_plans_larger_than_its_array():
    params = pa.make_params(pa.PA_MODE_DECODE, 8192, 64, 8, 128, 1, max_kv_len=4096)
    assert pa.pa_plan_workspace_size(params) > 16 << 20
    dummy = torch.zeros(16, dtype=torch.int32, device=DEV)
    st = pa.attn_decode_paged_noalloc(params, dummy, dummy, dummy, dummy, dummy, 1.0, dummy,
                                      num_slots=1, pt_pitch=4096, raise_on_error=False)
    assert st == pa.PA_ERR_WORKSPACE
    bad_mode = pa.make_params(pa.PA_MODE_EXTEND, 4, 8, 2, 128, 16, max_kv_len=64, max_q_tokens=64)
    st = pa.attn_decode_paged_noalloc(bad_mode, dummy, dummy, dummy, dummy, dummy, 1.0, dummy,
                                      num_slots=1, pt_pitch=4, raise_on_error=False)
    assert st == pa.PA_ERR_INVALID
