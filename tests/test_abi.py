"""Host-side checks of the C ABI (no GPU needed).

The shared library must load and export every function include/pagedattn.h
declares; parameter validation and workspace sizing are pure host code and
are exercised here without a device (num_sms given explicitly).
"""
import ctypes
import os
import re

import pytest

import paged_kv_flashattention_split_b200 as pa
from paged_kv_flashattention_split_b200 import build as pa_build
from tests.helpers import ws_offsets

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(pa.LIB_PATH):
        pa_build.build()
    return pa.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "pagedattn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:pa_status|const char\*|int32_t)\s+(\w+)\s*\(", src, flags=re.M)))


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert set(pa.EXPORTED) == set(names), names
    for n in names:
        assert hasattr(lib, n), n
    assert pa.pa_version() == 100


def test_status_strings(lib):
    for code, name in [(0, "PA_OK"), (1, "PA_ERR_INVALID"), (2, "PA_ERR_UNSUPPORTED"), (3, "PA_ERR_ARCH"),
                       (4, "PA_ERR_WORKSPACE"), (5, "PA_ERR_CUDA"), (6, "PA_ERR_DEVICE_INDEX")]:
        assert pa.status_string(code) == name
    assert pa.status_string(99) == "PA_ERR_UNKNOWN"


def P(**kw):
    base = dict(mode=0, batch=4, hq=8, hkv=2, head_dim=128, page_size=1, max_kv_len=300, num_sms=148)
    base.update(kw)
    return pa.make_params(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(head_dim=64), pa.PA_ERR_UNSUPPORTED),
    (dict(page_size=3), pa.PA_ERR_UNSUPPORTED),
    (dict(page_size=512), pa.PA_ERR_UNSUPPORTED),
    (dict(hq=6, hkv=4), pa.PA_ERR_INVALID),
    (dict(hq=32, hkv=2), pa.PA_ERR_UNSUPPORTED),        # 16 query heads per KV head
    (dict(batch=0), pa.PA_ERR_INVALID),
    (dict(batch=9000), pa.PA_ERR_INVALID),
    (dict(mode=7), pa.PA_ERR_INVALID),
    (dict(max_q_tokens=5), pa.PA_ERR_INVALID),          # decode plan given an extend-only input
    (dict(sage_k_block=64), pa.PA_ERR_INVALID),
    (dict(max_splits=4), pa.PA_ERR_INVALID),             # no split cap in DECODE (flat partition)
    (dict(mode=1, page_size=3, max_q_tokens=100), pa.PA_ERR_UNSUPPORTED),
    (dict(mode=2, page_size=64, sage_k_block=16), pa.PA_ERR_UNSUPPORTED),
    (dict(mode=2, page_size=64, sage_k_block=64, max_q_tokens=8), pa.PA_ERR_INVALID),
    (dict(mode=2, page_size=64, sage_k_block=64, max_splits=4), pa.PA_ERR_INVALID),   # no split cap in SAGE
    (dict(mode=2, page_size=64, sage_k_block=64, batch=8192, hq=4096, hkv=512, max_kv_len=1 << 30),
     pa.PA_ERR_UNSUPPORTED),                            # score rows beyond 2^46 bytes
    (dict(num_sms=-1), pa.PA_ERR_INVALID),
])
def test_parameter_validation(lib, kw, status):
    assert pa.pa_plan_workspace_size(P(**kw), raise_on_error=False) == status


@pytest.mark.parametrize("page_size", [1, 2, 4, 8, 256])
def test_extend_accepts_every_page_size(lib, page_size):
    """EXTEND plans for any power-of-two page size (below 8 the kernels gather slot by slot)."""
    assert pa.pa_plan_workspace_size(P(mode=1, page_size=page_size, max_q_tokens=100)) > 64


def test_workspace_size_matches_documented_layout(lib):
    for mode, extra in ((0, {}), (1, dict(page_size=16, max_q_tokens=9000)), (2, dict(page_size=64, sage_k_block=64, max_kv_len=4096))):
        p = P(mode=mode, batch=33, hq=32, hkv=8, **extra)
        n = pa.pa_plan_workspace_size(p)
        slots = 0
        if mode in (0, 2):
            slots = 148 * 2            # Hkv 8: one item covers the 8 KV heads, two slots per SM
            mi = slots + 33
        else:
            mi = -(-9000 // 128) + 33
        assert n == ws_offsets(mode, 33, 32, mi, hkv=8, max_kv_len=p.max_kv_len, slots=slots)["total"]


def test_host_checks_precede_device_use(lib):
    # NULL workspace / seq_lens are rejected before any CUDA call (works without a GPU)
    p = P()
    assert lib.attn_plan(ctypes.byref(p), None, None, None, 0, None) == pa.PA_ERR_INVALID
    # an EXTEND plan needs cu_seqlens_q, the other modes must not get one
    pe = P(mode=1, page_size=16, max_q_tokens=64)
    assert lib.attn_plan(ctypes.byref(pe), 16, None, 256, 1 << 20, None) == pa.PA_ERR_INVALID
    assert lib.attn_plan(ctypes.byref(p), 16, 32, 256, 1 << 20, None) == pa.PA_ERR_INVALID
    # short workspace
    assert lib.attn_plan(ctypes.byref(p), 16, None, 256, 64, None) == pa.PA_ERR_WORKSPACE
    # misaligned workspace
    assert lib.attn_plan(ctypes.byref(p), 16, None, 258, 1 << 20, None) == pa.PA_ERR_INVALID
    # a decode call given an extend plan
    assert lib.attn_decode_paged(ctypes.byref(pe), 256, 1 << 20, 256, 256, 256, 10, 256, 8, 1.0, 256, None,
                                 None) == pa.PA_ERR_WORKSPACE
    # page table pitch too small for max_kv_len
    assert lib.attn_decode_paged(ctypes.byref(p), 256, 1 << 30, 256, 256, 256, 10, 256, 8, 1.0, 256, None,
                                 None) == pa.PA_ERR_INVALID
