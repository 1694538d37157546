"""ctypes binding of libpagedattn.so: the C ABI under the same names.

This layer only marshals arguments: torch tensors become raw pointers, the
stream defaults to torch's current CUDA stream, and a non-zero status raises
``PagedAttnError``.  Every step of the attention path runs in the library's
CUDA kernels; there is no fallback.  If the shared library has not been built
the first call fails loudly with instructions.
"""
from __future__ import annotations

import ctypes
import os

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpagedattn.so")

PA_OK, PA_ERR_INVALID, PA_ERR_UNSUPPORTED, PA_ERR_ARCH = 0, 1, 2, 3
PA_ERR_WORKSPACE, PA_ERR_CUDA, PA_ERR_DEVICE_INDEX = 4, 5, 6
PA_MODE_DECODE, PA_MODE_EXTEND, PA_MODE_SAGE_DECODE, PA_MODE_SAGE_SPARSE = 0, 1, 2, 3

EXPORTED = ("pa_plan_workspace_size", "attn_plan", "attn_decode_paged", "attn_extend_paged",
            "attn_decode_paged_sage", "attn_debug_gather", "pa_read_device_error",
            "pa_status_string", "pa_version", "attn_decode_paged_noalloc", "attn_kv_store",
            "attn_kv_store_sage", "attn_decode_paged_fp8", "attn_plan_sage_sparse", "attn_extend_paged_sage",
            "pa_noalloc_read_device_error")


class pa_plan_params(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "mode", "batch", "hq", "hkv", "head_dim", "page_size", "max_kv_len", "max_q_tokens",
        "num_sms", "max_splits", "sage_k_block", "reserved")]


class PagedAttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


_lib = None
_P = ctypes.c_void_p
_I32, _I64, _F32, _SZ = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t


def lib() -> ctypes.CDLL:
    """Load (once) and return the shared library; raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is not built; run `python -m paged_kv_flashattention_split_b200.build` "
                "(or __graft_entry__.build()).  There is no CPU fallback.")
        L = ctypes.CDLL(LIB_PATH)
        PP = ctypes.POINTER(pa_plan_params)
        sig = {
            "pa_plan_workspace_size": (_I32, [PP, ctypes.POINTER(_SZ)]),
            "attn_plan": (_I32, [PP, _P, _P, _P, _SZ, _P]),
            "attn_plan_sage_sparse": (_I32, [PP, _P, _P, _I64, _P, _SZ, _P]),
            "attn_decode_paged": (_I32, [PP, _P, _SZ, _P, _P, _P, _I64, _P, _I64, _F32, _P, _P, _P]),
            "attn_extend_paged": (_I32, [PP, _P, _SZ, _P, _P, _P, _I64, _P, _I64, _F32, _P, _P, _P]),
            "attn_decode_paged_fp8": (_I32, [PP, _P, _SZ, _P, _P, _P, _F32, _F32, _I64, _P, _I64, _F32, _P, _P,
                                             _P]),
            "attn_decode_paged_sage": (_I32, [PP, _P, _SZ, _P, _P, _P, _P, _P, _P, _P, _I64, _P, _I64,
                                              _P, _P]),
            "attn_extend_paged_sage": (_I32, [PP, _P, _SZ, _P, _P, _P, _P, _P, _P, _P, _I64, _P, _I64, _P, _P]),
            "attn_debug_gather": (_I32, [_P, _I32, _I32, _I32, _I32, _I32, _I32, _P, _I64, _P, _I64,
                                         _P, _P, _P]),
            "pa_read_device_error": (_I32, [_P, _P]),
            "pa_noalloc_read_device_error": (_I32, [_P]),
            "attn_kv_store": (_I32, [_P, _P, _P, _I64, _I32, _I32, _P, _P, _I64, _P, _P]),
            "attn_kv_store_sage": (_I32, [_P, _P, _P, _P, _I64, _I32, _I32, _P, _P, _P, _I64, _P, _P]),
            "attn_decode_paged_noalloc": (_I32, [PP, _P, _P, _P, _P, _I64, _P, _I64, _F32, _P, _P, _P]),
            "pa_status_string": (ctypes.c_char_p, [_I32]),
            "pa_version": (_I32, []),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().pa_status_string(int(status)).decode()


def _ptr(t):
    """Device (or host) address of a tensor, an int address, or None -> NULL."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str, raise_on_error: bool):
    if raise_on_error and status != PA_OK:
        raise PagedAttnError(status, where)
    return status


def make_params(mode: int, batch: int, hq: int, hkv: int, head_dim: int = 128, page_size: int = 1,
                max_kv_len: int = 0, max_q_tokens: int = 0, num_sms: int = 0, max_splits: int = 0,
                sage_k_block: int = 0) -> pa_plan_params:
    return pa_plan_params(mode, batch, hq, hkv, head_dim, page_size, max_kv_len, max_q_tokens,
                          num_sms, max_splits, sage_k_block, 0)


def pa_plan_workspace_size(params: pa_plan_params, raise_on_error: bool = True):
    out = _SZ(0)
    st = lib().pa_plan_workspace_size(ctypes.byref(params), ctypes.byref(out))
    _check(st, "pa_plan_workspace_size", raise_on_error)
    return out.value if st == PA_OK else st


def attn_plan(params, seq_lens, cu_seqlens_q, ws, stream=None, raise_on_error=True) -> int:
    nbytes = ws.numel() * ws.element_size() if isinstance(ws, torch.Tensor) else 0
    st = lib().attn_plan(ctypes.byref(params), _ptr(seq_lens), _ptr(cu_seqlens_q), _ptr(ws), nbytes,
                         _stream(stream))
    return _check(st, "attn_plan", raise_on_error)


def attn_plan_sage_sparse(params, seq_lens, block_mask, ws, stream=None, raise_on_error=True) -> int:
    """Plan of the block-sparse Sage decode; block_mask uint8 [B, mask_pitch] (nonzero = attend)."""
    nbytes = ws.numel() * ws.element_size() if isinstance(ws, torch.Tensor) else 0
    st = lib().attn_plan_sage_sparse(ctypes.byref(params), _ptr(seq_lens), _ptr(block_mask),
                                     int(block_mask.shape[-1]), _ptr(ws), nbytes, _stream(stream))
    return _check(st, "attn_plan_sage_sparse", raise_on_error)


def attn_decode_paged(params, ws, q, k_pool, v_pool, page_table, sm_scale, out, lse_out=None,
                      num_slots=None, pt_pitch=None, stream=None, raise_on_error=True) -> int:
    num_slots = k_pool.shape[0] if num_slots is None else num_slots
    pt_pitch = page_table.shape[-1] if pt_pitch is None else pt_pitch
    st = lib().attn_decode_paged(ctypes.byref(params), _ptr(ws), ws.numel() * ws.element_size(),
                                 _ptr(q), _ptr(k_pool), _ptr(v_pool), int(num_slots), _ptr(page_table),
                                 int(pt_pitch), float(sm_scale), _ptr(out), _ptr(lse_out),
                                 _stream(stream))
    return _check(st, "attn_decode_paged", raise_on_error)


def attn_decode_paged_fp8(params, ws, q, k8_pool, v8_pool, k_scale, v_scale, page_table, sm_scale, out,
                          lse_out=None, num_slots=None, pt_pitch=None, stream=None, raise_on_error=True) -> int:
    """DECODE over E4M3 pools (uint8 codes) dequantised by k_scale / v_scale; q and out bf16."""
    num_slots = k8_pool.shape[0] if num_slots is None else num_slots
    pt_pitch = page_table.shape[-1] if pt_pitch is None else pt_pitch
    st = lib().attn_decode_paged_fp8(ctypes.byref(params), _ptr(ws), ws.numel() * ws.element_size(),
                                     _ptr(q), _ptr(k8_pool), _ptr(v8_pool), float(k_scale), float(v_scale),
                                     int(num_slots), _ptr(page_table), int(pt_pitch), float(sm_scale), _ptr(out),
                                     _ptr(lse_out), _stream(stream))
    return _check(st, "attn_decode_paged_fp8", raise_on_error)


def attn_extend_paged(params, ws, q, k_pool, v_pool, page_table, sm_scale, out, lse_out=None,
                      num_slots=None, pt_pitch=None, stream=None, raise_on_error=True) -> int:
    num_slots = k_pool.shape[0] if num_slots is None else num_slots
    pt_pitch = page_table.shape[-1] if pt_pitch is None else pt_pitch
    st = lib().attn_extend_paged(ctypes.byref(params), _ptr(ws), ws.numel() * ws.element_size(),
                                 _ptr(q), _ptr(k_pool), _ptr(v_pool), int(num_slots), _ptr(page_table),
                                 int(pt_pitch), float(sm_scale), _ptr(out), _ptr(lse_out),
                                 _stream(stream))
    return _check(st, "attn_extend_paged", raise_on_error)


def attn_decode_paged_sage(params, ws, q8, sf_q, k8_pool, v8_pool, sf_k, sf_v, v_mean, page_table,
                           out, num_slots=None, pt_pitch=None, stream=None, raise_on_error=True) -> int:
    num_slots = k8_pool.shape[0] if num_slots is None else num_slots
    pt_pitch = page_table.shape[-1] if pt_pitch is None else pt_pitch
    st = lib().attn_decode_paged_sage(ctypes.byref(params), _ptr(ws), ws.numel() * ws.element_size(),
                                      _ptr(q8), _ptr(sf_q), _ptr(k8_pool), _ptr(v8_pool), _ptr(sf_k),
                                      _ptr(sf_v), _ptr(v_mean), int(num_slots), _ptr(page_table),
                                      int(pt_pitch), _ptr(out), _stream(stream))
    return _check(st, "attn_decode_paged_sage", raise_on_error)


def attn_extend_paged_sage(params, ws, q8, sf_q, k8_pool, v8_pool, sf_k, sf_v, v_mean, page_table, out,
                           num_slots=None, pt_pitch=None, stream=None, raise_on_error=True) -> int:
    """8-bit Sage EXTEND over an EXTEND plan with page size 64; q8 int8 [T, Hq, D], out bf16."""
    num_slots = k8_pool.shape[0] if num_slots is None else num_slots
    pt_pitch = page_table.shape[-1] if pt_pitch is None else pt_pitch
    st = lib().attn_extend_paged_sage(ctypes.byref(params), _ptr(ws), ws.numel() * ws.element_size(),
                                      _ptr(q8), _ptr(sf_q), _ptr(k8_pool), _ptr(v8_pool), _ptr(sf_k),
                                      _ptr(sf_v), _ptr(v_mean), int(num_slots), _ptr(page_table),
                                      int(pt_pitch), _ptr(out), _stream(stream))
    return _check(st, "attn_extend_paged_sage", raise_on_error)


def attn_debug_gather(seq_lens, r, h_kv, hkv, page_size, max_len, k_pool, page_table, slots_out,
                      rows_out, head_dim=128, num_slots=None, pt_pitch=None, stream=None,
                      raise_on_error=True) -> int:
    num_slots = k_pool.shape[0] if num_slots is None else num_slots
    pt_pitch = page_table.shape[-1] if pt_pitch is None else pt_pitch
    st = lib().attn_debug_gather(_ptr(seq_lens), r, h_kv, hkv, head_dim, page_size, max_len,
                                 _ptr(k_pool), int(num_slots), _ptr(page_table), int(pt_pitch),
                                 _ptr(slots_out), _ptr(rows_out), _stream(stream))
    return _check(st, "attn_debug_gather", raise_on_error)


def attn_decode_paged_noalloc(params, seq_lens, q, k_pool, v_pool, page_table, sm_scale, out, lse_out=None,
                              num_slots=None, pt_pitch=None, stream=None, raise_on_error=True) -> int:
    """Plan and decode without a caller workspace (the library's fixed 16 MiB array is used)."""
    num_slots = k_pool.shape[0] if num_slots is None else num_slots
    pt_pitch = page_table.shape[-1] if pt_pitch is None else pt_pitch
    st = lib().attn_decode_paged_noalloc(ctypes.byref(params), _ptr(seq_lens), _ptr(q), _ptr(k_pool),
                                         _ptr(v_pool), int(num_slots), _ptr(page_table), int(pt_pitch),
                                         float(sm_scale), _ptr(out), _ptr(lse_out), _stream(stream))
    return _check(st, "attn_decode_paged_noalloc", raise_on_error)


def attn_kv_store(k_new, v_new, out_cache_loc, k_pool, v_pool, ws=None, n_tokens=None, num_slots=None,
                  stream=None, raise_on_error=True) -> int:
    """Scatter new tokens' K/V rows ([n, Hkv, D] bf16) into the pools at out_cache_loc (int32 [n])."""
    n = k_new.shape[0] if n_tokens is None else n_tokens
    num_slots = k_pool.shape[0] if num_slots is None else num_slots
    hkv = k_pool.shape[1]
    st = lib().attn_kv_store(_ptr(k_new), _ptr(v_new), _ptr(out_cache_loc), int(n), int(hkv), int(k_pool.shape[2]),
                             _ptr(k_pool), _ptr(v_pool), int(num_slots), _ptr(ws), _stream(stream))
    return _check(st, "attn_kv_store", raise_on_error)


def attn_kv_store_sage(k8_new, v8_new, sf_k_new, out_cache_loc, k8_pool, v8_pool, sf_k, ws=None, n_tokens=None,
                       num_slots=None, stream=None, raise_on_error=True) -> int:
    """Scatter new tokens' K8/V8 rows ([n, Hkv, D] bytes) into the 8-bit pools, and the block
    scales sf_k_new ([n, Hkv] fp32, or None) of the tokens that open a 64-slot block."""
    n = k8_new.shape[0] if n_tokens is None else n_tokens
    num_slots = k8_pool.shape[0] if num_slots is None else num_slots
    hkv = k8_pool.shape[1]
    st = lib().attn_kv_store_sage(_ptr(k8_new), _ptr(v8_new), _ptr(sf_k_new), _ptr(out_cache_loc), int(n), int(hkv),
                                  int(k8_pool.shape[2]), _ptr(k8_pool), _ptr(v8_pool), _ptr(sf_k), int(num_slots),
                                  _ptr(ws), _stream(stream))
    return _check(st, "attn_kv_store_sage", raise_on_error)


def pa_read_device_error(ws, stream=None) -> int:
    return lib().pa_read_device_error(_ptr(ws), _stream(stream))


def pa_noalloc_read_device_error(stream=None) -> int:
    """Read and clear the device error word of attn_decode_paged_noalloc's fixed array."""
    return lib().pa_noalloc_read_device_error(_stream(stream))


def pa_version() -> int:
    return lib().pa_version()
