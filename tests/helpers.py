"""Test-side helpers: run the library on workload inputs, read its plan back, compare with the oracle.

The tolerance reading for bf16 outputs: the kernels' output format is bf16,
whose own rounding (up to half a bf16 ulp of the true value) is not charged
to the kernel; on top of that the error may be at most 1e-2 (maximum) and
1e-3 (mean absolute error over all outputs).
"""
from __future__ import annotations

import numpy as np
import torch

from oracle.codecs import bf16_bits_to_f64, bf16_half_ulp

MAX_ABS = 1e-2
MEAN_ABS = 1e-3
LSE_ABS = 4e-3
SAGE_REL = 3e-2


def bits16(t: torch.Tensor) -> np.ndarray:
    """Raw 16-bit patterns of a bf16 tensor as a NumPy uint16 array (host copy)."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_errors(gpu_bf16: torch.Tensor, ref: np.ndarray):
    """(max of err - half ulp, mean err, raw max err) of a bf16 result against an fp64 reference."""
    got = bf16_bits_to_f64(bits16(gpu_bf16)).reshape(ref.shape)
    err = np.abs(got - ref)
    excess = err - bf16_half_ulp(ref)
    return float(np.max(excess, initial=0.0)), float(np.mean(err)) if err.size else 0.0, float(np.max(err, initial=0.0))


def assert_bf16_close(gpu_bf16, ref, what=""):
    assert np.all(np.isfinite(bf16_bits_to_f64(bits16(gpu_bf16)))), f"{what}: non-finite output"
    mx, mean, raw = bf16_errors(gpu_bf16, ref)
    assert mx <= MAX_ABS, f"{what}: max |err| beyond bf16 rounding {mx:.3e} (raw {raw:.3e})"
    assert mean <= MEAN_ABS, f"{what}: mean |err| {mean:.3e}"
    return mx, mean, raw


def sage_row_rel_error(gpu_bf16, ref):
    """max over rows (last axis = d) of ||O_gpu - O_ref||_inf / max(||O_ref||_inf, 1e-6)."""
    got = bf16_bits_to_f64(bits16(gpu_bf16)).reshape(ref.shape)
    num = np.max(np.abs(got - ref), axis=-1)
    den = np.maximum(np.max(np.abs(ref), axis=-1), 1e-6)
    return float(np.max(num / den))


def ws_offsets(mode: int, batch: int, hq: int, max_items: int, head_dim: int = 128, hkv: int = 8,
               max_kv_len: int = 0, slots: int = 0):
    """Byte offsets of the workspace arrays, from the layout documented at attn_plan."""
    off = 64
    o = {}
    for name, n in (("req_splits", batch), ("req_base", batch + 1), ("req_len", batch),
                    ("req_aux", batch), ("req_prefix", batch)):
        o[name] = off
        off += 4 * n
    off = (off + 15) // 16 * 16
    o["items"] = off
    off += 16 * max_items
    off = (off + 255) // 256 * 256
    if mode in (0, 2, 3):
        o["slot_first"] = off
        off += 4 * (slots + 1)
        off = (off + 255) // 256 * 256
    if mode == 3:
        mb = (max_kv_len + 63) // 64
        o["sel_base"] = off
        off += 4 * (batch + 1)
        off = (off + 255) // 256 * 256
        o["sel_block"] = off
        off += 4 * batch * mb
        off = (off + 255) // 256 * 256
    if mode in (0, 2, 3):
        o["partial_o"] = off
        off += 4 * max_items * hq * head_dim
        off = (off + 255) // 256 * 256
        o["partial_lse"] = off
        off += 4 * max_items * hq
        off = (off + 255) // 256 * 256
    if mode in (2, 3):
        o["item_max"] = off
        off += 4 * max_items * hq
        off = (off + 255) // 256 * 256
        o["score_pitch"] = (max(max_kv_len, 64) + 63) // 64 * 64
        o["scores"] = off
        off += 4 * batch * hq * o["score_pitch"]
        off = (off + 255) // 256 * 256
    o["total"] = off
    return o


def read_plan(ws: torch.Tensor, mode: int, batch: int, hq: int, max_kv_len: int = 0):
    """Parse the plan the GPU wrote into the workspace (host copy)."""
    raw = ws.cpu().numpy().view(np.uint8)
    hdr = raw[:64].view(np.int32)
    num_items, max_items, hkv, slots = int(hdr[7]), int(hdr[8]), int(hdr[4]), int(hdr[14])
    o = ws_offsets(mode, batch, hq, max_items, hkv=hkv, slots=slots, max_kv_len=max_kv_len)

    def arr(name, n):
        return raw[o[name]:o[name] + 4 * n].view(np.int32).tolist()

    items = raw[o["items"]:o["items"] + 16 * num_items].view(np.int32).reshape(-1, 4)
    return {"magic": int(hdr[0]), "mode": int(hdr[1]), "tile": int(hdr[9]), "chunk_tiles": int(hdr[10]),
            "error_word": int(hdr[11]), "num_items": num_items, "max_items": max_items,
            "req_splits": arr("req_splits", batch), "req_base": arr("req_base", batch + 1),
            "req_len": arr("req_len", batch), "slots": slots, "num_sms": int(hdr[12]),
            "slot_first": arr("slot_first", slots + 1) if mode in (0, 2, 3) else None,
            "sel_base": arr("sel_base", batch + 1) if mode == 3 else None,
            "items": [tuple(int(x) for x in it) for it in items]}


def alloc_ws(params, device="cuda"):
    from paged_kv_flashattention_split_b200 import pa_plan_workspace_size
    n = pa_plan_workspace_size(params)
    return torch.zeros(n, dtype=torch.uint8, device=device)
