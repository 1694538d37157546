"""fp64 reference for paged-KV attention in the DECODE and EXTEND modes (test infrastructure only).

What is computed, and where the pages say it:

* Two-level KV cache.  ``req_to_token`` maps (request, position) to a token
  slot and ``token_to_kv_pool`` maps a slot to that layer's K/V rows
  ("Implement Flash Attention Back End in SGLang - Basics and KV Cache",
  KV-cache passage; "Flash Attention Backend in SGLang: Grundlagen und KV Cache
  optimal nutzen", paragraph on the req_to_token and token_to_kv_pool levels).
  With a page size P > 1 the table holds page numbers and a logically
  contiguous sequence lives in fixed-size, non-contiguous blocks
  ("PagedAttention: 优化 KV Cache 的管理和利用率", section 2, 工作原理 items 1-3):
  slot(r, j) = page_table[r][j // P] * P + j % P.  With P = 1 the table is
  req_to_token itself.
* Attention itself is the standard definition softmax(scale * Q K^T) V
  ("FlashAttention: 优化计算过程中的临时显存占用", section 1 steps 1-2).  The
  tiled, online-softmax method reaches the same result without the N x N
  matrix in HBM (same page, section 2), so the oracle is the plain definition.
* DECODE has one query token per request and EXTEND adds new tokens that
  attend to the cached context (forward modes in "Implement Flash Attention
  Back End in SGLang", and in "Flash Attention Backend in SGLang: Grundlagen").

Readings where the pages are silent (each is listed in the design notes):
GQA query head h reads KV head h // (Hq // Hkv); EXTEND is causal aligned to
the bottom right (new query i at absolute position p + i sees keys
0 .. p + i); the new tokens' K/V are already in the pool; an empty sequence
gives O = 0 and lse = -inf.

All arithmetic is float64; inputs arrive as raw bit patterns and are decoded
exactly by ``oracle.codecs``.
"""
from __future__ import annotations

import numpy as np

from .codecs import bf16_bits_to_f64, e4m3_to_f64


def gather_slots(page_table: np.ndarray, seq_len: int, page_size: int, r: int) -> np.ndarray:
    """Token slots of request r, positions 0 .. seq_len-1 (int64).

    slot(r, j) = page_table[r][j // P] * P + j % P (see module docstring).
    """
    j = np.arange(int(seq_len), dtype=np.int64)
    pages = np.asarray(page_table[r], dtype=np.int64)[j // page_size]
    return pages * page_size + (j % page_size)


def gather_kv(pool_bits: np.ndarray, slots: np.ndarray, h_kv: int) -> np.ndarray:
    """Rows pool[slot][h_kv][:] for every slot, decoded from bfloat16 to float64: [len(slots), D]."""
    return bf16_bits_to_f64(pool_bits[slots, h_kv, :])


def softmax_attend(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float, visible=None):
    """O and natural-log LSE of softmax(scale * q k^T) v for a block of queries.

    q [M, D], k [N, D], v [N, D] in float64; ``visible`` is an optional boolean
    [M, N] mask (True = key may be attended).  Rows with no visible key return
    O = 0 and lse = -inf.
    """
    s = scale * (q @ k.T)                                   # [M, N]
    if visible is not None:
        s = np.where(visible, s, -np.inf)
    m = np.max(s, axis=1, initial=-np.inf)                  # row max
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    p = np.exp(s - m_safe[:, None])                         # exp(-inf) = 0 for masked keys
    p = np.where(np.isneginf(s), 0.0, p)
    l = p.sum(axis=1)
    with np.errstate(invalid="ignore", divide="ignore"):
        o = (p @ v) / l[:, None]
        lse = m_safe + np.log(l)
    o = np.where(empty[:, None], 0.0, o)
    lse = np.where(empty, -np.inf, lse)
    return o, lse


def decode(q_bits, k_pool_bits, v_pool_bits, page_table, seq_lens, page_size, sm_scale):
    """DECODE: one query token per request against its whole cached sequence.

    q_bits [B, Hq, D] uint16 (bf16), pools [num_slots, Hkv, D] uint16 (bf16),
    page_table [B, pitch] int, seq_lens [B] int.  Returns (O [B, Hq, D] float64,
    lse [B, Hq] float64, natural log).  No mask: every cached key 0 .. L-1 is
    visible, the decode token's own K/V being already in the pool.
    """
    B, Hq, D = q_bits.shape
    Hkv = k_pool_bits.shape[1]
    G = Hq // Hkv
    out = np.zeros((B, Hq, D))
    lse = np.full((B, Hq), -np.inf)
    q = bf16_bits_to_f64(q_bits)
    for r in range(B):
        L = int(seq_lens[r])
        if L == 0:
            continue
        slots = gather_slots(page_table, L, page_size, r)
        for hk in range(Hkv):
            k = gather_kv(k_pool_bits, slots, hk)
            v = gather_kv(v_pool_bits, slots, hk)
            heads = slice(hk * G, (hk + 1) * G)
            o, ls = softmax_attend(q[r, heads, :], k, v, sm_scale)
            out[r, heads, :] = o
            lse[r, heads] = ls
    return out, lse


def decode_fp8(q_bits, k8_pool, v8_pool, k_scale, v_scale, page_table, seq_lens, page_size, sm_scale):
    """DECODE over an FP8 KV cache: pools of E4M3 codes with one dequantisation scale each.

    The pages list FP8 among the FlashAttention backend's features ("Implement Flash
    Attention Back End in SGLang - Basics and KV Cache", feature list) without a formula;
    the reading taken: K = k_scale * E4M3(K8) and V = v_scale * E4M3(V8), decoded exactly
    (float64), then the standard definition as in ``decode``.  q_bits [B, Hq, D] uint16
    (bf16), k8_pool / v8_pool [num_slots, Hkv, D] uint8 codes.  Returns (O, lse).
    """
    B, Hq, D = q_bits.shape
    Hkv = k8_pool.shape[1]
    G = Hq // Hkv
    out = np.zeros((B, Hq, D))
    lse = np.full((B, Hq), -np.inf)
    q = bf16_bits_to_f64(q_bits)
    for r in range(B):
        L = int(seq_lens[r])
        if L == 0:
            continue
        slots = gather_slots(page_table, L, page_size, r)
        for hk in range(Hkv):
            k = float(k_scale) * e4m3_to_f64(k8_pool[slots, hk, :])
            v = float(v_scale) * e4m3_to_f64(v8_pool[slots, hk, :])
            heads = slice(hk * G, (hk + 1) * G)
            o, ls = softmax_attend(q[r, heads, :], k, v, sm_scale)
            out[r, heads, :] = o
            lse[r, heads] = ls
    return out, lse


def extend(q_bits, cu_seqlens_q, k_pool_bits, v_pool_bits, page_table, seq_lens, page_size, sm_scale):
    """EXTEND: new tokens of each request attend causally to the cached prefix and to themselves.

    q_bits [T, Hq, D] uint16 with request r's new tokens at rows
    cu_seqlens_q[r] .. cu_seqlens_q[r+1]-1; seq_lens[r] = p_r + n_r is the
    total length (prefix plus new tokens), whose K/V are all in the pool.
    New token i (0-based) sits at absolute position p_r + i and sees keys
    j <= p_r + i.  Returns (O [T, Hq, D], lse [T, Hq]).
    """
    T, Hq, D = q_bits.shape
    Hkv = k_pool_bits.shape[1]
    G = Hq // Hkv
    B = len(seq_lens)
    out = np.zeros((T, Hq, D))
    lse = np.full((T, Hq), -np.inf)
    q = bf16_bits_to_f64(q_bits)
    for r in range(B):
        q0, q1 = int(cu_seqlens_q[r]), int(cu_seqlens_q[r + 1])
        n = q1 - q0
        L = int(seq_lens[r])
        p = L - n
        if n == 0:
            continue
        slots = gather_slots(page_table, L, page_size, r)
        pos = p + np.arange(n)[:, None]                      # absolute position of each query
        visible = np.arange(L)[None, :] <= pos               # bottom-right aligned causal mask
        for hk in range(Hkv):
            k = gather_kv(k_pool_bits, slots, hk)
            v = gather_kv(v_pool_bits, slots, hk)
            for h in range(hk * G, (hk + 1) * G):
                o, ls = softmax_attend(q[q0:q1, h, :], k, v, sm_scale, visible)
                out[q0:q1, h, :] = o
                lse[q0:q1, h] = ls
    return out, lse


def merge_partials(o_parts: np.ndarray, lse_parts: np.ndarray):
    """Combine attention results over disjoint key subsets into the result over their union.

    o_parts [S, ..., D] are the per-subset normalised outputs and lse_parts
    [S, ...] their natural-log LSEs.  lse = log sum_s exp(lse_s) and
    O = sum_s exp(lse_s - lse) O_s.  Subsets with lse = -inf (no keys)
    contribute nothing; if all are empty the result is O = 0, lse = -inf.
    """
    m = np.max(lse_parts, axis=0)
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    w = np.exp(lse_parts - m_safe)                           # exp(-inf) = 0
    tot = w.sum(axis=0)
    with np.errstate(invalid="ignore", divide="ignore"):
        o = (w[..., None] * o_parts).sum(axis=0) / tot[..., None]
        lse = m_safe + np.log(tot)
    o = np.where(empty[..., None], 0.0, o)
    lse = np.where(empty, -np.inf, lse)
    return o, lse


def materialised_reference(q, k, v, scale, causal_offset=None):
    """Standard attention written out with plain Python loops, for tiny inputs.

    Builds the full score matrix P = Q K^T element by element, applies the
    row softmax and multiplies by V, following the three steps of standard
    attention in "FlashAttention: 优化计算过程中的临时显存占用", section 1.
    q [M][D], k [N][D], v [N][D] are nested sequences of floats.  If
    ``causal_offset`` is an int p, query i sees keys j <= p + i.
    Returns (O as a list of lists, lse as a list).
    """
    import math
    M, N, D = len(q), len(k), len(q[0])
    S = [[0.0] * N for _ in range(M)]
    for i in range(M):
        for j in range(N):
            acc = 0.0
            for d in range(D):
                acc += q[i][d] * k[j][d]
            S[i][j] = scale * acc
    O, LSE = [], []
    for i in range(M):
        vis = [j for j in range(N) if causal_offset is None or j <= causal_offset + i]
        if not vis:
            O.append([0.0] * D)
            LSE.append(-math.inf)
            continue
        mx = max(S[i][j] for j in vis)
        e = {j: math.exp(S[i][j] - mx) for j in vis}
        tot = sum(e.values())
        O.append([sum(e[j] * v[j][d] for j in vis) / tot for d in range(D)])
        LSE.append(mx + math.log(tot))
    return O, LSE


def materialised_score_bytes(seq_len: int, elem_bytes: int, batch: int = 1, heads: int = 1) -> int:
    """Bytes of the N x N score matrix standard attention keeps in HBM.

    "FlashAttention: 优化计算过程中的临时显存占用", section 2, worked example:
    N = 8192 in FP16 needs 8192 * 8192 * 2 bytes (about 128 MB) per head and
    sample, and 32 GB at batch 8 with 32 heads.
    """
    return seq_len * seq_len * elem_bytes * batch * heads


def kv_store(k_pool_bits, v_pool_bits, out_cache_loc, k_new_bits, v_new_bits):
    """The cache update before attention: pool[loc[t]] = new[t] for every new token t.

    "Flash Attention Backend in SGLang: Grundlagen und KV Cache optimal nutzen": the KV
    cache is updated within the forward methods; each new token's slot (out_cache_loc)
    comes from the caller.  Returns updated copies of the pools; a slot outside the pool
    is skipped.  Raw bit patterns are copied unchanged.
    """
    k = np.array(k_pool_bits, copy=True)
    v = np.array(v_pool_bits, copy=True)
    for t, slot in enumerate(np.asarray(out_cache_loc, dtype=np.int64)):
        if 0 <= slot < k.shape[0]:
            k[slot] = k_new_bits[t]
            v[slot] = v_new_bits[t]
    return k, v
