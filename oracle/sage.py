"""8-bit Sage decode, following the pages' formula step by step (test infrastructure only).

Source: "FlashInfer PrimTS, Sage Attention 도입으로 8비트 양자화 및 성능 최적화
달성", section "코드 분석" item 1 (README "Sage attention"):

    S[r][c] = sfQ[blkQ(r)] * sfK[blkK(c)] * (Q8 . K8^T)[r][c]
    P       = softmax_row(S), quantized to E4M3 as 448 * p
    O[r][d] = sfV[d] * (sum_c P8[r][c] * V8[c][d]) / (448 * l[r])  (+ v_mean[d])

and item 4 of the same section: the Q and K scales enter before the row max
and the exponential, P is E4M3 with the static factor 448, and the V scales
are applied per channel in the epilogue.  The caller supplies the 8-bit
tensors and all scales, which must be finite and positive and are not checked
(same item 1).

Layout (one decode token per request, DECODE mode):
  q8      int8  [B, Hq, D]           sf_q  float32 [B, Hq]       (blkQ = one row)
  k8 pool int8  [num_slots, Hkv, D]  sf_k  float32 [num_slots // k_block, Hkv]
  v8 pool uint8 [num_slots, Hkv, D]  (E4M3 codes)
  sf_v, v_mean float32 [Hkv, D]      (v_mean optional)

Readings where the formula leaves a step open (listed in the design notes):
* blkK(c) is the physical 64-key block of key c's slot, slot // k_block, so a
  scale travels with its page.
* softmax_row takes the maximum m over the request's whole row of keys; the
  top key therefore quantises to exactly 448.
* l[r] = sum_c exp(S[r][c] - m) of the unquantised probabilities.
* E4M3 rounding is round-to-nearest-even with saturation.
* The quantisation code is an integer decided by floating point, so it is
  decided in the kernel's precision: S is formed in float32 as
  fp32(fp32(sfQ * sfK) * fp32(dot)) (the integer dot is exact: |dot| <=
  127 * 127 * 128 < 2**24), and m is the float32 row maximum.  Everything
  after that (exp, 448 * p, the sums, the epilogue) is float64.
* There is no extra 1/sqrt(d) factor: the formula has none, so a caller folds
  any softmax scale into sfQ.
* An empty row (L = 0) gives O = v_mean (zero if absent).
"""
from __future__ import annotations

import numpy as np

from .attention import gather_slots
from .codecs import e4m3_to_f64, f64_to_e4m3


def sage_scores_f32(q8_row: np.ndarray, k8_rows: np.ndarray, sf_q: float, sf_k_rows: np.ndarray) -> np.ndarray:
    """S for one query row over keys: float32 (sfQ * sfK) * float32(exact int dot).

    q8_row [D] int8, k8_rows [N, D] int8, sf_k_rows [N] float32 (the scale of
    each key's block).  Returns float32 [N].
    """
    dot = k8_rows.astype(np.int64) @ q8_row.astype(np.int64)          # exact integers
    scale = np.float32(sf_q) * sf_k_rows.astype(np.float32)           # fp32 product, rounded
    return (scale * dot.astype(np.float32)).astype(np.float32)        # fp32 product, rounded


def sage_scores_f64(q8_row: np.ndarray, k8_rows: np.ndarray, sf_q: float, sf_k_rows: np.ndarray) -> np.ndarray:
    """S for one query row over keys with every step in float64: sfQ * sfK * (exact int dot).

    The literal formula without the float32 reading; used to show that the precision in
    which S is formed does not move the result beyond rounding.  Returns float64 [N].
    """
    dot = k8_rows.astype(np.int64) @ q8_row.astype(np.int64)
    return np.float64(sf_q) * sf_k_rows.astype(np.float64) * dot.astype(np.float64)


def sage_row(q8_row, k8_rows, v8_rows, sf_q, sf_k_rows, sf_v, v_mean, quantize_p: bool = True,
             score_f64: bool = False):
    """The Sage formula for one query row; returns O [D] float64.

    v8_rows [N, D] uint8 E4M3 codes, sf_v and v_mean [D].  ``quantize_p=False``
    replaces the E4M3 step on 448 * p by the identity (a switch used to tie
    this function to plain softmax attention in the tests).  ``score_f64=True``
    forms S and its row max in float64 instead of the kernel's float32 (the
    reading above), to measure what that reading moves.
    """
    D = v8_rows.shape[1] if v8_rows.ndim == 2 else len(sf_v)
    vm = np.zeros(D) if v_mean is None else np.asarray(v_mean, dtype=np.float64)
    if k8_rows.shape[0] == 0:
        return vm.copy()
    if score_f64:
        S = sage_scores_f64(q8_row, k8_rows, sf_q, sf_k_rows)         # step 1: scores (fp64)
        m = S.max()                                                   # step 2: row max (fp64)
    else:
        S = sage_scores_f32(q8_row, k8_rows, sf_q, sf_k_rows)         # step 1: scores
        m = np.float32(S.max())                                       # step 2: row max (fp32)
    p = np.exp(S.astype(np.float64) - np.float64(m))                  # step 3: exp(S - m) in (0, 1]
    l = p.sum()                                                       # unquantised row sum
    if quantize_p:
        P = e4m3_to_f64(f64_to_e4m3(448.0 * p))                       # step 4: E4M3(448 p)
    else:
        P = 448.0 * p
    V = e4m3_to_f64(v8_rows)                                          # exact decode of V8
    acc = P @ V                                                       # step 5: sum_c P8 V8
    return np.asarray(sf_v, dtype=np.float64) * acc / (448.0 * l) + vm   # step 6: epilogue


def selected_positions(seq_len: int, mask_row, k_block: int = 64) -> np.ndarray:
    """Key positions 0 .. L-1 of a request whose 64-key block j // k_block is selected.

    Block-sparse mode ("FlashInfer PrimTS, Sage Attention ...", README: the decode kernel
    runs in the dense and block-sparse modes): the reading taken is one mask per
    (request, logical key block), shared by every head; mask_row[b] != 0 selects block b.
    """
    j = np.arange(int(seq_len), dtype=np.int64)
    if mask_row is None:
        return j
    m = np.asarray(mask_row)
    return j[m[j // k_block] != 0]


def sage_decode(q8, sf_q, k8_pool, v8_pool, sf_k, sf_v, v_mean, page_table, seq_lens,
                page_size: int, k_block: int = 64, quantize_p: bool = True, block_mask=None,
                score_f64: bool = False) -> np.ndarray:
    """Sage DECODE over the paged cache; returns O [B, Hq, D] float64.

    Keys are gathered through the page table exactly as in the bf16 path
    (``oracle.attention.gather_slots``); key c's K scale is
    sf_k[slot(c) // k_block][h_kv]; query head h reads KV head h // (Hq // Hkv).
    With ``block_mask`` [B][n_blocks] (block-sparse mode), row r attends only to the keys
    of its selected blocks (``selected_positions``): the Sage formula, row max and row
    sum included, over that subset; a row with no selected key gives v_mean.
    ``score_f64`` as for ``sage_row``.
    """
    B, Hq, D = q8.shape
    Hkv = k8_pool.shape[1]
    G = Hq // Hkv
    out = np.zeros((B, Hq, D))
    for r in range(B):
        L = int(seq_lens[r])
        slots = gather_slots(page_table, L, page_size, r)
        if block_mask is not None:
            slots = slots[selected_positions(L, block_mask[r], k_block)]
        blocks = slots // k_block
        for hk in range(Hkv):
            k8 = k8_pool[slots, hk, :]
            v8 = v8_pool[slots, hk, :]
            sfk = sf_k[blocks, hk]
            vm = None if v_mean is None else v_mean[hk]
            for h in range(hk * G, (hk + 1) * G):
                out[r, h] = sage_row(q8[r, h], k8, v8, sf_q[r, h], sfk, sf_v[hk], vm, quantize_p, score_f64)
    return out


def kv_store_sage(k8_pool, v8_pool, sf_k, out_cache_loc, k8_new, v8_new, sf_k_new=None, k_block: int = 64):
    """The 8-bit cache update before a Sage attention call; returns updated copies.

    Each new token t is written to its slot s = out_cache_loc[t] (as in
    ``oracle.attention.kv_store``: the cache is updated within the forward methods,
    "Flash Attention Backend in SGLang: Grundlagen und KV Cache optimal nutzen"):
    k8_pool[s] = k8_new[t], v8_pool[s] = v8_new[t].  The K scales are per 64-key block
    of slots ("FlashInfer PrimTS, Sage Attention ..." README formula, sfK[blkK]); a block's
    scale is written by the token whose slot opens the block (s % k_block == 0):
    sf_k[s // k_block] = sf_k_new[t].  Later tokens of a block are quantised by the caller
    with the scale already there, so their scale rows are not written.  A slot outside the
    pool is skipped.  Raw bytes are copied unchanged.
    """
    k = np.array(k8_pool, copy=True)
    v = np.array(v8_pool, copy=True)
    sf = np.array(sf_k, copy=True)
    for t, slot in enumerate(np.asarray(out_cache_loc, dtype=np.int64)):
        if 0 <= slot < k.shape[0]:
            k[slot] = k8_new[t]
            v[slot] = v8_new[t]
            if sf_k_new is not None and slot % k_block == 0:
                sf[slot // k_block] = sf_k_new[t]
    return k, v, sf


def sage_extend(q8, sf_q, cu_seqlens_q, k8_pool, v8_pool, sf_k, sf_v, v_mean, page_table, seq_lens,
                page_size: int, k_block: int = 64, heads=None) -> np.ndarray:
    """Sage EXTEND (prefill over a cached prefix); returns O [T, Hq, D] float64.

    The Sage formula of ``sage_row`` for every new token: row i of request r (Q8 row
    cu_seqlens_q[r] + i, scale sf_q[row][h], blkQ = one row) sits at absolute position
    p_r + i, p_r = L_r - n_r, and sees keys 0 .. p_r + i (the bottom-right causal reading
    of ``oracle.attention.extend``); its row max and row sum run over those keys.  This
    is the variant the pages measure at S = 10800 ("FlashInfer PrimTS, Sage Attention ...",
    performance item 2); the kernel for it runs on the prefill path.

    The rows of one request and head are taken together as an [n, L] block with a
    visibility mask, each element through the same steps as ``sage_row`` (exact integer
    dot, float32 S and row max, float64 exp, E4M3(448 p), the unquantised row sum, the
    epilogue); only the order in which the float64 sums add their terms differs.  The
    integer dots run as float64 products, which are exact (every partial sum is an
    integer below 2**22).  ``heads`` restricts the query heads computed (the others are 0).
    """
    T, Hq, D = q8.shape
    Hkv = k8_pool.shape[1]
    G = Hq // Hkv
    out = np.zeros((T, Hq, D))
    heads = range(Hq) if heads is None else heads
    for r in range(len(seq_lens)):
        q0, q1 = int(cu_seqlens_q[r]), int(cu_seqlens_q[r + 1])
        n = q1 - q0
        if n == 0:
            continue
        L = int(seq_lens[r])
        p = L - n
        slots = gather_slots(page_table, L, page_size, r)
        blocks = slots // k_block
        visible = np.arange(L)[None, :] <= (p + np.arange(n))[:, None]      # [n, L]
        for h in heads:
            hk = h // G
            k8 = k8_pool[slots, hk, :].astype(np.float64)                    # [L, D]
            V = e4m3_to_f64(v8_pool[slots, hk, :])                           # [L, D]
            dot = q8[q0:q1, h, :].astype(np.float64) @ k8.T                  # exact integers [n, L]
            scale = sf_q[q0:q1, h].astype(np.float32)[:, None] * sf_k[blocks, hk].astype(np.float32)[None, :]
            S = (scale * dot.astype(np.float32)).astype(np.float32)          # step 1 (fp32 products)
            S = np.where(visible, S, np.float32(-np.inf))
            m = S.max(axis=1)                                                # step 2: fp32 row max
            pr = np.where(visible, np.exp(S.astype(np.float64) - m.astype(np.float64)[:, None]), 0.0)
            l = pr.sum(axis=1)                                               # step 3: unquantised l
            P = e4m3_to_f64(f64_to_e4m3(448.0 * pr))                         # step 4: E4M3(448 p)
            acc = P @ V                                                      # step 5
            vm = np.zeros(D) if v_mean is None else np.asarray(v_mean[hk], dtype=np.float64)
            out[q0:q1, h] = np.asarray(sf_v[hk], dtype=np.float64) * acc / (448.0 * l[:, None]) + vm   # step 6
    return out
