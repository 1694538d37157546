"""The per-batch scheduling plan, restated with plain integers (test infrastructure only).

The pages say the tile-scheduling metadata depends only on the sequence
lengths (and, for a prefill, the cumulative query lengths), so it is computed
once per batch and reused by every layer instead of being recomputed per
layer ("SGLang의 FA3 디코드 최적화: get_scheduler_metadata 도입", section
"코드 분석" items 1-3, and "왜 이게 좋은가" item 1; "Flash Attention Backend in
SGLang: Grundlagen", the FlashAttentionMetadata paragraph).  They give no
algorithm, so the algorithm below is this library's own; the CUDA plan kernel
must reproduce it bit for bit.

DECODE (split-KV work list)
  T        = max(64, page_size)                  keys per tile
  HG       = the largest of 8, 4, 2, 1 dividing Hkv   (KV heads one CTA covers)
  groups   = Hkv / HG                            CTAs per work item
  tiles_r  = ceil(L_r / T)
  total    = sum_r tiles_r * groups              units of work
  slots    = num_sms * 4                         CTAs one decode launch aims for
  chunk    = max(1, ceil(total / slots))         tiles per split
  L_r == 0 : one split, the empty range [0, 0)
  else     : splits_r = ceil(tiles_r / chunk), chunk_r = chunk;
             if splits_r > max_splits: chunk_r = ceil(tiles_r / max_splits),
                                       splits_r = ceil(tiles_r / chunk_r)
             split s covers keys [s*chunk_r*T, min((s+1)*chunk_r*T, L_r))
  items (r, s, kv_begin, kv_end), generated r-major then s, are sorted by
  key length descending, ties by generation order (longest first, so that the
  hardware's in-order block dispatch is a longest-processing-time schedule).
  req_base = exclusive prefix sum of splits_r (the merge's index of split 0).
  Bound used to size the grid and the workspace:
  num_items <= ceil(slots / groups) + B.

EXTEND (query-tile work list)
  n_r = cu[r+1] - cu[r], p_r = L_r - n_r, query tiles of 128 rows:
  tile t covers new tokens [128 t, min(128 (t+1), n_r)) and needs the key
  tiles 0 .. ceil((p_r + q_end) / 128) - 1; items (r, t, q_begin, q_end) are
  sorted by that key-tile count descending, ties by generation order.
  Bound: num_items <= ceil(max_q_tokens / 128) + B.

SAGE_DECODE (one item per request)
  items (r, 0, 0, L_r) sorted by L_r descending, ties by r.  num_items = B.
"""
from __future__ import annotations

MODE_DECODE, MODE_EXTEND, MODE_SAGE_DECODE = 0, 1, 2
DECODE_MIN_TILE = 64
DECODE_CTAS_PER_SM = 4
EXTEND_Q_TILE = 128
EXTEND_KV_TILE = 128


def _cdiv(a: int, b: int) -> int:
    return -(-a // b)


def decode_tile(page_size: int) -> int:
    return max(DECODE_MIN_TILE, page_size)


def decode_head_groups(hkv: int) -> int:
    """Number of CTAs per decode work item: Hkv / (largest of 8, 4, 2, 1 dividing Hkv)."""
    for hg in (8, 4, 2, 1):
        if hkv % hg == 0:
            return hkv // hg
    raise ValueError("hkv must be positive")


def max_items(mode: int, batch: int, hkv: int, num_sms: int, max_q_tokens: int = 0) -> int:
    """The host-side bound on the number of work items for a plan of this shape."""
    if mode == MODE_DECODE:
        return _cdiv(num_sms * DECODE_CTAS_PER_SM, decode_head_groups(hkv)) + batch
    if mode == MODE_EXTEND:
        return _cdiv(max_q_tokens, EXTEND_Q_TILE) + batch
    return batch


def plan(mode: int, seq_lens, cu_seqlens_q=None, *, hkv: int, page_size: int, num_sms: int,
         max_splits: int = 1 << 30, max_q_tokens: int = 0):
    """Return the plan as a dict of plain Python ints and lists.

    Keys: ``tile``, ``chunk_tiles`` (DECODE; 0 otherwise), ``req_splits``,
    ``req_base`` (length B + 1), ``items`` (list of 4-tuples, in execution
    order) and ``num_items``.
    """
    L = [int(x) for x in seq_lens]
    B = len(L)
    if any(x < 0 for x in L):
        raise ValueError("negative sequence length")
    gen = []                                  # (sort_key, generation index, item)
    splits = [0] * B
    chunk = 0
    tile = 0
    if mode == MODE_DECODE:
        tile = decode_tile(page_size)
        tiles = [_cdiv(x, tile) for x in L]
        total = sum(tiles) * decode_head_groups(hkv)
        slots = num_sms * DECODE_CTAS_PER_SM
        chunk = max(1, _cdiv(total, slots))
        for r in range(B):
            if tiles[r] == 0:
                splits[r] = 1
                gen.append((0, (r, 0, 0, 0)))
                continue
            chunk_r = chunk
            s_r = _cdiv(tiles[r], chunk_r)
            if s_r > max_splits:
                chunk_r = _cdiv(tiles[r], max_splits)
                s_r = _cdiv(tiles[r], chunk_r)
            splits[r] = s_r
            for s in range(s_r):
                a = s * chunk_r * tile
                b = min((s + 1) * chunk_r * tile, L[r])
                gen.append((b - a, (r, s, a, b)))
    elif mode == MODE_EXTEND:
        tile = EXTEND_KV_TILE
        cu = [int(x) for x in cu_seqlens_q]
        for r in range(B):
            n = cu[r + 1] - cu[r]
            p = L[r] - n
            if n < 0 or p < 0:
                raise ValueError("cu_seqlens_q inconsistent with seq_lens")
            qt = _cdiv(n, EXTEND_Q_TILE)
            splits[r] = qt
            for t in range(qt):
                q0 = t * EXTEND_Q_TILE
                q1 = min(q0 + EXTEND_Q_TILE, n)
                gen.append((_cdiv(p + q1, EXTEND_KV_TILE), (r, t, q0, q1)))
    elif mode == MODE_SAGE_DECODE:
        tile = 64
        for r in range(B):
            splits[r] = 1
            gen.append((L[r], (r, 0, 0, L[r])))
    else:
        raise ValueError("unknown mode")
    order = sorted(range(len(gen)), key=lambda i: (-gen[i][0], i))
    items = [gen[i][1] for i in order]
    base = [0] * (B + 1)
    for r in range(B):
        base[r + 1] = base[r] + splits[r]
    return {"tile": tile, "chunk_tiles": chunk, "req_splits": splits, "req_base": base,
            "items": items, "num_items": len(items)}
