"""The per-batch scheduling plan, restated with plain integers (test infrastructure only).

The pages say the tile-scheduling metadata depends only on the sequence
lengths (and, for a prefill, the cumulative query lengths), so it is computed
once per batch and reused by every layer instead of being recomputed per
layer ("SGLang의 FA3 디코드 최적화: get_scheduler_metadata 도입", section
"코드 분석" items 1-3, and "왜 이게 좋은가" item 1; "Flash Attention Backend in
SGLang: Grundlagen", the FlashAttentionMetadata paragraph).  They give no
algorithm, so the algorithm below is this library's own; the CUDA plan kernel
must reproduce it bit for bit.

DECODE (split-KV work list: a flat, balanced partition over CTA slots)
  T        = max(64, page_size)                  keys per unit (a tile)
  HG       = the largest of 8, 4, 2, 1 dividing Hkv   (KV heads one work item covers)
  groups   = Hkv / HG
  C        = max(1, floor(num_sms * 2 / groups)) CTA slots
  units_r  = ceil(L_r / T)
  the flat partition below (SAGE_DECODE) with unit T: slot c takes the global
  units [c per, (c+1) per), per = max(1, ceil(sum_r units_r / C)); each piece of a
  request inside one slot is an item (r, s, T u0, min(T u1, L_r)); an empty request
  is one item (r, 0, 0, 0); items r-major then s (slot order); slot_first; req_base.
  Every slot streams at most per tiles, so the slots finish together, and a request
  is split only where a slot boundary falls inside it (no split cap is needed).
  Bound: num_items <= C + B.

EXTEND (query-tile work list)
  n_r = cu[r+1] - cu[r], p_r = L_r - n_r, query tiles of 128 rows:
  tile t covers new tokens [128 t, min(128 (t+1), n_r)) and needs the key
  tiles 0 .. ceil((p_r + q_end) / 128) - 1; items (r, t, q_begin, q_end) are
  sorted by that key-tile count descending, ties by generation order.
  Bound: num_items <= ceil(max_q_tokens / 128) + B.

SAGE_DECODE (flat, balanced partition over CTA slots)
  U        = 32 keys per unit; units_r = ceil(L_r / U)
  HG, groups, C as for DECODE (a CTA covers HG KV heads of one slot; one wave of
                                                   two CTAs per SM)
  g_r      = sum_{r' < r} units_r'                 request r's first unit in
                                                   the concatenated sequence
  total    = sum_r units_r, per = max(1, ceil(total / C)) units per slot,
  used     = ceil(total / per)                     slots that get units
  slot c takes the global units [c per, (c+1) per); each maximal piece of that
  range inside one request is an item (r, s, U u0, min(U u1, L_r)) with u0, u1
  the piece's unit bounds relative to g_r and s its index among request r's
  pieces.  An empty request is one item (r, 0, 0, 0) in slot
  min(floor(g_r / per), max(used - 1, 0)).  Items are listed r-major then s,
  which is also slot order, so no sort is needed; slot_first[c] (c = 0 .. C)
  is the first item of slot c or later (num_items if none), and slot c runs
  items slot_first[c] .. slot_first[c+1] - 1.  req_base as for DECODE; every
  slot has at most per units, so the slots finish together.
  Bound: num_items <= C + B.

SAGE_SPARSE (the same partition over the selected blocks' units)
  A mask[r][b] (b < ceil(L_r / 64)) selects request r's 64-key blocks; sel_r is the
  ascending list of selected blocks, sel_base its exclusive prefix sum over requests
  (sel_block concatenates the lists).  A selected block holds 2 units, except a last
  block of L_r - 64 b <= 32 keys, which holds 1; U_r = the units of sel_r, in order.
  The SAGE_DECODE partition runs over the U_r, with items (r, s, u0, u1) in unit
  indices of request r (unit u is key positions 64 sel_r[u // 2] + 32 (u % 2) onward,
  up to 32 keys and not past L_r).  A request with no selected unit is one item
  (r, 0, 0, 0).  Bound: num_items <= C + B.
"""
from __future__ import annotations

MODE_DECODE, MODE_EXTEND, MODE_SAGE_DECODE, MODE_SAGE_SPARSE = 0, 1, 2, 3
DECODE_MIN_TILE = 64
SAGE_UNIT = 32
CTAS_PER_SM = 2
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


def flat_slots(hkv: int, num_sms: int) -> int:
    """CTA slots of a flat partition (DECODE, SAGE_DECODE, SAGE_SPARSE): max(1, floor(num_sms * 2 / groups))."""
    return max(1, num_sms * CTAS_PER_SM // decode_head_groups(hkv))


def max_items(mode: int, batch: int, hkv: int, num_sms: int, max_q_tokens: int = 0) -> int:
    """The host-side bound on the number of work items for a plan of this shape."""
    if mode in (MODE_DECODE, MODE_SAGE_DECODE, MODE_SAGE_SPARSE):
        return flat_slots(hkv, num_sms) + batch
    if mode == MODE_EXTEND:
        return _cdiv(max_q_tokens, EXTEND_Q_TILE) + batch
    raise ValueError("unknown mode")


def plan(mode: int, seq_lens, cu_seqlens_q=None, *, hkv: int, page_size: int, num_sms: int,
         max_q_tokens: int = 0, block_mask=None):
    """Return the plan as a dict of plain Python ints and lists.

    Keys: ``tile``, ``chunk_tiles`` (DECODE: tiles per slot; SAGE_DECODE: units per
    slot; 0 otherwise), ``req_splits``, ``req_base`` (length B + 1), ``items`` (list
    of 4-tuples, in execution order), ``num_items`` and, for DECODE, SAGE_DECODE and
    SAGE_SPARSE, ``slot_first`` (length C + 1); for SAGE_SPARSE also ``sel_base``
    (length B + 1) and ``sel_block``.
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
        return _flat_plan(L, decode_tile(page_size), flat_slots(hkv, num_sms))
    if mode == MODE_SAGE_DECODE:
        return _flat_plan(L, SAGE_UNIT, flat_slots(hkv, num_sms))
    if mode == MODE_SAGE_SPARSE:
        return _flat_plan(L, SAGE_UNIT, flat_slots(hkv, num_sms), block_mask)
    if mode == MODE_EXTEND:
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
    else:
        raise ValueError("unknown mode")
    order = sorted(range(len(gen)), key=lambda i: (-gen[i][0], i))
    items = [gen[i][1] for i in order]
    base = [0] * (B + 1)
    for r in range(B):
        base[r + 1] = base[r] + splits[r]
    return {"tile": tile, "chunk_tiles": chunk, "req_splits": splits, "req_base": base,
            "items": items, "num_items": len(items)}


def _flat_plan(L, U: int, C: int, block_mask=None):
    """The flat partition of DECODE / SAGE_DECODE / SAGE_SPARSE (module docstring) over
    C slots, with units of U keys, unit by unit."""
    B = len(L)
    sel = None
    if block_mask is None:
        units = [_cdiv(x, U) for x in L]
    else:
        sel, units = [], []
        for r in range(B):
            nb = _cdiv(L[r], 2 * SAGE_UNIT)
            blocks = [b for b in range(nb) if block_mask[r][b]]
            sel.append(blocks)
            units.append(sum(1 if L[r] - 2 * SAGE_UNIT * b <= SAGE_UNIT else 2 for b in blocks))
    total = sum(units)
    per = max(1, _cdiv(total, C))
    used = _cdiv(total, per)
    items, item_slot, splits = [], [], [0] * B
    g = 0
    for r in range(B):
        if units[r] == 0:
            splits[r] = 1
            items.append((r, 0, 0, 0))
            item_slot.append(min(g // per, max(used - 1, 0)))
            continue
        c_first, c_last = g // per, (g + units[r] - 1) // per
        splits[r] = c_last - c_first + 1
        for s, c in enumerate(range(c_first, c_last + 1)):
            u0 = max(g, c * per) - g
            u1 = min(g + units[r], (c + 1) * per) - g
            if sel is None:
                items.append((r, s, U * u0, min(U * u1, L[r])))
            else:
                items.append((r, s, u0, u1))
            item_slot.append(c)
        g += units[r]
    slot_first = []
    for c in range(C + 1):
        later = [i for i, sc in enumerate(item_slot) if sc >= c]
        slot_first.append(later[0] if later else len(items))
    base = [0] * (B + 1)
    for r in range(B):
        base[r + 1] = base[r] + splits[r]
    out = {"tile": U, "chunk_tiles": per, "req_splits": splits, "req_base": base,
           "items": items, "num_items": len(items), "slot_first": slot_first}
    if sel is not None:
        sb = [0] * (B + 1)
        for r in range(B):
            sb[r + 1] = sb[r] + len(sel[r])
        out["sel_base"] = sb
        out["sel_block"] = [b for blocks in sel for b in blocks]
    return out
