"""Seeded synthetic inputs for the paged-KV attention workloads.

This module only draws random numbers and lays them out; it holds none of
the attention arithmetic.  Both the CUDA library's callers (tests, bench) and
the CPU oracle's callers take their inputs from here, so the two sides always
see the same bits.

Recipe (all draws from ``torch.Generator``; integers uniform and inclusive):

* batch structure (lengths, slot/page permutation) from seed ``1000 + cfg``;
  layer ``l``'s tensors (Q, K and V pools) from seed ``1000 + 100 cfg + l``;
* Q, K, V ~ N(0, 1) drawn in float32 and rounded to bfloat16 (nearest-even);
* page_size 1: one ``randperm`` of the pool's slots, handed out to the
  requests in order, so each request's token slots are scattered;
  page_size P > 1: the same over whole pages;
* every pool row no request uses, including the tail of a request's last
  page, is NaN (bf16 0x7FC0; for the 8-bit pools V8 = 0x7F, the E4M3 NaN),
  so a kernel that gathers a wrong row produces NaN;
* page-table entries past a request's last page point at an unused page when
  one exists (else page 0), so a stray table read stays in bounds.
* long-context rows: a seeded Bernoulli mask scales 1% of the (token, kv-head)
  K rows by 8, which makes the softmax rows peaked;
* Sage: Q8, K8 uniform in [-127, 127]; V8 = E4M3(16 N(0, 1)); sfQ, sfK, sfV
  lognormal(mu=-4, sigma=0.5); v_mean ~ N(0, 0.1^2) (0.1 read as the standard
  deviation).
* block-sparse Sage: one Bernoulli(density) mask per (request, 64-key block), drawn
  from seed 9_000_000 + cfg (the pages measure density 0.10 and 0.125);
* FP8 KV cache: K8, V8 = E4M3(16 N(0, 1)) (clamped to +-448, nearest-even) with
  k_scale = v_scale = 1/16, so the dequantised K, V are N(0, 1) like the bf16 pools;
  Q ~ N(0, 1) in bf16.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

BF16_NAN = 0x7FC0
E4M3_NAN = 0x7F


@dataclass(frozen=True)
class Spec:
    """Shape of one workload.  ``len_lo``/``len_hi`` bound the total KV length
    (DECODE, SAGE) or the prefix length (EXTEND, with ``new_lo``/``new_hi`` for
    the new tokens)."""
    name: str
    cfg: int
    mode: str                 # "decode" | "extend" | "sage" | "fp8"
    batch: int
    len_lo: int
    len_hi: int
    hq: int
    hkv: int
    head_dim: int = 128
    page_size: int = 1
    pool_slots: int = 0       # page_size 1: slots in the pool (0 = exactly what the batch needs)
    spare_pages: float = 0.0  # page_size > 1: extra unused pages, as a fraction
    layers: int = 1
    distinct_pools: int = 0   # pools actually allocated (0 = one per layer); layers rotate over them
    new_lo: int = 0
    new_hi: int = 0
    peaked_frac: float = 0.0
    peaked_scale: float = 1.0
    density: float = 1.0      # block-sparse Sage: fraction of 64-key blocks attended

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    def scaled(self, **kw) -> "Spec":
        return replace(self, **kw)


CONFIGS = {
    1: Spec("decode_tiny", 1, "decode", batch=4, len_lo=17, len_hi=300, hq=8, hkv=2,
            page_size=1, pool_slots=2048),
    2: Spec("decode_llama3_8b", 2, "decode", batch=64, len_lo=512, len_hi=8192, hq=32, hkv=8,
            page_size=1, pool_slots=600_000, layers=32),
    3: Spec("extend_prefix", 3, "extend", batch=8, len_lo=0, len_hi=4096, hq=32, hkv=8,
            page_size=16, spare_pages=0.10, new_lo=128, new_hi=2048, layers=32),
    4: Spec("decode_long_llama3_70b", 4, "decode", batch=8, len_lo=131072, len_hi=131072, hq=64,
            hkv=8, page_size=64, layers=80, distinct_pools=8, peaked_frac=0.01, peaked_scale=8.0),
    5: Spec("sage_decode", 5, "sage", batch=32, len_lo=1024, len_hi=4096, hq=32, hkv=8,
            page_size=64, spare_pages=0.10, layers=32),
    6: Spec("decode_fp8_llama3_8b", 6, "fp8", batch=64, len_lo=512, len_hi=8192, hq=32, hkv=8,
            page_size=16, spare_pages=0.10, layers=32),
    7: Spec("sage_sparse_decode", 7, "sage", batch=32, len_lo=8192, len_hi=32768, hq=32, hkv=8,
            page_size=64, spare_pages=0.05, layers=32, distinct_pools=8, density=0.125),
    8: Spec("sage_extend_prefix", 8, "extend", batch=8, len_lo=0, len_hi=4096, hq=32, hkv=8,
            page_size=64, spare_pages=0.10, new_lo=128, new_hi=2048, layers=32),
    9: Spec("extend_prefix_page1", 9, "extend", batch=8, len_lo=0, len_hi=4096, hq=32, hkv=8,
            page_size=1, new_lo=128, new_hi=2048, layers=32),
}

# the workloads by name (the number of each is its seed id)
SPECS = {s.name: s for s in CONFIGS.values()}

FP8_SCALE = 1.0 / 16.0   # k_scale = v_scale of the FP8 pools


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randint(g, lo, hi, n, device):
    return torch.randint(lo, hi + 1, (n,), generator=g, device=device, dtype=torch.int64)


@dataclass
class Batch:
    """Lengths and the page table of one batch (shared by all layers)."""
    seq_lens: torch.Tensor        # int32 [B]  total KV length per request
    page_table: torch.Tensor      # int32 [B, pitch]
    num_slots: int
    used_slot_mask: torch.Tensor  # bool [num_slots]: rows some request reads
    cu_seqlens_q: torch.Tensor | None = None   # int32 [B+1] (EXTEND)
    new_lens: torch.Tensor | None = None       # int32 [B]   (EXTEND)


def make_batch(spec: Spec, device="cpu", seed: int | None = None) -> Batch:
    """Draw lengths and scatter each request over the pool (see module docstring)."""
    g = _gen(1000 + spec.cfg if seed is None else seed, "cpu")
    B, P = spec.batch, spec.page_size
    if spec.mode == "extend":
        prefix = _randint(g, spec.len_lo, spec.len_hi, B, "cpu")
        new = _randint(g, spec.new_lo, spec.new_hi, B, "cpu")
        L = prefix + new
    else:
        L = _randint(g, spec.len_lo, spec.len_hi, B, "cpu")
        new = None
    need = (L + P - 1) // P                                   # pages (or slots) per request
    total_need = int(need.sum())
    if P == 1:
        num_pages = max(spec.pool_slots, total_need)
    else:
        num_pages = total_need + int(math.ceil(total_need * spec.spare_pages))
    perm = torch.randperm(num_pages, generator=g, device="cpu")
    pitch = max(1, int(need.max()))
    spare = perm[total_need:]
    pad = int(spare[0]) if len(spare) else 0
    table = torch.full((B, pitch), pad, dtype=torch.int64)
    off = 0
    used = torch.zeros(num_pages * P, dtype=torch.bool)
    for r in range(B):
        n = int(need[r])
        pages = perm[off:off + n]
        table[r, :n] = pages
        off += n
        slots = (pages[:, None] * P + torch.arange(P)[None, :]).reshape(-1)[: int(L[r])]
        used[slots] = True
    cu = None
    if new is not None:
        cu = torch.zeros(B + 1, dtype=torch.int64)
        cu[1:] = torch.cumsum(new, 0)
        cu = cu.to(torch.int32).to(device)
        new = new.to(torch.int32).to(device)
    return Batch(L.to(torch.int32).to(device), table.to(torch.int32).to(device), num_pages * P,
                 used.to(device), cu, new)


def make_bf16_pools(spec: Spec, batch: Batch, layer: int, device="cpu", seed: int | None = None):
    """K and V pools [num_slots, Hkv, D] bf16 for one layer, unused rows NaN."""
    g = _gen(1000 + 100 * spec.cfg + layer if seed is None else seed, device)
    shape = (batch.num_slots, spec.hkv, spec.head_dim)
    k = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if spec.peaked_frac > 0:
        sel = torch.rand((batch.num_slots, spec.hkv, 1), generator=g, device=device) < spec.peaked_frac
        k = torch.where(sel, k * spec.peaked_scale, k)
    k = k.to(torch.bfloat16)
    v = torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    unused = ~batch.used_slot_mask.to(device)
    for t in (k, v):
        t.view(torch.int16)[unused] = BF16_NAN
    return k, v


def make_block_mask(spec: Spec, batch: Batch, device="cpu", seed: int | None = None) -> torch.Tensor:
    """uint8 [B, pitch] (pitch = the page table's, 64-key blocks = pages): 1 = block attended."""
    g = _gen(9_000_000 + spec.cfg if seed is None else seed, "cpu")
    m = (torch.rand(batch.page_table.shape, generator=g) < spec.density).to(torch.uint8)
    return m.to(device)


def make_fp8_pools(spec: Spec, batch: Batch, layer: int, device="cpu", seed: int | None = None):
    """K8 and V8 pools [num_slots, Hkv, D] of E4M3 codes (uint8) for one layer, unused rows NaN;
    dequantised by FP8_SCALE."""
    g = _gen(1000 + 100 * spec.cfg + layer if seed is None else seed, device)
    shape = (batch.num_slots, spec.hkv, spec.head_dim)
    out = []
    for _ in range(2):
        x = (16.0 * torch.randn(shape, generator=g, device=device, dtype=torch.float32)).clamp(-448, 448)
        c = x.to(torch.float8_e4m3fn).view(torch.uint8)
        c[~batch.used_slot_mask.to(device)] = E4M3_NAN
        out.append(c)
    return out[0], out[1]


def make_bf16_queries(spec: Spec, rows: int, layer: int, device="cpu", seed: int | None = None):
    """Q [rows, Hq, D] bf16 (rows = B for DECODE, sum of new tokens for EXTEND)."""
    g = _gen(7_000_000 + 1000 + 100 * spec.cfg + layer if seed is None else seed, device)
    return torch.randn((rows, spec.hq, spec.head_dim), generator=g, device=device,
                       dtype=torch.float32).to(torch.bfloat16)


@dataclass
class SageLayer:
    q8: torch.Tensor      # int8 [B, Hq, D]
    sf_q: torch.Tensor    # f32  [B, Hq]
    k8: torch.Tensor      # int8 [num_slots, Hkv, D]
    v8: torch.Tensor      # uint8 (E4M3 codes) [num_slots, Hkv, D]
    sf_k: torch.Tensor    # f32  [num_slots // 64, Hkv]
    sf_v: torch.Tensor    # f32  [Hkv, D]
    v_mean: torch.Tensor  # f32  [Hkv, D]


def make_sage_layer(spec: Spec, batch: Batch, layer: int, device="cpu", k_block: int = 64,
                    seed: int | None = None, q_rows: int | None = None) -> SageLayer:
    """8-bit Q/K/V, their scales and v_mean for one layer (see module docstring); q_rows query
    rows (default: one per request, the decode case; the new tokens for EXTEND)."""
    g = _gen(1000 + 100 * spec.cfg + layer if seed is None else seed, device)
    B, Hq, Hkv, D = spec.batch if q_rows is None else q_rows, spec.hq, spec.hkv, spec.head_dim
    S = batch.num_slots

    def ri(shape):
        return torch.randint(-127, 128, shape, generator=g, device=device, dtype=torch.int32).to(torch.int8)

    def lognormal(shape):
        return torch.exp(-4.0 + 0.5 * torch.randn(shape, generator=g, device=device, dtype=torch.float32))

    q8 = ri((B, Hq, D))
    k8 = ri((S, Hkv, D))
    v = (16.0 * torch.randn((S, Hkv, D), generator=g, device=device, dtype=torch.float32)).clamp(-448, 448)
    v8 = v.to(torch.float8_e4m3fn).view(torch.uint8)
    unused = ~batch.used_slot_mask.to(device)
    v8[unused] = E4M3_NAN
    k8[unused] = 127
    sf_q = lognormal((B, Hq))
    sf_k = lognormal((S // k_block, Hkv))
    sf_v = lognormal((Hkv, D))
    v_mean = 0.1 * torch.randn((Hkv, D), generator=g, device=device, dtype=torch.float32)
    return SageLayer(q8, sf_q, k8, v8, sf_k, sf_v, v_mean)


def decode_kv_bytes(seq_lens, hkv: int, head_dim: int, elem_bytes: int, page_size: int,
                    hq: int, q_bytes: int, o_bytes: int, extra_per_key: float = 0.0) -> float:
    """Algorithmic bytes of one decode call: K and V rows read once, the table
    entries read once (4 B per page), Q read and O written once."""
    L = [int(x) for x in seq_lens]
    kv = sum(L) * hkv * head_dim * elem_bytes * 2
    table = sum((x + page_size - 1) // page_size for x in L) * 4
    qo = len(L) * hq * head_dim * (q_bytes + o_bytes)
    return float(kv + table + qo + extra_per_key * sum(L))
