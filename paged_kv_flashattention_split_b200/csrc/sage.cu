// sage.cu - 8-bit "Sage" decode over the paged cache: a score pass, a value pass and a merge.
//
// The formula ("FlashInfer PrimTS, Sage Attention 도입으로 8비트 양자화 및 성능
// 최적화 달성", 코드 분석 item 1, README "Sage attention"):
//     S_j  = sfQ[r][h] * sfK[blk(j)][h_kv] * (Q8 . K8_j)
//     P    = softmax_row(S), quantised to E4M3 as 448 p
//     O[d] = sfV[h_kv][d] * (sum_j P8_j V8_j[d]) / (448 l) + v_mean[h_kv][d]
// with the scales applied before the row max and the exponential and sfV in
// the epilogue (same page, item 4).
//
// Quantising p needs the row max m over ALL keys of the row before any P8 is
// formed, so the work runs in two passes over the plan's CTA slots (a flat,
// balanced partition of every request's 32-key units, one wave of two CTAs per
// SM); a CTA takes one slot and one group of HG KV heads:
//   score pass: S for every key of its items and every query head of the
//     group, written to the workspace's score rows, and each head's maximum
//     over each item;
//   value pass (a programmatic dependent of the score pass): m = the maximum of
//     the request's item maxima, which is the exact row max; P8 = E4M3(448
//     exp(S - m)) from the stored S, l = sum exp(S - m), acc = P8 . V8.  A
//     request covered by one item writes its output; otherwise (acc, l) per item;
//   merge (a programmatic dependent of the value pass): O = sfV sum_s acc_s /
//     (448 sum_s l_s) + v_mean.  All items used the same m, so the merge is a
//     plain sum.
// The scores cost 4 bytes per key and query head on top of the 128-byte K8 and
// V8 rows per key and KV head (1/8 more at G = 4); they are written and read
// back while they are still in L2.
//
// Each CTA is one producer warp and eight consumer warps around a 3-stage ring.
// A tile is 32 slots of one 64-slot page: the producer reads the page ids (and,
// for the score pass, the K scales) of 32 tiles at once, one per lane, and
// loads each tile with ONE TMA box {128 B, 32 slots, HG heads} of a 3-D tensor
// map over the pool [slot][head][128 B], 128-byte swizzled, so shared memory
// holds [head][slot][128 B] and the ldmatrix reads of 8 consecutive slots hit
// 8 different bank groups.  In the value pass a second box brings the tile's
// scores [query head][32 keys] (fp32, swizzled) from the score rows.  Consumer
// warp w takes KV head w of the group (the value pass spreads a head's 8
// 16-byte d-blocks over 8 / HG warps when HG < 8):
//   score: S^T[16 keys x 8 heads] = K8[16 x 128] . Q8^T on the INT8 tensor cores
//          (mma.m16n8k32.s8, exact int32 dot), S = fp32(fp32(sfQ sfK) fp32(dot));
//   value: O^T[16 d x 8 heads] += V8^T[16 d x 32 keys] . P8^T on the FP8 tensor
//          cores (mma.m16n8k32.e4m3, fp32 accumulation); ldmatrix.trans on byte
//          pairs plus one byte permute gives 4 keys of one d per register, in a
//          fixed key order that P8's fragment uses too (the sum over keys does
//          not depend on their order).
// Rows past the end of a request's last page share its box; their K8 only
// produce scores that are never stored, and their V8 rows are zeroed in shared
// memory before use.  Every mbarrier wait is bounded: on timeout the CTA
// records PA_ERR_DEVICE_INDEX, its roles stop, and the producer waits for the
// copies it issued before it exits.
#include "kernels.h"
#include "tma.cuh"

namespace pa {

namespace {
constexpr int kConsumerWarps = 8;
constexpr int kThreads = 32 * (kConsumerWarps + 1);
constexpr int kStages = 3;
constexpr int kTileKeys = 32;
constexpr uint32_t kWaitLimit = 1u << 20;
constexpr float kLog2e = 1.4426950408889634f;

// What the producer tells the consumers about the tile in a stage.
struct StageInfo {
  int kstart;      // first key of the tile
  int nvalid;      // keys of the item in the tile (1 .. 32)
  int page;        // the tile's page, -1 if its table entry was bad (nothing loaded)
  int pad;
};

template <int HG, int G, bool VPASS>
struct SageSmem {
  static constexpr int KV = HG * kTileKeys * kHeadDim;            // [head][slot][128 B]
  static constexpr int SB = VPASS ? HG * G * kTileKeys * 4 : 0;   // [query head][32] fp32
  static constexpr int STAGE = (KV + SB + 1023) / 1024 * 1024;
  static constexpr int OFF_SFK = kStages * STAGE;                              // [k][32] fp32, 128 B each
  static constexpr int OFF_INFO = OFF_SFK + kStages * 128;
  static constexpr int OFF_BAR = OFF_INFO + kStages * (int)sizeof(StageInfo);   // full[k], empty[k]
  static constexpr int OFF_FLAG = OFF_BAR + 2 * kStages * 8;
  static constexpr int OFF_RED = OFF_FLAG + 16;                                 // [8 warps][8] floats
  static constexpr int BYTES = OFF_RED + kConsumerWarps * 8 * 4 + 1024;         // + alignment slack
  static_assert(OFF_BAR % 8 == 0, "barrier alignment");
};

__device__ __forceinline__ void mma_s8_16832(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_e4m3_16832(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Two floats to E4M3 (round to nearest even, saturating); `lo` in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t v;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;\n" : "=h"(v) : "f"(hi), "f"(lo));
  return v;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;\n" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

struct SageLaunch {
  CUtensorMap tm_kv;   // K8 (score pass) or V8 (value pass) pool, box {128, 32, HG}
  CUtensorMap tm_s;    // score rows [B * Hq][score_pitch] fp32, box {32, HG * G}
  CUtensorMap tm_sfk;  // score pass, HG >= 4: sfK [num_slots / 64][Hkv] fp32, box {HG, 1}
  WsView ws;
  const int8_t* q8;
  const float* sf_q;
  const float* sf_k;
  const float* sf_v;
  const float* v_mean;
  int64_t num_slots;
  const int32_t* page_table;
  int64_t pt_pitch;
  uint16_t* out;
  int batch, hq, hkv;
};

__device__ __forceinline__ bool sage_ws_ok(const PlanHeader* hdr) {
  return hdr->magic == kMagic && sage_mode(hdr->mode);
}

// Tiles of an item: SAGE_DECODE items are key ranges [a0, a1), SAGE_SPARSE items unit
// ranges [a0, a1) of the request's selected blocks (one 32-key tile per unit).
__device__ __forceinline__ int item_tiles(bool sparse, int a0, int a1) {
  return sparse ? a1 - a0 : (a1 - a0 + kTileKeys - 1) / kTileKeys;
}

// Tile t of an item: its first key, its key count (0 past the item) and the raw table entry
// of its page (checked where it is used).
struct TileRef {
  int ks, nv, e;
};
__device__ __forceinline__ TileRef tile_ref(const SageLaunch& a, bool sparse, int r, int a0, int a1, int len,
                                            int selb, int t) {
  TileRef x{0, 0, -1};
  const int32_t* table = a.page_table + (size_t)r * a.pt_pitch;
  if (!sparse) {
    x.ks = a0 + kTileKeys * t;
    if (x.ks < a1) {
      x.nv = min(kTileKeys, a1 - x.ks);
      x.e = __ldg(table + (x.ks >> 6));
    }
  } else if (a0 + t < a1) {
    const int u = a0 + t;
    const int blk = __ldg(a.ws.sel_block + selb + (u >> 1));
    x.ks = blk * kSageBlock + (u & 1) * kTileKeys;
    x.nv = min(kTileKeys, len - x.ks);
    x.e = __ldg(table + blk);
  }
  return x;
}

// The items of this CTA's slot: [first, last).
__device__ __forceinline__ bool slot_items(const SageLaunch& a, int groups, int& first, int& last) {
  const int slot = blockIdx.x / groups;
  if (slot >= a.ws.hdr->slots) return false;
  first = a.ws.slot_first[slot];
  last = min(a.ws.slot_first[slot + 1], a.ws.hdr->num_items);
  return first < last;
}

// Item metadata of a slot, 32 items at a time, one item per lane; every warp keeps its own
// window, so no role waits on a chain of dependent reads at an item boundary.
struct ItemWindow {
  int w0 = -(1 << 30);
  int r = 0, kv0 = 0, kv1 = 0, base = 0, splits = 0;   // item w0 + lane
  int len = 0, selb = 0;                                // SAGE_SPARSE producer: L_r and sel_base[r]
  __device__ __forceinline__ void load(const SageLaunch& a, int w, int last, bool with_req, bool with_sel = false) {
    w0 = w;
    const int i = w + (threadIdx.x & 31);
    r = kv0 = kv1 = base = splits = len = selb = 0;
    if (i < last) {
      const int4 it = a.ws.items[i];
      r = it.x;
      kv0 = it.z;
      kv1 = it.w;
      if (with_req) {
        base = a.ws.req_base[r];
        splits = min(a.ws.req_splits[r], a.ws.hdr->max_items - base);   // clamped only after a flagged overflow
      }
      if (with_sel) {
        len = a.ws.req_len[r];
        selb = a.ws.sel_base[r];
      }
    }
  }
  // item i for the producer: request, item bounds, L_r and sel_base[r]
  __device__ __forceinline__ void get_sel(const SageLaunch& a, int i, int last, bool with_sel, int& ri, int& k0,
                                          int& k1, int& li, int& sbi) {
    if (i < w0 || i >= w0 + 32) load(a, i, last, false, with_sel);
    const int l = i - w0;
    ri = __shfl_sync(0xffffffffu, r, l);
    k0 = __shfl_sync(0xffffffffu, kv0, l);
    k1 = __shfl_sync(0xffffffffu, kv1, l);
    li = __shfl_sync(0xffffffffu, len, l);
    sbi = __shfl_sync(0xffffffffu, selb, l);
  }
  // item i (the same i on every lane): request, key range, first item and item count of its request
  __device__ __forceinline__ void get(const SageLaunch& a, int i, int last, bool with_req, int& ri, int& k0, int& k1,
                                      int& bi, int& si) {
    if (i < w0 || i >= w0 + 32) load(a, i, last, with_req);
    const int l = i - w0;
    ri = __shfl_sync(0xffffffffu, r, l);
    k0 = __shfl_sync(0xffffffffu, kv0, l);
    k1 = __shfl_sync(0xffffffffu, kv1, l);
    bi = __shfl_sync(0xffffffffu, base, l);
    si = __shfl_sync(0xffffffffu, splits, l);
  }
};

// Shared-memory handles of one CTA.
template <int HG, int G, bool VPASS>
struct Ring {
  using L = SageSmem<HG, G, VPASS>;
  uint32_t base;
  uint8_t* ptr;
  __device__ __forceinline__ Ring() {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    base = (raw + 1023u) & ~1023u;
    ptr = smem_raw + (base - raw);
  }
  __device__ __forceinline__ uint32_t stage(int s) const { return base + s * L::STAGE; }
  __device__ __forceinline__ uint32_t full(int s) const { return base + L::OFF_BAR + 8 * s; }
  __device__ __forceinline__ uint32_t empty(int s) const { return base + L::OFF_BAR + 8 * (kStages + s); }
  __device__ __forceinline__ StageInfo* info() const { return reinterpret_cast<StageInfo*>(ptr + L::OFF_INFO); }
  // score pass: sfK of stage s's page for each head of the group (128-byte aligned: a TMA target)
  __device__ __forceinline__ float* sfk(int s) const { return reinterpret_cast<float*>(ptr + L::OFF_SFK + 128 * s); }
  __device__ __forceinline__ volatile int* abort_flag() const {
    return reinterpret_cast<volatile int*>(ptr + L::OFF_FLAG);
  }
  __device__ __forceinline__ float* red() const { return reinterpret_cast<float*>(ptr + L::OFF_RED); }
  __device__ __forceinline__ void init() const {
    if (threadIdx.x == 0) {
      for (int s = 0; s < kStages; ++s) {
        mbar_init(full(s), 1);
        mbar_init(empty(s), kConsumerWarps);
      }
      *abort_flag() = 0;
      mbar_fence_init();
    }
    __syncthreads();
  }
  // bounded, warp-uniform wait: every lane observes the phase itself, the warp agrees on
  // the outcome; false (and the CTA-wide abort flag set) if the phase never completes
  __device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity, PlanHeader* hdr) const {
    for (uint32_t i = 0; i < kWaitLimit; ++i) {
      const bool done = mbar_try_wait(bar, parity);
      if (__all_sync(0xffffffffu, done)) return true;
      if (__any_sync(0xffffffffu, *abort_flag() != 0)) return false;
    }
    if ((threadIdx.x & 31) == 0) {
      *abort_flag() = 1;
      set_device_error(hdr, PA_ERR_DEVICE_INDEX);
    }
    return false;
  }
};

// The producer warp: page ids of 32 tiles per round, one per lane, then one TMA box per tile;
// in the score pass also the page's K scales (one box {HG, 1} when HG >= 4, which keeps a
// dependent global read off the path to the first copy; else read by the lanes), in the
// value pass one box of the tile's scores.  The value pass requests the V8 of its first
// kStages tiles before it waits for the score pass, their scores after.
template <int HG, int G, bool VPASS>
__device__ __forceinline__ void produce(const SageLaunch& a, const Ring<HG, G, VPASS>& rg, int first, int last,
                                        int grp) {
  using L = SageSmem<HG, G, VPASS>;
  const int lane = threadIdx.x & 31;
  PlanHeader* hdr = a.ws.hdr;
  StageInfo* info = rg.info();
  uint32_t q = 0;   // ring uses so far
  bool ok = true;
  bool waited = !VPASS;
  int pend_n = 0, pend_x[kStages], pend_y[kStages];   // value pass: deferred score boxes (lane 0)
  auto flush = [&]() {
    asm volatile("griddepcontrol.wait;\n" ::: "memory");   // the score pass has completed
    if (lane == 0)
      for (int k = 0; k < pend_n; ++k)
        tma_load_2d(rg.stage(k) + L::KV, &a.tm_s, pend_x[k], pend_y[k], rg.full(k));
    waited = true;
  };
  ItemWindow win;
  const bool sparse = hdr->mode == PA_MODE_SAGE_SPARSE;
  int r = 0, a0 = 0, a1 = 0, len = 0, selb = 0;
  if (first < last) win.get_sel(a, first, last, sparse, r, a0, a1, len, selb);
  TileRef pre = tile_ref(a, sparse, r, a0, a1, len, selb, lane);   // first round of the next item
  for (int item = first; item < last && ok; ++item) {
    const int n_tiles = item_tiles(sparse, a0, a1);
    const int srow = r * a.hq + grp * HG * G;
    int rn = 0, a0n = 0, a1n = 0, lenn = 0, selbn = 0;
    if (item + 1 < last) win.get_sel(a, item + 1, last, sparse, rn, a0n, a1n, lenn, selbn);
    if (n_tiles == 0 && item + 1 < last) pre = tile_ref(a, sparse, rn, a0n, a1n, lenn, selbn, lane);   // no round
    for (int tb = 0; tb < n_tiles && ok; tb += 32) {
      const TileRef tr = tb == 0 ? pre : tile_ref(a, sparse, r, a0, a1, len, selb, tb + lane);
      // the next item's first page ids, read behind this item's last round
      if (tb + 32 >= n_tiles && item + 1 < last) pre = tile_ref(a, sparse, rn, a0n, a1n, lenn, selbn, lane);
      int pg = -1;
      if (tb + lane < n_tiles) {
        if (tr.e >= 0 && ((long long)tr.e + 1) * kSageBlock <= a.num_slots) pg = tr.e;
        else set_device_error(hdr, PA_ERR_DEVICE_INDEX);
      }
      constexpr bool kSfkLanes = !VPASS && HG < 4;   // K scales read by the lanes
      float sfk[HG];
#pragma unroll
      for (int h = 0; h < HG; ++h)
        sfk[h] = kSfkLanes && pg >= 0 ? __ldg(a.sf_k + (size_t)pg * a.hkv + grp * HG + h) : 0.f;
      const int nt = min(32, n_tiles - tb);
      for (int i = 0; i < nt; ++i, ++q) {
        const int s = q % kStages;
        if (VPASS && !waited && q == kStages) flush();
        if (q >= kStages && !rg.wait(rg.empty(s), ((q / kStages) - 1) & 1, hdr)) {
          ok = false;
          break;
        }
        const int p = __shfl_sync(0xffffffffu, pg, i);
        const int ks = __shfl_sync(0xffffffffu, tr.ks, i);
        const int nv = __shfl_sync(0xffffffffu, tr.nv, i);
        float sf[HG];
#pragma unroll
        for (int h = 0; h < HG; ++h) sf[h] = __shfl_sync(0xffffffffu, sfk[h], i);
        if (lane == 0) {
          StageInfo& in = info[s];
          in.kstart = ks;
          in.nvalid = nv;
          in.page = p;
          if (kSfkLanes) {
#pragma unroll
            for (int h = 0; h < HG; ++h) rg.sfk(s)[h] = sf[h];
          }
          const bool sfk_box = !VPASS && !kSfkLanes && p >= 0;
          mbar_expect_tx(rg.full(s), (p >= 0 ? L::KV : 0) + L::SB + (sfk_box ? HG * 4 : 0));
          if (p >= 0)   // K8 / V8 stream through once: first out of L2, ahead of the score rows
            tma_load_3d_hint(rg.stage(s), &a.tm_kv, 0, p * kSageBlock + (ks & (kSageBlock - 1)), grp * HG, rg.full(s),
                             l2_evict_first());
          if (sfk_box) tma_load_2d(smem_u32(rg.sfk(s)), &a.tm_sfk, grp * HG, p, rg.full(s));
          if (VPASS) {
            if (waited) {
              tma_load_2d(rg.stage(s) + L::KV, &a.tm_s, ks, srow, rg.full(s));
            } else {
              pend_x[pend_n] = ks;
              pend_y[pend_n] = srow;
              ++pend_n;
            }
          }
        }
      }
    }
    r = rn;
    a0 = a0n;
    a1 = a1n;
    len = lenn;
    selb = selbn;
  }
  if (VPASS && !waited) flush();
  if (!ok && lane == 0) {
    // drain: wait (bounded) for the copies this warp issued into the last kStages uses
    const uint32_t q0 = q > (uint32_t)kStages ? q - kStages : 0;
    for (uint32_t u = q0; u < q; ++u)
      for (uint32_t i = 0; i < kWaitLimit && !mbar_try_wait(rg.full(u % kStages), (u / kStages) & 1); ++i) {}
  }
}

// ---------------------------------------------------------------- score pass
template <int HG, int G>
__global__ void __launch_bounds__(kThreads, 2) sage_score_kernel(const __grid_constant__ SageLaunch a) {
  // the value pass (a programmatic dependent) may be scheduled now; it waits for this
  // whole grid to finish before it reads the scores
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  // this grid is itself a programmatic dependent of whatever precedes it on the stream (the
  // previous layer's merge lets it start early): nothing is read before that grid is done
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, tig = lane & 3, mat = lane >> 3;
  PlanHeader* hdr = a.ws.hdr;
  if (!sage_ws_ok(hdr)) {
    if (tid == 0 && blockIdx.x == 0) set_device_error(hdr, PA_ERR_WORKSPACE);
    return;
  }
  const int groups = a.hkv / HG, grp = blockIdx.x % groups;
  int first = 0, last = 0;
  if (!slot_items(a, groups, first, last)) return;
  Ring<HG, G, false> rg;
  rg.init();
  if (warp == kConsumerWarps) {
    produce<HG, G, false>(a, rg, first, last, grp);
    return;
  }
  // consumer warp `warp` owns KV head `warp` of the group (warps HG.. idle when HG < 8)
  const bool active = warp < HG;
  const int hl = active ? warp : 0;
  const int hkv = grp * HG + hl;
  const float NEG_INF = -__int_as_float(0x7f800000);
  const StageInfo* info = rg.info();
  const bool sparse = hdr->mode == PA_MODE_SAGE_SPARSE;
  const int c0 = 2 * tig, c1 = 2 * tig + 1;          // this thread's query-head columns of S^T
  // Q8^T as the B operand: b0 = Q8[head gid][32 ks + 4 tig .. +3], b1 = the same at +16; the
  // next item's are read while this item's tiles are processed
  uint32_t qn0[4], qn1[4];
  float sfqn0 = 0.f, sfqn1 = 0.f;
  auto load_q = [&](int rq) {
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(a.q8 + ((size_t)rq * a.hq + (size_t)hkv * G + gid) * kHeadDim);
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      qn0[ks] = active && gid < G ? __ldg(qrow + 8 * ks + tig) : 0u;
      qn1[ks] = active && gid < G ? __ldg(qrow + 8 * ks + 4 + tig) : 0u;
    }
    sfqn0 = active && c0 < G ? __ldg(a.sf_q + (size_t)rq * a.hq + (size_t)hkv * G + c0) : 0.f;
    sfqn1 = active && c1 < G ? __ldg(a.sf_q + (size_t)rq * a.hq + (size_t)hkv * G + c1) : 0.f;
  };
  ItemWindow win;
  int rn = 0, kv0n = 0, kv1n = 0, b_, s_;
  win.get(a, first, last, false, rn, kv0n, kv1n, b_, s_);
  load_q(rn);
  uint32_t q = 0;
  for (int item = first; item < last; ++item) {
    const int r = rn, kv0 = kv0n, kv1 = kv1n;
    const int n_tiles = item_tiles(sparse, kv0, kv1);
    uint32_t qb0[4], qb1[4];
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      qb0[ks] = qn0[ks];
      qb1[ks] = qn1[ks];
    }
    const float sfq0 = sfqn0, sfq1 = sfqn1;
    if (item + 1 < last) {
      win.get(a, item + 1, last, false, rn, kv0n, kv1n, b_, s_);
      load_q(rn);
    }
    float* srow0 = a.ws.scores + ((size_t)r * a.hq + (size_t)hkv * G + (c0 < G ? c0 : 0)) * a.ws.score_pitch;
    float* srow1 = a.ws.scores + ((size_t)r * a.hq + (size_t)hkv * G + (c1 < G ? c1 : 0)) * a.ws.score_pitch;
    float mx0 = NEG_INF, mx1 = NEG_INF;
    for (int t = 0; t < n_tiles; ++t, ++q) {
      const int s = q % kStages;
      if (!rg.wait(rg.full(s), (q / kStages) & 1, hdr)) return;
      const int ks0 = info[s].kstart, page = info[s].page, nv = info[s].nvalid;
      if (active && page >= 0) {
        const float sfk = rg.sfk(s)[hl];
        const float sc0 = sfq0 * sfk, sc1 = sfq1 * sfk;      // fp32(sfQ sfK)
        const uint32_t kst = rg.stage(s) + hl * kTileKeys * kHeadDim;
#pragma unroll
        for (int kb = 0; kb < 2; ++kb) {
          const int row = 16 * kb + (lane & 7) + ((mat & 1) << 3);
          int acc[4] = {0, 0, 0, 0};
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            uint32_t af[4];
            const int chunk = 2 * kk + (mat >> 1);
            ldmatrix_x4(af, kst + row * kHeadDim + ((chunk ^ (row & 7)) << 4));
            mma_s8_16832(acc, af, qb0[kk], qb1[kk]);
          }
          const int j0 = 16 * kb + gid, j1 = j0 + 8;                 // key offsets in the tile
          const int key0 = ks0 + j0, key1 = ks0 + j1;
          // S = fp32(fp32(sfQ sfK) fp32(dot)); the int32 dot is exact and |dot| < 2^24
          const float s00 = sc0 * (float)acc[0], s01 = sc1 * (float)acc[1];
          const float s10 = sc0 * (float)acc[2], s11 = sc1 * (float)acc[3];
          if (c0 < G) {
            if (j0 < nv) { srow0[key0] = s00; mx0 = fmaxf(mx0, s00); }
            if (j1 < nv) { srow0[key1] = s10; mx0 = fmaxf(mx0, s10); }
          }
          if (c1 < G) {
            if (j0 < nv) { srow1[key0] = s01; mx1 = fmaxf(mx1, s01); }
            if (j1 < nv) { srow1[key1] = s11; mx1 = fmaxf(mx1, s11); }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(rg.empty(s));
    }
    // this head's maxima over the item (the 8 key rows of the fragments)
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
    }
    if (active && gid == 0) {
      float* im = a.ws.item_max + (size_t)item * a.hq + (size_t)hkv * G;
      if (c0 < G) im[c0] = mx0;
      if (c1 < G) im[c1] = mx1;
    }
  }
}

// ---------------------------------------------------------------- value pass
// two CTAs per SM where their shared memory fits (G = 8 with HG = 8 takes one)
template <int HG, int G>
__global__ void __launch_bounds__(kThreads, 2 * SageSmem<HG, G, true>::BYTES <= 227 * 1024 ? 2 : 1)
    sage_value_kernel(const __grid_constant__ SageLaunch a) {
  using L = SageSmem<HG, G, true>;
  constexpr int WPH = kConsumerWarps / HG;   // warps per KV head
  constexpr int NDB = 8 / WPH;               // 16-byte d-blocks per warp
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");   // lets the merge be scheduled
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, tig = lane & 3;
  PlanHeader* hdr = a.ws.hdr;
  if (!sage_ws_ok(hdr)) return;   // the score pass has flagged it
  const int groups = a.hkv / HG, grp = blockIdx.x % groups;
  int first = 0, last = 0;
  if (!slot_items(a, groups, first, last)) return;
  Ring<HG, G, true> rg;
  rg.init();
  if (warp == kConsumerWarps) {
    produce<HG, G, true>(a, rg, first, last, grp);
    return;
  }
  const int hl = warp % HG, db0 = (warp / HG) * NDB;
  const int hkv = grp * HG + hl;
  const bool p_lane = gid < G;
  const float NEG_INF = -__int_as_float(0x7f800000);
  const StageInfo* info = rg.info();
  const bool sparse = hdr->mode == PA_MODE_SAGE_SPARSE;
  float* mw = rg.red() + warp * 8;
  asm volatile("griddepcontrol.wait;\n" ::: "memory");   // the score pass has completed and its writes are visible
  // m for the G query heads of this KV head is the maximum of the request's item maxima: each
  // lane reads those of items base + lane, base + lane + 32, ...; the first 32 of the next
  // item's request are read while this item's tiles are processed
  float mv[G];
  auto load_m = [&](int b, int sp) {
#pragma unroll
    for (int g = 0; g < G; ++g)
      mv[g] = lane < sp ? __ldcg(a.ws.item_max + (size_t)(b + lane) * a.hq + (size_t)hkv * G + g) : NEG_INF;
  };
  ItemWindow win;
  int rn = 0, kv0n = 0, kv1n = 0, basen = 0, splitsn = 0;
  win.get(a, first, last, true, rn, kv0n, kv1n, basen, splitsn);
  load_m(basen, splitsn);
  uint32_t q = 0;
  for (int item = first; item < last; ++item) {
    const int r = rn, kv0 = kv0n, kv1 = kv1n, base = basen, splits = splitsn;
    const int n_tiles = item_tiles(sparse, kv0, kv1);
    {
      float m[G];
#pragma unroll
      for (int g = 0; g < G; ++g) m[g] = mv[g];
      for (int sp = lane + 32; sp < splits; sp += 32) {   // requests of more than 32 items
#pragma unroll
        for (int g = 0; g < G; ++g) m[g] = fmaxf(m[g], __ldcg(a.ws.item_max + (size_t)(base + sp) * a.hq + (size_t)hkv * G + g));
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m[g] = fmaxf(m[g], __shfl_xor_sync(0xffffffffu, m[g], off));
        if (lane == 0) mw[g] = m[g] == NEG_INF ? 0.f : m[g];
      }
    }
    __syncwarp();
    if (item + 1 < last) {
      win.get(a, item + 1, last, true, rn, kv0n, kv1n, basen, splitsn);
      load_m(basen, splitsn);
    }
    const float m_use = p_lane ? mw[gid] : 0.f;
    float o[NDB][4];
#pragma unroll
    for (int b = 0; b < NDB; ++b) o[b][0] = o[b][1] = o[b][2] = o[b][3] = 0.f;
    float lsum = 0.f;
    const int srow = hl * G + (p_lane ? gid : 0);   // this lane's row of the stage's score box
    for (int t = 0; t < n_tiles; ++t, ++q) {
      const int s = q % kStages;
      if (!rg.wait(rg.full(s), (q / kStages) & 1, hdr)) return;
      const uint32_t vst = rg.stage(s) + hl * kTileKeys * kHeadDim;
      const int nv = info[s].page >= 0 ? info[s].nvalid : 0;   // keys of the item in this tile
      if (nv < kTileKeys) {
        // rows past the item (or of a page that was not loaded) become zero in this warp's d-blocks
        uint8_t* vp = rg.ptr + (vst - rg.base);
        for (int idx = lane; idx < (kTileKeys - nv) * NDB; idx += 32) {
          const int row = nv + idx / NDB, chunk = db0 + idx % NDB;
          *reinterpret_cast<uint4*>(vp + row * kHeadDim + ((chunk ^ (row & 7)) << 4)) = make_uint4(0, 0, 0, 0);
        }
        __syncwarp();
      }
      // P8 for query head gid at the keys {2tig, 2tig+1, 8+2tig, 9+2tig} (+16): the key order
      // of the V8 fragments below
      uint32_t pb0 = 0u, pb1 = 0u;
      if (p_lane) {
        const uint8_t* sp = rg.ptr + (rg.stage(s) - rg.base) + L::KV + srow * 128;
        float p[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int key = 2 * tig + 8 * i;
          const float2 sv = *reinterpret_cast<const float2*>(sp + (((key >> 2) ^ (srow & 7)) << 4) + (key & 3) * 4);
          const float sx = key < nv ? sv.x : NEG_INF;
          const float sy = key + 1 < nv ? sv.y : NEG_INF;
          p[2 * i] = ex2((sx - m_use) * kLog2e);      // exp(S - m), 0 for masked keys
          p[2 * i + 1] = ex2((sy - m_use) * kLog2e);
          lsum += p[2 * i] + p[2 * i + 1];
        }
        pb0 = e4m3x2(448.f * p[0], 448.f * p[1]) | (e4m3x2(448.f * p[2], 448.f * p[3]) << 16);
        pb1 = e4m3x2(448.f * p[4], 448.f * p[5]) | (e4m3x2(448.f * p[6], 448.f * p[7]) << 16);
      }
#pragma unroll
      for (int b = 0; b < NDB; ++b) {
        const int db = db0 + b;
        uint32_t vr[4];
        ldmatrix_x4_trans(vr, vst + lane * kHeadDim + ((db ^ (lane & 7)) << 4));
        uint32_t af[4];
        af[0] = prmt(vr[0], vr[1], 0x6420);   // d = 16 db + 2 gid,     keys 0-15
        af[1] = prmt(vr[0], vr[1], 0x7531);   // d = 16 db + 2 gid + 1, keys 0-15
        af[2] = prmt(vr[2], vr[3], 0x6420);   // keys 16-31
        af[3] = prmt(vr[2], vr[3], 0x7531);
        mma_e4m3_16832(o[b], af, pb0, pb1);
      }
      if (nv < kTileKeys) fence_proxy_async();   // the zeroing writes before the next TMA into this stage
      __syncwarp();
      if (lane == 0) mbar_arrive(rg.empty(s));
    }
    // l of query head gid (summed over the 4 lanes that split its keys), then per column
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 1);
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);
    const float l0 = __shfl_sync(0xffffffffu, lsum, (2 * tig) * 4);
    const float l1 = __shfl_sync(0xffffffffu, lsum, (2 * tig + 1) * 4);
    const int c0 = 2 * tig, c1 = 2 * tig + 1;          // this thread's query-head columns of O^T
    if (splits == 1) {
#pragma unroll
      for (int b = 0; b < NDB; ++b) {
        const int d = 16 * (db0 + b) + 2 * gid;
        const float2 sfv = *reinterpret_cast<const float2*>(a.sf_v + (size_t)hkv * kHeadDim + d);
        const float2 vm = a.v_mean ? *reinterpret_cast<const float2*>(a.v_mean + (size_t)hkv * kHeadDim + d)
                                   : make_float2(0.f, 0.f);
        if (c0 < G) {
          const float inv = l0 > 0.f ? 1.f / (448.f * l0) : 0.f;
          *reinterpret_cast<uint32_t*>(a.out + ((size_t)r * a.hq + (size_t)hkv * G + c0) * kHeadDim + d) =
              pack_bf16x2(sfv.x * o[b][0] * inv + vm.x, sfv.y * o[b][2] * inv + vm.y);
        }
        if (c1 < G) {
          const float inv = l1 > 0.f ? 1.f / (448.f * l1) : 0.f;
          *reinterpret_cast<uint32_t*>(a.out + ((size_t)r * a.hq + (size_t)hkv * G + c1) * kHeadDim + d) =
              pack_bf16x2(sfv.x * o[b][1] * inv + vm.x, sfv.y * o[b][3] * inv + vm.y);
        }
      }
    } else {
      const size_t prow = (size_t)item * a.hq + (size_t)hkv * G;
#pragma unroll
      for (int b = 0; b < NDB; ++b) {
        const int d = 16 * (db0 + b) + 2 * gid;
        if (c0 < G) *reinterpret_cast<float2*>(a.ws.partial_o + (prow + c0) * kHeadDim + d) = make_float2(o[b][0], o[b][2]);
        if (c1 < G) *reinterpret_cast<float2*>(a.ws.partial_o + (prow + c1) * kHeadDim + d) = make_float2(o[b][1], o[b][3]);
      }
      if (db0 == 0 && tig == 0 && p_lane) a.ws.partial_lse[prow + gid] = lsum;
    }
  }
}

// One warp per (request, query head) of a request that was split:
// O = sfV sum_s acc_s / (448 sum_s l_s) + v_mean.  Each lane owns 4 of the 128 outputs and
// issues the loads of 8 items before it adds them (in item order).
__global__ void __launch_bounds__(256) sage_merge_kernel(const __grid_constant__ SageLaunch a) {
  asm volatile("griddepcontrol.wait;\n" ::: "memory");   // the value pass has completed
  // the next layer's score pass (a programmatic dependent) may be scheduled: it waits for this grid
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  PlanHeader* hdr = a.ws.hdr;
  if (!sage_ws_ok(hdr)) return;
  const int gw = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (gw >= a.batch * a.hq) return;
  const int r = gw / a.hq, h = gw % a.hq;
  const int splits = a.ws.req_splits[r];
  if (splits <= 1) return;
  const int base = a.ws.req_base[r];
  if (base + splits > hdr->max_items) return;
  const int h_kv = h / (a.hq / a.hkv);
  const float4 sfv = __ldg(reinterpret_cast<const float4*>(a.sf_v + (size_t)h_kv * kHeadDim) + lane);
  const float4 vm = a.v_mean ? __ldg(reinterpret_cast<const float4*>(a.v_mean + (size_t)h_kv * kHeadDim) + lane)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
  const float4* po = reinterpret_cast<const float4*>(a.ws.partial_o + ((size_t)base * a.hq + h) * kHeadDim) + lane;
  const float* pl = a.ws.partial_lse + (size_t)base * a.hq + h;
  const size_t row4 = (size_t)a.hq * kHeadDim / 4;   // float4s from one item's row to the next
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float l = 0.f;
  for (int s0 = 0; s0 < splits; s0 += 8) {
    float4 v[8];
    float lv[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const bool in = s0 + j < splits;
      v[j] = in ? __ldcg(po + (size_t)(s0 + j) * row4) : make_float4(0.f, 0.f, 0.f, 0.f);
      lv[j] = in ? __ldcg(pl + (size_t)(s0 + j) * a.hq) : 0.f;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      acc.x += v[j].x;
      acc.y += v[j].y;
      acc.z += v[j].z;
      acc.w += v[j].w;
      l += lv[j];
    }
  }
  const float inv = l > 0.f ? 1.f / (448.f * l) : 0.f;
  uint2 packed;
  packed.x = pack_bf16x2(sfv.x * acc.x * inv + vm.x, sfv.y * acc.y * inv + vm.y);
  packed.y = pack_bf16x2(sfv.z * acc.z * inv + vm.z, sfv.w * acc.w * inv + vm.w);
  reinterpret_cast<uint2*>(a.out + ((size_t)r * a.hq + h) * kHeadDim)[lane] = packed;
}

cudaError_t launch_pdl(void (*kernel)(const SageLaunch), dim3 grid, dim3 block, size_t smem, const SageLaunch& a,
                       cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, a);
}

// [num_slots][hkv][128] bytes as 3-D {128, slots, heads}; box {128, 32, HG}, 128-byte swizzle
bool encode_pool(CUtensorMap* tm, const void* ptr, int64_t num_slots, int hkv, int hg) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {128, (cuuint64_t)num_slots, (cuuint64_t)hkv};
  const cuuint64_t strides[2] = {(cuuint64_t)hkv * 128, 128};
  const cuuint32_t box[3] = {128, (cuuint32_t)kTileKeys, (cuuint32_t)hg};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// score rows [rows][pitch] fp32 as 2-D {pitch, rows}; box {32, box_rows}, 128-byte swizzle
bool encode_scores(CUtensorMap* tm, const float* ptr, int64_t pitch, int64_t rows, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)pitch, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)pitch * 4};
  const cuuint32_t box[2] = {(cuuint32_t)kTileKeys, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// sfK [pages][hkv] fp32 as 2-D {hkv, pages}; box {hg, 1}
bool encode_sfk(CUtensorMap* tm, const float* ptr, int64_t pages, int hkv, int hg) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)hkv, (cuuint64_t)pages};
  const cuuint64_t strides[1] = {(cuuint64_t)hkv * 4};
  const cuuint32_t box[2] = {(cuuint32_t)hg, 1};
  const cuuint32_t estr[2] = {1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int HG, int G>
cudaError_t launch_sage_hg(SageLaunch& a, const int8_t* k8, const uint8_t* v8, int slots, cudaStream_t s) {
  using LS = SageSmem<HG, G, false>;
  using LV = SageSmem<HG, G, true>;
  static std::atomic<bool> score_set[kMaxDevices], value_set[kMaxDevices];
  cudaError_t e0 = raise_smem_limit(sage_score_kernel<HG, G>, LS::BYTES, score_set);
  if (e0 == cudaSuccess) e0 = raise_smem_limit(sage_value_kernel<HG, G>, LV::BYTES, value_set);
  if (e0 != cudaSuccess) return e0;
  const dim3 grid(slots * (a.hkv / HG));
  if (!encode_scores(&a.tm_s, a.ws.scores, a.ws.score_pitch, (int64_t)a.batch * a.hq, HG * G) ||
      !encode_pool(&a.tm_kv, k8, a.num_slots, a.hkv, HG) ||
      (HG >= 4 && !encode_sfk(&a.tm_sfk, a.sf_k, a.num_slots / kSageBlock, a.hkv, HG)))
    return cudaErrorInvalidValue;
  cudaError_t e = launch_pdl(sage_score_kernel<HG, G>, grid, dim3(kThreads), LS::BYTES, a, s);
  if (e != cudaSuccess) return e;
  if (!encode_pool(&a.tm_kv, v8, a.num_slots, a.hkv, HG)) return cudaErrorInvalidValue;
  e = launch_pdl(sage_value_kernel<HG, G>, grid, dim3(kThreads), LV::BYTES, a, s);
  if (e != cudaSuccess) return e;
  return launch_pdl(sage_merge_kernel, dim3((a.batch * a.hq + 7) / 8), dim3(256), 0, a, s);
}

template <int G>
cudaError_t launch_sage_g(SageLaunch& a, const int8_t* k8, const uint8_t* v8, int slots, cudaStream_t s) {
  switch (decode_heads_per_cta(a.hkv)) {
    case 8: return launch_sage_hg<8, G>(a, k8, v8, slots, s);
    case 4: return launch_sage_hg<4, G>(a, k8, v8, slots, s);
    case 2: return launch_sage_hg<2, G>(a, k8, v8, slots, s);
    default: return launch_sage_hg<1, G>(a, k8, v8, slots, s);
  }
}

}  // namespace

cudaError_t launch_sage(const SageLaunchArgs& in, cudaStream_t s) {
  SageLaunch a;
  a.ws = in.ws;
  a.q8 = in.q8;
  a.sf_q = in.sf_q;
  a.sf_k = in.sf_k;
  a.sf_v = in.sf_v;
  a.v_mean = in.v_mean;
  a.num_slots = in.num_slots;
  a.page_table = in.page_table;
  a.pt_pitch = in.pt_pitch;
  a.out = in.out;
  a.batch = in.batch;
  a.hq = in.hq;
  a.hkv = in.hkv;
  switch (in.hq / in.hkv) {
    case 1: return launch_sage_g<1>(a, in.k8, in.v8, in.slots, s);
    case 2: return launch_sage_g<2>(a, in.k8, in.v8, in.slots, s);
    case 4: return launch_sage_g<4>(a, in.k8, in.v8, in.slots, s);
    case 8: return launch_sage_g<8>(a, in.k8, in.v8, in.slots, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace pa
