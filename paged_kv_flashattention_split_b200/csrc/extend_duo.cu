// extend_duo.cu - bf16 causal EXTEND on a pair of CTAs that share every K/V tile through
// the tensor cores' two-SM form (tcgen05 cta_group::2).
//
// The operation is that of extend.cu: new token i of request r (absolute position
// p_r + i) attends to keys 0 .. p_r + i, O = softmax(scale Q K^T + causal mask) V,
// without the score matrix ever reaching HBM ("FlashAttention: 优化计算过程中的临时显存占用",
// sections 1-2; the forward modes of "Implement Flash Attention Back End in SGLang").
// This kernel serves head groups of 4 or 8 query heads per KV head.
//
// One cluster of two CTAs per (query tile of 128 new tokens, quad of query heads of one
// KV group): CTA rank c holds the 128-row query tiles of heads 4 q + 2 c and 4 q + 2 c + 1.
// Each MMA is issued once, by the rank-0 CTA, for M = 256 rows (the two CTAs' query tiles):
//     S_t = Q_t K^T   B = K tile, split by keys: rank c loads keys 64 c .. 64 c + 63
//     O_t += P_t V    B = V tile, split by d:    rank c loads d 64 c .. 64 c + 63
// so each SM loads a quarter of the K/V bytes the four heads use, half of what a CTA
// serving two heads alone would load.  Per CTA (10 warps):
//   warp 0      producer: Q once, then K/V key tiles into 3-stage rings, one TMA box
//               per page (K boxes complete on the rank-0 CTA's barrier, V boxes on this
//               CTA's own), or, for pages below 8 slots, 16-byte cp.async gathers of K that
//               the warp announces itself once they have landed (V is then gathered by an
//               eleventh warp, warp 10, the same way: one warp's gathers alone held the
//               slot-granular cache at half the rate);
//   warp 1      TMEM (512 columns: S_0, S_1, O_0, O_1) and, in the rank-0 CTA, the MMA
//               issuer;
//   warps 2-9   one softmax warpgroup per head: thread i owns query row i, reads S_t from
//               TMEM, tells the issuer at once that S_t is free (so S_t(j+1) runs on the
//               tensor cores during this tile's softmax), writes P_t (bf16) to shared
//               memory in the MMA's swizzled layout, and keeps a running max with a lazy
//               O rescale in TMEM.
// With P in shared memory instead of over S in TMEM, the next score tile no longer waits
// for this tile's PV: per head the chain is softmax(j) -> softmax(j + 1), and the tensor
// cores run S(j + 1) and PV(j) of both heads in its shadow.
//
// Every wait is bounded: on timeout the CTA records PA_ERR_DEVICE_INDEX, its roles stop,
// the issuer drains the tensor cores, and both CTAs meet at the final cluster barrier
// before TMEM is freed (neither exits while the other may still touch its memory).
#include "gather.cuh"
#include "kernels.h"
#include "tma.cuh"

namespace pa {
namespace {

constexpr int kThreads = 320;
constexpr int kThreadsGather = 352;               // + one warp that gathers V (page sizes below 8)
constexpr int kTileKeys = 128;
constexpr int kStages = 3;
constexpr int kQTile = 128 * 256;                    // 128 rows x 128 d bf16 = 32 KB (2 chunks of 64 d)
constexpr int kQChunk = 128 * 128;
constexpr int kKStage = 64 * 256;                    // this CTA's 64 keys x 128 d = 16 KB (2 chunks)
constexpr int kKChunk = 64 * 128;
constexpr int kVStage = 128 * 128;                   // 128 keys x this CTA's 64 d = 16 KB
constexpr int kPTile = 128 * 256;                    // 128 rows x 128 keys bf16 = 32 KB (2 chunks of 64 keys)
constexpr int kPChunk = 128 * 128;
constexpr uint32_t kTmemCols = 512;                  // S_0 [0,128), S_1 [128,256), O_0 [256,384), O_1 [384,512)
constexpr uint32_t kWaitLimit = 1u << 20;
constexpr float kLn2 = 0.693147180559945309f;
constexpr float kRescaleThreshold = 8.f;             // log2 units

constexpr int kOffQ = 0;                             // Q_0, Q_1
constexpr int kOffK = kOffQ + 2 * kQTile;
constexpr int kOffV = kOffK + kStages * kKStage;
constexpr int kOffP = kOffV + kStages * kVStage;     // P_0, P_1
constexpr int kOffBar = kOffP + 2 * kPTile;
constexpr int kSmemBytes = kOffBar + 256 + 1024;     // barriers, TMEM address, flag, alignment slack
static_assert(kSmemBytes <= 232448, "shared memory per CTA");

enum Bar {
  B_Q = 0,                          // (rank 0) both CTAs' Q tiles landed
  B_KFULL = 1,                      // [3] (rank 0) both CTAs' K halves landed (TMA bytes, or 2 gather arrivals)
  B_VLAND = B_KFULL + kStages,      // [3] this CTA's V half landed
  B_KEMPTY = B_VLAND + kStages,     // [3] S(j) done with the K stage (multicast to both CTAs)
  B_VEMPTY = B_KEMPTY + kStages,    // [3] PV(j) of both heads done with the V stage (multicast)
  B_SFULL = B_VEMPTY + kStages,     // [2] S_t in TMEM (multicast)
  B_SFREE = B_SFULL + 2,            // [2] (rank 0) both CTAs' softmax t read S_t: 8 warp arrivals
  B_PFULL = B_SFREE + 2,            // [2] (rank 0) both CTAs' P_t written: 8 warp arrivals
  B_PVDONE = B_PFULL + 2,           // [2] PV_t done: P_t free, O_t stable (multicast)
  B_DRAIN = B_PVDONE + 2,
  B_COUNT
};
static_assert(B_COUNT * 8 + 16 <= 256, "barrier area");

struct DuoLaunch {
  CUtensorMap tm_q, tm_k, tm_v;   // 64-byte aligned kernel parameters
  const uint16_t* k_pool;         // for the slot-by-slot gather (page sizes below 8)
  const uint16_t* v_pool;
  int gather;                     // 1: K/V halves by 16-byte cp.async gathers, 0: one TMA box per page
  WsView ws;
  const int32_t* page_table;
  int64_t pt_pitch;
  int64_t num_slots;
  uint16_t* out;
  float* lse_out;
  float scale_log2;
  int64_t q_rows;
  int hq, hkv, page_size, page_shift, box_k, box_v;
};

// ---------------------------------------------------------------- PTX helpers

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
  return r;
}
// Address in the shared::cluster window of the same shared-memory offset in CTA `rank`.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}
// Arrive on an mbarrier of either CTA of the cluster (`cluster_addr` in the shared::cluster
// window; the default release semantics, as for a local arrive).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];\n" ::"r"(cluster_addr) : "memory");
}
// Try-wait that acquires at cluster scope: the MMA issuer's barriers that count the peer
// CTA's arrivals and copies.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n.reg .pred p;\nmbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\nselp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Non-blocking test of a phase, acquiring at cluster scope (the issuer polls several barriers).
__device__ __forceinline__ bool mbar_test_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n.reg .pred p;\nmbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\nselp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;\n" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
// 4-D tiled load into this CTA's shared memory completing on an mbarrier of either CTA of
// the pair (`bar` in the shared::cluster window).  No multicast.
__device__ __forceinline__ void tma_load_4d_pair(uint32_t dst, const CUtensorMap* tm, int c0, int c1, int c2, int c3,
                                                 uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], [%6];\n"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(tm)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
      : "memory");
}

// smem matrix descriptor: 128B swizzle, 8-row groups 1024 B apart (SBO), LBO as given
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo_bytes) {
  return (uint64_t)((addr & 0x3FFFF) >> 4) | ((uint64_t)(lbo_bytes >> 4) << 16) | ((uint64_t)(1024 >> 4) << 32) |
         (1ull << 46) | (2ull << 61);
}
// D (TMEM of both CTAs) (+)= A (shared, both CTAs) x B (shared, half of N in each CTA)
__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\ntcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n}\n"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on the mbarrier at `bar`'s offset in both CTAs once this thread's MMAs are done.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;\n"
      ::"r"(bar), "h"((uint16_t)0x3)
      : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
        "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
        "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&v)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
               : "r"(taddr));
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&v)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};\n"
               ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }

// instruction descriptor, kind::f16: bf16 A and B, fp32 D, M = 256 (the pair), N = 128
constexpr uint32_t kIdescBase = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((256u >> 4) << 24);
constexpr uint32_t kIdescS = kIdescBase;                 // A (Q) and B (K) K-major
constexpr uint32_t kIdescPV = kIdescBase | (1u << 16);   // A (P) K-major, B (V) MN-major: d contiguous

// GATHER: the page-size-below-8 path (cp.async gathers); a separate instantiation, so the TMA
// path's register allocation carries none of the gather code.
template <bool GATHER>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(GATHER ? kThreadsGather : kThreads, 1)
    extend_duo_kernel(const __grid_constant__ DuoLaunch a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  const uint32_t bars = base + kOffBar;
  auto bar = [&](int i) -> uint32_t { return bars + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + kOffBar + 8 * B_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base_ptr + kOffBar + 8 * B_COUNT + 8);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  PlanHeader* hdr = a.ws.hdr;
  // both CTAs of a cluster take the same early exits (they share the work item)
  if (hdr->magic != kMagic || hdr->mode != PA_MODE_EXTEND) {
    if (tid == 0 && blockIdx.x == 0) set_device_error(hdr, PA_ERR_WORKSPACE);
    return;
  }
  const int quads = a.hq / 4;
  const int pair = blockIdx.x >> 1;
  const int item = pair / quads, quad = pair % quads;
  if (item >= hdr->num_items) return;
  const int4 it = a.ws.items[item];
  const int r = it.x, q_begin = it.z, q_end = it.w;
  const int L = a.ws.req_len[r], prefix = a.ws.req_prefix[r], q_start = a.ws.req_aux[r];
  const int h0 = 4 * quad + 2 * (int)rank;                   // this CTA's heads h0, h0 + 1
  const int h_kv = (4 * quad) / (a.hq / a.hkv);
  const int kv_end = prefix + q_end;
  const int n_kv = (kv_end + kTileKeys - 1) / kTileKeys;

  if (tid == 0) {
    for (int i = 0; i < B_COUNT; ++i) {
      const bool warp_arrivals = (i >= B_SFREE && i < B_SFREE + 2) || (i >= B_PFULL && i < B_PFULL + 2);
      const bool gathered_k = GATHER && i >= B_KFULL && i < B_KFULL + kStages;
      mbar_init(bar(i), warp_arrivals ? 8u : gathered_k ? 2u : 1u);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;\n"
                 ::"r"(smem_u32(tmem_slot)), "r"(kTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;\n" ::: "memory");
  }
  tc_fence_before();
  cluster_sync();                                             // barriers of both CTAs initialised
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // bounded waits: `wait` for barriers completed by this CTA's own copies and arrivals or by the
  // issuer's commits, `wait_cl` (cluster-scope acquire) for the issuer's barriers that count the
  // peer CTA's copies and arrivals
  auto wait_impl = [&](uint32_t b, uint32_t parity, bool cluster) -> bool {
    for (uint32_t i = 0; i < kWaitLimit; ++i) {
      if (cluster ? mbar_try_wait_cluster(b, parity) : mbar_try_wait(b, parity)) return true;
      if (*abort_flag) return false;
    }
    *abort_flag = 1;
    set_device_error(hdr, PA_ERR_DEVICE_INDEX);
    return false;
  };
  auto wait = [&](uint32_t b, uint32_t parity) -> bool { return wait_impl(b, parity, false); };
  auto wait_cl = [&](uint32_t b, uint32_t parity) -> bool { return wait_impl(b, parity, true); };
  auto stage_parity = [](int j) -> uint32_t { return (uint32_t)(j / kStages) & 1u; };
  // keys of tile j: [128 j, 128 j + 128) clipped to L; this CTA's K half starts 64 rank further
  auto tile_keys = [&](int j) { return min(kTileKeys, L - j * kTileKeys); };
  auto half_keys = [&](int j, int c) { return max(0, min(64, L - j * kTileKeys - 64 * c)); };

  if (warp == 0) {
    // ------------------------------------------------------------ producer (whole warp)
    const int32_t* table = a.page_table + (size_t)r * a.pt_pitch;
    const uint32_t lead_q = map_to_rank(bar(B_Q), 0);
    if (lane == 0) {
      if (leader) mbar_expect_tx(bar(B_Q), 2u * 2u * kQTile);  // both CTAs' two query tiles
      const int row0 = q_start + q_begin;
      for (int t = 0; t < 2; ++t)
        for (int ch = 0; ch < 2; ++ch)
          tma_load_4d_pair(base + kOffQ + t * kQTile + ch * kQChunk, &a.tm_q, 0, row0, ch, h0 + t, lead_q);
    }
    // slot of the first row of box `o` (box_rows rows) starting `key0` keys into the request
    auto box_slot = [&](int key0, int o, int box_rows) -> int {
      const int key = key0 + o * box_rows;
      const int page = __ldg(table + (key >> a.page_shift));
      const long long slot = ((long long)page << a.page_shift) + (key & (a.page_size - 1));
      if (page < 0 || slot + box_rows > a.num_slots) {         // keep the copy in bounds, flag the id
        set_device_error(hdr, PA_ERR_DEVICE_INDEX);
        return 0;
      }
      return (int)slot;
    };
    int issued = 0;
    if (GATHER) {
      // the copies complete on no barrier, so the warp announces them: once K(j) is issued it
      // waits for K(j - 1)'s copies, fences them for the tensor cores (async proxy) and arrives
      // on the rank-0 CTA's KFULL (V is gathered the same way by warp 10, on this CTA's VLAND).
      for (int j = 0; j < n_kv; ++j) {
        const int s = j % kStages;
        const int nk = half_keys(j, (int)rank);
        bool ok = true;
        if (lane == 0) ok = j < kStages || wait(bar(B_KEMPTY + s), stage_parity(j) ^ 1u);
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        gather_rows<2, 64>(base + kOffK + s * kKStage, kKChunk, 0, a.k_pool, table, j * kTileKeys + 64 * (int)rank, nk,
                       (nk + 15) & ~15, a.page_shift, a.page_size, a.hkv, h_kv, a.num_slots, hdr, lane);
        cp_async_commit();
        if (j > 0) {
          cp_async_wait<1>();
          fence_proxy_async();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(map_to_rank(bar(B_KFULL + (j - 1) % kStages), 0));
        }
        issued = j + 1;
      }
      cp_async_wait<0>();
      fence_proxy_async();
      __syncwarp();
      if (lane == 0 && issued > 0) mbar_arrive_cluster(map_to_rank(bar(B_KFULL + (issued - 1) % kStages), 0));
      issued = 0;                                                // nothing left in flight
    }
    for (int j = 0; !GATHER && j < n_kv; ++j) {
      const int s = j % kStages;
      // K: this CTA's 64-key half, one box per page (box_k rows), both d chunks
      const int kk0 = j * kTileKeys + 64 * (int)rank;
      const int ops_k = (half_keys(j, (int)rank) + a.box_k - 1) / a.box_k;
      const int kslot = lane < ops_k ? box_slot(kk0, lane, a.box_k) : 0;
      bool ok = true;
      if (lane == 0) {
        ok = j < kStages || wait(bar(B_KEMPTY + s), stage_parity(j) ^ 1u);
        if (ok && leader) {
          const int ops_all = (half_keys(j, 0) + a.box_k - 1) / a.box_k + (half_keys(j, 1) + a.box_k - 1) / a.box_k;
          mbar_expect_tx(bar(B_KFULL + s), (uint32_t)ops_all * a.box_k * 256u);
        }
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      const uint32_t lead_k = map_to_rank(bar(B_KFULL + s), 0);
      if (lane < ops_k)
        for (int ch = 0; ch < 2; ++ch)
          tma_load_4d_pair(base + kOffK + s * kKStage + ch * kKChunk + lane * a.box_k * 128, &a.tm_k, 0, kslot, ch,
                           h_kv, lead_k);
      // V: all 128 keys of the tile, this CTA's 64 d (chunk = rank), one box per page (box_v rows)
      const int ops_v = (tile_keys(j) + a.box_v - 1) / a.box_v;
      const int vslot = lane < ops_v ? box_slot(j * kTileKeys, lane, a.box_v) : 0;
      if (lane == 0) {
        ok = j < kStages || wait(bar(B_VEMPTY + s), stage_parity(j) ^ 1u);
        if (ok) mbar_expect_tx(bar(B_VLAND + s), (uint32_t)ops_v * a.box_v * 128u);
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      if (lane < ops_v)
        tma_load_4d(base + kOffV + s * kVStage + lane * a.box_v * 128, &a.tm_v, 0, vslot, (int)rank, h_kv,
                    bar(B_VLAND + s));
      issued = j + 1;
    }
    // copies still in flight when the CTA gives up: wait (bounded) until they land
    if (lane == 0 && *abort_flag) {
      for (int j = max(0, issued - kStages); j < issued; ++j) {
        if (leader)
          for (uint32_t i = 0; i < kWaitLimit && !mbar_try_wait_cluster(bar(B_KFULL + j % kStages), stage_parity(j)); ++i) {}
        for (uint32_t i = 0; i < kWaitLimit && !mbar_try_wait(bar(B_VLAND + j % kStages), stage_parity(j)); ++i) {}
      }
    }
  } else if (GATHER && warp == 10) {
    // ------------------------------------------------------------ V gathers (page sizes below 8)
    const int32_t* table = a.page_table + (size_t)r * a.pt_pitch;
    int vissued = 0;
    for (int j = 0; j < n_kv; ++j) {
      const int s = j % kStages;
      const int nv = tile_keys(j);
      bool ok = true;
      if (lane == 0) ok = j < kStages || wait(bar(B_VEMPTY + s), stage_parity(j) ^ 1u);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      gather_rows<1, 128>(base + kOffV + s * kVStage, kVStage, (int)rank, a.v_pool, table, j * kTileKeys, nv,
                          (nv + 15) & ~15, a.page_shift, a.page_size, a.hkv, h_kv, a.num_slots, hdr, lane);
      cp_async_commit();
      if (j > 0) {
        cp_async_wait<1>();
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_VLAND + (j - 1) % kStages));
      }
      vissued = j + 1;
    }
    cp_async_wait<0>();
    fence_proxy_async();
    __syncwarp();
    if (lane == 0 && vissued > 0) mbar_arrive(bar(B_VLAND + (vissued - 1) % kStages));
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (rank 0 only)
    if (leader && lane == 0) {
      auto issue_s = [&](int t, int j) {                         // S_t = Q_t K(j)^T, M = 256
        const uint32_t qb = base + kOffQ + t * kQTile;
        const uint32_t kb = base + kOffK + (j % kStages) * kKStage;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {                          // 8 steps of 16 over d
          tc_mma_pair(tmem + 128 * t, smem_desc(qb + (kk >> 2) * kQChunk + (kk & 3) * 32, 16),
                      smem_desc(kb + (kk >> 2) * kKChunk + (kk & 3) * 32, 16), kIdescS, kk > 0);
        }
        tc_commit_pair(bar(B_SFULL + t));
      };
      auto issue_pv = [&](int t, int j) {                        // O_t += P_t V(j), M = 256
        const int nsteps = (tile_keys(j) + 15) / 16;              // 16-key steps that hold live keys
        const uint32_t pb = base + kOffP + t * kPTile;
        const uint32_t vb = base + kOffV + (j % kStages) * kVStage;
        for (int kk = 0; kk < nsteps; ++kk)
          tc_mma_pair(tmem + 256 + 128 * t, smem_desc(pb + (kk >> 2) * kPChunk + (kk & 3) * 32, 16),
                      smem_desc(vb + kk * 16 * 128, kVStage), kIdescPV, (j > 0 || kk > 0) ? 1u : 0u);
        tc_commit_pair(bar(B_PVDONE + t));
      };
      bool ok = wait_cl(bar(B_Q), 0) && wait_cl(bar(B_KFULL), 0);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        issue_s(1, 0);
        tc_commit_pair(bar(B_KEMPTY));
      }
      // Event-driven issue: each head's next S (needs its K tile and both CTAs' softmax to have
      // read the previous S) and next PV (needs both CTAs' P) go to the tensor cores as soon as
      // they are ready, so one head's softmax never holds up the other head's MMAs.  A K stage
      // is released once both heads' S of that tile are issued, a V stage once both PVs are.
      int ns[2] = {1, 1}, npv[2] = {0, 0}, k_rel = 1, v_rel = 0;
      uint32_t idle = 0;
      while (ok && (npv[0] < n_kv || npv[1] < n_kv)) {
        bool progress = false;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (npv[t] < n_kv && mbar_test_wait_cluster(bar(B_PFULL + t), (uint32_t)npv[t] & 1u)) {
            tc_fence_after();
            issue_pv(t, npv[t]++);
            progress = true;
          }
          if (ns[t] < n_kv && mbar_test_wait_cluster(bar(B_SFREE + t), (uint32_t)(ns[t] - 1) & 1u) &&
              mbar_test_wait_cluster(bar(B_KFULL + ns[t] % kStages), stage_parity(ns[t]))) {
            tc_fence_after();
            issue_s(t, ns[t]++);
            progress = true;
          }
        }
        while (k_rel < n_kv && ns[0] > k_rel && ns[1] > k_rel) tc_commit_pair(bar(B_KEMPTY + (k_rel++) % kStages));
        while (v_rel < n_kv && npv[0] > v_rel && npv[1] > v_rel) tc_commit_pair(bar(B_VEMPTY + (v_rel++) % kStages));
        if (progress) {
          idle = 0;
        } else if (++idle > 4 * kWaitLimit || *abort_flag) {
          if (!*abort_flag) {
            *abort_flag = 1;
            set_device_error(hdr, PA_ERR_DEVICE_INDEX);
          }
          ok = false;
        } else {
          __nanosleep(32);
        }
      }
      // all issued tensor-core work has finished before TMEM is released
      tc_commit_pair(bar(B_DRAIN));
      for (uint32_t i = 0; i < kWaitLimit && !mbar_try_wait(bar(B_DRAIN), 0); ++i) {}
    }
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    const int t = (warp - 2) >> 2;                              // head h0 + t of this CTA
    const int h = h0 + t;
    const int row = 32 * (warp & 3) + lane;                    // TMEM lane = query row of the tile
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t tmem_s = tmem + 128 * t, tmem_o = tmem + 256 + 128 * t;
    const int q_local = q_begin + row;
    const bool row_valid = q_local < q_end && q_start + q_local < a.q_rows;   // never store past the O buffer
    const int limit = row_valid ? prefix + q_local : L - 1;    // last visible key (inclusive)
    const float NEG_INF = -__int_as_float(0x7f800000);
    const float c = a.scale_log2;                              // > 0: the max commutes with the scale
    const uint32_t lead_sfree = map_to_rank(bar(B_SFREE + t), 0);
    const uint32_t lead_pfull = map_to_rank(bar(B_PFULL + t), 0);
    uint8_t* prow_base = base_ptr + kOffP + t * kPTile;
    float m_used = NEG_INF, l = 0.f;
    bool ok = true;
    // tcgen05.ld/st are warp-collective: every wait result is made uniform across the warp
    auto wwait = [&](uint32_t b, uint32_t parity) { return __all_sync(0xffffffffu, wait(b, parity)) != 0; };
    for (int j = 0; j < n_kv && ok; ++j) {
      if (!(ok = wwait(bar(B_SFULL + t), (uint32_t)j & 1u))) break;
      tc_fence_after();
      uint32_t sv[4][32];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) tmem_ld32(tmem_s + lane_off + 32 * cc, sv[cc]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(lead_sfree);         // S_t may be overwritten by S_t(j + 1)
      // raw-score row max, causal mask on tiles that reach past this tile's first row
      const int key0 = j * kTileKeys;
      const bool diag = key0 + kTileKeys - 1 > prefix + q_begin || key0 + kTileKeys > L;
      if (diag) {
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (key0 + 32 * cc + e > limit) sv[cc][e] = __float_as_uint(NEG_INF);
      }
      // row max over four independent 3-input chains
      float mxp[4] = {NEG_INF, NEG_INF, NEG_INF, NEG_INF};
#pragma unroll
      for (int cc = 0; cc < 4; ++cc)
#pragma unroll
        for (int e = 0; e < 32; e += 2)
          mxp[cc] = max3(mxp[cc], __uint_as_float(sv[cc][e]), __uint_as_float(sv[cc][e + 1]));
      float mx = max3(mxp[0], mxp[1], fmaxf(mxp[2], mxp[3]));
      mx *= c;                                                  // log2 units
      float alpha = 1.f;
      if (m_used == NEG_INF) {
        m_used = mx;
      } else if (mx > m_used + kRescaleThreshold) {
        alpha = ex2(m_used - mx);
        m_used = mx;
      }
      // P = 2^(c s - m) packed to bf16 pairs (in the low half of each 32-register row); the row sum
      // adds the same bf16-rounded values the PV MMA multiplies, so O is a convex combination of V
      // rows whatever the rounding of P
      const float neg_m = m_used == NEG_INF ? 0.f : -m_used;
      const float2 c2 = make_float2(c, c), nm2 = make_float2(neg_m, neg_m);
      float2 lsum[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int cc = 0; cc < 4; ++cc)
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const float2 x = __ffma2_rn(make_float2(__uint_as_float(sv[cc][e]), __uint_as_float(sv[cc][e + 1])), c2, nm2);
          const uint32_t w = pack_bf16x2(ex2(x.x), ex2(x.y));
          lsum[(e >> 1) & 3] = __fadd2_rn(lsum[(e >> 1) & 3], make_float2(bf16lo_to_f32(w), bf16hi_to_f32(w)));
          sv[cc][e >> 1] = w;
        }
      const float2 ls = __fadd2_rn(__fadd2_rn(lsum[0], lsum[1]), __fadd2_rn(lsum[2], lsum[3]));
      const float lt = ls.x + ls.y;
      // PV_t(j-1) done: the P_t buffer is free and O_t holds every earlier tile
      if (j > 0 && !(ok = wwait(bar(B_PVDONE + t), (uint32_t)(j - 1) & 1u))) break;
      if (__any_sync(0xffffffffu, alpha != 1.f)) {              // rescale rows of O_t in TMEM
        tc_fence_after();
#pragma unroll 1
        for (int cc = 0; cc < 16; ++cc) {                        // 8 columns at a time keeps registers low
          uint32_t ov[8];
          tmem_ld8(tmem_o + lane_off + 8 * cc, ov);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 8; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
          tmem_st8(tmem_o + lane_off + 8 * cc, ov);
        }
        tmem_wait_st();
      }
      l = l * alpha + lt;
      // P_t (K-major over keys, 128-byte swizzle): row `row`, keys 0-63 in chunk 0, 64-127 in chunk 1
#pragma unroll
      for (int u = 0; u < 16; ++u) {                             // 16-byte units of 8 keys
        const int p0 = 4 * u;                                    // packed pair index: keys 2 p0 ..
        const uint32_t w0 = sv[p0 >> 4][p0 & 15], w1 = sv[(p0 + 1) >> 4][(p0 + 1) & 15];
        const uint32_t w2 = sv[(p0 + 2) >> 4][(p0 + 2) & 15], w3 = sv[(p0 + 3) >> 4][(p0 + 3) & 15];
        const int chunk = u >> 3, unit = u & 7;
        *reinterpret_cast<uint4*>(prow_base + chunk * kPChunk + row * 128 + ((unit ^ (row & 7)) << 4)) =
            make_uint4(w0, w1, w2, w3);
      }
      // this CTA's V half of tile j has landed; rows past L inside the last 16-key step must read
      // as zero.  Either head's PV(j) may run first, so the first warp of each warpgroup writes the
      // same zeros before its own P_FULL arrival.
      if (!(ok = wwait(bar(B_VLAND + j % kStages), stage_parity(j)))) break;
      const int nk = tile_keys(j);
      if ((warp & 3) == 2 && nk < kTileKeys && (nk & 15)) {
        uint8_t* vt = base_ptr + kOffV + (j % kStages) * kVStage;
        const int z0 = nk, z1 = (nk + 15) & ~15;
        for (int idx = lane; idx < (z1 - z0) * 8; idx += 32) {   // 16-byte units of rows z0 .. z1 - 1
          const int rr = z0 + idx / 8, un = idx & 7;
          *reinterpret_cast<uint4*>(vt + rr * 128 + un * 16) = make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async();                                       // P (and zeroed V rows) before the MMA reads
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(lead_pfull);
    }
    // every PV of this head has finished
    if (ok) ok = wwait(bar(B_PVDONE + t), (uint32_t)(n_kv - 1) & 1u);
    if (ok) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      uint16_t* orow = a.out + ((size_t)(q_start + q_local) * a.hq + h) * kHeadDim;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t ov[32];
        tmem_ld32(tmem_o + lane_off + 32 * cc, ov);
        tmem_wait_ld();
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(ov[8 * g + 0]) * inv, __uint_as_float(ov[8 * g + 1]) * inv);
          w.y = pack_bf16x2(__uint_as_float(ov[8 * g + 2]) * inv, __uint_as_float(ov[8 * g + 3]) * inv);
          w.z = pack_bf16x2(__uint_as_float(ov[8 * g + 4]) * inv, __uint_as_float(ov[8 * g + 5]) * inv);
          w.w = pack_bf16x2(__uint_as_float(ov[8 * g + 6]) * inv, __uint_as_float(ov[8 * g + 7]) * inv);
          if (row_valid) *reinterpret_cast<uint4*>(orow + 32 * cc + 8 * g) = w;
        }
      }
      if (a.lse_out && row_valid)
        a.lse_out[(size_t)(q_start + q_local) * a.hq + h] = l > 0.f ? (m_used + __log2f(l)) * kLn2 : NEG_INF;
    }
  }
  // neither CTA leaves (or frees TMEM) while the other may still read its shared memory,
  // arrive on its barriers or run MMAs into its TMEM
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// [rows][heads][128] bf16 viewed as 4-D {64 d, rows, 2 halves of d, heads}; box {64, box_rows, 1, 1}
bool encode_rows(CUtensorMap* tm, const void* ptr, int64_t rows, int heads, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {64, (cuuint64_t)rows, 2, (cuuint64_t)heads};
  const cuuint64_t strides[3] = {(cuuint64_t)heads * 256, 128, 256};
  const cuuint32_t box[4] = {64, (cuuint32_t)box_rows, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_extend_duo(const ExtendArgs& in, cudaStream_t s) {
  static std::atomic<bool> smem_set[kMaxDevices], smem_set_g[kMaxDevices];
  cudaError_t e = in.page_size < 8 ? raise_smem_limit(extend_duo_kernel<true>, kSmemBytes, smem_set_g)
                                   : raise_smem_limit(extend_duo_kernel<false>, kSmemBytes, smem_set);
  if (e != cudaSuccess) return e;
  DuoLaunch a;
  a.gather = in.page_size < 8 ? 1 : 0;
  a.k_pool = in.k_pool;
  a.v_pool = in.v_pool;
  const int box_k = in.page_size < 64 ? in.page_size : 64;
  const int box_v = in.page_size < kTileKeys ? in.page_size : kTileKeys;
  if (!encode_rows(&a.tm_q, in.q, in.q_rows, in.hq, 128) ||
      (!a.gather && (!encode_rows(&a.tm_k, in.k_pool, in.num_slots, in.hkv, box_k) ||
                     !encode_rows(&a.tm_v, in.v_pool, in.num_slots, in.hkv, box_v))))
    return cudaErrorInvalidValue;
  a.ws = in.ws;
  a.page_table = in.page_table;
  a.pt_pitch = in.pt_pitch;
  a.num_slots = in.num_slots;
  a.out = in.out;
  a.lse_out = in.lse_out;
  a.scale_log2 = in.scale_log2;
  a.q_rows = in.q_rows;
  a.hq = in.hq;
  a.hkv = in.hkv;
  a.page_size = in.page_size;
  a.page_shift = in.page_shift;
  a.box_k = box_k;
  a.box_v = box_v;
  if (a.gather)
    extend_duo_kernel<true><<<in.max_items * (in.hq / 4) * 2, kThreadsGather, kSmemBytes, s>>>(a);
  else
    extend_duo_kernel<false><<<in.max_items * (in.hq / 4) * 2, kThreads, kSmemBytes, s>>>(a);
  return cudaGetLastError();
}

}  // namespace pa
