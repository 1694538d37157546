// extend.cu - bf16 causal EXTEND over the paged cache on the 5th-generation tensor cores.
//
// New token i of request r (absolute position p_r + i) attends to keys
// 0 .. p_r + i of its cached prefix and of the new tokens, all already in the
// pool: O = softmax(scale Q K^T + causal mask) V.  The tiled online softmax
// gives the standard result without the score matrix ever reaching HBM
// ("FlashAttention: 优化计算过程中的临时显存占用", sections 1-2); the two
// forward modes are those of "Implement Flash Attention Back End in SGLang".
//
// One CTA per (query tile of 128 new tokens, query head), 6 warps:
//   warp 0      producer: TMA loads of the Q tile once and of K/V key tiles
//               (128 keys, i.e. 128 / P pages) into 2-stage rings, each page
//               one box of a 4-D tensor map over the pool [slot][head][d];
//               lane o reads box o's page id one tile ahead, and a K stage is
//               refilled as soon as its S MMA is done (a V stage after its PV);
//   warp 1      allocates TMEM and issues, from one thread,
//                   S  = Q K^T   (tcgen05.mma kind::f16, M 128, N 128, S in TMEM)
//                   O += P V     (P from shared memory, O accumulated in TMEM);
//   warps 2-5   softmax: thread i owns query row i (TMEM lane i), reads its
//               128 scores with tcgen05.ld, applies the causal mask on the
//               diagonal tiles, keeps a running max (rescaling O in TMEM only
//               when the max grows by more than 2^8) and writes P (bf16) to
//               one of two shared-memory buffers in the MMA's swizzled layout,
//               so P(j+1) is written while PV(j) reads P(j); at the end it
//               normalises its O row and stores it.
// The issue order S(0), then per tile S(j+1) before PV(j), lets the tensor
// cores compute the next scores while the softmax works on the current ones.
// Key tiles past the last one any row of the query tile can see are never
// loaded (causal tile skipping).
//
// Every wait on an mbarrier is bounded: on timeout the CTA records
// PA_ERR_DEVICE_INDEX in the workspace, every role stops, the MMA issuer
// drains its tensor-core work, and TMEM is freed before the CTA exits.
#include "gather.cuh"
#include "kernels.h"
#include "tma.cuh"

namespace pa {
namespace {

constexpr int kThreads = 192;
constexpr int kTileKeys = 128;
constexpr int kNumStages = 2;
constexpr int kChunkBytes = 128 * 128;           // one 64-column half of a 128 x 128 bf16 tile
constexpr int kTileBytes = 2 * kChunkBytes;      // 32 KB
constexpr uint32_t kTmemCols = 256;              // S: columns [0,128), O: [128, 256)
constexpr uint32_t kWaitLimit = 1u << 20;
constexpr float kLn2 = 0.693147180559945309f;
constexpr float kRescaleThreshold = 8.f;         // log2 units

// shared-memory plan (offsets from a 1024-aligned base)
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kTileBytes;
constexpr int kOffV = kOffK + kNumStages * kTileBytes;
constexpr int kOffP = kOffV + kNumStages * kTileBytes;   // two P buffers
constexpr int kOffBar = kOffP + 2 * kTileBytes;
constexpr int kSmemBytes = kOffBar + 256 + 1024;  // barriers, TMEM address, flags, alignment slack

struct ExtendLaunch {
  CUtensorMap tm_q, tm_k, tm_v;   // 64-byte aligned kernel parameters
  const uint16_t* k_pool;         // for the slot-by-slot gather (page sizes below 8)
  const uint16_t* v_pool;
  int gather;                     // 1: K/V tiles by 16-byte cp.async gathers, 0: one TMA box per page
  WsView ws;
  const int32_t* page_table;
  int64_t pt_pitch;
  int64_t num_slots;
  uint16_t* out;
  float* lse_out;
  float scale_log2;
  int64_t q_rows;
  int hq, hkv, page_size, page_shift, box_rows, max_items;
};

// ---------------------------------------------------------------- PTX helpers

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }

// smem matrix descriptor: 128B swizzle, 8-row groups 1024 B apart (SBO), LBO as given
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo_bytes) {
  return (uint64_t)((addr & 0x3FFFF) >> 4) | ((uint64_t)(lbo_bytes >> 4) << 16) | ((uint64_t)(1024 >> 4) << 32) |
         (1ull << 46) | (2ull << 61);
}
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\ntcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar) : "memory");
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
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n"
      ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]),
        "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]),
        "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
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
// stores v[0..15] (the packed half of a 32-register row)
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n"
      ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}
// D (TMEM) += A (TMEM, K-major bf16 pairs) x B (shared memory descriptor)
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\ntcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }

// instruction descriptor, kind::f16: bf16 A and B, fp32 D, M = 128, N = 128
constexpr uint32_t kIdescBase = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescS = kIdescBase;                 // A (Q) and B (K) K-major
constexpr uint32_t kIdescPV = kIdescBase | (1u << 16);   // B (V) MN-major: d contiguous

// mbarriers, 8 bytes each, in this order after the tile buffers
enum Bar {
  B_Q = 0,
  B_K_FULL = 1,                       // [2] K tile landed
  B_V_FULL = B_K_FULL + kNumStages,   // [2] V tile landed
  B_K_EMPTY = B_V_FULL + kNumStages,  // [2] S MMA done with the K stage
  B_V_EMPTY = B_K_EMPTY + kNumStages, // [2] PV MMA done with the V stage
  B_S_FULL = B_V_EMPTY + kNumStages,  // S in TMEM
  B_S_FREE,                           // softmax has read S (128 arrivals)
  B_P_FULL,                           // [2] P buffer written (128 arrivals)
  B_P_FREE = B_P_FULL + 2,            // [2] PV(j) finished (P buffer j % 2 free, O stable)
  B_DRAIN = B_P_FREE + 2,
  B_COUNT
};
static_assert(B_COUNT * 8 + 16 <= 256, "barrier area");

// Producer warp, page sizes below 8: K and V tiles of 128 keys gathered slot by slot with
// cp.async into the same [2 chunks][128 rows][128 B] layout the TMA boxes produce.  The
// copies complete on no barrier, so the warp announces them itself: once K(j) is issued it
// waits for K(j - 1)'s copies, fences them for the tensor cores (async proxy) and arrives on
// K_FULL(j - 1); the same for V after V(j) is issued.  K's announcement never waits for a V
// stage (the MMA issuer needs K(j) before it can finish with V(j - 1)).  Rows past the
// request's end, up to the 16-key step the MMAs read, are zero-filled.
template <typename WaitFn>
__device__ __forceinline__ void produce_gathered(const ExtendLaunch& a, const int32_t* table, int L, int n_kv,
                                                 int h_kv, uint32_t k_base, uint32_t v_base, uint32_t bar_kfull,
                                                 uint32_t bar_vfull, uint32_t bar_kempty, uint32_t bar_vempty,
                                                 int lane, WaitFn&& wait) {
  constexpr int kTileBytes = 2 * 128 * 128;
  // copy groups are committed in the order K(0), V(0), K(1), V(1), ...
  auto announce = [&](uint32_t full_bar, int tile) {
    cp_async_wait<2>();                           // all but the two newest groups have landed
    fence_proxy_async();
    __syncwarp();
    if (lane == 0) mbar_arrive(full_bar + 8u * (tile & 1));
  };
  int issued = 0;
  for (int j = 0; j < n_kv; ++j) {
    const int s = j & 1;
    const uint32_t par = ((uint32_t)(j >> 1) & 1u) ^ 1u;
    const int nk = min(128, L - j * 128);
    const int pad = (nk + 15) & ~15;
    bool ok = true;
    if (lane == 0) ok = j < 2 || wait(bar_kempty + 8u * s, par);
    if (!__shfl_sync(0xffffffffu, ok, 0)) break;
    gather_rows<2, 128>(k_base + s * kTileBytes, 128 * 128, 0, a.k_pool, table, j * 128, nk, pad, a.page_shift,
                   a.page_size, a.hkv, h_kv, a.num_slots, a.ws.hdr, lane);
    cp_async_commit();
    if (j > 0) announce(bar_kfull, j - 1);        // groups after K(j - 1): V(j - 1), K(j)
    if (lane == 0) ok = j < 2 || wait(bar_vempty + 8u * s, par);
    if (!__shfl_sync(0xffffffffu, ok, 0)) break;
    gather_rows<2, 128>(v_base + s * kTileBytes, 128 * 128, 0, a.v_pool, table, j * 128, nk, pad, a.page_shift,
                   a.page_size, a.hkv, h_kv, a.num_slots, a.ws.hdr, lane);
    cp_async_commit();
    if (j > 0) announce(bar_vfull, j - 1);        // groups after V(j - 1): K(j), V(j)
    issued = j + 1;
  }
  cp_async_wait<0>();
  fence_proxy_async();
  __syncwarp();
  if (lane == 0 && issued > 0) {
    mbar_arrive(bar_kfull + 8u * ((issued - 1) & 1));
    mbar_arrive(bar_vfull + 8u * ((issued - 1) & 1));
  }
}

__global__ void __launch_bounds__(kThreads, 1) extend_kernel(const __grid_constant__ ExtendLaunch a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  const uint32_t bars = base + kOffBar;
  auto bar = [&](int i) -> uint32_t { return bars + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + kOffBar + 8 * B_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base_ptr + kOffBar + 8 * B_COUNT + 8);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  PlanHeader* hdr = a.ws.hdr;
  if (hdr->magic != kMagic || hdr->mode != PA_MODE_EXTEND) {
    if (tid == 0 && blockIdx.x == 0) set_device_error(hdr, PA_ERR_WORKSPACE);
    return;
  }
  const int item = blockIdx.x / a.hq, h = blockIdx.x % a.hq;
  if (item >= hdr->num_items) return;
  const int4 it = a.ws.items[item];
  const int r = it.x, q_begin = it.z, q_end = it.w;
  const int L = a.ws.req_len[r], prefix = a.ws.req_prefix[r], q_start = a.ws.req_aux[r];
  const int h_kv = h / (a.hq / a.hkv);
  const int kv_end = prefix + q_end;                          // keys any row of this tile can see
  const int n_kv = (kv_end + kTileKeys - 1) / kTileKeys;

  if (tid == 0) {
    for (int i = 0; i < B_COUNT; ++i) mbar_init(bar(i), (i == B_S_FREE || i == B_P_FULL || i == B_P_FULL + 1) ? 128 : 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n"
                 ::"r"(smem_u32(tmem_slot)), "r"(kTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_s = tmem, tmem_o = tmem + 128;

  // bounded wait: false (and the CTA-wide abort flag set) if the barrier never completes
  auto wait = [&](uint32_t b, uint32_t parity) -> bool {
    for (uint32_t i = 0; i < kWaitLimit; ++i) {
      if (mbar_try_wait(b, parity)) return true;
      if (*abort_flag) return false;
    }
    *abort_flag = 1;
    set_device_error(hdr, PA_ERR_DEVICE_INDEX);
    return false;
  };
  // key tile j: keys [128 j, 128 j + 128) clipped to L
  auto tile_keys = [&](int j) { return min(kTileKeys, L - j * kTileKeys); };
  // parity of the completion of a 2-deep ring barrier that tile j waits for / releases
  auto ring_parity = [](int j) -> uint32_t { return (uint32_t)(j >> 1) & 1u; };

  if (warp == 0) {
    // ------------------------------------------------------------ producer (whole warp)
    const int32_t* table = a.page_table + (size_t)r * a.pt_pitch;
    if (lane == 0) {
      mbar_expect_tx(bar(B_Q), 2 * kChunkBytes);
      const int row0 = q_start + q_begin;
      tma_load_4d(base + kOffQ, &a.tm_q, 0, row0, 0, h, bar(B_Q));
      tma_load_4d(base + kOffQ + kChunkBytes, &a.tm_q, 0, row0, 1, h, bar(B_Q));
    }
    // lane o owns box o of each tile: its slot comes from one table read, issued before the waits
    auto box_slot = [&](int j) -> int {
      const int n_ops = (tile_keys(j) + a.box_rows - 1) / a.box_rows;
      if (lane >= n_ops) return -1;
      const int key = j * kTileKeys + lane * a.box_rows;
      const int page = __ldg(table + (key >> a.page_shift));
      const long long slot = ((long long)page << a.page_shift) + (key & (a.page_size - 1));
      if (page < 0 || slot + a.box_rows > a.num_slots) {       // keep the copy in bounds, flag the id
        set_device_error(hdr, PA_ERR_DEVICE_INDEX);
        return 0;
      }
      return (int)slot;
    };
    int issued = 0;
    if (a.gather) {
      produce_gathered(a, table, L, n_kv, h_kv, base + kOffK, base + kOffV, bar(B_K_FULL), bar(B_V_FULL),
                       bar(B_K_EMPTY), bar(B_V_EMPTY), lane, wait);
    }
    int next_slot = a.gather ? 0 : box_slot(0);
    for (int j = 0; !a.gather && j < n_kv; ++j) {
      const int s = j & 1;
      const int slot = next_slot;
      const int n_ops = (tile_keys(j) + a.box_rows - 1) / a.box_rows;
      const uint32_t bytes = (uint32_t)n_ops * a.box_rows * 128u * 2u;
      const uint32_t off = (uint32_t)lane * a.box_rows * 128u;
      // K stage s is free once S(j-2) is done
      bool ok = true;
      if (lane == 0) {
        ok = j < kNumStages || wait(bar(B_K_EMPTY + s), ring_parity(j) ^ 1u);
        if (ok) mbar_expect_tx(bar(B_K_FULL + s), bytes);
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      if (lane < n_ops)
        for (int ch = 0; ch < 2; ++ch)
          tma_load_4d(base + kOffK + s * kTileBytes + ch * kChunkBytes + off, &a.tm_k, 0, slot, ch, h_kv,
                      bar(B_K_FULL + s));
      // V stage s is free once PV(j-2) is done
      if (lane == 0) {
        ok = j < kNumStages || wait(bar(B_V_EMPTY + s), ring_parity(j) ^ 1u);
        if (ok) mbar_expect_tx(bar(B_V_FULL + s), bytes);
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      if (lane < n_ops)
        for (int ch = 0; ch < 2; ++ch)
          tma_load_4d(base + kOffV + s * kTileBytes + ch * kChunkBytes + off, &a.tm_v, 0, slot, ch, h_kv,
                      bar(B_V_FULL + s));
      issued = j + 1;
      if (j + 1 < n_kv) next_slot = box_slot(j + 1);
    }
    // copies still in flight when the CTA gives up: wait (bounded) until they land
    if (lane == 0 && *abort_flag && !a.gather) {
      for (int j = max(0, issued - kNumStages); j < issued; ++j) {
        for (uint32_t i = 0; i < kWaitLimit && !mbar_try_wait(bar(B_K_FULL + (j & 1)), ring_parity(j)); ++i) {}
        for (uint32_t i = 0; i < kWaitLimit && !mbar_try_wait(bar(B_V_FULL + (j & 1)), ring_parity(j)); ++i) {}
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      auto issue_s = [&](int j) {
        const uint32_t kb = base + kOffK + (j & 1) * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {   // 8 steps of 16 over d
          const uint32_t off = (kk >> 2) * kChunkBytes + (kk & 3) * 32;
          tc_mma(tmem_s, smem_desc(base + kOffQ + off, 16), smem_desc(kb + off, 16), kIdescS, kk > 0);
        }
        tc_commit(bar(B_S_FULL));
        tc_commit(bar(B_K_EMPTY + (j & 1)));
      };
      bool ok = wait(bar(B_Q), 0) && wait(bar(B_K_FULL), 0);
      if (ok) {
        tc_fence_after();
        issue_s(0);
      }
      for (int j = 0; ok && j < n_kv; ++j) {
        const int s = j & 1;
        if (j + 1 < n_kv) {
          ok = wait(bar(B_S_FREE), j & 1) && wait(bar(B_K_FULL + ((j + 1) & 1)), ring_parity(j + 1));
          if (!ok) break;
          tc_fence_after();
          issue_s(j + 1);
        }
        ok = wait(bar(B_P_FULL + s), ring_parity(j)) && wait(bar(B_V_FULL + s), ring_parity(j));
        if (!ok) break;
        tc_fence_after();
        const int nsteps = (tile_keys(j) + 15) / 16;           // 16-key steps that hold live keys
        const uint32_t vb = base + kOffV + s * kTileBytes;
        const uint32_t pb = base + kOffP + s * kTileBytes;
        for (int kk = 0; kk < nsteps; ++kk) {
          const uint32_t pa_off = (kk >> 2) * kChunkBytes + (kk & 3) * 32;   // P: K-major over keys
          tc_mma(tmem_o, smem_desc(pb + pa_off, 16), smem_desc(vb + kk * 16 * 128, kChunkBytes), kIdescPV,
                 (j > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(bar(B_V_EMPTY + s));
        tc_commit(bar(B_P_FREE + s));
      }
      // all issued tensor-core work has finished before TMEM is released
      tc_commit(bar(B_DRAIN));
      for (uint32_t i = 0; i < kWaitLimit && !mbar_try_wait(bar(B_DRAIN), 0); ++i) {}
    }
  } else {
    // ------------------------------------------------------------ softmax warpgroup
    const int row = 32 * (warp & 3) + lane;                    // TMEM lane = query row of the tile
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const int q_local = q_begin + row;
    const bool row_valid = q_local < q_end && q_start + q_local < a.q_rows;   // never store past the O buffer
    const int limit = row_valid ? prefix + q_local : L - 1;    // last visible key (inclusive)
    const float NEG_INF = -__int_as_float(0x7f800000);
    const float c = a.scale_log2;                              // > 0: the max commutes with the scale
    float m_used = NEG_INF, l = 0.f;
    bool ok = true;
    // tcgen05.ld/st are warp-collective: every wait result is made uniform across the warp
    auto wwait = [&](uint32_t b, uint32_t parity) { return __all_sync(0xffffffffu, wait(b, parity)) != 0; };
    for (int j = 0; j < n_kv && ok; ++j) {
      const int s = j & 1;
      if (!(ok = wwait(bar(B_S_FULL), j & 1))) break;
      tc_fence_after();
      uint32_t sv[4][32];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) tmem_ld32(tmem_s + lane_off + 32 * cc, sv[cc]);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar(B_S_FREE));
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
      // 8 independent partial maxima keep the reduction off a 128-long dependency chain
      float mxp[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mxp[i] = NEG_INF;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc)
#pragma unroll
        for (int e = 0; e < 32; ++e) mxp[e & 7] = fmaxf(mxp[e & 7], __uint_as_float(sv[cc][e]));
      float mx = fmaxf(fmaxf(fmaxf(mxp[0], mxp[1]), fmaxf(mxp[2], mxp[3])),
                       fmaxf(fmaxf(mxp[4], mxp[5]), fmaxf(mxp[6], mxp[7])));
      mx *= c;                                                  // log2 units
      float alpha = 1.f;
      if (m_used == NEG_INF) {
        m_used = mx;
      } else if (mx > m_used + kRescaleThreshold) {
        alpha = ex2(m_used - mx);
        m_used = mx;
      }
      // P = 2^(c s - m) as bf16 (overwriting the scores), row sum of the same rounded values
      const float neg_m = m_used == NEG_INF ? 0.f : -m_used;
      float ltp[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) ltp[i] = 0.f;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc)
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const uint32_t w = pack_bf16x2(ex2(fmaf(__uint_as_float(sv[cc][e]), c, neg_m)),
                                         ex2(fmaf(__uint_as_float(sv[cc][e + 1]), c, neg_m)));
          ltp[(e >> 1) & 7] += bf16lo_to_f32(w) + bf16hi_to_f32(w);
          sv[cc][e >> 1] = w;                                   // packed pairs in the low half of each row
        }
      const float lt = ((ltp[0] + ltp[1]) + (ltp[2] + ltp[3])) + ((ltp[4] + ltp[5]) + (ltp[6] + ltp[7]));
      if (j >= 2 && !(ok = wwait(bar(B_P_FREE + s), ring_parity(j) ^ 1u))) break;   // PV(j-2) released buffer s
      if (__any_sync(0xffffffffu, alpha != 1.f)) {                                   // rescale rows of O in TMEM
        // PV(j-1) done, so O is stable.  "PV(i) done" is always read from P_FREE[i % 2], whose
        // phases this warpgroup observes in order, so a wait can never match an older phase.
        if (j > 0 && !(ok = wwait(bar(B_P_FREE + ((j - 1) & 1)), ring_parity(j - 1)))) break;
        tc_fence_after();
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t ov[32];
          tmem_ld32(tmem_o + lane_off + 32 * cc, ov);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
          tmem_st32(tmem_o + lane_off + 32 * cc, ov);
        }
        tmem_wait_st();
      }
      l = l * alpha + lt;
      uint8_t* prow = base_ptr + kOffP + s * kTileBytes;
#pragma unroll
      for (int u = 0; u < 16; ++u) {   // 16-byte units of 8 keys; pairs 4u .. 4u+3 of the row
        const int p0 = 4 * u;          // pair index: row element 2 p0
        const uint32_t w0 = sv[p0 >> 4][p0 & 15], w1 = sv[(p0 + 1) >> 4][(p0 + 1) & 15];
        const uint32_t w2 = sv[(p0 + 2) >> 4][(p0 + 2) & 15], w3 = sv[(p0 + 3) >> 4][(p0 + 3) & 15];
        const int chunk = u >> 3, unit = u & 7;
        const uint32_t off = chunk * kChunkBytes + row * 128 + ((unit ^ (row & 7)) << 4);
        *reinterpret_cast<uint4*>(prow + off) = make_uint4(w0, w1, w2, w3);
      }
      // the last tile: V rows past L inside the last 16-key step must read as zero
      const int nk = tile_keys(j);
      if (nk < kTileKeys && (nk & 15) && warp == 2) {
        if (!(ok = wwait(bar(B_V_FULL + s), ring_parity(j)))) break;
        const int z0 = nk, z1 = (nk + 15) & ~15;
        uint8_t* vt = base_ptr + kOffV + s * kTileBytes;
        for (int idx = lane; idx < (z1 - z0) * 16; idx += 32) {   // 16-byte units of rows z0..z1-1, both halves
          const int rr = z0 + idx / 16, ch = (idx / 8) & 1, un = idx & 7;
          *reinterpret_cast<uint4*>(vt + ch * kChunkBytes + rr * 128 + un * 16) = make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async();
      tc_fence_before();
      mbar_arrive(bar(B_P_FULL + s));
    }
    // every PV has finished: PV(n-2) and PV(n-1) on their P_FREE barriers
    if (ok && n_kv >= 2) ok = wwait(bar(B_P_FREE + ((n_kv - 2) & 1)), ring_parity(n_kv - 2));
    if (ok) ok = wwait(bar(B_P_FREE + ((n_kv - 1) & 1)), ring_parity(n_kv - 1));
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
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}


// ======================================================================================
// Two query tiles per CTA: heads h0 = 2 hp and h1 = 2 hp + 1 of the same KV group share
// every K/V tile.  Warp 0 loads, warp 1 issues the MMAs, warps 2-5 and 6-9 are one
// softmax warpgroup per query tile.  TMEM (512 columns): S0 [0,128), S1 [128,256),
// O0 [256,384), O1 [384,512); P_t (bf16, two per 32-bit column) is written over the
// first 64 columns of S_t once S_t has been read, and PV_t takes A from TMEM.  The
// tensor cores execute one thread's MMAs in issue order, so S_t(j+1), issued after
// PV_t(j), never overwrites P_t(j) before it has been read; and S_t(j) complete
// implies PV_t(j-1) complete, so O_t is stable whenever softmax t reads S_t.
// While one warpgroup runs its softmax the tensor cores work on the other tile.
constexpr int kPairThreads = 320;
constexpr int kPairOffQ = 0;                                   // Q0, Q1
constexpr int kPairOffK = 2 * kTileBytes;
constexpr int kPairOffV = kPairOffK + kNumStages * kTileBytes;
constexpr int kPairOffBar = kPairOffV + kNumStages * kTileBytes;
constexpr int kPairSmemBytes = kPairOffBar + 256 + 1024;
constexpr uint32_t kPairTmemCols = 512;

enum PairBar {
  PB_Q = 0,
  PB_K_FULL = 1,
  PB_V_FULL = PB_K_FULL + kNumStages,
  PB_K_EMPTY = PB_V_FULL + kNumStages,
  PB_V_EMPTY = PB_K_EMPTY + kNumStages,
  PB_S_FULL = PB_V_EMPTY + kNumStages,  // [2] per query tile
  PB_P_FULL = PB_S_FULL + 2,            // [2] per query tile, 128 arrivals
  PB_O_DONE = PB_P_FULL + 2,            // [2] per query tile
  PB_DRAIN = PB_O_DONE + 2,
  PB_COUNT
};
static_assert(PB_COUNT * 8 + 16 <= 256, "barrier area");

__global__ void __launch_bounds__(kPairThreads, 1) extend_pair_kernel(const __grid_constant__ ExtendLaunch a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  const uint32_t bars = base + kPairOffBar;
  auto bar = [&](int i) -> uint32_t { return bars + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + kPairOffBar + 8 * PB_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base_ptr + kPairOffBar + 8 * PB_COUNT + 8);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  PlanHeader* hdr = a.ws.hdr;
  if (hdr->magic != kMagic || hdr->mode != PA_MODE_EXTEND) {
    if (tid == 0 && blockIdx.x == 0) set_device_error(hdr, PA_ERR_WORKSPACE);
    return;
  }
  const int pairs = a.hq / 2;
  const int item = blockIdx.x / pairs, hp = blockIdx.x % pairs;
  if (item >= hdr->num_items) return;
  const int4 it = a.ws.items[item];
  const int r = it.x, q_begin = it.z, q_end = it.w;
  const int L = a.ws.req_len[r], prefix = a.ws.req_prefix[r], q_start = a.ws.req_aux[r];
  const int h0 = 2 * hp;
  const int h_kv = h0 / (a.hq / a.hkv);
  const int kv_end = prefix + q_end;
  const int n_kv = (kv_end + kTileKeys - 1) / kTileKeys;

  if (tid == 0) {
    for (int i = 0; i < PB_COUNT; ++i) mbar_init(bar(i), (i == PB_P_FULL || i == PB_P_FULL + 1) ? 128 : 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n"
                 ::"r"(smem_u32(tmem_slot)), "r"(kPairTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto wait = [&](uint32_t b, uint32_t parity) -> bool {
    for (uint32_t i = 0; i < kWaitLimit; ++i) {
      if (mbar_try_wait(b, parity)) return true;
      if (*abort_flag) return false;
    }
    *abort_flag = 1;
    set_device_error(hdr, PA_ERR_DEVICE_INDEX);
    return false;
  };
  auto tile_keys = [&](int j) { return min(kTileKeys, L - j * kTileKeys); };
  auto ring_parity = [](int j) -> uint32_t { return (uint32_t)(j >> 1) & 1u; };

  if (warp == 0) {
    // ------------------------------------------------------------ producer (whole warp)
    const int32_t* table = a.page_table + (size_t)r * a.pt_pitch;
    if (lane == 0) {
      mbar_expect_tx(bar(PB_Q), 4 * kChunkBytes);
      const int row0 = q_start + q_begin;
      for (int t = 0; t < 2; ++t)
        for (int ch = 0; ch < 2; ++ch)
          tma_load_4d(base + kPairOffQ + t * kTileBytes + ch * kChunkBytes, &a.tm_q, 0, row0, ch, h0 + t, bar(PB_Q));
    }
    auto box_slot = [&](int j) -> int {
      const int n_ops = (tile_keys(j) + a.box_rows - 1) / a.box_rows;
      if (lane >= n_ops) return -1;
      const int key = j * kTileKeys + lane * a.box_rows;
      const int page = __ldg(table + (key >> a.page_shift));
      const long long slot = ((long long)page << a.page_shift) + (key & (a.page_size - 1));
      if (page < 0 || slot + a.box_rows > a.num_slots) {
        set_device_error(hdr, PA_ERR_DEVICE_INDEX);
        return 0;
      }
      return (int)slot;
    };
    int issued = 0;
    if (a.gather) {
      produce_gathered(a, table, L, n_kv, h_kv, base + kPairOffK, base + kPairOffV, bar(PB_K_FULL), bar(PB_V_FULL),
                       bar(PB_K_EMPTY), bar(PB_V_EMPTY), lane, wait);
    }
    int next_slot = a.gather ? 0 : box_slot(0);
    for (int j = 0; !a.gather && j < n_kv; ++j) {
      const int s = j & 1;
      const int slot = next_slot;
      const int n_ops = (tile_keys(j) + a.box_rows - 1) / a.box_rows;
      const uint32_t bytes = (uint32_t)n_ops * a.box_rows * 128u * 2u;
      const uint32_t off = (uint32_t)lane * a.box_rows * 128u;
      bool ok = true;
      if (lane == 0) {
        ok = j < kNumStages || wait(bar(PB_K_EMPTY + s), ring_parity(j) ^ 1u);
        if (ok) mbar_expect_tx(bar(PB_K_FULL + s), bytes);
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      if (lane < n_ops)
        for (int ch = 0; ch < 2; ++ch)
          tma_load_4d(base + kPairOffK + s * kTileBytes + ch * kChunkBytes + off, &a.tm_k, 0, slot, ch, h_kv,
                      bar(PB_K_FULL + s));
      if (lane == 0) {
        ok = j < kNumStages || wait(bar(PB_V_EMPTY + s), ring_parity(j) ^ 1u);
        if (ok) mbar_expect_tx(bar(PB_V_FULL + s), bytes);
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      if (lane < n_ops)
        for (int ch = 0; ch < 2; ++ch)
          tma_load_4d(base + kPairOffV + s * kTileBytes + ch * kChunkBytes + off, &a.tm_v, 0, slot, ch, h_kv,
                      bar(PB_V_FULL + s));
      issued = j + 1;
      if (j + 1 < n_kv) next_slot = box_slot(j + 1);
    }
    if (lane == 0 && *abort_flag && !a.gather) {
      for (int j = max(0, issued - kNumStages); j < issued; ++j) {
        for (uint32_t i = 0; i < kWaitLimit && !mbar_try_wait(bar(PB_K_FULL + (j & 1)), ring_parity(j)); ++i) {}
        for (uint32_t i = 0; i < kWaitLimit && !mbar_try_wait(bar(PB_V_FULL + (j & 1)), ring_parity(j)); ++i) {}
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      auto issue_s = [&](int t, int j) {            // S_t = Q_t K(j)^T
        const uint32_t qb = base + kPairOffQ + t * kTileBytes;
        const uint32_t kb = base + kPairOffK + (j & 1) * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kChunkBytes + (kk & 3) * 32;
          tc_mma(tmem + 128 * t, smem_desc(qb + off, 16), smem_desc(kb + off, 16), kIdescS, kk > 0);
        }
        tc_commit(bar(PB_S_FULL + t));
      };
      auto issue_pv = [&](int t, int j) {           // O_t += P_t V(j), P_t from TMEM
        const int nsteps = (tile_keys(j) + 15) / 16;
        const uint32_t vb = base + kPairOffV + (j & 1) * kTileBytes;
        for (int kk = 0; kk < nsteps; ++kk)
          tc_mma_ts(tmem + 256 + 128 * t, tmem + 128 * t + 8 * kk, smem_desc(vb + kk * 16 * 128, kChunkBytes),
                    kIdescPV, (j > 0 || kk > 0) ? 1u : 0u);
        tc_commit(bar(PB_O_DONE + t));
      };
      bool ok = wait(bar(PB_Q), 0) && wait(bar(PB_K_FULL), 0);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        issue_s(1, 0);
        tc_commit(bar(PB_K_EMPTY));
      }
      for (int j = 0; ok && j < n_kv; ++j) {
        const int s = j & 1, s1 = (j + 1) & 1;
        const bool more = j + 1 < n_kv;
        if (!(ok = wait(bar(PB_V_FULL + s), ring_parity(j)) && wait(bar(PB_P_FULL), j & 1))) break;
        tc_fence_after();
        issue_pv(0, j);
        if (more) {
          if (!(ok = wait(bar(PB_K_FULL + s1), ring_parity(j + 1)))) break;
          tc_fence_after();
          issue_s(0, j + 1);
        }
        if (!(ok = wait(bar(PB_P_FULL + 1), j & 1))) break;
        tc_fence_after();
        issue_pv(1, j);
        tc_commit(bar(PB_V_EMPTY + s));
        if (more) {
          issue_s(1, j + 1);
          tc_commit(bar(PB_K_EMPTY + s1));
        }
      }
      tc_commit(bar(PB_DRAIN));
      for (uint32_t i = 0; i < kWaitLimit && !mbar_try_wait(bar(PB_DRAIN), 0); ++i) {}
    }
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    const int t = (warp - 2) >> 2;                             // query tile of this warpgroup
    const int h = h0 + t;
    const int row = 32 * (warp & 3) + lane;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t tmem_s = tmem + 128 * t, tmem_o = tmem + 256 + 128 * t;
    const int q_local = q_begin + row;
    const bool row_valid = q_local < q_end && q_start + q_local < a.q_rows;
    const int limit = row_valid ? prefix + q_local : L - 1;
    const float NEG_INF = -__int_as_float(0x7f800000);
    const float c = a.scale_log2;
    float m_used = NEG_INF, l = 0.f;
    bool ok = true;
    auto wwait = [&](uint32_t b, uint32_t parity) { return __all_sync(0xffffffffu, wait(b, parity)) != 0; };
    for (int j = 0; j < n_kv && ok; ++j) {
      const int s = j & 1;
      if (!(ok = wwait(bar(PB_S_FULL + t), j & 1))) break;
      // PV_t(j-1) finished before S_t(j); its O_DONE phase is observed here so that every
      // phase of that barrier is waited in order (the final wait below can never alias)
      if (j > 0 && !(ok = wwait(bar(PB_O_DONE + t), (j - 1) & 1))) break;
      tc_fence_after();
      uint32_t sv[4][32];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) tmem_ld32(tmem_s + lane_off + 32 * cc, sv[cc]);
      tmem_wait_ld();
      const int key0 = j * kTileKeys;
      const bool diag = key0 + kTileKeys - 1 > prefix + q_begin || key0 + kTileKeys > L;
      if (diag) {
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (key0 + 32 * cc + e > limit) sv[cc][e] = __float_as_uint(NEG_INF);
      }
      float mxp[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mxp[i] = NEG_INF;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc)
#pragma unroll
        for (int e = 0; e < 32; ++e) mxp[e & 7] = fmaxf(mxp[e & 7], __uint_as_float(sv[cc][e]));
      float mx = fmaxf(fmaxf(fmaxf(mxp[0], mxp[1]), fmaxf(mxp[2], mxp[3])),
                       fmaxf(fmaxf(mxp[4], mxp[5]), fmaxf(mxp[6], mxp[7])));
      mx *= c;
      float alpha = 1.f;
      if (m_used == NEG_INF) {
        m_used = mx;
      } else if (mx > m_used + kRescaleThreshold) {
        alpha = ex2(m_used - mx);
        m_used = mx;
      }
      const float neg_m = m_used == NEG_INF ? 0.f : -m_used;
      float ltp[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) ltp[i] = 0.f;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc)
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const uint32_t w = pack_bf16x2(ex2(fmaf(__uint_as_float(sv[cc][e]), c, neg_m)),
                                         ex2(fmaf(__uint_as_float(sv[cc][e + 1]), c, neg_m)));
          ltp[(e >> 1) & 7] += bf16lo_to_f32(w) + bf16hi_to_f32(w);
          sv[cc][e >> 1] = w;
        }
      const float lt = ((ltp[0] + ltp[1]) + (ltp[2] + ltp[3])) + ((ltp[4] + ltp[5]) + (ltp[6] + ltp[7]));
      if (__any_sync(0xffffffffu, alpha != 1.f)) {             // O_t is stable: PV_t(j-1) finished before S_t(j)
#pragma unroll 1
        for (int cc = 0; cc < 16; ++cc) {                        // 8 columns at a time keeps registers low
          uint32_t ov[8];
          tmem_ld8(tmem_o + lane_off + 8 * cc, ov);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 8; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
          tmem_st8(tmem_o + lane_off + 8 * cc, ov);
        }
      }
      l = l * alpha + lt;
      // P_t over the first 64 columns of S_t: column p holds keys 2p (low half) and 2p + 1
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) tmem_st16(tmem_s + lane_off + 16 * cc, sv[cc]);
      tmem_wait_st();
      const int nk = tile_keys(j);
      if (t == 0 && nk < kTileKeys && (nk & 15) && warp == 2) {   // V rows past L in the last 16-key step
        if (!(ok = wwait(bar(PB_V_FULL + s), ring_parity(j)))) break;
        const int z0 = nk, z1 = (nk + 15) & ~15;
        uint8_t* vt = base_ptr + kPairOffV + s * kTileBytes;
        for (int idx = lane; idx < (z1 - z0) * 16; idx += 32) {
          const int rr = z0 + idx / 16, ch = (idx / 8) & 1, un = idx & 7;
          *reinterpret_cast<uint4*>(vt + ch * kChunkBytes + rr * 128 + un * 16) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async();
      }
      tc_fence_before();
      mbar_arrive(bar(PB_P_FULL + t));
    }
    if (ok) ok = wwait(bar(PB_O_DONE + t), (n_kv - 1) & 1);
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
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kPairTmemCols) : "memory");
  }
}

// ---------------------------------------------------------------- host: tensor maps

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

cudaError_t launch_extend(const ExtendArgs& in, cudaStream_t s) {
  // four heads of one KV group over a pair of CTAs sharing every K/V tile (extend_duo.cu)
  if ((in.hq / in.hkv) % 4 == 0) return launch_extend_duo(in, s);
  static std::atomic<bool> single_set[kMaxDevices], pair_set[kMaxDevices];
  ExtendLaunch a;
  a.gather = in.page_size < 8 ? 1 : 0;
  a.k_pool = in.k_pool;
  a.v_pool = in.v_pool;
  const int box_rows = in.page_size < kTileKeys ? in.page_size : kTileKeys;
  if (!encode_rows(&a.tm_q, in.q, in.q_rows, in.hq, 128) ||
      (!a.gather && (!encode_rows(&a.tm_k, in.k_pool, in.num_slots, in.hkv, box_rows) ||
                     !encode_rows(&a.tm_v, in.v_pool, in.num_slots, in.hkv, box_rows))))
    return cudaErrorInvalidValue;
  a.ws = in.ws;
  a.page_table = in.page_table;
  a.pt_pitch = in.pt_pitch;
  a.num_slots = in.num_slots;
  a.out = in.out;
  a.lse_out = in.lse_out;
  a.scale_log2 = in.scale_log2;
  a.hq = in.hq;
  a.hkv = in.hkv;
  a.page_size = in.page_size;
  a.page_shift = in.page_shift;
  a.box_rows = box_rows;
  a.max_items = in.max_items;
  a.q_rows = in.q_rows;
  if ((in.hq / in.hkv) % 2 == 0) {   // two heads of one KV group per CTA
    cudaError_t e = raise_smem_limit(extend_pair_kernel, kPairSmemBytes, pair_set);
    if (e != cudaSuccess) return e;
    extend_pair_kernel<<<in.max_items * (in.hq / 2), kPairThreads, kPairSmemBytes, s>>>(a);
  } else {
    cudaError_t e = raise_smem_limit(extend_kernel, kSmemBytes, single_set);
    if (e != cudaSuccess) return e;
    extend_kernel<<<in.max_items * in.hq, kThreads, kSmemBytes, s>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace pa
