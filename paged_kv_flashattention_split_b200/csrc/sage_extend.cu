// sage_extend.cu - 8-bit "Sage" EXTEND (prefill over a cached prefix) on the 5th-generation
// tensor cores, in their native 8-bit kinds.
//
// The formula ("FlashInfer PrimTS, Sage Attention 도입으로 8비트 양자화 및 성능 최적화
// 달성", 코드 분석 item 1, README "Sage attention") for every new token: row i of request r
// (absolute position p_r + i) over its visible keys j <= p_r + i,
//     S_j  = sfQ[row][h] * sfK[blk(j)][h_kv] * (Q8 . K8_j),  m = max_j S_j,
//     P8_j = E4M3(448 exp(S_j - m)),  l = sum_j exp(S_j - m),
//     O[d] = sfV[h_kv][d] * (sum_j P8_j V8_j[d]) / (448 l) + v_mean[h_kv][d];
// the dense Sage variant the pages measure at S = 10800 (same page, performance item 2).
//
// P8 needs the exact row max before any probability is formed, so a CTA makes two passes
// over its key tiles: pass 1 computes S = Q K^T and each row's maximum, pass 2 computes S
// again, P8 and O += P8 V.  A CTA owns one query tile of 128 new tokens and NH query heads
// of one KV group (NH = 2 when the group size is even, else 1): every K8 and V8 tile it
// loads serves all NH heads, which halves the tile traffic per head against one head per
// CTA.  Both contractions run on the 8-bit tensor cores: S on tcgen05.mma kind::i8 (int8 x
// int8 into int32, exact), P8 V on kind::f8f6f4 (E4M3 x E4M3 into fp32) with P8 from a
// shared-memory tile (K-major, 128-byte swizzle) and V8 read in place as an MN-major
// operand.  The 8-bit tiles land from TMA in the operands' 128-byte-swizzled layouts, so
// nothing is converted on chip.  TMEM holds one S buffer and the O accumulator per head;
// pass 1, which has no O yet, uses the O columns as a second S buffer.
// Roles (2 + 4 NH warps):
//   warp 0      producer: Q8 of the NH heads once, then TMA boxes of 64 slots (one page) x
//               128 bytes into an 8-stage ring of 16 KB tiles, in the order K8(0..n-1)
//               (pass 1), then K8(0), V8(0), K8(1), V8(1), ... (pass 2);
//   warp 1      MMA issuer: S(g) of every head (g = 0 .. 2n-1 over both passes) as soon as
//               the softmax has taken the previous S of its buffer into registers, so the
//               next S runs while the softmax works on the current one; in pass 2, O +=
//               P8 V(j) per head once P8(j) is written; a stage is released when the MMAs
//               that read it complete;
//   warps 2..   softmax, one warpgroup per head: thread i owns query row i (TMEM lane i);
//               pass 1 reduces the row maximum of the causally masked scores, pass 2
//               writes P8 into the head's P buffer j % 2 and sums l; at the end it applies
//               the epilogue.  V8 rows past the request's last key inside the last 32-key
//               step are zeroed before PV reads them (0 x NaN would poison O).
// Every wait on an mbarrier is bounded: on timeout the CTA records PA_ERR_DEVICE_INDEX,
// its roles stop, the producer waits for its copies, the MMA issuer drains the tensor
// cores, and TMEM is freed before exit.
#include <climits>

#include "kernels.h"
#include "tma.cuh"

namespace pa {
namespace {

constexpr int kTileRows = 128;                     // query rows and keys per tile
constexpr int kTile8 = 128 * 128;                  // 128 rows x 128 bytes of 8-bit data (16 KB)
constexpr int kStg = 8;                            // ring stages
constexpr uint32_t kWaitLimit = 1u << 20;
constexpr float kLog2e = 1.4426950408889634f;
// int32 -> fp32 without the conversion unit: for |v| < 2^22 the bits 0x4B400000 + v are the
// float 1.5 * 2^23 + v exactly, and subtracting 1.5 * 2^23 leaves fp32(v) exactly (the
// dots here are at most 128 * 128 * 128 = 2^21 in magnitude)
constexpr int kCvtBiasBits = 0x4B400000;
constexpr float kCvtBias = 12582912.f;

// NH query heads of one KV group per CTA (2 when the group size is even, else 1)
template <int NH>
struct Cfg {
  static constexpr int kThreads = 64 + 128 * NH;           // producer, MMA issuer, NH softmax warpgroups
  static constexpr uint32_t kTmemCols = 256 * NH;          // S (int32) of each head, then O (fp32) of each head
  static constexpr int kOffQ = 0;                          // [NH] Q8 tiles
  static constexpr int kOffP = kOffQ + NH * kTile8;        // [NH][2] P8 tiles
  static constexpr int kOffStg = kOffP + 2 * NH * kTile8;  // [kStg] K8 / V8 ring
  static constexpr int kOffBar = kOffStg + kStg * kTile8;
  static constexpr int kSmemBytes = kOffBar + 512 + 1024;
};
static_assert(Cfg<2>::kSmemBytes <= 227 * 1024, "shared memory per CTA");

enum Bar {
  B_STG_FULL = 0,                  // [kStg] tile landed (TMA)
  B_STG_EMPTY = B_STG_FULL + kStg, // [kStg] the MMA that read it has completed (commit)
  B_Q = B_STG_EMPTY + kStg,        // Q8 of the NH heads landed
  B_S_FULL,                        // [2] S(g) of every head in TMEM buffer b (commit)
  B_S_READ = B_S_FULL + 2,         // [2] every softmax thread has taken S(g) from buffer b (128 NH)
  B_P_FULL = B_S_READ + 2,         // [2] P8(j) of every head in its shared-memory buffer j % 2 (128 NH)
  B_PV_DONE = B_P_FULL + 2,        // [2] PV(j) of every head done: buffer j % 2 is free (commit)
  B_O_DONE = B_PV_DONE + 2,        // every PV done (commit)
  B_DRAIN,
  B_COUNT
};
static_assert(B_COUNT * 8 + 16 <= 512, "barrier area");

// instruction descriptors, M = 128, N = 128
//   S:  kind::i8, s32 D, s8 A and B, both K-major
//   PV: kind::f8f6f4, f32 D, E4M3 A (P8, K-major) and B (V8, MN-major)
constexpr uint32_t kIdescS = (2u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescPV = (1u << 4) | (1u << 16) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

struct SageExtendLaunch {
  CUtensorMap tm_q8;    // q8 [rows][Hq][128] bytes as {128, rows, Hq}, box {128, 128, 1}
  CUtensorMap tm_k8;    // pools [slots][Hkv][128] as {128, slots, Hkv}, box {128, 64, 1}
  CUtensorMap tm_v8;
  WsView ws;
  const float* sf_q;
  const float* sf_k;
  const float* sf_v;
  const float* v_mean;
  const int32_t* page_table;
  int64_t pt_pitch;
  int64_t num_slots;
  int64_t q_rows;
  uint16_t* out;
  int hq, hkv;
};

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }

// smem matrix descriptor: 128-byte swizzle, 8-row groups 1024 bytes apart (SBO); the
// operands here are 128 bytes wide, one swizzle atom, so the LBO is never used
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr) {
  return (uint64_t)((addr & 0x3FFFF) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) | (1ull << 46) |
         (2ull << 61);
}
// D (TMEM, s32) += A (smem, s8) x B (smem, s8)
__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t accumulate) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\ntcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n}\n"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(kIdescS), "r"(accumulate)
      : "memory");
}
// D (TMEM, f32) += A (smem, E4M3) x B (smem, E4M3)
__device__ __forceinline__ void mma_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t accumulate) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\ntcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n}\n"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(kIdescPV), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
        "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
        "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }

// Two floats to E4M3 codes (nearest even, saturating); `lo` in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t v;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;\n" : "=h"(v) : "f"(hi), "f"(lo));
  return v;
}

template <int NH>
__global__ void __launch_bounds__(Cfg<NH>::kThreads, 1) sage_extend_kernel(const __grid_constant__ SageExtendLaunch a) {
  using C = Cfg<NH>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  const uint32_t bars = base + C::kOffBar;
  auto bar = [&](int i) -> uint32_t { return bars + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + C::kOffBar + 8 * B_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base_ptr + C::kOffBar + 8 * B_COUNT + 8);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  PlanHeader* hdr = a.ws.hdr;
  if (hdr->magic != kMagic || hdr->mode != PA_MODE_EXTEND || hdr->page_size != kSageBlock) {
    if (tid == 0 && blockIdx.x == 0) set_device_error(hdr, PA_ERR_WORKSPACE);
    return;
  }
  const int ctas_per_item = a.hq / NH;
  const int item = blockIdx.x / ctas_per_item, h0 = (blockIdx.x % ctas_per_item) * NH;
  if (item >= hdr->num_items) return;
  const int4 it = a.ws.items[item];
  const int r = it.x, q_begin = it.z, q_end = it.w;
  const int L = a.ws.req_len[r], prefix = a.ws.req_prefix[r], q_start = a.ws.req_aux[r];
  const int h_kv = h0 / (a.hq / a.hkv);                    // shared by the CTA's NH heads
  const int kv_end = prefix + q_end;                         // keys any row of this tile can see
  const int n = (kv_end + kTileRows - 1) / kTileRows;       // key tiles
  const int32_t* table = a.page_table + (size_t)r * a.pt_pitch;

  if (tid == 0) {
    for (int i = 0; i < B_COUNT; ++i) {
      const bool many = (i >= B_S_READ && i < B_S_READ + 2) || i == B_P_FULL || i == B_P_FULL + 1;
      mbar_init(bar(i), many ? 128 * NH : 1);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n"
                 ::"r"(smem_u32(tmem_slot)), "r"(C::kTmemCols) : "memory");
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
  // warp-uniform: every lane observes the phase, and all take the same branch
  auto wwait = [&](uint32_t b, uint32_t parity) { return __all_sync(0xffffffffu, wait(b, parity)) != 0; };
  // raw table entry of page b of the request, checked: -1 if out of range
  auto page_of = [&](int b) -> int {
    if (b * kSageBlock >= L) return -1;
    const int e = __ldg(table + b);
    if (e < 0 || ((long long)e + 1) * kSageBlock > a.num_slots) {
      set_device_error(hdr, PA_ERR_DEVICE_INDEX);
      return -1;
    }
    return e;
  };
  // ring items: t < n is K8(t) of pass 1; then K8(j) at n + 2j and V8(j) at n + 2j + 1
  const int n_items = 3 * n;
  auto stage_of = [](int t) { return t % kStg; };
  auto full_parity = [](int t) { return (uint32_t)(t / kStg) & 1u; };
  // S buffers: pass 1 (g < n, no O yet) alternates between buffer 0 and buffer 1, which is
  // the O region; pass 2 uses buffer 0.  u = how many earlier S went through the same buffer.
  auto s_buf = [n](int g) { return g < n ? (g & 1) : 0; };
  auto s_use = [n](int g) { return g < n ? (g >> 1) : ((n + 1) >> 1) + (g - n); };

  if (warp == 0) {
    // ------------------------------------------------------------ producer (whole warp)
    if (lane == 0) {
      mbar_expect_tx(bar(B_Q), NH * kTile8);
      for (int hh = 0; hh < NH; ++hh)
        tma_load_3d(base + C::kOffQ + hh * kTile8, &a.tm_q8, 0, q_start + q_begin, h0 + hh, bar(B_Q));
    }
    int issued = 0;
    int pg_lo = -1, pg_hi = -1;   // this lane's pages for the tile j = tb + lane of the current round
    int round_tb = -1;
    for (int t = 0; t < n_items; ++t) {
      const int s = stage_of(t);
      const int j = t < n ? t : (t - n) >> 1;
      const bool is_v = t >= n && ((t - n) & 1);
      if ((j >> 5) << 5 != round_tb) {                         // page ids of 32 tiles, one per lane
        round_tb = (j >> 5) << 5;
        const int jj = round_tb + lane;
        pg_lo = jj < n ? page_of(2 * jj) : -1;
        pg_hi = jj < n ? page_of(2 * jj + 1) : -1;
      }
      const int plo = __shfl_sync(0xffffffffu, pg_lo, j & 31);
      const int phi = __shfl_sync(0xffffffffu, pg_hi, j & 31);
      bool ok = true;
      if (lane == 0) {
        ok = t < kStg || wait(bar(B_STG_EMPTY + s), (uint32_t)((t / kStg) - 1) & 1u);
        if (ok) {
          const uint32_t dst = base + C::kOffStg + s * kTile8;
          const uint32_t bytes = (plo >= 0 ? kTile8 / 2 : 0) + (phi >= 0 ? kTile8 / 2 : 0);
          mbar_expect_tx(bar(B_STG_FULL + s), bytes);
          const CUtensorMap* tm = is_v ? &a.tm_v8 : &a.tm_k8;
          if (plo >= 0) tma_load_3d(dst, tm, 0, plo * kSageBlock, h_kv, bar(B_STG_FULL + s));
          if (phi >= 0) tma_load_3d(dst + kTile8 / 2, tm, 0, phi * kSageBlock, h_kv, bar(B_STG_FULL + s));
        }
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      issued = t + 1;
    }
    if (lane == 0 && *abort_flag) {   // copies still in flight: wait (bounded) until they land
      for (uint32_t i = 0; i < kWaitLimit && !mbar_try_wait(bar(B_Q), 0); ++i) {}
      for (int t = max(0, issued - kStg); t < issued; ++t)
        for (uint32_t i = 0; i < kWaitLimit && !mbar_try_wait(bar(B_STG_FULL + stage_of(t)), full_parity(t)); ++i) {}
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = wait(bar(B_Q), 0);
      // descriptors of the first tile of each operand region; a tile or 32-byte step further
      // on is the same descriptor with its start address (bits 0-13, 16-byte units) advanced
      const uint64_t d_q = smem_desc(base + C::kOffQ), d_p = smem_desc(base + C::kOffP);
      const uint64_t d_stg = smem_desc(base + C::kOffStg);
      // S(g) of every head of the CTA (g = 0 .. 2n-1 over both passes) into its buffer, once
      // every softmax thread has taken the buffer's previous S into registers
      auto issue_s = [&](int g) -> bool {
        const int t = g < n ? g : n + 2 * (g - n);
        const int b = s_buf(g), u = s_use(g);
        if (!wait(bar(B_STG_FULL + stage_of(t)), full_parity(t))) return false;
        if (u > 0 && !wait(bar(B_S_READ + b), (uint32_t)(u - 1) & 1u)) return false;
        tc_fence_after();
        const uint64_t d_k = d_stg + (uint64_t)((stage_of(t) * kTile8) >> 4);
        const uint32_t d_s = tmem + 128 * NH * b;
#pragma unroll
        for (int hh = 0; hh < NH; ++hh)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)   // 4 steps of 32 bytes over d
            mma_i8(d_s + 128 * hh, d_q + (uint64_t)((hh * kTile8 + kk * 32) >> 4), d_k + (uint64_t)(kk * 2), kk > 0);
        tc_commit(bar(B_S_FULL + b));
        tc_commit(bar(B_STG_EMPTY + stage_of(t)));
        return true;
      };
      for (int g = 0; ok && g <= n; ++g) ok = issue_s(g);   // pass 1, then S(0) of pass 2
      for (int j = 0; ok && j < n; ++j) {
        // S(j + 1) runs on the tensor cores while the softmax turns S(j) into P8(j)
        if (j + 1 < n && !(ok = issue_s(n + j + 1))) break;
        const int t = n + 2 * j + 1;   // V8(j)
        if (!(ok = wait(bar(B_P_FULL + (j & 1)), (uint32_t)(j >> 1) & 1u) && wait(bar(B_STG_FULL + stage_of(t)), full_parity(t))))
          break;
        tc_fence_after();
        const int nsteps = (min(kTileRows, L - j * kTileRows) + 31) / 32;   // 32-key steps that hold live keys
        const uint64_t d_v = d_stg + (uint64_t)((stage_of(t) * kTile8) >> 4);
        const uint64_t d_pj = d_p + (uint64_t)(((j & 1) * kTile8) >> 4);
#pragma unroll
        for (int hh = 0; hh < NH; ++hh)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)   // 32 keys per step: 32 bytes of P8, 32 rows (4 KB) of V8
            if (kk < nsteps)
              mma_f8(tmem + 128 * (NH + hh), d_pj + (uint64_t)((2 * hh * kTile8 + kk * 32) >> 4),
                     d_v + (uint64_t)(kk * 256), (j > 0 || kk > 0) ? 1u : 0u);
        tc_commit(bar(B_PV_DONE + (j & 1)));
        tc_commit(bar(B_STG_EMPTY + stage_of(t)));
      }
      if (ok) tc_commit(bar(B_O_DONE));
      // all issued tensor-core work has finished before TMEM is released
      tc_commit(bar(B_DRAIN));
      for (uint32_t i = 0; i < kWaitLimit && !mbar_try_wait(bar(B_DRAIN), 0); ++i) {}
    }
  } else {
    // ------------------------------------------------------------ softmax (one warpgroup per head)
    const int wg = (warp - 2) >> 2, h = h0 + wg;
    const int row = 32 * (warp & 3) + lane;                    // TMEM lane = query row of the tile
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t tmem_s = tmem + 128 * wg + lane_off, tmem_o = tmem + 128 * (NH + wg) + lane_off;   // buffer 0
    // this row of a P8 tile: K-major, 128-byte swizzle (16-byte chunk c at c ^ (row & 7))
    const uint32_t p_row = (uint32_t)((row >> 3) * 1024 + (row & 7) * 128);
    const int sw = row & 7;
    const int q_local = q_begin + row;
    const bool row_valid = q_local < q_end && q_start + q_local < a.q_rows;
    const int limit = row_valid ? prefix + q_local : -1;       // last visible key (inclusive)
    const float NEG_INF = -__int_as_float(0x7f800000);
    const float sfq = row_valid ? __ldg(a.sf_q + (size_t)(q_start + q_local) * a.hq + h) : 0.f;
    // sfK of the two pages of 32 tiles per round, one tile per lane; each thread then forms
    // fp32(sfQ sfK) with its own row's sfQ
    float sk_lo = 0.f, sk_hi = 0.f;
    int round_tb = -1;
    auto scales = [&](int j, float& s0, float& s1) {
      if ((j >> 5) << 5 != round_tb) {
        round_tb = (j >> 5) << 5;
        const int jj = round_tb + lane;
        const int plo = jj < n ? page_of(2 * jj) : -1, phi = jj < n ? page_of(2 * jj + 1) : -1;
        sk_lo = plo >= 0 ? __ldg(a.sf_k + (size_t)plo * a.hkv + h_kv) : 0.f;
        sk_hi = phi >= 0 ? __ldg(a.sf_k + (size_t)phi * a.hkv + h_kv) : 0.f;
      }
      s0 = sfq * __shfl_sync(0xffffffffu, sk_lo, j & 31);
      s1 = sfq * __shfl_sync(0xffffffffu, sk_hi, j & 31);
    };
    // S(g) into registers; the MMA issuer may then overwrite the buffer with S(g + 1)
    auto take_s = [&](int g, uint32_t (&sv)[4][32]) -> bool {
      const int b = s_buf(g);
      if (!wwait(bar(B_S_FULL + b), (uint32_t)s_use(g) & 1u)) return false;
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) tmem_ld32(tmem_s + 128 * NH * b + 32 * cc, sv[cc]);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar(B_S_READ + b));
      return true;
    };
    bool ok = true;
    float m = NEG_INF;
    // pass 1: the row maximum of the visible scores, S = fp32(sfQ sfK) fp32(dot) (the dot is
    // exact).  Rounding is monotonic, so over one page half (one scale sc) the maximum of
    // fp32(sc x) is fp32(sc max x) for sc >= 0 and fp32(sc min x) for sc < 0: the reduction
    // runs on the int32 dots and converts two values per tile.
    for (int j = 0; j < n && ok; ++j) {
      float s0, s1;
      scales(j, s0, s1);
      uint32_t sv[4][32];
      if (!(ok = take_s(j, sv))) break;
      const int key0 = j * kTileRows;
      const bool nonneg = __all_sync(0xffffffffu, s0 >= 0.f && s1 >= 0.f);
      int mx[2] = {INT_MIN, INT_MIN}, mn[2] = {INT_MAX, INT_MAX};
      if (__all_sync(0xffffffffu, key0 + kTileRows - 1 <= limit)) {   // every key visible to the warp's rows
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          int a0 = INT_MIN, a1 = INT_MIN, b0 = INT_MAX, b1 = INT_MAX;
#pragma unroll
          for (int e = 0; e < 64; e += 4) {
            const int* v = reinterpret_cast<const int*>(sv[2 * hf + (e >> 5)]) + (e & 31);
            a0 = __vimax3_s32(a0, v[0], v[1]);
            a1 = __vimax3_s32(a1, v[2], v[3]);
            if (!nonneg) {
              b0 = __vimin3_s32(b0, v[0], v[1]);
              b1 = __vimin3_s32(b1, v[2], v[3]);
            }
          }
          mx[hf] = max(a0, a1);
          mn[hf] = min(b0, b1);
        }
      } else {
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int v = (int)sv[cc][e];
            const bool vis = key0 + 32 * cc + e <= limit;
            mx[cc >> 1] = vis ? max(mx[cc >> 1], v) : mx[cc >> 1];
            mn[cc >> 1] = vis ? min(mn[cc >> 1], v) : mn[cc >> 1];
          }
      }
      // a dot is at most 2^21 in magnitude, so INT_MIN marks a half with no visible key
      if (mx[0] != INT_MIN) m = fmaxf(m, s0 * (float)(s0 >= 0.f ? mx[0] : mn[0]));
      if (mx[1] != INT_MIN) m = fmaxf(m, s1 * (float)(s1 >= 0.f ? mx[1] : mn[1]));
    }
    const float m_use = m == NEG_INF ? 0.f : m;
    // P8 = E4M3(448 exp(S - m)) with S = fp32(sc * dot) formed exactly as the row max was, so
    // S - m is exact for every key near the max (Sterbenz) and the code each key gets is the
    // one its float32 score decides: 448 p carries only the rounding of (S - m) log2 e, of
    // ex2 and of the product by 448 (well under 1e-6 relative), not the error of a score
    // folded into one fused multiply-add (about 1e-5 near the max at these magnitudes)
    const float2 neg_m2 = make_float2(-m_use, -m_use), log2e2 = make_float2(kLog2e, kLog2e);
    const float2 k448 = make_float2(448.f, 448.f);
    float2 l2 = make_float2(0.f, 0.f);   // l, the sum of the unquantised p
    // pass 2: P8 = E4M3(448 exp(S - m)) into a shared-memory P tile; l of the unquantised p
    for (int j = 0; j < n && ok; ++j) {
      float s0, s1;
      scales(j, s0, s1);
      uint32_t sv[4][32];
      if (!(ok = take_s(n + j, sv))) break;
      // the P buffer's previous tile (j - 2) has been multiplied
      if (j >= 2 && !(ok = wwait(bar(B_PV_DONE + (j & 1)), (uint32_t)((j >> 1) - 1) & 1u))) break;
      uint8_t* prow = base_ptr + C::kOffP + (2 * wg + (j & 1)) * kTile8 + p_row;
      const int key0 = j * kTileRows;
      const bool full = __all_sync(0xffffffffu, key0 + kTileRows - 1 <= limit);
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        const float sc = cc < 2 ? s0 : s1;
        const float2 sc2 = make_float2(sc, sc), nb = make_float2(-kCvtBias, -kCvtBias);
        uint32_t pw[8];
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          float q[4];
#pragma unroll
          for (int u = 0; u < 4; u += 2) {
            float2 x = make_float2(__int_as_float((int)sv[cc][e + u] + kCvtBiasBits),
                                   __int_as_float((int)sv[cc][e + u + 1] + kCvtBiasBits));
            x = __fadd2_rn(x, nb);                                        // the exact fp32 dots
            const float2 t = __fmul2_rn(__fadd2_rn(__fmul2_rn(x, sc2), neg_m2), log2e2);   // (S - m) log2 e
            float2 p = make_float2(ex2(t.x), ex2(t.y));
            if (!full) {
              const int k = key0 + 32 * cc + e + u;
              if (k > limit) p.x = 0.f;
              if (k + 1 > limit) p.y = 0.f;
            }
            l2 = __fadd2_rn(l2, p);
            const float2 p448 = __fmul2_rn(p, k448);
            q[u] = p448.x;
            q[u + 1] = p448.y;
          }
          pw[e >> 2] = e4m3x2(q[0], q[1]) | (e4m3x2(q[2], q[3]) << 16);
        }
        // keys 32 cc .. 32 cc + 31 are the 16-byte chunks 2 cc and 2 cc + 1 of the row
        *reinterpret_cast<uint4*>(prow + (((2 * cc) ^ sw) << 4)) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
        *reinterpret_cast<uint4*>(prow + (((2 * cc + 1) ^ sw) << 4)) = make_uint4(pw[4], pw[5], pw[6], pw[7]);
      }
      // the last tile: V8 rows past L inside the last 32-key step must read as zero (each
      // warpgroup's first warp writes the same zeros before its own P_FULL arrival)
      const int live = min(kTileRows, L - j * kTileRows);
      if ((live & 31) && (warp & 3) == 2) {
        const int t = n + 2 * j + 1;
        if (!(ok = wwait(bar(B_STG_FULL + stage_of(t)), full_parity(t)))) break;
        const int z1 = (live + 31) & ~31;
        uint8_t* vt = base_ptr + C::kOffStg + stage_of(t) * kTile8;
        for (int idx = lane; idx < (z1 - live) * 8; idx += 32) {   // 16-byte units of rows live .. z1-1
          const int rr = live + idx / 8, un = idx & 7;
          *reinterpret_cast<uint4*>(vt + rr * 128 + un * 16) = make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async();   // the P8 stores (and zeroed V8 rows) are read by the tensor cores
      mbar_arrive(bar(B_P_FULL + (j & 1)));
    }
    if (ok) ok = wwait(bar(B_O_DONE), 0);
    if (ok) {
      tc_fence_after();
      const float l448 = 448.f * (l2.x + l2.y);
      const float inv = l448 > 0.f ? 1.f / l448 : 0.f;
      uint16_t* orow = a.out + ((size_t)(q_start + q_local) * a.hq + h) * kHeadDim;
      const float* sfv = a.sf_v + (size_t)h_kv * kHeadDim;
      const float* vm = a.v_mean ? a.v_mean + (size_t)h_kv * kHeadDim : nullptr;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t ov[32];
        tmem_ld32(tmem_o + 32 * cc, ov);
        tmem_wait_ld();
#pragma unroll
        for (int g4 = 0; g4 < 4; ++g4) {
          float o8[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int d = 32 * cc + 8 * g4 + e;
            o8[e] = __ldg(sfv + d) * __uint_as_float(ov[8 * g4 + e]) * inv + (vm ? __ldg(vm + d) : 0.f);
          }
          uint4 w;
          w.x = pack_bf16x2(o8[0], o8[1]);
          w.y = pack_bf16x2(o8[2], o8[3]);
          w.z = pack_bf16x2(o8[4], o8[5]);
          w.w = pack_bf16x2(o8[6], o8[7]);
          if (row_valid) *reinterpret_cast<uint4*>(orow + 32 * cc + 8 * g4) = w;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(C::kTmemCols) : "memory");
  }
}

// [rows][heads][128] bytes as 3-D {128, rows, heads}; box {128, box_rows, 1}, 128-byte swizzle
bool encode_rows8(CUtensorMap* tm, const void* ptr, int64_t rows, int heads, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {128, (cuuint64_t)rows, (cuuint64_t)heads};
  const cuuint64_t strides[2] = {(cuuint64_t)heads * 128, 128};
  const cuuint32_t box[3] = {128, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_sage_extend(const SageExtendArgs& in, cudaStream_t s) {
  static std::atomic<bool> one_set[kMaxDevices], two_set[kMaxDevices];
  cudaError_t e0 = raise_smem_limit(sage_extend_kernel<1>, Cfg<1>::kSmemBytes, one_set);
  if (e0 == cudaSuccess) e0 = raise_smem_limit(sage_extend_kernel<2>, Cfg<2>::kSmemBytes, two_set);
  if (e0 != cudaSuccess) return e0;
  SageExtendLaunch a;
  if (!encode_rows8(&a.tm_q8, in.q8, in.q_rows, in.hq, 128) ||
      !encode_rows8(&a.tm_k8, in.k8, in.num_slots, in.hkv, kSageBlock) ||
      !encode_rows8(&a.tm_v8, in.v8, in.num_slots, in.hkv, kSageBlock))
    return cudaErrorInvalidValue;
  a.ws = in.ws;
  a.sf_q = in.sf_q;
  a.sf_k = in.sf_k;
  a.sf_v = in.sf_v;
  a.v_mean = in.v_mean;
  a.page_table = in.page_table;
  a.pt_pitch = in.pt_pitch;
  a.num_slots = in.num_slots;
  a.q_rows = in.q_rows;
  a.out = in.out;
  a.hq = in.hq;
  a.hkv = in.hkv;
  if ((in.hq / in.hkv) % 2 == 0)
    sage_extend_kernel<2><<<in.max_items * (in.hq / 2), Cfg<2>::kThreads, Cfg<2>::kSmemBytes, s>>>(a);
  else
    sage_extend_kernel<1><<<in.max_items * in.hq, Cfg<1>::kThreads, Cfg<1>::kSmemBytes, s>>>(a);
  return cudaGetLastError();
}

}  // namespace pa
