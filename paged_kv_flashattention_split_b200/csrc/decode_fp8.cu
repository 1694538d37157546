// decode_fp8.cu - split-KV decode over an FP8 (E4M3) KV cache with bf16 queries.
//
// The FlashAttention backend lists FP8 among its features ("Implement Flash
// Attention Back End in SGLang - Basics and KV Cache", feature list); the operation
// taken is the standard decode on the dequantised cache,
//     K = k_scale * E4M3(K8),  V = v_scale * E4M3(V8),
//     O = softmax(sm_scale * q K^T) V,  lse = log sum_j exp(sm_scale q . K_j),
// with one scale per pool.  The plan, its split partials and the merge are those of the
// bf16 decode.
//
// One CTA (8 warps, 97 KB of shared memory, two CTAs per SM) per (slot of the plan's flat
// partition, group of HG KV heads), HG = 8 at Hkv = 8, walking the work items of its slot:
// a token slot's 8-bit rows of the group are one contiguous
// HG * 128-byte run (1 KB), gathered with 16-byte cp.async into a 3-stage XOR-swizzled
// ring of TK = 16 * 8 / HG keys, like the bf16 kernel.  Warp (hw, kb) takes KV head hw and
// keys [16 kb, 16 kb + 16) of every tile.  E4M3 converts exactly to f16, and f16 products
// accumulate exactly in fp32, so the tensor-core path is f16 mma.sync m16n8k16:
//     S^T[16 keys x 8 heads] = K[16 x 128] . Q^T     (K8 bytes -> f16 pairs in registers)
//     O^T[128 d x 8 heads]  += V^T[128 x 16 keys] . P^T
// with Q converted from bf16 to f16 once (|q| < 65504 is required; values below 2^-24
// flush).  The 8-bit ldmatrix fragments hold 4 consecutive d of one key (QK) or 2 keys of
// two d (PV); the MMAs take the d (and key) index order those fragments come in, with Q and
// P arranged to match — a dot product does not depend on the order of its terms.
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "kernels.h"

namespace pa {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;
constexpr int kStages = 3;
constexpr int kHalfStage = 16 * 1024;                      // K8 (or V8) bytes of one tile
constexpr int kStageBytes = 2 * kHalfStage;
constexpr int kSlotBufBytes = 2 * 128 * 4;                 // slot ids of two tiles
constexpr int kSmem = kStages * kStageBytes + kSlotBufBytes;   // 97 KB: two CTAs per SM
constexpr float kLn2 = 0.693147180559945309f;

// D = A(16x16, row) * B(16x8, col) + D, f16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Two E4M3 codes (low byte first) to a packed f16 pair, exactly.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_codes) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(two_codes & 0xFFFFu), __NV_E4M3);
  return (uint32_t)h.x | ((uint32_t)h.y << 16);
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;\n" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  const __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}
__device__ __forceinline__ float f16lo_to_f32(uint32_t x) { return __half2float(__ushort_as_half((unsigned short)(x & 0xFFFFu))); }
__device__ __forceinline__ float f16hi_to_f32(uint32_t x) { return __half2float(__ushort_as_half((unsigned short)(x >> 16))); }

template <int HG, int G>
__global__ void __launch_bounds__(kThreads, 2) decode_fp8_kernel(Fp8DecodeLaunch a) {
  constexpr int WPH = kWarps / HG;            // warps per KV head
  constexpr int TK = 16 * WPH;                // keys per tile
  constexpr int CH = HG * 8;                  // 16-byte chunks in one key's 8-bit row of HG heads
  constexpr int ROW = CH * 16;                // bytes of that row
  constexpr int LOADS = kHalfStage / 16 / kThreads;   // copies per thread per tile, K8 and V8 each
  constexpr int KEY_STEP = kThreads / CH;     // keys one pass of the block covers
  static_assert(TK * ROW == kHalfStage && KEY_STEP * LOADS == TK && TK <= 128, "tile geometry");

  extern __shared__ __align__(128) uint8_t smem[];
  // the merge (a programmatic dependent) may be scheduled now; it waits for this grid to finish
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  // a programmatic dependent of whatever precedes it on the stream: nothing is read before
  // that grid is done
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  int32_t* sbuf = reinterpret_cast<int32_t*>(smem + kStages * kStageBytes);   // [2][TK]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, tig = lane & 3;
  PlanHeader* hdr = a.ws.hdr;
  if (hdr->magic != kMagic || hdr->mode != PA_MODE_DECODE) {
    if (tid == 0 && blockIdx.x == 0) set_device_error(hdr, PA_ERR_WORKSPACE);
    return;
  }
  const int groups = a.hkv / HG;
  const int slot = blockIdx.x / groups, grp = blockIdx.x % groups;
  if (slot >= hdr->slots) return;
  // this CTA's head group of every item of its slot of the plan's flat partition
  const int first = a.ws.slot_first[slot], last = min(a.ws.slot_first[slot + 1], hdr->num_items);
  for (int item = first; item < last; ++item) {
    const int4 it = a.ws.items[item];
    const int r = it.x, split = it.y, kv0 = it.z, kv1 = it.w;
    const int n_tiles = (kv1 - kv0 + TK - 1) / TK;
    const int hw = warp % HG, kb = warp / HG;
    const int h_kv = grp * HG + hw;

    // Q^T as the B operand, in f16, d in the order of the K fragments: for the 16-d chunk c,
    // b0 = Q[head gid][16c + 4tig, +1], b1 = Q[head gid][16c + 4tig + 2, +3].
    uint32_t qb0[8], qb1[8];
    {
      const uint2* qrow = reinterpret_cast<const uint2*>(a.q + ((size_t)r * a.hq + (size_t)h_kv * G + gid) * kHeadDim);
      #pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint2 v = gid < G ? __ldg(qrow + 4 * c + tig) : make_uint2(0u, 0u);   // 4 bf16 at 16c + 4tig
        qb0[c] = pack_f16x2(bf16lo_to_f32(v.x), bf16hi_to_f32(v.x));
        qb1[c] = pack_f16x2(bf16lo_to_f32(v.y), bf16hi_to_f32(v.y));
      }
    }

    const int page_shift = a.page_shift;
    const int page_mask = (1 << page_shift) - 1;
    const int32_t* table = a.page_table + (size_t)r * a.pt_pitch;
    auto table_entry = [&](int j) -> int { return j < kv1 ? __ldg(table + (j >> page_shift)) : -1; };
    auto entry_to_slot = [&](int page, int j) -> int {
      if (j >= kv1) return -1;
      const long long slot = ((long long)page << page_shift) + (j & page_mask);
      if (page < 0 || slot >= a.num_slots) {
        set_device_error(hdr, PA_ERR_DEVICE_INDEX);
        return -1;                                   // skipped: the row reads as zero
      }
      return (int)slot;
    };

    const int ld_c = tid % CH, ld_k0 = tid / CH;
    const size_t slot_stride = (size_t)a.hkv * kHeadDim;
    const size_t grp_off = (size_t)grp * HG * kHeadDim + (size_t)ld_c * 16;
    const uint32_t smem_base = smem_u32(smem);
    const uint64_t policy = l2_evict_first();   // KV rows stream through once
    auto issue = [&](int tile) {
      const uint32_t kst = smem_base + (tile % kStages) * kStageBytes;
      const int32_t* sl = sbuf + (tile & 1) * TK;
      #pragma unroll
      for (int i = 0; i < LOADS; ++i) {
        const int key = ld_k0 + KEY_STEP * i;
        const int slot = sl[key];
        const size_t off = slot >= 0 ? (size_t)slot * slot_stride + grp_off : 0;
        const int bytes = slot >= 0 ? 16 : 0;      // rows past the split (or bad ids) are zero-filled
        const uint32_t dst = kst + key * ROW + ((ld_c ^ (key & 7)) << 4);
        cp_async_16_hint(dst, a.k8_pool + off, bytes, policy);
        cp_async_16_hint(dst + kHalfStage, a.v8_pool + off, bytes, policy);
      }
    };

    if (tid < TK) {
      const int j0 = kv0 + tid, j1 = kv0 + TK + tid;
      sbuf[tid] = entry_to_slot(table_entry(j0), j0);
      sbuf[TK + tid] = entry_to_slot(table_entry(j1), j1);
    }
    __syncthreads();
    if (0 < n_tiles) issue(0);
    cp_async_commit();
    if (1 < n_tiles) issue(1);
    cp_async_commit();
    __syncthreads();
    if (tid < TK) {
      const int j2 = kv0 + 2 * TK + tid;
      sbuf[tid] = entry_to_slot(table_entry(j2), j2);
    }

    const float NEG_INF = -__int_as_float(0x7f800000);
    float m_run0 = NEG_INF, m_run1 = NEG_INF, l_run0 = 0.f, l_run1 = 0.f;
    float o[8][4];
    #pragma unroll
    for (int mt = 0; mt < 8; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;

    const int mat = lane >> 3;
    const int f_row = kb * 16 + (lane & 7) + ((mat & 1) << 3);   // fragment row (key) of this lane's ldmatrix address
    const uint32_t f_row_off = f_row * ROW;
    const int head_chunk = hw * 8;

    for (int t = 0; t < n_tiles; ++t) {
      cp_async_wait<kStages - 2>();
      __syncthreads();
      if (t + 2 < n_tiles) issue(t + 2);
      cp_async_commit();
      const int j_next = kv0 + (t + 3) * TK + tid;
      const int page_next = tid < TK ? table_entry(j_next) : -1;   // latency hidden by this tile

      const uint32_t kst = smem_base + (t % kStages) * kStageBytes;
      const uint32_t vst = kst + kHalfStage;
      // S^T = K . Q^T: one ldmatrix.x4 brings 16 keys x 32 d (two 16-d chunks)
      float s[4] = {0.f, 0.f, 0.f, 0.f};
      #pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        uint32_t kr[4];
        const int chunk = head_chunk + 2 * ks + (mat >> 1);
        ldmatrix_x4(kr, kst + f_row_off + ((chunk ^ (f_row & 7)) << 4));
        // kr[0]: key gid, d 32ks + 4tig .. +3; kr[1]: key gid + 8; kr[2], kr[3]: the same at d + 16
        uint32_t af[4];
        af[0] = e4m3x2_to_f16x2(kr[0]);
        af[1] = e4m3x2_to_f16x2(kr[1]);
        af[2] = e4m3x2_to_f16x2(kr[0] >> 16);
        af[3] = e4m3x2_to_f16x2(kr[1] >> 16);
        mma_f16_16816(s, af, qb0[2 * ks], qb1[2 * ks]);
        af[0] = e4m3x2_to_f16x2(kr[2]);
        af[1] = e4m3x2_to_f16x2(kr[3]);
        af[2] = e4m3x2_to_f16x2(kr[2] >> 16);
        af[3] = e4m3x2_to_f16x2(kr[3] >> 16);
        mma_f16_16816(s, af, qb0[2 * ks + 1], qb1[2 * ks + 1]);
      }
      const int key0 = kv0 + t * TK + kb * 16 + gid;
      const int key1 = key0 + 8;
      const float x00 = key0 < kv1 ? s[0] * a.scale_log2 : NEG_INF;
      const float x01 = key0 < kv1 ? s[1] * a.scale_log2 : NEG_INF;
      const float x10 = key1 < kv1 ? s[2] * a.scale_log2 : NEG_INF;
      const float x11 = key1 < kv1 ? s[3] * a.scale_log2 : NEG_INF;
      float mx0 = fmaxf(x00, x10), mx1 = fmaxf(x01, x11);
      #pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
      }
      const float mn0 = fmaxf(m_run0, mx0), mn1 = fmaxf(m_run1, mx1);
      const float mu0 = mn0 == NEG_INF ? 0.f : mn0;
      const float mu1 = mn1 == NEG_INF ? 0.f : mn1;
      const float al0 = ex2(m_run0 - mu0), al1 = ex2(m_run1 - mu1);
      m_run0 = mn0;
      m_run1 = mn1;
      const uint32_t pk0 = pack_f16x2(ex2(x00 - mu0), ex2(x01 - mu1));
      const uint32_t pk1 = pack_f16x2(ex2(x10 - mu0), ex2(x11 - mu1));
      // the row sum uses the same f16-rounded probabilities as the PV product
      l_run0 = l_run0 * al0 + f16lo_to_f32(pk0) + f16lo_to_f32(pk1);
      l_run1 = l_run1 * al1 + f16hi_to_f32(pk0) + f16hi_to_f32(pk1);
      #pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        o[mt][0] *= al0;
        o[mt][1] *= al1;
        o[mt][2] *= al0;
        o[mt][3] *= al1;
      }
      const uint32_t pb0 = movmatrix_trans(pk0);  // P^T[key 2tig..+1][head gid], keys 0-7
      const uint32_t pb1 = movmatrix_trans(pk1);  // keys 8-15
      // O^T += V^T . P^T: one ldmatrix.x4.trans brings 16 keys x two 16-byte d-blocks
      #pragma unroll
      for (int mp = 0; mp < 4; ++mp) {
        uint32_t vr[4];
        const int chunk = head_chunk + 2 * mp + (mat >> 1);
        ldmatrix_x4_trans(vr, vst + f_row_off + ((chunk ^ (f_row & 7)) << 4));
        // vr[0]: keys 2tig, 2tig+1 at d 2gid, 2gid+1 of block 2mp (keys 0-7); vr[1]: keys 8-15;
        // vr[2], vr[3]: the same for block 2mp + 1.  Row gid of the MMA is d 2gid, row gid + 8 is
        // d 2gid + 1.
        #pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t x = prmt(vr[2 * h], vr[2 * h], 0x3120);       // (k 2tig, k 2tig+1) at d 2gid | at d 2gid+1
          const uint32_t y = prmt(vr[2 * h + 1], vr[2 * h + 1], 0x3120);
          uint32_t af[4];
          af[0] = e4m3x2_to_f16x2(x);
          af[1] = e4m3x2_to_f16x2(x >> 16);
          af[2] = e4m3x2_to_f16x2(y);
          af[3] = e4m3x2_to_f16x2(y >> 16);
          mma_f16_16816(o[2 * mp + h], af, pb0, pb1);
        }
      }
      if (tid < TK) sbuf[((t + 3) & 1) * TK + tid] = entry_to_slot(page_next, j_next);
    }
    cp_async_wait<0>();
    __syncthreads();

    // Combine the warps of each head through shared memory.
    float* red_o = reinterpret_cast<float*>(smem);   // [warps][8 heads][128 d]
    float* red_m = red_o + kWarps * 8 * kHeadDim;    // [warps][8]
    float* red_l = red_m + kWarps * 8;               // [warps][8]
    #pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l_run0 += __shfl_xor_sync(0xffffffffu, l_run0, off);
      l_run1 += __shfl_xor_sync(0xffffffffu, l_run1, off);
    }
    if (gid == 0) {
      red_m[warp * 8 + 2 * tig] = m_run0;
      red_m[warp * 8 + 2 * tig + 1] = m_run1;
      red_l[warp * 8 + 2 * tig] = l_run0;
      red_l[warp * 8 + 2 * tig + 1] = l_run1;
    }
    #pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      const int d = 16 * mt + 2 * gid;
      float* h0 = red_o + (warp * 8 + 2 * tig) * kHeadDim;
      float* h1 = h0 + kHeadDim;
      *reinterpret_cast<float2*>(h0 + d) = make_float2(o[mt][0], o[mt][2]);
      *reinterpret_cast<float2*>(h1 + d) = make_float2(o[mt][1], o[mt][3]);
    }
    __syncthreads();

    const int splits = a.ws.req_splits[r];
    for (int idx = tid; idx < HG * G * kHeadDim; idx += kThreads) {
      const int hl = idx / (G * kHeadDim), g = (idx / kHeadDim) % G, d = idx % kHeadDim;
      float M = NEG_INF;
      #pragma unroll
      for (int k2 = 0; k2 < WPH; ++k2) M = fmaxf(M, red_m[(k2 * HG + hl) * 8 + g]);
      float O = 0.f, lse2 = NEG_INF;
      if (M != NEG_INF) {
        float wsum = 0.f, acc = 0.f;
        #pragma unroll
        for (int k2 = 0; k2 < WPH; ++k2) {
          const int wi = (k2 * HG + hl) * 8 + g;
          const float f = ex2(red_m[wi] - M);
          wsum += red_l[wi] * f;
          acc += red_o[wi * kHeadDim + d] * f;
        }
        O = a.v_scale * acc / wsum;
        lse2 = M + __log2f(wsum);
      }
      const int hq_idx = (grp * HG + hl) * G + g;
      if (splits == 1) {
        a.out[((size_t)r * a.hq + hq_idx) * kHeadDim + d] = __bfloat16_as_ushort(__float2bfloat16_rn(O));
        if (d == 0 && a.lse_out) a.lse_out[(size_t)r * a.hq + hq_idx] = lse2 * kLn2;
      } else {
        const size_t p = (size_t)(a.ws.req_base[r] + split) * a.hq + hq_idx;
        a.ws.partial_o[p * kHeadDim + d] = O;
        if (d == 0) a.ws.partial_lse[p] = lse2;
      }
    }
  }
}

template <int HG, int G>
cudaError_t launch_fp8_hg(const Fp8DecodeLaunch& a, cudaStream_t s) {
  static std::atomic<bool> smem_set[kMaxDevices];
  cudaError_t e = raise_smem_limit(decode_fp8_kernel<HG, G>, kSmem, smem_set);
  if (e != cudaSuccess) return e;
  e = launch_programmatic(decode_fp8_kernel<HG, G>, dim3(a.slots * (a.hkv / HG)), dim3(kThreads), kSmem, a, s);
  if (e != cudaSuccess) return e;
  DecodeLaunch m{};
  m.ws = a.ws;
  m.out = a.out;
  m.lse_out = a.lse_out;
  m.batch = a.batch;
  m.hq = a.hq;
  m.hkv = a.hkv;
  m.max_items = a.max_items;
  return launch_decode_merge(m, s);
}

template <int G>
cudaError_t launch_fp8_g(const Fp8DecodeLaunch& a, cudaStream_t s) {
  switch (decode_heads_per_cta(a.hkv)) {
    case 8: return launch_fp8_hg<8, G>(a, s);
    case 4: return launch_fp8_hg<4, G>(a, s);
    case 2: return launch_fp8_hg<2, G>(a, s);
    default: return launch_fp8_hg<1, G>(a, s);
  }
}

}  // namespace

cudaError_t launch_decode_fp8(const Fp8DecodeLaunch& a, cudaStream_t s) {
  switch (a.hq / a.hkv) {
    case 1: return launch_fp8_g<1>(a, s);
    case 2: return launch_fp8_g<2>(a, s);
    case 4: return launch_fp8_g<4>(a, s);
    case 8: return launch_fp8_g<8>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace pa
