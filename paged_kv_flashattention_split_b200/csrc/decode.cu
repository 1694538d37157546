// decode.cu - bf16 split-KV decode over the paged cache, and the log-sum-exp merge.
//
// One CTA (4 warps, 97 KB of shared memory, two CTAs per SM) per (slot of the
// plan's flat partition, group of HG KV heads), HG = 4 at Hkv = 8; the CTA walks
// the work items of its slot (pieces of requests of at most the slot's share of
// key tiles) one after the other.  It gathers each token slot's K
// and V rows of its heads as one contiguous HG * 256-byte run (1 KB): a warp's
// 16-byte cp.async copies cover 512 consecutive bytes, and the slots' rows are
// fetched from HBM once for all query heads that read them.  Tiles of
// TK = 16 * 4 / HG keys flow through a 3-stage, XOR-swizzled shared-memory ring;
// the slot ids of a tile are read from the table one tile ahead, by TK threads,
// with the load's latency hidden behind a tile of compute.  Warp (hw, kb) takes
// KV head hw of the group and keys [16 kb, 16 kb + 16) of every tile and
// computes, on the tensor cores,
//     S^T[16 keys x 8 heads] = K[16 x 128] . Q^T      (mma.m16n8k16, keys as M)
// for the G = Hq / Hkv <= 8 query heads that read this KV head.  The online
// softmax keeps a running max and sum per head (warp shuffles over the 8 key
// rows); the probabilities are rounded to bf16, transposed in registers with
// movmatrix and used as the B operand of
//     O^T[128 d x 8 heads] += V^T[128 x 16 keys] . P^T
// The warps of a head are combined through shared memory at the end.  A
// request covered by one split writes its bf16 output directly; otherwise
// each split writes (O_s, lse_s) and merge_kernel computes
//     lse = log2 sum_s 2^lse_s,  O = sum_s 2^(lse_s - lse) O_s.
//
// This is the tiled online-softmax evaluation of softmax(scale q K^T) V that
// "FlashAttention: 优化计算过程中的临时显存占用" (sections 1-2) describes:
// no score matrix ever reaches HBM, and the result equals the standard one.
#include "kernels.h"

namespace pa {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;
constexpr int kStages = 3;
constexpr int kHalfStage = 16 * 1024;                      // K (or V) bytes of one tile
constexpr int kStageBytes = 2 * kHalfStage;
constexpr int kSlotBufBytes = 2 * 64 * 4;                  // slot ids of two tiles
constexpr int kDecodeSmem = kStages * kStageBytes + kSlotBufBytes;   // 97 KB: two CTAs per SM
constexpr float kLn2 = 0.693147180559945309f;

__device__ __forceinline__ bool workspace_ok(const PlanHeader* hdr, int mode) {
  return hdr->magic == kMagic && hdr->mode == mode;
}

template <int HG, int G>
__global__ void __launch_bounds__(kThreads, 2) decode_splitkv_kernel(DecodeLaunch a) {
  constexpr int WPH = kWarps / HG;            // warps per KV head
  constexpr int TK = 16 * WPH;                // keys per tile
  constexpr int CH = HG * 16;                 // 16-byte chunks in one key's row of HG heads
  constexpr int ROW = CH * 16;                // bytes of that row
  constexpr int LOADS = kHalfStage / 16 / kThreads;   // copies per thread per tile, K and V each
  constexpr int KEY_STEP = kThreads / CH;     // keys one pass of the block covers
  static_assert(TK * ROW == kHalfStage && KEY_STEP * LOADS == TK, "tile geometry");

  extern __shared__ __align__(128) uint8_t smem[];
  // the merge kernel (launched as a programmatic dependent) may be scheduled now; it
  // waits for this whole grid to finish before it reads anything
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  // this grid is itself a programmatic dependent of whatever precedes it on the stream (the
  // previous layer's merge lets it start early): nothing is read before that grid is done
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  int32_t* sbuf = reinterpret_cast<int32_t*>(smem + kStages * kStageBytes);   // [2][TK]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, tig = lane & 3;
  PlanHeader* hdr = a.ws.hdr;
  if (!workspace_ok(hdr, PA_MODE_DECODE)) {
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

    // Q^T as the B operand: b0 = Q[head gid][16kk + 2tig .. +1], b1 = the same at +8.
    uint32_t qb0[8], qb1[8];
    {
      const uint32_t* qrow =
          reinterpret_cast<const uint32_t*>(a.q + ((size_t)r * a.hq + (size_t)h_kv * G + gid) * kHeadDim);
      #pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        qb0[kk] = gid < G ? __ldg(qrow + 8 * kk + tig) : 0u;
        qb1[kk] = gid < G ? __ldg(qrow + 8 * kk + 4 + tig) : 0u;
      }
    }

    const int page_shift = a.page_shift;
    const int page_mask = (1 << page_shift) - 1;
    const int32_t* table = a.page_table + (size_t)r * a.pt_pitch;
    // raw table entry for key j (or -1 past the split); checked when it is stored
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

    // Gather roles: thread -> chunk ld_c of keys ld_k0 + KEY_STEP * i.
    const int ld_c = tid % CH, ld_k0 = tid / CH;
    const size_t slot_stride = (size_t)a.hkv * kHeadDim;
    const size_t grp_off = (size_t)grp * HG * kHeadDim + (size_t)ld_c * 8;
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
        cp_async_16_hint(dst, a.k_pool + off, bytes, policy);
        cp_async_16_hint(dst + kHalfStage, a.v_pool + off, bytes, policy);
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

    // ldmatrix row/chunk roles of this lane (fragment layouts of mma.m16n8k16)
    const int mat = lane >> 3;
    const int k_row = kb * 16 + (lane & 7) + ((mat & 1) << 3);   // K as A: chunk + (mat >> 1)
    const int v_row = kb * 16 + (lane & 7) + ((mat >> 1) << 3);  // V^T as A: chunk + (mat & 1)
    const uint32_t k_row_off = k_row * ROW, v_row_off = v_row * ROW;
    const int head_chunk = hw * 16;

    for (int t = 0; t < n_tiles; ++t) {
      cp_async_wait<kStages - 2>();
      __syncthreads();
      if (t + 2 < n_tiles) issue(t + 2);
      cp_async_commit();
      const int j_next = kv0 + (t + 3) * TK + tid;
      const int page_next = tid < TK ? table_entry(j_next) : -1;   // latency hidden by this tile

      const uint32_t kst = smem_base + (t % kStages) * kStageBytes;
      const uint32_t vst = kst + kHalfStage;
      float s[4] = {0.f, 0.f, 0.f, 0.f};
      #pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        uint32_t af[4];
        const int chunk = head_chunk + 2 * kk + (mat >> 1);
        ldmatrix_x4(af, kst + k_row_off + ((chunk ^ (k_row & 7)) << 4));
        mma_bf16_16816(s, af, qb0[kk], qb1[kk]);
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
      const uint32_t pk0 = pack_bf16x2(ex2(x00 - mu0), ex2(x01 - mu1));
      const uint32_t pk1 = pack_bf16x2(ex2(x10 - mu0), ex2(x11 - mu1));
      // the row sum uses the same bf16-rounded probabilities as the PV product
      l_run0 = l_run0 * al0 + bf16lo_to_f32(pk0) + bf16lo_to_f32(pk1);
      l_run1 = l_run1 * al1 + bf16hi_to_f32(pk0) + bf16hi_to_f32(pk1);
      #pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        o[mt][0] *= al0;
        o[mt][1] *= al1;
        o[mt][2] *= al0;
        o[mt][3] *= al1;
      }
      const uint32_t pb0 = movmatrix_trans(pk0);  // P^T[key 2tig..+1][head gid], keys 0-7
      const uint32_t pb1 = movmatrix_trans(pk1);  // keys 8-15
      #pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        uint32_t af[4];
        const int chunk = head_chunk + 2 * mt + (mat & 1);
        ldmatrix_x4_trans(af, vst + v_row_off + ((chunk ^ (v_row & 7)) << 4));
        mma_bf16_16816(o[mt], af, pb0, pb1);
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
      const int d = 16 * mt + gid;
      float* h0 = red_o + (warp * 8 + 2 * tig) * kHeadDim;
      float* h1 = h0 + kHeadDim;
      h0[d] = o[mt][0];
      h1[d] = o[mt][1];
      h0[d + 8] = o[mt][2];
      h1[d + 8] = o[mt][3];
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
        O = acc / wsum;
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

// One warp per (request, query head) of a request that was split: combine the
// split partials, lse = log2 sum_s 2^lse_s, O = sum_s 2^(lse_s - lse) O_s.
// Lanes read the split LSEs in parallel; each lane owns 4 of the 128 outputs
// and keeps up to 8 splits' loads in flight.
__global__ void __launch_bounds__(256) merge_kernel(DecodeLaunch a) {
  asm volatile("griddepcontrol.wait;\n" ::: "memory");   // the decode grid has completed and its writes are visible
  // the next layer's decode grid (a programmatic dependent) may be scheduled: it waits for this one
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  PlanHeader* hdr = a.ws.hdr;
  if (!workspace_ok(hdr, PA_MODE_DECODE)) return;
  const int gw = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (gw >= a.batch * a.hq) return;
  const int r = gw / a.hq, h = gw % a.hq;
  const int splits = a.ws.req_splits[r];
  if (splits <= 1) return;
  const int base = a.ws.req_base[r];
  if (base + splits > a.max_items) return;  // only after a plan overflow, which the plan flags
  const float NEG_INF = -__int_as_float(0x7f800000);
  const float* lse = a.ws.partial_lse + (size_t)base * a.hq + h;      // stride hq per split
  const float* po = a.ws.partial_o + ((size_t)base * a.hq + h) * kHeadDim + 4 * lane;
  float M = NEG_INF;
  for (int sp = lane; sp < splits; sp += 32) M = fmaxf(M, lse[(size_t)sp * a.hq]);
  #pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float wpart = 0.f;
  if (M != NEG_INF) {
    for (int s0 = 0; s0 < splits; s0 += 32) {
      const float w_l = s0 + lane < splits ? ex2(lse[(size_t)(s0 + lane) * a.hq] - M) : 0.f;
      wpart += w_l;
      const int n = min(32, splits - s0);
      #pragma unroll 8
      for (int j = 0; j < n; ++j) {
        const float w = __shfl_sync(0xffffffffu, w_l, j);
        const float4 v = *reinterpret_cast<const float4*>(po + (size_t)(s0 + j) * a.hq * kHeadDim);
        acc.x += w * v.x;
        acc.y += w * v.y;
        acc.z += w * v.z;
        acc.w += w * v.w;
      }
    }
  }
  #pragma unroll
  for (int off = 16; off > 0; off >>= 1) wpart += __shfl_xor_sync(0xffffffffu, wpart, off);
  const float inv = M == NEG_INF ? 0.f : 1.f / wpart;
  uint2 packed;
  packed.x = pack_bf16x2(acc.x * inv, acc.y * inv);
  packed.y = pack_bf16x2(acc.z * inv, acc.w * inv);
  reinterpret_cast<uint2*>(a.out + ((size_t)r * a.hq + h) * kHeadDim)[lane] = packed;
  if (lane == 0 && a.lse_out)
    a.lse_out[(size_t)r * a.hq + h] = M == NEG_INF ? NEG_INF : (M + __log2f(wpart)) * kLn2;
}

__global__ void debug_gather_kernel(GatherLaunch a) {
  const int L = min(a.seq_lens[a.r], a.max_len);
  const int P = 1 << a.page_shift;
  const int32_t* table = a.page_table + (size_t)a.r * a.pt_pitch;
  for (int j = blockIdx.x; j < L; j += gridDim.x) {
    const int page = table[j >> a.page_shift];
    long long slot = (long long)page * P + (j & (P - 1));
    const bool ok = page >= 0 && slot < a.num_slots;
    if (threadIdx.x == 0) a.slots_out[j] = ok ? (int32_t)slot : -1;
    const uint16_t* src = a.k_pool + ((size_t)(ok ? slot : 0) * a.hkv + a.h_kv) * kHeadDim;
    for (int d = threadIdx.x; d < kHeadDim; d += blockDim.x)
      a.rows_out[(size_t)j * kHeadDim + d] = ok ? src[d] : (uint16_t)0;
  }
}

template <int HG, int G>
cudaError_t launch_decode_hg(const DecodeLaunch& a, cudaStream_t s) {
  static std::atomic<bool> smem_set[kMaxDevices];
  cudaError_t e = raise_smem_limit(decode_splitkv_kernel<HG, G>, kDecodeSmem, smem_set);
  if (e != cudaSuccess) return e;
  e = launch_programmatic(decode_splitkv_kernel<HG, G>, dim3(a.slots * (a.hkv / HG)), dim3(kThreads), kDecodeSmem, a, s);
  if (e != cudaSuccess) return e;
  return launch_decode_merge(a, s);
}

}  // namespace

// The merge is a programmatic dependent of the decode grid just launched on `s` (that grid
// executes griddepcontrol.launch_dependents): its launch overlaps the decode's tail.
cudaError_t launch_decode_merge(const DecodeLaunch& a, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((a.batch * a.hq + 7) / 8);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, merge_kernel, a);
}

namespace {

// A plan item covers decode_heads_per_cta(Hkv) <= 8 KV heads; a CTA of four warps takes at
// most four of them, so an item of eight heads is two CTAs.
template <int G>
cudaError_t launch_decode_g(const DecodeLaunch& a, cudaStream_t s) {
  switch (decode_heads_per_cta(a.hkv)) {
    case 8:
    case 4: return launch_decode_hg<4, G>(a, s);
    case 2: return launch_decode_hg<2, G>(a, s);
    default: return launch_decode_hg<1, G>(a, s);
  }
}

}  // namespace

cudaError_t launch_decode(const DecodeLaunch& a, cudaStream_t s) {
  switch (a.hq / a.hkv) {
    case 1: return launch_decode_g<1>(a, s);
    case 2: return launch_decode_g<2>(a, s);
    case 4: return launch_decode_g<4>(a, s);
    case 8: return launch_decode_g<8>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_debug_gather(const GatherLaunch& a, cudaStream_t s) {
  debug_gather_kernel<<<256, 128, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace pa
