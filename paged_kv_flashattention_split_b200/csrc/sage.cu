// sage.cu - 8-bit "Sage" decode over the paged cache.
//
// The formula ("FlashInfer PrimTS, Sage Attention 도입으로 8비트 양자화 및 성능
// 최적화 달성", 코드 분석 item 1, README "Sage attention"):
//     S_j  = sfQ[r][h] * sfK[blk(j)][h_kv] * (Q8 . K8_j)
//     P    = softmax_row(S), quantised to E4M3 as 448 p
//     O[d] = sfV[h_kv][d] * (sum_j P8_j V8_j[d]) / (448 l) + v_mean[h_kv][d]
// with the scales applied before the row max and the exponential and sfV in
// the epilogue (same page, item 4).
//
// Quantising p needs the row max m over ALL keys before any P8 is formed.
// A thread-block cluster of 4 CTAs takes one (request, KV head): CTA q scores
// the q-th quarter of the keys, keeps its scores in shared memory, and the
// four CTAs exchange their maxima through distributed shared memory, so every
// CTA quantises against the exact global m.  Then each CTA streams its V8
// rows, and the four partial sums are reduced through distributed shared
// memory by CTA 0, which applies the epilogue.  No score ever reaches HBM and
// no CTA waits on anything but the cluster barrier (its CTAs are co-scheduled).
//
// Per CTA (4 warps), in 64-key tiles (one 64-slot page each):
//   QK: S^T[16 keys x 8 heads] = K8[16 x 128] . Q8^T on the INT8 tensor cores
//       (mma.m16n8k32.s8, exact int32 dot), S = fp32(fp32(sfQ sfK) fp32(dot));
//   PV: O[16 (G heads used) x 8 d] += P8[16 x 32 keys] . V8[32 keys x 8 d] on
//       the FP8 tensor cores (mma.m16n8k32.e4m3, fp32 accumulation).  V8 is
//       key-major in memory; ldmatrix.trans on byte pairs plus one byte
//       permute gives 4 keys per register, with the keys of a register in a
//       fixed order that P8's A fragment uses too (the sum over keys does not
//       depend on their order).
#include "kernels.h"

namespace pa {

namespace {
constexpr int kThreads = 128;
constexpr int kClusterCtas = 4;
constexpr int kTileKeys = 64;                      // = one sfK block = one page
constexpr int kRowBytes = kHeadDim;                // 8-bit rows: 128 bytes per (slot, head)
constexpr int kTileBytes = kTileKeys * kRowBytes;  // 8 KB
constexpr int kStages = 4;
constexpr float kLog2e = 1.4426950408889634f;
}  // namespace

// Keys of score storage per CTA and head: a quarter of max_kv_len, rounded up to whole tiles.
int sage_cap(int max_kv_len) {
  const int per = (max_kv_len + kClusterCtas - 1) / kClusterCtas;
  return (per + kTileKeys - 1) / kTileKeys * kTileKeys;
}
size_t sage_smem_bytes(int G, int cap) {
  return (size_t)kStages * kTileBytes + (size_t)G * cap * 4 + (32 + 8 + 8) * 4 + (size_t)G * kHeadDim * 4 +
         (size_t)(cap / kTileKeys) * 8;
}
static size_t sage_smem_bytes_max() { return sage_smem_bytes(8, (int)(kSageScoreBudget / (8 * 4))); }

namespace {

__device__ __forceinline__ void mma_s8_16832(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_e4m3_16832(float (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
  const uint32_t zero = 0u;   // A rows 8..15 (heads 8..15) are empty for G <= 8
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(zero), "r"(a2), "r"(zero), "r"(b0), "r"(b1));
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

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}

// Load a float from CTA `rank`'s shared memory at the address `local` has in this CTA.
__device__ __forceinline__ float ld_dsmem_f32(const float* local, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];\n" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

struct SageLaunch {
  WsView ws;  // same fields as SageLaunchArgs, with cap in place of max_kv_len
  const int8_t* q8;
  const float* sf_q;
  const int8_t* k8;
  const uint8_t* v8;
  const float* sf_k;
  const float* sf_v;
  const float* v_mean;
  int64_t num_slots;
  const int32_t* page_table;
  int64_t pt_pitch;
  uint16_t* out;
  int batch, hq, hkv, cap;        // cap: score capacity per CTA per head (keys, multiple of 64)
};

template <int G>
__global__ void __cluster_dims__(kClusterCtas, 1, 1) __launch_bounds__(kThreads)
sage_decode_kernel(SageLaunch a) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* ring = smem;                                             // [kStages][64 keys][128 B]
  float* S = reinterpret_cast<float*>(smem + kStages * kTileBytes);  // [G][cap]
  float* red = S + G * a.cap;                                       // [4 warps][8] maxima
  float* cta_max = red + 32;                                        // [8]
  float* part_l = cta_max + 8;                                      // [8]
  float* part_o = part_l + 8;                                       // [G][128]
  int32_t* tile_page = reinterpret_cast<int32_t*>(part_o + G * kHeadDim);   // [cap / 64] page of each tile
  float* tile_sfk = reinterpret_cast<float*>(tile_page + a.cap / kTileKeys);  // [cap / 64] its K scale

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const float NEG_INF = -__int_as_float(0x7f800000);
  PlanHeader* hdr = a.ws.hdr;
  const bool ok = hdr->magic == kMagic && hdr->mode == PA_MODE_SAGE_DECODE;
  const int cluster = blockIdx.x / kClusterCtas;
  const uint32_t rank = cluster_ctarank();
  const int item = cluster / a.hkv, h_kv = cluster % a.hkv;
  // Every CTA of a cluster takes the same branch here, so the cluster barriers below always pair up.
  if (!ok || item >= hdr->num_items) {
    if (!ok && tid == 0 && blockIdx.x == 0) set_device_error(hdr, PA_ERR_WORKSPACE);
    return;
  }
  const int4 it = a.ws.items[item];
  const int r = it.x, L = it.w;
  const int C = ((L + kClusterCtas - 1) / kClusterCtas + kTileKeys - 1) / kTileKeys * kTileKeys;
  const int k0 = min((int)rank * C, L), k1 = min(k0 + C, L);
  const int n_tiles = (k1 - k0 + kTileKeys - 1) / kTileKeys;
  const int32_t* table = a.page_table + (size_t)r * a.pt_pitch;
  const size_t slot_stride = (size_t)a.hkv * kRowBytes;
  const uint32_t ring_base = smem_u32(ring);

  // Tile t covers keys k0 + 64 t .. +63, all in one page (k0 is a multiple of 64).  The page
  // ids and K scales of all this CTA's tiles are read once, up front, so no copy ever waits
  // on a table read.
  for (int t = tid; t < n_tiles; t += kThreads) {
    const int page = __ldg(table + ((k0 + t * kTileKeys) >> 6));
    const bool good = page >= 0 && ((long long)page + 1) * kTileKeys <= a.num_slots;
    if (!good) set_device_error(hdr, PA_ERR_DEVICE_INDEX);
    tile_page[t] = good ? page : -1;
    tile_sfk[t] = good ? __ldg(a.sf_k + (size_t)page * a.hkv + h_kv) : 0.f;
  }
  __syncthreads();
  // 64 rows x 128 B: thread -> chunk (tid % 8) of rows tid / 8 + 16 i
  auto issue = [&](const uint8_t* pool, int t) {
    const int stage = t % kStages;
    const int page = tile_page[t];
    const uint32_t dst0 = ring_base + stage * kTileBytes;
    const int c = tid & 7;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int row = (tid >> 3) + 16 * i;
      const int j = k0 + t * kTileKeys + row;
      const bool valid = page >= 0 && j < k1;   // keys past the range read as zero
      const size_t off = valid ? ((size_t)page * kTileKeys + row) * slot_stride + (size_t)h_kv * kRowBytes + c * 16 : 0;
      cp_async_16(dst0 + row * kRowBytes + ((c ^ (row & 7)) << 4), pool + off, valid ? 16 : 0);
    }
  };

  // ---------------- phase 1: scores into shared memory, per-head maxima
  uint32_t qb0[4], qb1[4];
  {
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(a.q8 + ((size_t)r * a.hq + (size_t)h_kv * G + gid) * kHeadDim);
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      qb0[ks] = gid < G ? __ldg(qrow + 8 * ks + tig) : 0u;
      qb1[ks] = gid < G ? __ldg(qrow + 8 * ks + 4 + tig) : 0u;
    }
  }
  const int col0 = 2 * tig, col1 = 2 * tig + 1;           // this thread's head columns of S^T
  const float sfq0 = col0 < G ? __ldg(a.sf_q + (size_t)r * a.hq + h_kv * G + col0) : 0.f;
  const float sfq1 = col1 < G ? __ldg(a.sf_q + (size_t)r * a.hq + h_kv * G + col1) : 0.f;
  const int mat = lane >> 3;
  const int k_row = warp * 16 + (lane & 7) + ((mat & 1) << 3);
  float mx0 = NEG_INF, mx1 = NEG_INF;

  for (int t = 0; t < kStages - 1; ++t) {
    if (t < n_tiles) issue(reinterpret_cast<const uint8_t*>(a.k8), t);
    cp_async_commit();
  }
  for (int t = 0; t < n_tiles; ++t) {
    cp_async_wait<kStages - 2>();
    __syncthreads();
    if (t + kStages - 1 < n_tiles) issue(reinterpret_cast<const uint8_t*>(a.k8), t + kStages - 1);
    cp_async_commit();
    const int stage = t % kStages;
    const uint32_t kst = ring_base + stage * kTileBytes;
    int acc[4] = {0, 0, 0, 0};
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      uint32_t af[4];
      const int chunk = 2 * ks + (mat >> 1);
      ldmatrix_x4(af, kst + k_row * kRowBytes + ((chunk ^ (k_row & 7)) << 4));
      mma_s8_16832(acc, af, qb0[ks], qb1[ks]);
    }
    const float sfk = tile_sfk[t];
    const int jl0 = t * kTileKeys + warp * 16 + gid, jl1 = jl0 + 8;   // key index within this CTA's range
    const bool v0 = k0 + jl0 < k1, v1 = k0 + jl1 < k1;
    // S = fp32(fp32(sfQ sfK) fp32(dot)); the int32 dot is exact and |dot| < 2^24
    const float s00 = v0 ? (sfq0 * sfk) * (float)acc[0] : NEG_INF;
    const float s01 = v0 ? (sfq1 * sfk) * (float)acc[1] : NEG_INF;
    const float s10 = v1 ? (sfq0 * sfk) * (float)acc[2] : NEG_INF;
    const float s11 = v1 ? (sfq1 * sfk) * (float)acc[3] : NEG_INF;
    if (col0 < G) {
      S[col0 * a.cap + jl0] = s00;
      S[col0 * a.cap + jl1] = s10;
      mx0 = fmaxf(mx0, fmaxf(s00, s10));
    }
    if (col1 < G) {
      S[col1 * a.cap + jl0] = s01;
      S[col1 * a.cap + jl1] = s11;
      mx1 = fmaxf(mx1, fmaxf(s01, s11));
    }
  }
  cp_async_wait<0>();
  __syncthreads();                                             // every warp is done with the K8 ring
  // the first V8 tiles do not depend on the maximum: start them before the exchange
  for (int t = 0; t < kStages - 1; ++t) {
    if (t < n_tiles) issue(a.v8, t);
    cp_async_commit();
  }
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
  }
  if (gid == 0) {
    red[warp * 8 + col0] = mx0;
    red[warp * 8 + col1] = mx1;
  }
  __syncthreads();
  if (tid < 8) cta_max[tid] = fmaxf(fmaxf(red[tid], red[8 + tid]), fmaxf(red[16 + tid], red[24 + tid]));
  cluster_sync();                                              // #1: every CTA's maxima are visible

  // ---------------- phase 2: P8 = E4M3(448 exp(S - m)), l, and O = P8 . V8
  // This thread forms P8 for head gid (gid < G) at the keys {2tig, 2tig+1, 8+2tig, 9+2tig}
  // (+16) of each 32-key step: the key order the V8 fragments below come in.
  float m_h = NEG_INF;
  if (gid < G)
    for (uint32_t q = 0; q < kClusterCtas; ++q) m_h = fmaxf(m_h, ld_dsmem_f32(cta_max + gid, q));
  const float m_use = m_h == NEG_INF ? 0.f : m_h;
  const float* Sh = S + (gid < G ? gid : 0) * a.cap;
  float lsum = 0.f;
  float oe[2][4], oo[2][4];          // d-blocks 2 warp and 2 warp + 1: even / odd d columns
#pragma unroll
  for (int b = 0; b < 2; ++b)
#pragma unroll
    for (int i = 0; i < 4; ++i) oe[b][i] = oo[b][i] = 0.f;

  for (int t = 0; t < n_tiles; ++t) {
    cp_async_wait<kStages - 2>();
    __syncthreads();
    if (t + kStages - 1 < n_tiles) issue(a.v8, t + kStages - 1);
    cp_async_commit();
    const uint32_t vst = ring_base + (t % kStages) * kTileBytes;
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      uint32_t pa0 = 0u, pa2 = 0u;
      if (gid < G) {
        const int base = t * kTileKeys + 32 * ks;
        float p[8];
        const int keys[8] = {2 * tig, 2 * tig + 1, 8 + 2 * tig, 9 + 2 * tig,
                             16 + 2 * tig, 17 + 2 * tig, 24 + 2 * tig, 25 + 2 * tig};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int jl = base + keys[i];
          const float sv = k0 + jl < k1 ? Sh[jl] : NEG_INF;
          p[i] = ex2((sv - m_use) * kLog2e);                  // exp(S - m), 0 for masked keys
          lsum += p[i];
        }
        pa0 = e4m3x2(448.f * p[0], 448.f * p[1]) | (e4m3x2(448.f * p[2], 448.f * p[3]) << 16);
        pa2 = e4m3x2(448.f * p[4], 448.f * p[5]) | (e4m3x2(448.f * p[6], 448.f * p[7]) << 16);
      }
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        const int db = 2 * warp + b;                          // 16-byte d-block of this warp
        const int vkey = 32 * ks + 8 * mat + (lane & 7);
        uint32_t vr[4];
        ldmatrix_x4_trans(vr, vst + vkey * kRowBytes + ((db ^ (vkey & 7)) << 4));
        const uint32_t be0 = prmt(vr[0], vr[1], 0x6420), bo0 = prmt(vr[0], vr[1], 0x7531);
        const uint32_t be1 = prmt(vr[2], vr[3], 0x6420), bo1 = prmt(vr[2], vr[3], 0x7531);
        mma_e4m3_16832(oe[b], pa0, pa2, be0, be1);
        mma_e4m3_16832(oo[b], pa0, pa2, bo0, bo1);
      }
    }
  }
  cp_async_wait<0>();
  // l for head gid: every warp formed the same probabilities; warp 0's sum is used
  lsum += __shfl_xor_sync(0xffffffffu, lsum, 1);
  lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);
  if (warp == 0 && tig == 0 && gid < G) part_l[gid] = lsum;
  if (gid < G) {
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      const int d = 16 * (2 * warp + b) + 4 * tig;
      float* row = part_o + gid * kHeadDim;
      row[d] = oe[b][0];
      row[d + 2] = oe[b][1];
      row[d + 1] = oo[b][0];
      row[d + 3] = oo[b][1];
    }
  }
  cluster_sync();                                              // #2: partials are visible

  if (rank == 0) {
    for (int idx = tid; idx < G * kHeadDim; idx += kThreads) {
      const int h = idx / kHeadDim, d = idx % kHeadDim;
      float acc = 0.f, l = 0.f;
      for (uint32_t q = 0; q < kClusterCtas; ++q) {
        acc += ld_dsmem_f32(part_o + idx, q);
        l += ld_dsmem_f32(part_l + h, q);
      }
      const float vm = a.v_mean ? __ldg(a.v_mean + (size_t)h_kv * kHeadDim + d) : 0.f;
      const float sfv = __ldg(a.sf_v + (size_t)h_kv * kHeadDim + d);
      const float o = l > 0.f ? sfv * acc / (448.f * l) + vm : vm;
      a.out[((size_t)r * a.hq + h_kv * G + h) * kHeadDim + d] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
    }
  }
  cluster_sync();                                              // #3: CTA 0 is done reading the others
}

template <int G>
cudaError_t launch_sage_g(const SageLaunch& a, size_t smem, cudaStream_t s) {
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(sage_decode_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)sage_smem_bytes_max());
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  sage_decode_kernel<G><<<a.batch * a.hkv * kClusterCtas, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sage(const SageLaunchArgs& in, cudaStream_t s) {
  SageLaunch a;
  a.ws = in.ws;
  a.q8 = in.q8;
  a.sf_q = in.sf_q;
  a.k8 = in.k8;
  a.v8 = in.v8;
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
  a.cap = sage_cap(in.max_kv_len);
  const int G = in.hq / in.hkv;
  const size_t smem = sage_smem_bytes(G, a.cap);
  switch (G) {
    case 1: return launch_sage_g<1>(a, smem, s);
    case 2: return launch_sage_g<2>(a, smem, s);
    case 4: return launch_sage_g<4>(a, smem, s);
    case 8: return launch_sage_g<8>(a, smem, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace pa
