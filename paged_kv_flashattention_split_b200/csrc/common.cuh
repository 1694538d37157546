// common.cuh - workspace layout and small device helpers shared by the kernels.
//
// The PTX wrappers below are thin spellings of documented sm_80+/sm_100a
// instructions (cp.async, ldmatrix, mma.sync, movmatrix, ex2.approx) so that
// the kernels read as the algorithm.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "pagedattn.h"

namespace pa {

constexpr int32_t kMagic = 0x4C504150;          // "PAPL"
constexpr int kHeadDim = 128;
constexpr int kDecodeMinTile = 64;               // keys per decode tile (and split granularity floor)
constexpr int kExtendQTile = 128;
constexpr int kExtendKvTile = 128;
constexpr int kSageBlock = 64;
constexpr int kSageUnit = 32;                    // keys per unit of the Sage partition
constexpr int kFlatCtasPerSm = 2;                // CTAs per SM a flat partition's slots are sized for
constexpr int kMaxBatch = 8192;
constexpr int kMaxSortItems = 16384;             // single-CTA bitonic sort capacity

// 64-byte header at the start of the workspace (layout documented in pagedattn.h).
struct PlanHeader {
  int32_t magic, mode, batch, hq, hkv, head_dim, page_size, num_items;
  int32_t max_items, tile, chunk_tiles, error_word;
  int32_t num_sms, max_splits, slots, reserved1;   // slots: CTA slots of a flat partition, else 0
};
static_assert(sizeof(PlanHeader) == 64, "header is 64 bytes");

// Byte offsets of the workspace arrays.
struct WsLayout {
  size_t req_splits, req_base, req_len, req_aux, req_prefix, items, slot_first, sel_base, sel_block, partial_o,
      partial_lse, item_max, scores, total;
  int64_t score_pitch;   // SAGE: keys per (request, head) row of the score scratch
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// KV heads one decode CTA covers: the largest of 8, 4, 2, 1 that divides Hkv.
__host__ __device__ inline int decode_heads_per_cta(int hkv) {
  return hkv % 8 == 0 ? 8 : hkv % 4 == 0 ? 4 : hkv % 2 == 0 ? 2 : 1;
}

// The Sage modes (dense and block-sparse) share the flat partition and the run kernels.
__host__ __device__ inline bool sage_mode(int mode) {
  return mode == PA_MODE_SAGE_DECODE || mode == PA_MODE_SAGE_SPARSE;
}

// Modes whose run kernels write split partials for a merge.
__host__ __device__ inline bool splitkv_mode(int mode) {
  return mode == PA_MODE_DECODE || sage_mode(mode);
}

// Modes planned as a flat partition of the requests' units over CTA slots.
__host__ __device__ inline bool flat_mode(int mode) { return splitkv_mode(mode); }

// CTA slots of a flat partition: max(1, floor(num_sms * 2 / groups)).
__host__ __device__ inline int flat_slots(int hkv, int num_sms) {
  const int groups = hkv / decode_heads_per_cta(hkv);
  const int c = num_sms * kFlatCtasPerSm / groups;
  return c > 1 ? c : 1;
}

inline WsLayout ws_layout(int mode, int batch, int hq, int hkv, int head_dim, int max_items, int max_kv_len,
                          int slots) {
  WsLayout w{};
  size_t off = sizeof(PlanHeader);
  w.req_splits = off; off += 4 * (size_t)batch;
  w.req_base = off;   off += 4 * (size_t)(batch + 1);
  w.req_len = off;    off += 4 * (size_t)batch;
  w.req_aux = off;    off += 4 * (size_t)batch;
  w.req_prefix = off; off += 4 * (size_t)batch;
  off = align_up(off, 16);
  w.items = off;      off += 16 * (size_t)max_items;
  off = align_up(off, 256);
  if (flat_mode(mode)) {
    w.slot_first = off; off += 4 * (size_t)(slots + 1);
    off = align_up(off, 256);
  }
  if (mode == PA_MODE_SAGE_SPARSE) {
    const size_t max_blocks = ((size_t)max_kv_len + kSageBlock - 1) / kSageBlock;
    w.sel_base = off;  off += 4 * (size_t)(batch + 1);
    off = align_up(off, 256);
    w.sel_block = off; off += 4 * (size_t)batch * max_blocks;
    off = align_up(off, 256);
  }
  if (splitkv_mode(mode)) {
    w.partial_o = off;   off += 4 * (size_t)max_items * hq * head_dim;
    off = align_up(off, 256);
    w.partial_lse = off; off += 4 * (size_t)max_items * hq;
    off = align_up(off, 256);
  }
  if (sage_mode(mode)) {
    w.item_max = off;    off += 4 * (size_t)max_items * hq;
    off = align_up(off, 256);
    w.score_pitch = (int64_t)align_up((size_t)(max_kv_len > kSageBlock ? max_kv_len : kSageBlock), kSageBlock);
    w.scores = off;      off += 4 * (size_t)batch * hq * (size_t)w.score_pitch;
    off = align_up(off, 256);
  }
  w.total = off;
  return w;
}

// Plain-data view of the workspace that kernels receive by value.
struct WsView {
  PlanHeader* hdr;
  int32_t* req_splits;
  int32_t* req_base;
  int32_t* req_len;
  int32_t* req_aux;
  int32_t* req_prefix;
  int4* items;
  int32_t* slot_first;  // DECODE, SAGE: [slots + 1] first item of each CTA slot
  int32_t* sel_base;    // SAGE_SPARSE: [B + 1] first selected block of each request in sel_block
  int32_t* sel_block;   // SAGE_SPARSE: the selected 64-key blocks, request by request
  float* partial_o;
  float* partial_lse;   // DECODE: split LSE (log2); SAGE: split row sum l
  float* item_max;      // SAGE: [max_items][Hq] maximum score of each split
  float* scores;        // SAGE: [B][Hq][score_pitch] the scores S
  int64_t score_pitch;
};

inline WsView ws_view(void* ws, const WsLayout& w) {
  char* b = static_cast<char*>(ws);
  WsView v;
  v.hdr = reinterpret_cast<PlanHeader*>(b);
  v.req_splits = reinterpret_cast<int32_t*>(b + w.req_splits);
  v.req_base = reinterpret_cast<int32_t*>(b + w.req_base);
  v.req_len = reinterpret_cast<int32_t*>(b + w.req_len);
  v.req_aux = reinterpret_cast<int32_t*>(b + w.req_aux);
  v.req_prefix = reinterpret_cast<int32_t*>(b + w.req_prefix);
  v.items = reinterpret_cast<int4*>(b + w.items);
  v.slot_first = w.slot_first ? reinterpret_cast<int32_t*>(b + w.slot_first) : nullptr;
  v.sel_base = w.sel_base ? reinterpret_cast<int32_t*>(b + w.sel_base) : nullptr;
  v.sel_block = w.sel_block ? reinterpret_cast<int32_t*>(b + w.sel_block) : nullptr;
  v.partial_o = w.partial_o ? reinterpret_cast<float*>(b + w.partial_o) : nullptr;
  v.partial_lse = w.partial_lse ? reinterpret_cast<float*>(b + w.partial_lse) : nullptr;
  v.item_max = w.item_max ? reinterpret_cast<float*>(b + w.item_max) : nullptr;
  v.scores = w.scores ? reinterpret_cast<float*>(b + w.scores) : nullptr;
  v.score_pitch = w.score_pitch;
  return v;
}

// Records the first device-side error in the header (later ones are dropped).
__device__ __forceinline__ void set_device_error(PlanHeader* hdr, int code) {
  atomicCAS(&hdr->error_word, 0, code);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte global->shared copy; src_bytes = 0 writes zeros without reading.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
// An L2 cache policy that marks the lines an access brings in as the first to evict: for data
// streamed through once (KV tiles), so it does not push out what is read again (partials,
// score rows, page tables).
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;\n" : "=l"(p));
  return p;
}
// The same with an L2 cache policy (createpolicy) for the line it reads.
__device__ __forceinline__ void cp_async_16_hint(uint32_t dst, const void* src, int src_bytes, uint64_t policy) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2, %3;\n" ::"r"(dst), "l"(src),
               "r"(src_bytes), "l"(policy)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// D = A(16x16, row) * B(16x8, col) + D, bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Transpose an 8x8 matrix of 16-bit elements held one row pair per thread.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}

// 2^x (hardware approximation; 2^-inf = 0).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// Two floats to a packed bf16 pair, round to nearest even; `lo` lands in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float bf16lo_to_f32(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t x) { return __uint_as_float(x & 0xFFFF0000u); }

}  // namespace pa
