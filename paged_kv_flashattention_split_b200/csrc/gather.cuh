// gather.cuh - slot-by-slot gather of K/V rows into the tensor cores' shared-memory layout.
//
// With pages of fewer than 8 slots (page size 1 makes the table the per-token
// req_to_token map itself: "Implement Flash Attention Back End in SGLang - Basics and
// KV Cache", KV-cache passage) a TMA box per page would move too few bytes per copy, so
// the extend kernels gather such tiles with 16-byte cp.async, one warp, straight into the
// same 128-byte-swizzled K-major / MN-major layout their TMA boxes produce:
//     [chunk c][row][128 B],  16-byte unit u of a row at ((u ^ (row & 7)) << 4).
#pragma once

#include "common.cuh"

namespace pa {

// Gathers rows [0, nrows_pad) (nrows_pad <= MAXROWS) of a tile whose row `row` is key
// key0 + row of the request (slot(key) = table[key >> page_shift] << page_shift +
// key % page_size) from KV head h_kv of a [num_slots][hkv][128] bf16 pool: NCHUNKS
// 64-element chunks per row starting at chunk0, chunk c at dst + c * chunk_bytes.  Rows
// >= nvalid and rows whose slot lies outside the pool are zero-filled (the latter also
// set PA_ERR_DEVICE_INDEX).  Called by all 32 lanes of one warp; the copies are left in
// flight (the caller commits and waits on them).  The rows' slot ids are read first, all
// at once (lane l reads rows l, l + 32, ...), and handed to the copying lanes by shuffles,
// so the table reads' latency is paid once per tile rather than once per copy.
template <int NCHUNKS, int MAXROWS>
__device__ __forceinline__ void gather_rows(uint32_t dst, uint32_t chunk_bytes, int chunk0, const uint16_t* pool,
                                            const int32_t* table, int key0, int nvalid, int nrows_pad,
                                            int page_shift, int page_size, int hkv, int h_kv, int64_t num_slots,
                                            PlanHeader* hdr, int lane) {
  constexpr int kUnits = NCHUNKS * 8;                    // 16-byte units per row
  constexpr int kRowsPerIter = 32 / kUnits;              // rows one warp-wide step covers
  static_assert(MAXROWS % 32 == 0 && kUnits <= 32, "gather geometry");
  int slot_of[MAXROWS / 32];                             // slot of row lane + 32 i, -1 if none
#pragma unroll
  for (int i = 0; i < MAXROWS / 32; ++i) {
    const int row = lane + 32 * i;
    slot_of[i] = -1;
    if (row < nvalid) {
      const int key = key0 + row;
      const int page = __ldg(table + (key >> page_shift));
      const long long slot = ((long long)page << page_shift) + (key & (page_size - 1));
      if (page >= 0 && slot < num_slots) slot_of[i] = (int)slot;
      else set_device_error(hdr, PA_ERR_DEVICE_INDEX);
    }
  }
#pragma unroll
  for (int it = 0; it < MAXROWS / kRowsPerIter; ++it) {
    const int row = it * kRowsPerIter + lane / kUnits;   // row / 32 is the same for the whole warp
    if (it * kRowsPerIter >= nrows_pad) break;
    const int slot = __shfl_sync(0xffffffffu, slot_of[(it * kRowsPerIter) / 32], row & 31);
    const int c = (lane % kUnits) >> 3, u = lane & 7;
    const uint32_t d = dst + c * chunk_bytes + row * 128 + ((u ^ (row & 7)) << 4);
    const bool live = row < nrows_pad && slot >= 0;
    const uint16_t* src = live ? pool + ((size_t)slot * hkv + h_kv) * kHeadDim + (chunk0 + c) * 64 + u * 8 : pool;
    if (row < nrows_pad) cp_async_16(d, src, live ? 16 : 0);
  }
}

}  // namespace pa
