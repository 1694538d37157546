// plan.cu - the per-batch scheduling plan (one CTA, integer arithmetic only).
//
// The scheduling metadata is a function of the sequence lengths (and, for a
// prefill, the cumulative query lengths) alone, so it is built once per batch
// and reused by every layer ("SGLang의 FA3 디코드 최적화: get_scheduler_metadata
// 도입", 코드 분석 items 1-3, 왜 이게 좋은가 item 1).  The algorithm is the one
// stated at attn_plan in pagedattn.h; every step is integer so the result is
// exact and identical on recomputation.
#include <algorithm>

#include "kernels.h"

namespace pa {
namespace {

constexpr int kPlanThreads = 1024;

__device__ __forceinline__ long long cdiv_ll(long long a, long long b) { return (a + b - 1) / b; }

// Block-wide exclusive scan of one int per thread (blockDim.x a multiple of 32, at most 1024);
// returns this thread's prefix.  Warps scan by shuffles, one warp scans the warp totals:
// two barriers (and one more before `scratch`, 33 ints, may be reused).
__device__ int block_exclusive_scan(int v, int* scratch, int* total) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nw ? scratch[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    scratch[lane] = w;                            // inclusive over warps 0 .. lane
    if (lane == 31) scratch[32] = w;
  }
  __syncthreads();
  const int before = warp > 0 ? scratch[warp - 1] : 0;
  *total = scratch[32];
  __syncthreads();
  return before + x - v;
}

// The block mask of one request, 512 blocks per warp-wide step: lane l holds blocks
// b0 + 16 l .. b0 + 16 l + 15 as bits 0..15 (16 independent byte loads, so one load latency).
__device__ __forceinline__ uint32_t mask_bits(const uint8_t* m, int b0, int nb, int lane) {
  uint32_t bits = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int b = b0 + 16 * lane + i;
    if (b < nb && __ldg(m + b) != 0) bits |= 1u << i;
  }
  return bits;
}

// EXTEND: work of query tile s (key tiles it needs) for the sort key; items run longest first.
__device__ __forceinline__ int item_work(int s, int prefix, int n) {
  const int q1 = min((s + 1) * kExtendQTile, n);
  return (int)cdiv_ll(prefix + q1, kExtendKvTile);
}

// DECODE, SAGE_DECODE, SAGE_SPARSE: the flat partition of the requests' units (T-key tiles
// for DECODE, 32-key units for Sage, of the selected 64-key blocks only for SAGE_SPARSE)
// over CTA slots (the algorithm at attn_plan).  Items come out r-major, which is also slot
// order, so no sort.  Each thread owns the requests [r0, r1) through every step; the
// per-request values live in shared memory (`sm`, 3 B + max_items ints), so the only global
// reads are the lengths and the masks, issued together, and the workspace is written once.
__device__ void flat_plan(const PlanLaunch& a, int* sm, int* scan, int* chunk_out, int* n_out) {
  const int tid = threadIdx.x, nt = blockDim.x;
  WsView ws = a.ws;
  PlanHeader* hdr = ws.hdr;
  const int B = a.batch;
  const bool sparse = a.mode == PA_MODE_SAGE_SPARSE;
  const int U = a.mode == PA_MODE_DECODE ? a.tile : kSageUnit;   // keys per unit
  int* s_len = sm;               // L_r
  int* s_units = sm + B;         // units of request r
  int* s_sel = sm + 2 * B;       // SAGE_SPARSE: selected blocks of r, then sel_base[r]
  int* item_slot = sm + 3 * B;   // [max_items]
  const int warp = tid >> 5, lane = tid & 31, nwarps = nt >> 5;
  const int per_t = (B + nt - 1) / nt;
  const int r0 = min(B, tid * per_t), r1 = min(B, r0 + per_t);
  auto clamp_len = [&](int L) {
    if (L < 0 || L > a.max_kv_len) {
      set_device_error(hdr, PA_ERR_DEVICE_INDEX);
      L = max(0, min(L, a.max_kv_len));
    }
    return L;
  };
  // 1. lengths (clamped and flagged when out of range), the units of each request, and its
  //    selected block count (SAGE_SPARSE)
  uint32_t kept_bits = 0;        // SAGE_SPARSE: this lane's mask bits of the warp's one request
  const bool keep = sparse && B <= nwarps;
  if (!sparse) {
    for (int r = r0; r < r1; ++r) {
      const int L = clamp_len(a.seq_lens[r]);
      s_len[r] = L;
      s_units[r] = (int)cdiv_ll(L, U);
      ws.req_len[r] = L;
      ws.req_prefix[r] = 0;
    }
  } else {
    // one warp per request; the first 512 mask bytes are read together with the length (the
    // row holds mask_pitch >= ceil(max_kv_len / 64) bytes) and cut to ceil(L / 64) blocks
    const int first_chunk = (int)min(a.mask_pitch, (int64_t)512);
    for (int r = warp; r < B; r += nwarps) {
      const uint8_t* m = a.block_mask + (size_t)r * a.mask_pitch;
      const int L_raw = a.seq_lens[r];
      uint32_t bits = mask_bits(m, 0, first_chunk, lane);
      int L = L_raw;
      if (L < 0 || L > a.max_kv_len) {
        if (lane == 0) set_device_error(hdr, PA_ERR_DEVICE_INDEX);
        L = max(0, min(L, a.max_kv_len));
      }
      const int nb = (int)cdiv_ll(L, kSageBlock);
      const int live = nb - 16 * lane;                   // blocks of this lane's 16 inside the row
      bits &= live >= 16 ? 0xFFFFu : live > 0 ? (1u << live) - 1u : 0u;
      int nsel = __popc(bits);
      bool last_sel = live >= 1 && live <= 16 && ((bits >> (live - 1)) & 1u);
      if (keep) kept_bits = bits;
      for (int b0 = 512; b0 < nb; b0 += 512) {           // rows of more than 512 blocks
        const uint32_t more = mask_bits(m, b0, nb, lane);
        nsel += __popc(more);
        const int i_last = nb - 1 - b0 - 16 * lane;
        if (i_last >= 0 && i_last < 16) last_sel = (more >> i_last) & 1u;
      }
      for (int o = 16; o > 0; o >>= 1) nsel += __shfl_xor_sync(0xffffffffu, nsel, o);
      // two 32-key units per selected block; a last block of <= 32 keys is one unit
      const bool short_last = __any_sync(0xffffffffu, last_sel) && L - kSageBlock * (nb - 1) <= kSageUnit;
      if (lane == 0) {
        s_len[r] = L;
        s_units[r] = 2 * nsel - (short_last ? 1 : 0);
        s_sel[r] = nsel;
        ws.req_len[r] = L;
        ws.req_prefix[r] = 0;
      }
    }
  }
  __syncthreads();
  if (sparse) {
    // sel_base = exclusive prefix sum of the selected block counts; then the block lists
    int local_b = 0;
    for (int r = r0; r < r1; ++r) local_b += s_sel[r];
    int total_b = 0;
    int run_b = block_exclusive_scan(local_b, scan, &total_b);
    for (int r = r0; r < r1; ++r) {
      const int n = s_sel[r];
      s_sel[r] = run_b;
      ws.sel_base[r] = run_b;
      run_b += n;
    }
    if (tid == 0) ws.sel_base[B] = total_b;
    __syncthreads();
    for (int r = warp; r < B; r += nwarps) {    // the selected blocks in ascending order, a warp per request
      const int nb = (int)cdiv_ll(s_len[r], kSageBlock);
      const uint8_t* m = a.block_mask + (size_t)r * a.mask_pitch;
      int k = s_sel[r];
      for (int b0 = 0; b0 < nb; b0 += 512) {
        uint32_t bits = keep && b0 == 0 ? kept_bits : mask_bits(m, b0, nb, lane);
        const int cnt = __popc(bits);
        int incl = cnt;                                     // lanes before this one hold lower blocks
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        int at = k + incl - cnt;
        while (bits) {
          const int i = __ffs(bits) - 1;
          ws.sel_block[at++] = b0 + 16 * lane + i;
          bits &= bits - 1;
        }
        k += __shfl_sync(0xffffffffu, incl, 31);
      }
    }
  }
  // 2. g_r = exclusive prefix sum of the units (written to req_aux), total
  int local = 0;
  for (int r = r0; r < r1; ++r) local += s_units[r];
  int total = 0;
  const int run_u = block_exclusive_scan(local, scan, &total);
  const int per = (int)max(1LL, cdiv_ll(total, a.slots));
  const int used = (int)cdiv_ll(total, per);
  // 3. pieces per request, then req_base
  auto pieces = [&](int u, int g) { return u > 0 ? (g + u - 1) / per - g / per + 1 : 1; };
  int local_s = 0;
  for (int r = r0, g = run_u; r < r1; ++r) {
    const int u = s_units[r];
    const int sp = pieces(u, g);
    ws.req_aux[r] = g;
    ws.req_splits[r] = sp;
    local_s += sp;
    g += u;
  }
  int n_items = 0;
  const int run_s = block_exclusive_scan(local_s, scan, &n_items);
  if (tid == 0) ws.req_base[B] = n_items;
  if (n_items > a.max_items) {  // cannot happen (bound slots + B); keep the grid safe
    if (tid == 0) set_device_error(hdr, PA_ERR_DEVICE_INDEX);
    n_items = a.max_items;
  }
  // 4. the items (key ranges; SAGE_SPARSE: unit ranges) and the slot of each
  for (int r = r0, g = run_u, base = run_s; r < r1; ++r) {
    const int L = s_len[r], u = s_units[r];
    ws.req_base[r] = base;
    if (u == 0) {
      if (base < n_items) {
        ws.items[base] = make_int4(r, 0, 0, 0);
        item_slot[base] = min(g / per, max(used - 1, 0));
      }
    } else {
      const int c_first = g / per, c_last = (g + u - 1) / per;
      for (int c = c_first; c <= c_last; ++c) {
        const int i = base + (c - c_first);
        if (i >= n_items) break;
        const int u0 = max(g, c * per) - g, u1 = min(g + u, (c + 1) * per) - g;
        ws.items[i] = sparse ? make_int4(r, c - c_first, u0, u1)
                             : make_int4(r, c - c_first, u0 * U, (int)min((long long)u1 * U, (long long)L));
        item_slot[i] = c;
      }
    }
    base += pieces(u, g);
    g += u;
  }
  for (int c = tid; c <= a.slots; c += nt) ws.slot_first[c] = n_items;
  __syncthreads();
  // 5. slot_first[c] = first item whose slot is >= c (slots are non-decreasing along the list)
  for (int i = tid; i < n_items; i += nt) {
    const int c_prev = i > 0 ? item_slot[i - 1] : -1;
    for (int c = c_prev + 1; c <= item_slot[i]; ++c) ws.slot_first[c] = i;
  }
  *chunk_out = per;
  *n_out = n_items;
}

__global__ void __launch_bounds__(kPlanThreads) plan_kernel(PlanLaunch a) {
  extern __shared__ unsigned long long keys[];
  __shared__ int scan[kPlanThreads];
  const int tid = threadIdx.x, nt = blockDim.x;
  WsView ws = a.ws;
  PlanHeader* hdr = ws.hdr;
  const int B = a.batch;
  if (tid == 0) hdr->error_word = 0;  // every new plan starts with a clean error word
  __syncthreads();
  int chunk = 0, n_items = 0;
  if (flat_mode(a.mode)) {
    flat_plan(a, reinterpret_cast<int*>(keys), scan, &chunk, &n_items);
  } else {

  // 1. lengths (clamped and flagged when out of range), query tiles per request
  for (int r = tid; r < B; r += nt) {
    int L = a.seq_lens[r];
    if (L < 0 || L > a.max_kv_len) {
      set_device_error(hdr, PA_ERR_DEVICE_INDEX);
      L = max(0, min(L, a.max_kv_len));
    }
    ws.req_len[r] = L;
    const int q0 = a.cu_seqlens_q[r], q1 = a.cu_seqlens_q[r + 1];
    int n = q1 - q0;
    if (n < 0 || n > L) {
      set_device_error(hdr, PA_ERR_DEVICE_INDEX);
      n = max(0, min(n, L));
    }
    ws.req_splits[r] = (int)cdiv_ll(n, kExtendQTile);
    ws.req_aux[r] = q0;
    ws.req_prefix[r] = L - n;
  }
  __syncthreads();

  // 2. req_base = exclusive prefix sum of the per-request item counts
  const int per = (B + nt - 1) / nt;
  const int r0 = min(B, tid * per), r1 = min(B, r0 + per);
  int local = 0;
  for (int r = r0; r < r1; ++r) local += ws.req_splits[r];
  int total_items = 0;
  int run = block_exclusive_scan(local, scan, &total_items);
  for (int r = r0; r < r1; ++r) {
    ws.req_base[r] = run;
    run += ws.req_splits[r];
  }
  if (tid == 0) ws.req_base[B] = total_items;
  n_items = total_items;
  if (n_items > a.max_items) {  // cannot happen for lengths within bounds; keep the grid safe
    if (tid == 0) set_device_error(hdr, PA_ERR_DEVICE_INDEX);
    n_items = a.max_items;
  }
  for (int i = tid; i < a.sort_n; i += nt) keys[i] = ~0ull;
  __syncthreads();

  // 3. sort keys: (0x7FFFFFFF - work) in the high word, generation index in the low word
  for (int r = tid; r < B; r += nt) {
    const int base = ws.req_base[r], splits = ws.req_splits[r];
    const int L = ws.req_len[r], prefix = ws.req_prefix[r];
    const int n = L - prefix;
    for (int s = 0; s < splits; ++s) {
      const int g = base + s;
      if (g >= n_items) break;
      const unsigned work = (unsigned)item_work(s, prefix, n);
      keys[g] = ((unsigned long long)(0x7FFFFFFFu - work) << 32) | (unsigned)g;
    }
  }
  __syncthreads();

  // 4. bitonic sort, ascending (unique keys, so the order is fully determined)
  for (int k = 2; k <= a.sort_n; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < a.sort_n; i += nt) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const unsigned long long x = keys[i], y = keys[ixj];
          const bool up = (i & k) == 0;
          if ((x > y) == up) {
            keys[i] = y;
            keys[ixj] = x;
          }
        }
      }
      __syncthreads();
    }
  }

  // 5. items in execution order
  for (int i = tid; i < n_items; i += nt) {
    const int g = (int)(keys[i] & 0xFFFFFFFFu);
    int lo = 0, hi = B;  // find r with req_base[r] <= g < req_base[r+1]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (ws.req_base[mid] <= g) lo = mid; else hi = mid;
    }
    const int r = lo, s = g - ws.req_base[r];
    const int L = ws.req_len[r], prefix = ws.req_prefix[r];
    const int n = L - prefix;
    ws.items[i] = make_int4(r, s, s * kExtendQTile, min((s + 1) * kExtendQTile, n));
  }
  }  // EXTEND

  // 6. header
  if (tid == 0) {
    hdr->magic = kMagic;
    hdr->mode = a.mode;
    hdr->batch = B;
    hdr->hq = a.hq;
    hdr->hkv = a.hkv;
    hdr->head_dim = a.head_dim;
    hdr->page_size = a.page_size;
    hdr->num_items = n_items;
    hdr->max_items = a.max_items;
    hdr->tile = a.tile;
    hdr->chunk_tiles = chunk;
    hdr->num_sms = a.num_sms;
    hdr->max_splits = a.max_splits;
    hdr->slots = flat_mode(a.mode) ? a.slots : 0;
    hdr->reserved1 = 0;
  }
}

}  // namespace

cudaError_t launch_plan(const PlanLaunch& a, cudaStream_t s) {
  // EXTEND: the sort keys; flat modes: 3 ints per request and one per item
  size_t smem = sizeof(unsigned long long) * (size_t)a.sort_n;
  if (flat_mode(a.mode)) smem = std::max(smem, sizeof(int) * (3 * (size_t)a.batch + (size_t)a.max_items));
  constexpr int kSmemMax = (int)std::max(sizeof(unsigned long long) * kMaxSortItems,
                                         sizeof(int) * (3 * (size_t)kMaxBatch + kMaxSortItems));
  static std::atomic<bool> smem_set[kMaxDevices];
  cudaError_t e = raise_smem_limit(plan_kernel, kSmemMax, smem_set);
  if (e != cudaSuccess) return e;
  plan_kernel<<<1, kPlanThreads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace pa
