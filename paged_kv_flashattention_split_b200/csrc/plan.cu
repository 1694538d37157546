// plan.cu - the per-batch scheduling plan (one CTA, integer arithmetic only).
//
// The scheduling metadata is a function of the sequence lengths (and, for a
// prefill, the cumulative query lengths) alone, so it is built once per batch
// and reused by every layer ("SGLang의 FA3 디코드 최적화: get_scheduler_metadata
// 도입", 코드 분석 items 1-3, 왜 이게 좋은가 item 1).  The algorithm is the one
// stated at attn_plan in pagedattn.h; every step is integer so the result is
// exact and identical on recomputation.
#include "kernels.h"

namespace pa {
namespace {

constexpr int kPlanThreads = 1024;

__device__ __forceinline__ long long cdiv_ll(long long a, long long b) { return (a + b - 1) / b; }

// Block-wide exclusive scan of one int per thread; returns this thread's prefix.
__device__ int block_exclusive_scan(int v, int* scratch, int* total) {
  const int tid = threadIdx.x;
  scratch[tid] = v;
  __syncthreads();
  for (int off = 1; off < blockDim.x; off <<= 1) {
    int add = tid >= off ? scratch[tid - off] : 0;
    __syncthreads();
    scratch[tid] += add;
    __syncthreads();
  }
  int incl = scratch[tid];
  *total = scratch[blockDim.x - 1];
  __syncthreads();
  return incl - v;
}

// EXTEND: work of query tile s (key tiles it needs) for the sort key; items run longest first.
__device__ __forceinline__ int item_work(int s, int prefix, int n) {
  const int q1 = min((s + 1) * kExtendQTile, n);
  return (int)cdiv_ll(prefix + q1, kExtendKvTile);
}

// DECODE, SAGE_DECODE, SAGE_SPARSE: the flat partition of the requests' units (T-key tiles
// for DECODE, 32-key units for Sage, of the selected 64-key blocks only for SAGE_SPARSE)
// over CTA slots (the algorithm at attn_plan).  Items come out r-major, which is also slot
// order, so no sort.
__device__ void flat_plan(const PlanLaunch& a, int* item_slot, int* scan, int* chunk_out, int* n_out) {
  const int tid = threadIdx.x, nt = blockDim.x;
  WsView ws = a.ws;
  PlanHeader* hdr = ws.hdr;
  const int B = a.batch;
  const bool sparse = a.mode == PA_MODE_SAGE_SPARSE;
  const int U = a.mode == PA_MODE_DECODE ? a.tile : kSageUnit;   // keys per unit
  // 1. lengths (clamped and flagged when out of range); the units of each request
  //    (req_prefix holds them during the plan), and its selected block count (SAGE_SPARSE)
  const int warp = tid >> 5, lane = tid & 31, nwarps = nt >> 5;
  if (!sparse) {
    for (int r = tid; r < B; r += nt) {
      int L = a.seq_lens[r];
      if (L < 0 || L > a.max_kv_len) {
        set_device_error(hdr, PA_ERR_DEVICE_INDEX);
        L = max(0, min(L, a.max_kv_len));
      }
      ws.req_len[r] = L;
      ws.req_prefix[r] = (int)cdiv_ll(L, U);
      ws.req_splits[r] = 0;
    }
  } else {
    // one warp per request scans its block mask 32 blocks at a time (coalesced byte loads, ballots)
    for (int r = warp; r < B; r += nwarps) {
      int L = a.seq_lens[r];
      if (L < 0 || L > a.max_kv_len) {
        if (lane == 0) set_device_error(hdr, PA_ERR_DEVICE_INDEX);
        L = max(0, min(L, a.max_kv_len));
      }
      const int nb = (int)cdiv_ll(L, kSageBlock);
      const uint8_t* m = a.block_mask + (size_t)r * a.mask_pitch;
      int units = 0, nsel = 0;
      for (int b0 = 0; b0 < nb; b0 += 32) {
        const int b = b0 + lane;
        const bool sel = b < nb && m[b] != 0;
        nsel += __popc(__ballot_sync(0xffffffffu, sel));
        if (sel) units += L - kSageBlock * b <= kSageUnit ? 1 : 2;   // a last block of <= 32 keys is one unit
      }
      for (int o = 16; o > 0; o >>= 1) units += __shfl_xor_sync(0xffffffffu, units, o);
      if (lane == 0) {
        ws.req_len[r] = L;
        ws.req_prefix[r] = units;
        ws.req_splits[r] = nsel;   // scratch until step 3
      }
    }
  }
  __syncthreads();
  const int per_t = (B + nt - 1) / nt;
  const int r0 = min(B, tid * per_t), r1 = min(B, r0 + per_t);
  if (sparse) {
    // sel_base = exclusive prefix sum of the selected block counts; the block lists
    int local_b = 0;
    for (int r = r0; r < r1; ++r) local_b += ws.req_splits[r];
    int total_b = 0;
    int run_b = block_exclusive_scan(local_b, scan, &total_b);
    for (int r = r0; r < r1; ++r) {
      ws.sel_base[r] = run_b;
      run_b += ws.req_splits[r];
    }
    if (tid == 0) ws.sel_base[B] = total_b;
    __syncthreads();
    for (int r = warp; r < B; r += nwarps) {    // the selected blocks in ascending order, a warp per request
      const int L = ws.req_len[r], nb = (int)cdiv_ll(L, kSageBlock);
      const uint8_t* m = a.block_mask + (size_t)r * a.mask_pitch;
      int k = ws.sel_base[r];
      for (int b0 = 0; b0 < nb; b0 += 32) {
        const int b = b0 + lane;
        const bool sel = b < nb && m[b] != 0;
        const unsigned ballot = __ballot_sync(0xffffffffu, sel);
        if (sel) ws.sel_block[k + __popc(ballot & ((1u << lane) - 1u))] = b;
        k += __popc(ballot);
      }
    }
  }
  // 2. g_r = exclusive prefix sum of the units (kept in req_aux), total
  long long local = 0;
  for (int r = r0; r < r1; ++r) local += ws.req_prefix[r];
  int total = 0;
  int run = block_exclusive_scan((int)local, scan, &total);
  for (int r = r0; r < r1; ++r) {
    ws.req_aux[r] = run;
    run += ws.req_prefix[r];
  }
  const int per = (int)max(1LL, cdiv_ll(total, a.slots));
  const int used = (int)cdiv_ll(total, per);
  __syncthreads();
  // 3. pieces per request, then req_base
  for (int r = tid; r < B; r += nt) {
    const int u = ws.req_prefix[r], g = ws.req_aux[r];
    ws.req_splits[r] = u > 0 ? (g + u - 1) / per - g / per + 1 : 1;
  }
  __syncthreads();
  int local_s = 0;
  for (int r = r0; r < r1; ++r) local_s += ws.req_splits[r];
  int n_items = 0;
  int run_s = block_exclusive_scan(local_s, scan, &n_items);
  for (int r = r0; r < r1; ++r) {
    ws.req_base[r] = run_s;
    run_s += ws.req_splits[r];
  }
  if (tid == 0) ws.req_base[B] = n_items;
  if (n_items > a.max_items) {  // cannot happen (bound slots + B); keep the grid safe
    if (tid == 0) set_device_error(hdr, PA_ERR_DEVICE_INDEX);
    n_items = a.max_items;
  }
  __syncthreads();
  // 4. the items (key ranges; SAGE_SPARSE: unit ranges) and the slot of each
  for (int r = tid; r < B; r += nt) {
    const int L = ws.req_len[r], u = ws.req_prefix[r], g = ws.req_aux[r], base = ws.req_base[r];
    if (u == 0) {
      if (base < n_items) {
        ws.items[base] = make_int4(r, 0, 0, 0);
        item_slot[base] = min(g / per, max(used - 1, 0));
      }
      continue;
    }
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
  for (int c = tid; c <= a.slots; c += nt) ws.slot_first[c] = n_items;
  __syncthreads();
  // 5. slot_first[c] = first item whose slot is >= c (slots are non-decreasing along the list)
  for (int i = tid; i < n_items; i += nt) {
    const int c_prev = i > 0 ? item_slot[i - 1] : -1;
    for (int c = c_prev + 1; c <= item_slot[i]; ++c) ws.slot_first[c] = i;
  }
  __syncthreads();
  for (int r = tid; r < B; r += nt) ws.req_prefix[r] = 0;
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
  const size_t smem = sizeof(unsigned long long) * (size_t)a.sort_n;
  static std::atomic<bool> smem_set[kMaxDevices];
  cudaError_t e = raise_smem_limit(plan_kernel, (int)(sizeof(unsigned long long) * kMaxSortItems), smem_set);
  if (e != cudaSuccess) return e;
  plan_kernel<<<1, kPlanThreads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace pa
