// api.cu - the C ABI: parameter validation, workspace sizing and kernel launches.
//
// Host-side checks run before any CUDA call, so invalid arguments are reported
// without touching the device.  Validation follows the pages' conventions:
// inputs a mode does not use must not be passed (a dense plan rejects
// block-sparse-only inputs, "FlashInfer PrimTS, Sage Attention ..." 코드 분석
// item 2), 8-bit Sage needs SM100 (item 3 of the same section), the Sage
// shared-memory budget is checked before launch (same item), and scale values
// are never checked (item 1).
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "kernels.h"

using namespace pa;

namespace {

struct Derived {
  int G = 0, num_sms = 0, max_splits = 0, max_items = 0, tile = 0, sort_n = 0, page_shift = 0, slots = 0;
  WsLayout layout{};
};

int ilog2(int x) {
  int s = 0;
  while ((1 << s) < x) ++s;
  return s;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

pa_status device_sms(int* sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
  if (cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return PA_ERR_CUDA;
  return PA_OK;
}

// PAGEDATTN_TEST_FORCE_ARCH=<major*10+minor> replaces the queried compute
// capability; a test hook for the wrong-architecture error path.
pa_status check_arch() {
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return PA_ERR_CUDA;
  if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return PA_ERR_CUDA;
  if (const char* f = std::getenv("PAGEDATTN_TEST_FORCE_ARCH")) {
    const int cc = std::atoi(f);
    major = cc / 10;
    minor = cc % 10;
  }
  return (major == 10 && minor == 0) ? PA_OK : PA_ERR_ARCH;
}

pa_status derive(const pa_plan_params* p, Derived* d) {
  if (!p) return PA_ERR_INVALID;
  if (p->mode < PA_MODE_DECODE || p->mode > PA_MODE_SAGE_SPARSE) return PA_ERR_INVALID;
  if (p->batch < 1 || p->batch > kMaxBatch) return PA_ERR_INVALID;
  if (p->hq < 1 || p->hkv < 1 || p->hq % p->hkv != 0) return PA_ERR_INVALID;
  if (p->max_kv_len < 0 || p->max_q_tokens < 0 || p->num_sms < 0 || p->max_splits < 0) return PA_ERR_INVALID;
  if (p->reserved != 0) return PA_ERR_INVALID;
  const int G = p->hq / p->hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return PA_ERR_UNSUPPORTED;
  if (p->head_dim != kHeadDim) return PA_ERR_UNSUPPORTED;
  const int P = p->page_size;
  if (P < 1 || P > 256 || (P & (P - 1)) != 0) return PA_ERR_UNSUPPORTED;
  d->G = G;
  d->page_shift = ilog2(P);
  switch (p->mode) {
    case PA_MODE_DECODE:
      // the flat partition balances the slots itself: no split cap
      if (p->max_q_tokens != 0 || p->sage_k_block != 0 || p->max_splits != 0) return PA_ERR_INVALID;
      d->max_splits = 0;
      // the plan counts tiles in int32
      if ((long long)p->batch * ((p->max_kv_len + kDecodeMinTile - 1) / kDecodeMinTile) >= (1LL << 31))
        return PA_ERR_UNSUPPORTED;
      d->tile = P > kDecodeMinTile ? P : kDecodeMinTile;
      break;
    case PA_MODE_EXTEND:
      if (p->sage_k_block != 0 || p->max_splits > 1) return PA_ERR_INVALID;
      d->max_splits = 1;
      d->tile = kExtendKvTile;
      break;
    case PA_MODE_SAGE_DECODE:
    case PA_MODE_SAGE_SPARSE:
      // the flat partition balances the slots itself: no split cap
      if (p->max_q_tokens != 0 || p->max_splits != 0) return PA_ERR_INVALID;
      if (p->sage_k_block != kSageBlock || P != kSageBlock) return PA_ERR_UNSUPPORTED;
      d->max_splits = 0;
      // the score rows ([B][Hq][max_kv_len rounded up to 64] fp32) stay below 2^46 bytes
      if ((double)p->batch * p->hq * ((double)p->max_kv_len + kSageBlock) * 4.0 > 7.0e13) return PA_ERR_UNSUPPORTED;
      // the plan counts 32-key units in int32
      if ((long long)p->batch * ((p->max_kv_len + kSageUnit - 1) / kSageUnit) >= (1LL << 31)) return PA_ERR_UNSUPPORTED;
      d->tile = kSageUnit;
      break;
  }
  int sms = p->num_sms;
  if (sms == 0) {
    pa_status st = device_sms(&sms);
    if (st != PA_OK) return st;
  }
  d->num_sms = sms;
  long long mi = 0;
  if (flat_mode(p->mode))
  {
    d->slots = flat_slots(p->hkv, sms);
    mi = (long long)d->slots + p->batch;
  }
  else
    mi = ((long long)p->max_q_tokens + kExtendQTile - 1) / kExtendQTile + p->batch;
  if (mi > kMaxSortItems) return PA_ERR_UNSUPPORTED;
  d->max_items = (int)mi;
  int n = 2;
  while (n < d->max_items) n <<= 1;
  d->sort_n = n;
  d->layout = ws_layout(p->mode, p->batch, p->hq, p->hkv, p->head_dim, d->max_items, p->max_kv_len, d->slots);
  return PA_OK;
}

pa_status from_cuda(cudaError_t e) { return e == cudaSuccess ? PA_OK : PA_ERR_CUDA; }

}  // namespace

extern "C" {

int32_t pa_version(void) { return 100; }

const char* pa_status_string(pa_status s) {
  switch (s) {
    case PA_OK: return "PA_OK";
    case PA_ERR_INVALID: return "PA_ERR_INVALID";
    case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
    case PA_ERR_ARCH: return "PA_ERR_ARCH";
    case PA_ERR_WORKSPACE: return "PA_ERR_WORKSPACE";
    case PA_ERR_CUDA: return "PA_ERR_CUDA";
    case PA_ERR_DEVICE_INDEX: return "PA_ERR_DEVICE_INDEX";
  }
  return "PA_ERR_UNKNOWN";
}

pa_status pa_plan_workspace_size(const pa_plan_params* params, size_t* bytes) {
  if (!bytes) return PA_ERR_INVALID;
  Derived d;
  pa_status st = derive(params, &d);
  if (st != PA_OK) return st;
  *bytes = d.layout.total;
  return PA_OK;
}

static pa_status plan_common(const pa_plan_params* params, const int32_t* d_seq_lens, const int32_t* d_cu_seqlens_q,
                             const uint8_t* d_block_mask, int64_t mask_pitch, void* d_ws, size_t ws_bytes,
                             pa_stream_t stream);

pa_status attn_plan(const pa_plan_params* params, const int32_t* d_seq_lens,
                    const int32_t* d_cu_seqlens_q, void* d_ws, size_t ws_bytes, pa_stream_t stream) {
  if (params && params->mode == PA_MODE_SAGE_SPARSE) return PA_ERR_INVALID;   // needs attn_plan_sage_sparse
  return plan_common(params, d_seq_lens, d_cu_seqlens_q, nullptr, 0, d_ws, ws_bytes, stream);
}

pa_status attn_plan_sage_sparse(const pa_plan_params* params, const int32_t* d_seq_lens,
                                const uint8_t* d_block_mask, int64_t mask_pitch, void* d_ws, size_t ws_bytes,
                                pa_stream_t stream) {
  if (!params || params->mode != PA_MODE_SAGE_SPARSE || !d_block_mask) return PA_ERR_INVALID;
  if (mask_pitch < ((int64_t)params->max_kv_len + kSageBlock - 1) / kSageBlock || mask_pitch < 1)
    return PA_ERR_INVALID;
  return plan_common(params, d_seq_lens, nullptr, d_block_mask, mask_pitch, d_ws, ws_bytes, stream);
}

static pa_status plan_common(const pa_plan_params* params, const int32_t* d_seq_lens, const int32_t* d_cu_seqlens_q,
                             const uint8_t* d_block_mask, int64_t mask_pitch, void* d_ws, size_t ws_bytes,
                             pa_stream_t stream) {
  Derived d;
  pa_status st = derive(params, &d);
  if (st != PA_OK) return st;
  if (!d_seq_lens || !d_ws) return PA_ERR_INVALID;
  if ((params->mode == PA_MODE_EXTEND) != (d_cu_seqlens_q != nullptr)) return PA_ERR_INVALID;
  if (!aligned16(d_ws)) return PA_ERR_INVALID;
  if (ws_bytes < d.layout.total) return PA_ERR_WORKSPACE;
  if ((st = check_arch()) != PA_OK) return st;
  PlanLaunch a;
  a.ws = ws_view(d_ws, d.layout);
  a.seq_lens = d_seq_lens;
  a.cu_seqlens_q = d_cu_seqlens_q;
  a.mode = params->mode;
  a.batch = params->batch;
  a.hq = params->hq;
  a.hkv = params->hkv;
  a.head_dim = params->head_dim;
  a.page_size = params->page_size;
  a.max_kv_len = params->max_kv_len;
  a.num_sms = d.num_sms;
  a.max_splits = d.max_splits;
  a.max_items = d.max_items;
  a.tile = d.tile;
  a.sort_n = d.sort_n;
  a.slots = d.slots;
  a.block_mask = d_block_mask;
  a.mask_pitch = mask_pitch;
  return from_cuda(launch_plan(a, (cudaStream_t)stream));
}

pa_status attn_decode_paged(const pa_plan_params* params, const void* d_ws, size_t ws_bytes,
                            const uint16_t* d_q, const uint16_t* d_k_pool, const uint16_t* d_v_pool,
                            int64_t num_slots, const int32_t* d_page_table, int64_t pt_pitch,
                            float sm_scale, uint16_t* d_out, float* d_lse_out, pa_stream_t stream) {
  Derived d;
  pa_status st = derive(params, &d);
  if (st != PA_OK) return st;
  if (params->mode != PA_MODE_DECODE) return PA_ERR_WORKSPACE;
  if (!d_ws || !d_q || !d_k_pool || !d_v_pool || !d_page_table || !d_out) return PA_ERR_INVALID;
  if (!aligned16(d_ws) || !aligned16(d_q) || !aligned16(d_k_pool) || !aligned16(d_v_pool) ||
      !aligned16(d_out))
    return PA_ERR_INVALID;
  if (d_lse_out && (reinterpret_cast<uintptr_t>(d_lse_out) & 3u)) return PA_ERR_INVALID;
  if (num_slots < 1 || pt_pitch < 1) return PA_ERR_INVALID;
  const long long need_pitch = ((long long)params->max_kv_len + params->page_size - 1) / params->page_size;
  if (pt_pitch < need_pitch) return PA_ERR_INVALID;
  if (ws_bytes < d.layout.total) return PA_ERR_WORKSPACE;
  if ((st = check_arch()) != PA_OK) return st;
  DecodeLaunch a;
  a.ws = ws_view(const_cast<void*>(d_ws), d.layout);
  a.q = d_q;
  a.k_pool = d_k_pool;
  a.v_pool = d_v_pool;
  a.num_slots = num_slots;
  a.page_table = d_page_table;
  a.pt_pitch = pt_pitch;
  a.scale_log2 = sm_scale * 1.4426950408889634f;
  a.out = d_out;
  a.lse_out = d_lse_out;
  a.batch = params->batch;
  a.hq = params->hq;
  a.hkv = params->hkv;
  a.page_shift = d.page_shift;
  a.max_items = d.max_items;
  a.slots = d.slots;
  return from_cuda(launch_decode(a, (cudaStream_t)stream));
}

pa_status attn_decode_paged_fp8(const pa_plan_params* params, const void* d_ws, size_t ws_bytes,
                                const uint16_t* d_q, const uint8_t* d_k8_pool, const uint8_t* d_v8_pool,
                                float k_scale, float v_scale, int64_t num_slots, const int32_t* d_page_table,
                                int64_t pt_pitch, float sm_scale, uint16_t* d_out, float* d_lse_out,
                                pa_stream_t stream) {
  Derived d;
  pa_status st = derive(params, &d);
  if (st != PA_OK) return st;
  if (params->mode != PA_MODE_DECODE) return PA_ERR_WORKSPACE;
  if (!d_ws || !d_q || !d_k8_pool || !d_v8_pool || !d_page_table || !d_out) return PA_ERR_INVALID;
  if (!aligned16(d_ws) || !aligned16(d_q) || !aligned16(d_k8_pool) || !aligned16(d_v8_pool) ||
      !aligned16(d_out))
    return PA_ERR_INVALID;
  if (d_lse_out && (reinterpret_cast<uintptr_t>(d_lse_out) & 3u)) return PA_ERR_INVALID;
  if (num_slots < 1 || pt_pitch < 1) return PA_ERR_INVALID;
  const long long need_pitch = ((long long)params->max_kv_len + params->page_size - 1) / params->page_size;
  if (pt_pitch < need_pitch) return PA_ERR_INVALID;
  if (ws_bytes < d.layout.total) return PA_ERR_WORKSPACE;
  if ((st = check_arch()) != PA_OK) return st;
  Fp8DecodeLaunch a;
  a.ws = ws_view(const_cast<void*>(d_ws), d.layout);
  a.q = d_q;
  a.k8_pool = d_k8_pool;
  a.v8_pool = d_v8_pool;
  a.num_slots = num_slots;
  a.page_table = d_page_table;
  a.pt_pitch = pt_pitch;
  a.scale_log2 = sm_scale * k_scale * 1.4426950408889634f;
  a.v_scale = v_scale;
  a.out = d_out;
  a.lse_out = d_lse_out;
  a.batch = params->batch;
  a.hq = params->hq;
  a.hkv = params->hkv;
  a.page_shift = d.page_shift;
  a.max_items = d.max_items;
  a.slots = d.slots;
  return from_cuda(launch_decode_fp8(a, (cudaStream_t)stream));
}

pa_status attn_extend_paged(const pa_plan_params* params, const void* d_ws, size_t ws_bytes,
                            const uint16_t* d_q, const uint16_t* d_k_pool, const uint16_t* d_v_pool,
                            int64_t num_slots, const int32_t* d_page_table, int64_t pt_pitch,
                            float sm_scale, uint16_t* d_out, float* d_lse_out, pa_stream_t stream) {
  Derived d;
  pa_status st = derive(params, &d);
  if (st != PA_OK) return st;
  if (params->mode != PA_MODE_EXTEND) return PA_ERR_WORKSPACE;
  if (!d_ws || !d_q || !d_k_pool || !d_v_pool || !d_page_table || !d_out) return PA_ERR_INVALID;
  if (!aligned16(d_ws) || !aligned16(d_q) || !aligned16(d_k_pool) || !aligned16(d_v_pool) || !aligned16(d_out))
    return PA_ERR_INVALID;
  if (d_lse_out && (reinterpret_cast<uintptr_t>(d_lse_out) & 3u)) return PA_ERR_INVALID;
  if (num_slots < params->page_size || num_slots >= (1LL << 31) || pt_pitch < 1 || params->max_q_tokens < 1)
    return PA_ERR_INVALID;
  const long long need_pitch = ((long long)params->max_kv_len + params->page_size - 1) / params->page_size;
  if (pt_pitch < need_pitch) return PA_ERR_INVALID;
  if (ws_bytes < d.layout.total) return PA_ERR_WORKSPACE;
  if ((st = check_arch()) != PA_OK) return st;
  ExtendArgs a;
  a.ws = ws_view(const_cast<void*>(d_ws), d.layout);
  a.q = d_q;
  a.k_pool = d_k_pool;
  a.v_pool = d_v_pool;
  a.q_rows = params->max_q_tokens;
  a.num_slots = num_slots;
  a.page_table = d_page_table;
  a.pt_pitch = pt_pitch;
  a.out = d_out;
  a.lse_out = d_lse_out;
  a.scale_log2 = sm_scale * 1.4426950408889634f;
  a.hq = params->hq;
  a.hkv = params->hkv;
  a.page_size = params->page_size;
  a.page_shift = d.page_shift;
  a.max_items = d.max_items;
  return from_cuda(launch_extend(a, (cudaStream_t)stream));
}

pa_status attn_decode_paged_sage(const pa_plan_params* params, const void* d_ws, size_t ws_bytes,
                                 const int8_t* d_q8, const float* d_sf_q, const int8_t* d_k8_pool,
                                 const uint8_t* d_v8_pool, const float* d_sf_k, const float* d_sf_v,
                                 const float* d_v_mean, int64_t num_slots, const int32_t* d_page_table,
                                 int64_t pt_pitch, uint16_t* d_out, pa_stream_t stream) {
  Derived d;
  pa_status st = derive(params, &d);
  if (st != PA_OK) return st;
  if (!sage_mode(params->mode)) return PA_ERR_WORKSPACE;
  if (!d_ws || !d_q8 || !d_sf_q || !d_k8_pool || !d_v8_pool || !d_sf_k || !d_sf_v || !d_page_table || !d_out)
    return PA_ERR_INVALID;
  if (!aligned16(d_ws) || !aligned16(d_q8) || !aligned16(d_k8_pool) || !aligned16(d_v8_pool) || !aligned16(d_out) ||
      !aligned16(d_sf_k) || !aligned16(d_sf_v) || (d_v_mean && !aligned16(d_v_mean)))
    return PA_ERR_INVALID;
  if (num_slots < kSageBlock || num_slots % kSageBlock != 0 || num_slots >= (1LL << 31) || pt_pitch < 1)
    return PA_ERR_INVALID;
  const long long need_pitch = ((long long)params->max_kv_len + params->page_size - 1) / params->page_size;
  if (pt_pitch < need_pitch) return PA_ERR_INVALID;
  if (ws_bytes < d.layout.total) return PA_ERR_WORKSPACE;
  if ((st = check_arch()) != PA_OK) return st;
  SageLaunchArgs a;
  a.ws = ws_view(const_cast<void*>(d_ws), d.layout);
  a.q8 = d_q8;
  a.sf_q = d_sf_q;
  a.k8 = d_k8_pool;
  a.v8 = d_v8_pool;
  a.sf_k = d_sf_k;
  a.sf_v = d_sf_v;
  a.v_mean = d_v_mean;
  a.num_slots = num_slots;
  a.page_table = d_page_table;
  a.pt_pitch = pt_pitch;
  a.out = d_out;
  a.batch = params->batch;
  a.hq = params->hq;
  a.hkv = params->hkv;
  a.slots = d.slots;
  return from_cuda(launch_sage(a, (cudaStream_t)stream));
}

pa_status attn_extend_paged_sage(const pa_plan_params* params, const void* d_ws, size_t ws_bytes,
                                 const int8_t* d_q8, const float* d_sf_q, const int8_t* d_k8_pool,
                                 const uint8_t* d_v8_pool, const float* d_sf_k, const float* d_sf_v,
                                 const float* d_v_mean, int64_t num_slots, const int32_t* d_page_table,
                                 int64_t pt_pitch, uint16_t* d_out, pa_stream_t stream) {
  Derived d;
  pa_status st = derive(params, &d);
  if (st != PA_OK) return st;
  if (params->mode != PA_MODE_EXTEND) return PA_ERR_WORKSPACE;
  if (params->page_size != kSageBlock) return PA_ERR_UNSUPPORTED;   // a page is one sfK block
  if (!d_ws || !d_q8 || !d_sf_q || !d_k8_pool || !d_v8_pool || !d_sf_k || !d_sf_v || !d_page_table || !d_out)
    return PA_ERR_INVALID;
  if (!aligned16(d_ws) || !aligned16(d_q8) || !aligned16(d_k8_pool) || !aligned16(d_v8_pool) || !aligned16(d_out))
    return PA_ERR_INVALID;
  if (num_slots < kSageBlock || num_slots % kSageBlock != 0 || num_slots >= (1LL << 31) || pt_pitch < 1)
    return PA_ERR_INVALID;
  const long long need_pitch = ((long long)params->max_kv_len + params->page_size - 1) / params->page_size;
  if (pt_pitch < need_pitch) return PA_ERR_INVALID;
  if (ws_bytes < d.layout.total) return PA_ERR_WORKSPACE;
  if ((st = check_arch()) != PA_OK) return st;
  SageExtendArgs a;
  a.ws = ws_view(const_cast<void*>(d_ws), d.layout);
  a.q8 = d_q8;
  a.sf_q = d_sf_q;
  a.k8 = d_k8_pool;
  a.v8 = d_v8_pool;
  a.sf_k = d_sf_k;
  a.sf_v = d_sf_v;
  a.v_mean = d_v_mean;
  a.num_slots = num_slots;
  a.page_table = d_page_table;
  a.pt_pitch = pt_pitch;
  a.q_rows = params->max_q_tokens;
  a.out = d_out;
  a.hq = params->hq;
  a.hkv = params->hkv;
  a.max_items = d.max_items;
  return from_cuda(launch_sage_extend(a, (cudaStream_t)stream));
}

pa_status attn_kv_store(const uint16_t* d_k_new, const uint16_t* d_v_new, const int32_t* d_out_cache_loc,
                        int64_t n_tokens, int32_t hkv, int32_t head_dim, uint16_t* d_k_pool, uint16_t* d_v_pool,
                        int64_t num_slots, void* d_ws, pa_stream_t stream) {
  if (n_tokens < 0 || hkv < 1 || num_slots < 1) return PA_ERR_INVALID;
  if (head_dim != kHeadDim) return PA_ERR_UNSUPPORTED;
  if (n_tokens == 0) return PA_OK;
  if (!d_k_new || !d_v_new || !d_out_cache_loc || !d_k_pool || !d_v_pool) return PA_ERR_INVALID;
  if (!aligned16(d_k_new) || !aligned16(d_v_new) || !aligned16(d_k_pool) || !aligned16(d_v_pool) ||
      (d_ws && !aligned16(d_ws)))
    return PA_ERR_INVALID;
  pa_status st = check_arch();
  if (st != PA_OK) return st;
  StoreLaunch a;
  a.k_new = d_k_new;
  a.v_new = d_v_new;
  a.loc = d_out_cache_loc;
  a.n_tokens = n_tokens;
  a.hkv = hkv;
  a.elem_bytes = 2;
  a.k_pool = d_k_pool;
  a.v_pool = d_v_pool;
  a.num_slots = num_slots;
  a.sf_k_new = nullptr;
  a.sf_k = nullptr;
  a.hdr = static_cast<PlanHeader*>(d_ws);
  return from_cuda(launch_kv_store(a, (cudaStream_t)stream));
}

pa_status attn_kv_store_sage(const int8_t* d_k8_new, const uint8_t* d_v8_new, const float* d_sf_k_new,
                             const int32_t* d_out_cache_loc, int64_t n_tokens, int32_t hkv, int32_t head_dim,
                             int8_t* d_k8_pool, uint8_t* d_v8_pool, float* d_sf_k, int64_t num_slots, void* d_ws,
                             pa_stream_t stream) {
  if (n_tokens < 0 || hkv < 1 || num_slots < 1) return PA_ERR_INVALID;
  if (head_dim != kHeadDim) return PA_ERR_UNSUPPORTED;
  if (d_sf_k_new && (!d_sf_k || num_slots % kSageBlock != 0)) return PA_ERR_INVALID;
  if (n_tokens == 0) return PA_OK;
  if (!d_k8_new || !d_v8_new || !d_out_cache_loc || !d_k8_pool || !d_v8_pool) return PA_ERR_INVALID;
  if (!aligned16(d_k8_new) || !aligned16(d_v8_new) || !aligned16(d_k8_pool) || !aligned16(d_v8_pool) ||
      (d_ws && !aligned16(d_ws)))
    return PA_ERR_INVALID;
  pa_status st = check_arch();
  if (st != PA_OK) return st;
  StoreLaunch a;
  a.k_new = d_k8_new;
  a.v_new = d_v8_new;
  a.loc = d_out_cache_loc;
  a.n_tokens = n_tokens;
  a.hkv = hkv;
  a.elem_bytes = 1;
  a.k_pool = d_k8_pool;
  a.v_pool = d_v8_pool;
  a.num_slots = num_slots;
  a.sf_k_new = d_sf_k_new;
  a.sf_k = d_sf_k;
  a.hdr = static_cast<PlanHeader*>(d_ws);
  return from_cuda(launch_kv_store(a, (cudaStream_t)stream));
}

pa_status attn_debug_gather(const int32_t* d_seq_lens, int32_t r, int32_t h_kv, int32_t hkv,
                            int32_t head_dim, int32_t page_size, int32_t max_len,
                            const uint16_t* d_k_pool, int64_t num_slots, const int32_t* d_page_table,
                            int64_t pt_pitch, int32_t* d_slots_out, uint16_t* d_rows_out,
                            pa_stream_t stream) {
  if (!d_seq_lens || !d_k_pool || !d_page_table || !d_slots_out || !d_rows_out) return PA_ERR_INVALID;
  if (head_dim != kHeadDim) return PA_ERR_UNSUPPORTED;
  if (page_size < 1 || page_size > 256 || (page_size & (page_size - 1))) return PA_ERR_UNSUPPORTED;
  if (r < 0 || hkv < 1 || h_kv < 0 || h_kv >= hkv || max_len < 0 || num_slots < 1 || pt_pitch < 1)
    return PA_ERR_INVALID;
  pa_status st = check_arch();
  if (st != PA_OK) return st;
  GatherLaunch a;
  a.seq_lens = d_seq_lens;
  a.r = r;
  a.h_kv = h_kv;
  a.hkv = hkv;
  a.page_shift = ilog2(page_size);
  a.max_len = max_len;
  a.k_pool = d_k_pool;
  a.num_slots = num_slots;
  a.page_table = d_page_table;
  a.pt_pitch = pt_pitch;
  a.slots_out = d_slots_out;
  a.rows_out = d_rows_out;
  return from_cuda(launch_debug_gather(a, (cudaStream_t)stream));
}

pa_status pa_read_device_error(void* d_ws, pa_stream_t stream) {
  if (!d_ws) return PA_ERR_INVALID;
  PlanHeader h;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemcpyAsync(&h, d_ws, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess) return PA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return PA_ERR_CUDA;
  const int32_t zero = 0;
  char* word = static_cast<char*>(d_ws) + offsetof(PlanHeader, error_word);
  if (cudaMemcpyAsync(word, &zero, sizeof(zero), cudaMemcpyHostToDevice, s) != cudaSuccess) return PA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return PA_ERR_CUDA;
  if (h.error_word != 0) return (pa_status)h.error_word;
  return h.magic == kMagic ? PA_OK : PA_ERR_WORKSPACE;
}

}  // extern "C"
