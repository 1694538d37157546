// noalloc.cu - a DECODE entry point for callers that cannot allocate device memory.
//
// attn_decode_paged needs a caller-allocated workspace: the plan's work list
// and, above all, the fp32 split partials that the decode kernel writes and
// the merge kernel reads.  Some callers have no way to provide one: code that
// runs inside a host framework which owns all device allocations and exposes
// no allocator, plugins loaded into a process whose memory pool must not be
// touched, or call sites where allocating would synchronise the device or
// break a pre-sized memory budget.  attn_decode_paged_noalloc serves them:
// it plans and decodes in one call, and its workspace (header, work list,
// split partials) lives in one file-scope device array, so the call itself
// allocates nothing.
//
// The array costs kNoAllocBytes of device memory on every GPU that loads the
// library, for as long as the process lives.  All calls share it and it keeps
// the last call's contents, so two calls that overlap on the GPU (different
// streams, or different host threads) race on it; callers must order them.
#include <mutex>

#include "kernels.h"

namespace {

constexpr size_t kNoAllocBytes = 16u << 20;   // 16 MiB of workspace

static __device__ __align__(256) unsigned char g_noalloc_ws[kNoAllocBytes];

// Device address of g_noalloc_ws, looked up once per device (with that device current).
constexpr int kMaxDevices = 64;
void* g_ws_addr[kMaxDevices] = {};
std::mutex g_ws_mutex;

pa_status noalloc_workspace(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_ws_mutex);
  if (!g_ws_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_ws) != cudaSuccess || !p) return PA_ERR_CUDA;
    g_ws_addr[dev] = p;
  }
  *out = g_ws_addr[dev];
  return PA_OK;
}

}  // namespace

extern "C" pa_status attn_decode_paged_noalloc(const pa_plan_params* params, const int32_t* d_seq_lens,
                                               const uint16_t* d_q, const uint16_t* d_k_pool,
                                               const uint16_t* d_v_pool, int64_t num_slots,
                                               const int32_t* d_page_table, int64_t pt_pitch,
                                               float sm_scale, uint16_t* d_out, float* d_lse_out,
                                               pa_stream_t stream) {
  if (!params || params->mode != PA_MODE_DECODE) return PA_ERR_INVALID;
  size_t need = 0;
  pa_status st = pa_plan_workspace_size(params, &need);
  if (st != PA_OK) return st;
  if (need > kNoAllocBytes) return PA_ERR_WORKSPACE;   // plan too large for the fixed array
  if (!d_seq_lens) return PA_ERR_INVALID;
  void* ws = nullptr;
  if ((st = noalloc_workspace(&ws)) != PA_OK) return st;
  // The plan kernel rewrites the header, the per-request arrays and the work
  // list, and every partial is written before it is read; only the header is
  // cleared here, so that a failed plan can never leave a stale one behind.
  if (cudaMemsetAsync(ws, 0, sizeof(pa::PlanHeader), (cudaStream_t)stream) != cudaSuccess) return PA_ERR_CUDA;
  if ((st = attn_plan(params, d_seq_lens, nullptr, ws, kNoAllocBytes, stream)) != PA_OK) return st;
  return attn_decode_paged(params, ws, kNoAllocBytes, d_q, d_k_pool, d_v_pool, num_slots, d_page_table,
                           pt_pitch, sm_scale, d_out, d_lse_out, stream);
}

// The error word of the fixed array's plan header: the no-allocation decode's own
// pa_read_device_error (the caller has no workspace pointer to pass to that one).
extern "C" pa_status pa_noalloc_read_device_error(pa_stream_t stream) {
  void* ws = nullptr;
  pa_status st = noalloc_workspace(&ws);
  if (st != PA_OK) return st;
  return pa_read_device_error(ws, stream);
}
