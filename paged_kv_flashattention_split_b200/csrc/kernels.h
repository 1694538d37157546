// kernels.h - host-side launchers implemented by the .cu files (internal).
#pragma once

#include "common.cuh"

namespace pa {

struct PlanLaunch {
  WsView ws;
  const int32_t* seq_lens;
  const int32_t* cu_seqlens_q;
  int mode, batch, hq, hkv, head_dim, page_size, max_kv_len, num_sms, max_splits, max_items, tile;
  int sort_n;  // power of two >= max_items
};
cudaError_t launch_plan(const PlanLaunch& a, cudaStream_t s);

struct DecodeLaunch {
  WsView ws;
  const uint16_t* q;
  const uint16_t* k_pool;
  const uint16_t* v_pool;
  int64_t num_slots;
  const int32_t* page_table;
  int64_t pt_pitch;
  float scale_log2;   // sm_scale * log2(e)
  uint16_t* out;
  float* lse_out;
  int batch, hq, hkv, page_shift, max_items;
};
cudaError_t launch_decode(const DecodeLaunch& a, cudaStream_t s);

struct GatherLaunch {
  const int32_t* seq_lens;
  int r, h_kv, hkv, page_shift, max_len;
  const uint16_t* k_pool;
  int64_t num_slots;
  const int32_t* page_table;
  int64_t pt_pitch;
  int32_t* slots_out;
  uint16_t* rows_out;
};
cudaError_t launch_debug_gather(const GatherLaunch& a, cudaStream_t s);

}  // namespace pa
