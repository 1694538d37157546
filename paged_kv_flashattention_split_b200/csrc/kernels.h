// kernels.h - host-side launchers implemented by the .cu files (internal).
#pragma once

#include <atomic>

#include "common.cuh"

namespace pa {

constexpr int kMaxDevices = 64;

// Launches `kernel` as a programmatic dependent of the grid before it on `s`: it may start
// once that grid executes griddepcontrol.launch_dependents (or exits), and must itself
// execute griddepcontrol.wait before it reads anything that grid (or any earlier work) wrote.
template <typename K, typename A>
cudaError_t launch_programmatic(K kernel, dim3 grid, dim3 block, size_t smem, const A& args, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args);
}

// Raises `kernel`'s dynamic shared-memory limit to `bytes` on the current device, once per
// device.  Host threads may launch at the same time: the per-device flags are atomic, and
// setting the attribute twice is harmless.  Devices beyond kMaxDevices set it on every call.
template <typename K>
cudaError_t raise_smem_limit(K kernel, int bytes, std::atomic<bool>* done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool cached = dev >= 0 && dev < kMaxDevices;
  if (cached && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && cached) done[dev].store(true, std::memory_order_release);
  return e;
}

struct PlanLaunch {
  WsView ws;
  const int32_t* seq_lens;
  const int32_t* cu_seqlens_q;
  int mode, batch, hq, hkv, head_dim, page_size, max_kv_len, num_sms, max_splits, max_items, tile;
  int sort_n;  // power of two >= max_items
  int slots;   // DECODE, SAGE: CTA slots of the flat partition
  const uint8_t* block_mask;   // SAGE_SPARSE: [B][mask_pitch], nonzero = the 64-key block is attended
  int64_t mask_pitch;
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
  int slots;          // CTA slots of the plan's flat partition
};
cudaError_t launch_decode(const DecodeLaunch& a, cudaStream_t s);
cudaError_t launch_decode_merge(const DecodeLaunch& a, cudaStream_t s);   // the split merge alone

struct Fp8DecodeLaunch {
  WsView ws;
  const uint16_t* q;       // bf16 [B][Hq][D]
  const uint8_t* k8_pool;  // E4M3 [num_slots][Hkv][D]
  const uint8_t* v8_pool;
  int64_t num_slots;
  const int32_t* page_table;
  int64_t pt_pitch;
  float scale_log2;        // sm_scale * k_scale * log2(e)
  float v_scale;
  uint16_t* out;
  float* lse_out;
  int batch, hq, hkv, page_shift, max_items;
  int slots;               // CTA slots of the plan's flat partition
};
cudaError_t launch_decode_fp8(const Fp8DecodeLaunch& a, cudaStream_t s);

struct SageLaunchArgs {
  WsView ws;
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
  int batch, hq, hkv, slots;
};
cudaError_t launch_sage(const SageLaunchArgs& a, cudaStream_t s);

struct ExtendArgs {
  WsView ws;
  const uint16_t* q;
  const uint16_t* k_pool;
  const uint16_t* v_pool;
  int64_t q_rows;          // rows of the Q / O buffers (max_q_tokens)
  int64_t num_slots;
  const int32_t* page_table;
  int64_t pt_pitch;
  uint16_t* out;
  float* lse_out;
  float scale_log2;
  int hq, hkv, page_size, page_shift, max_items;
};
cudaError_t launch_extend(const ExtendArgs& a, cudaStream_t s);
cudaError_t launch_extend_duo(const ExtendArgs& a, cudaStream_t s);   // head groups of 4 or 8, a CTA pair per quad

struct SageExtendArgs {
  WsView ws;
  const int8_t* q8;        // [q_rows][Hq][D]
  const float* sf_q;       // [q_rows][Hq]
  const int8_t* k8;
  const uint8_t* v8;
  const float* sf_k;
  const float* sf_v;
  const float* v_mean;
  int64_t num_slots;
  const int32_t* page_table;
  int64_t pt_pitch;
  int64_t q_rows;
  uint16_t* out;           // bf16 [q_rows][Hq][D]
  int hq, hkv, max_items;
};
cudaError_t launch_sage_extend(const SageExtendArgs& a, cudaStream_t s);

struct StoreLaunch {
  const void* k_new;
  const void* v_new;
  const int32_t* loc;
  int64_t n_tokens;
  int hkv;
  int elem_bytes;      // 2: bf16 pools; 1: Sage K8 / V8 pools
  void* k_pool;
  void* v_pool;
  int64_t num_slots;
  const float* sf_k_new;   // Sage: [n_tokens][hkv] block scales, or NULL
  float* sf_k;             // Sage: [num_slots / 64][hkv]
  PlanHeader* hdr;     // optional: where to record an out-of-range slot
};
cudaError_t launch_kv_store(const StoreLaunch& a, cudaStream_t s);

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
