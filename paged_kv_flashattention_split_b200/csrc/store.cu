// store.cu - KV cache update: scatter new tokens' K/V rows into their pool slots.
//
// The cache is updated inside the forward pass before attention reads it
// ("Flash Attention Backend in SGLang: Grundlagen und KV Cache optimal nutzen").
// A token's row of all Hkv heads is one contiguous run both in the new-token tensor
// and in its pool slot (Hkv * 256 bytes in bf16, Hkv * 128 in the 8-bit Sage pools), so
// consecutive threads copy consecutive 16-byte pieces: coalesced reads, and writes in
// whole rows.  For the Sage pools the token that opens a 64-slot block also writes the
// block's K scales.
#include "kernels.h"

namespace pa {
namespace {

__global__ void __launch_bounds__(256) kv_store_kernel(StoreLaunch a) {
  const int64_t chunks_per_row = (int64_t)a.hkv * kHeadDim * a.elem_bytes / 16;   // 16-byte pieces per token row
  const int64_t total = a.n_tokens * chunks_per_row;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / chunks_per_row, c = i % chunks_per_row;
    const int32_t slot = __ldg(a.loc + t);
    if (slot < 0 || slot >= a.num_slots) {
      if (c == 0 && a.hdr) set_device_error(a.hdr, PA_ERR_DEVICE_INDEX);
      continue;
    }
    const uint4 kv = __ldg(reinterpret_cast<const uint4*>(a.k_new) + i);
    const uint4 vv = __ldg(reinterpret_cast<const uint4*>(a.v_new) + i);
    reinterpret_cast<uint4*>(a.k_pool)[(int64_t)slot * chunks_per_row + c] = kv;
    reinterpret_cast<uint4*>(a.v_pool)[(int64_t)slot * chunks_per_row + c] = vv;
  }
  if (!a.sf_k_new) return;
  // Sage: sfK[slot / 64][h] = sf_k_new[t][h] for the tokens whose slot opens its block
  const int64_t n_sf = a.n_tokens * a.hkv;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_sf; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / a.hkv, h = i % a.hkv;
    const int32_t slot = __ldg(a.loc + t);
    if (slot < 0 || slot >= a.num_slots || slot % kSageBlock != 0) continue;
    a.sf_k[(int64_t)(slot / kSageBlock) * a.hkv + h] = __ldg(a.sf_k_new + i);
  }
}

}  // namespace

cudaError_t launch_kv_store(const StoreLaunch& a, cudaStream_t s) {
  const int64_t total = a.n_tokens * a.hkv * kHeadDim * a.elem_bytes / 16;
  int dev = 0, sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int64_t want = (total + 255) / 256;
  const int blocks = (int)(want < (int64_t)sms * 8 ? (want > 0 ? want : 1) : (int64_t)sms * 8);
  kv_store_kernel<<<blocks, 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace pa
