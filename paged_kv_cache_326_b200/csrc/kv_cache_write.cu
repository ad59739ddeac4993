// kv_cache_write: scatter each new token's key and value into its slot.
//
// "KV cache", section "How it works": each generated token's key and value
// join the cache; "The KV Cache and PagedAttention", section "One Token at a
// Time": a step computes keys and values for the new token alone.
//
// One thread moves one 16-byte vector of K and the matching one of V.  A
// token's H*D elements are contiguous in the input and land in H tiles of the
// pool (one per head, stride block_size*head_dim), each a contiguous row of
// head_dim elements, so both the loads and the stores are full 16-byte
// transactions and consecutive threads touch consecutive bytes of a row.
#include <cuda_runtime.h>

#include <cstdint>

#include "dtype.cuh"
#include "fp8.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace pa {

__global__ void __launch_bounds__(256)
kv_cache_write_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                      uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                      const int64_t* __restrict__ slot_mapping, int num_tokens, int num_heads,
                      int vec_per_row, int block_size, int64_t num_slots, int32_t* status) {
  // Programmatic dependent launch: wait for the previous kernel's writes
  // (for example the last decode still reading this pool), then let the
  // decode kernel that follows get its CTAs resident.
  griddep_wait();
  griddep_launch_dependents();
  const int64_t per_token = static_cast<int64_t>(num_heads) * vec_per_row;
  const int64_t total = per_token * num_tokens;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / per_token;
    const int64_t r = i - t * per_token;
    const int64_t h = r / vec_per_row;
    const int64_t c = r - h * vec_per_row;
    const int64_t slot = __ldg(slot_mapping + t);
    if (slot < 0) continue;
    if (slot >= num_slots) {
      if (r == 0) set_status(status, -9 /* PA_ERR_BAD_SLOT */);
      continue;
    }
    const int64_t blk = slot / block_size;
    const int64_t place = slot - blk * block_size;
    const int64_t dst = ((blk * num_heads + h) * block_size + place) * vec_per_row + c;
    k_cache[dst] = __ldg(k + i);
    v_cache[dst] = __ldg(v + i);
  }
}

// The 8-bit cache's write ("The KV Cache and PagedAttention", section "What
// Came After": one byte per cached number): each element x of the new key
// (value) is stored as the E4M3 code of the fp32 quotient x / k_scale
// (x / v_scale), IEEE division, round to nearest even, saturating.  One
// thread turns one 16-byte vector of 8 input elements into 8 codes.
template <typename T>
__global__ void __launch_bounds__(256)
kv_cache_write_fp8_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                          uint2* __restrict__ k_cache, uint2* __restrict__ v_cache,
                          const int64_t* __restrict__ slot_mapping, float k_scale, float v_scale,
                          int num_tokens, int num_heads, int vec_per_row, int block_size,
                          int64_t num_slots, int32_t* status) {
  griddep_wait();
  griddep_launch_dependents();
  const int64_t per_token = static_cast<int64_t>(num_heads) * vec_per_row;
  const int64_t total = per_token * num_tokens;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / per_token;
    const int64_t r = i - t * per_token;
    const int64_t h = r / vec_per_row;
    const int64_t c = r - h * vec_per_row;
    const int64_t slot = __ldg(slot_mapping + t);
    if (slot < 0) continue;
    if (slot >= num_slots) {
      if (r == 0) set_status(status, -9 /* PA_ERR_BAD_SLOT */);
      continue;
    }
    const int64_t blk = slot / block_size;
    const int64_t place = slot - blk * block_size;
    const int64_t dst = ((blk * num_heads + h) * block_size + place) * vec_per_row + c;
    float x[8];
    unpack8<T>(__ldg(k + i), x);
    k_cache[dst] = e4m3x8_quantize(x, k_scale);
    unpack8<T>(__ldg(v + i), x);
    v_cache[dst] = e4m3x8_quantize(x, v_scale);
  }
}

cudaError_t launch_kv_cache_write_fp8(const void* k, const void* v, void* k_cache, void* v_cache,
                                      const int64_t* slot_mapping, float k_scale, float v_scale,
                                      int num_tokens, int num_heads, int head_dim, int block_size,
                                      int64_t num_blocks, bool bf16, int32_t* status,
                                      cudaStream_t stream) {
  const int vec_per_row = head_dim / 8;  // input: 8 two-byte elements per 16 bytes
  const int64_t total = static_cast<int64_t>(num_tokens) * num_heads * vec_per_row;
  if (total == 0) return cudaSuccess;
  const int threads = 256;
  int64_t blocks = (total + threads - 1) / threads;
  if (blocks > (1 << 20)) blocks = 1 << 20;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks));
  cfg.blockDim = dim3(threads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const auto kernel = bf16 ? kv_cache_write_fp8_kernel<__nv_bfloat16> : kv_cache_write_fp8_kernel<__half>;
  cudaError_t err = cudaLaunchKernelEx(
      &cfg, kernel, static_cast<const uint4*>(k), static_cast<const uint4*>(v),
      static_cast<uint2*>(k_cache), static_cast<uint2*>(v_cache), slot_mapping, k_scale, v_scale,
      num_tokens, num_heads, vec_per_row, block_size, num_blocks * block_size, status);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

cudaError_t launch_kv_cache_write(const void* k, const void* v, void* k_cache, void* v_cache,
                                  const int64_t* slot_mapping, int num_tokens, int num_heads,
                                  int head_dim, int block_size, int64_t num_blocks,
                                  int32_t* status, cudaStream_t stream) {
  const int vec_per_row = head_dim / 8;  // 8 two-byte elements per 16 bytes
  const int64_t total = static_cast<int64_t>(num_tokens) * num_heads * vec_per_row;
  if (total == 0) return cudaSuccess;
  const int threads = 256;
  int64_t blocks = (total + threads - 1) / threads;
  if (blocks > (1 << 20)) blocks = 1 << 20;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks));
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t err = cudaLaunchKernelEx(
      &cfg, kv_cache_write_kernel, static_cast<const uint4*>(k), static_cast<const uint4*>(v),
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), slot_mapping, num_tokens,
      num_heads, vec_per_row, block_size, num_blocks * block_size, status);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace pa
