// read_probe: a read-only streaming kernel, for measuring the HBM read
// ceiling beside the decode kernels (a diagnostic; the pages have no
// counterpart).  A persistent grid reads every 16-byte vector of a buffer
// once, four vectors in flight per thread, and folds them with XOR into one
// word per CTA so that no load can be optimised away.
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.h"

namespace pa {

namespace {

constexpr int kProbeThreads = 512;

__global__ void __launch_bounds__(kProbeThreads)
read_probe_kernel(const uint4* __restrict__ buf, int64_t nvec, uint32_t* __restrict__ sink) {
  uint32_t acc = 0;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kProbeThreads;
  int64_t i = static_cast<int64_t>(blockIdx.x) * kProbeThreads + threadIdx.x;
  for (; i + 3 * stride < nvec; i += 4 * stride) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = __ldcs(buf + i + u * stride);
#pragma unroll
    for (int u = 0; u < 4; ++u) acc ^= v[u].x ^ v[u].y ^ v[u].z ^ v[u].w;
  }
  for (; i < nvec; i += stride) {
    const uint4 v = __ldcs(buf + i);
    acc ^= v.x ^ v.y ^ v.z ^ v.w;
  }
  __shared__ uint32_t red[kProbeThreads / 32];
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, off);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t r = 0;
    for (int w = 0; w < kProbeThreads / 32; ++w) r ^= red[w];
    sink[blockIdx.x] = r;
  }
}

}  // namespace

cudaError_t launch_read_probe(const void* buf, int64_t bytes, uint32_t* sink, int sink_words,
                              cudaStream_t stream) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaGetLastError();
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return cudaGetLastError();
  const int grid = sms * 4 < sink_words ? sms * 4 : sink_words;  // 4 CTAs of 512 per SM
  if (grid <= 0) return cudaErrorInvalidValue;
  read_probe_kernel<<<grid, kProbeThreads, 0, stream>>>(static_cast<const uint4*>(buf), bytes / 16,
                                                        sink);
  return cudaGetLastError();
}

}  // namespace pa
