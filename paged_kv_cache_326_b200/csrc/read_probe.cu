// read_probe: a read-only streaming kernel, for measuring the HBM read
// ceiling beside the decode kernels, and a write-only one for the block
// copies (diagnostics; the pages have no counterpart).  A persistent grid reads every 16-byte vector of a buffer
// once, four vectors in flight per thread, and folds them with XOR into one
// word per CTA so that no load can be optimised away.
#include <cuda_runtime.h>

#include <cstdint>

#include "exp2poly.cuh"
#include "kernels.h"
#include "ptx.cuh"

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

// Write-only stream: every 16-byte vector of the buffer receives a pattern
// derived from its index (streaming stores, four per thread per round).
__global__ void __launch_bounds__(kProbeThreads)
write_probe_kernel(uint4* __restrict__ buf, int64_t nvec) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kProbeThreads;
  int64_t i = static_cast<int64_t>(blockIdx.x) * kProbeThreads + threadIdx.x;
  for (; i + 3 * stride < nvec; i += 4 * stride) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t x = static_cast<uint32_t>(i + u * stride);
      __stcs(buf + i + u * stride, make_uint4(x, x ^ 0x9e3779b9u, ~x, x + 1u));
    }
  }
  for (; i < nvec; i += stride) {
    const uint32_t x = static_cast<uint32_t>(i);
    __stcs(buf + i, make_uint4(x, x ^ 0x9e3779b9u, ~x, x + 1u));
  }
}

// y[i] = 2^x[i], by the FMA-pipe polynomial of exp2poly.cuh (method 0) or by
// the exponential unit's ex2.approx (method 1).
__global__ void __launch_bounds__(256)
exp2_probe_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t n, int method) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x * 2;
  for (int64_t i = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 2; i < n;
       i += stride) {
    const float a = x[i];
    const float b = i + 1 < n ? x[i + 1] : 0.f;
    float2 r;
    if (method == 0) {
      r = exp2_poly2(make_float2(a, b));
    } else {
      r = make_float2(fast_exp2(a), fast_exp2(b));
    }
    y[i] = r.x;
    if (i + 1 < n) y[i + 1] = r.y;
  }
}

}  // namespace

cudaError_t launch_exp2_probe(const float* x, float* y, int64_t n, int method,
                              cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  int64_t blocks = (n + 511) / 512;
  if (blocks > 4096) blocks = 4096;
  exp2_probe_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(x, y, n, method);
  return cudaGetLastError();
}

cudaError_t launch_write_probe(void* buf, int64_t bytes, cudaStream_t stream) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaGetLastError();
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return cudaGetLastError();
  write_probe_kernel<<<sms * 4, kProbeThreads, 0, stream>>>(static_cast<uint4*>(buf), bytes / 16);
  return cudaGetLastError();
}

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
