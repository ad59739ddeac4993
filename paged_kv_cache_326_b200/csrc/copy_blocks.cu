// copy_blocks: whole-block copies between two pools (or within one): the
// device side of copy-on-write ("The KV Cache and PagedAttention", section
// "Shared, Copied on Write": a text that must change a block it shares
// first receives a duplicate of it) and of moving blocks out of a pool and back
// (section "When Memory Runs Out").
//
// A block of one pool tensor is one contiguous run of H * B * D elements, so
// a copy is a plain stream of 16-byte vectors.  All copies of a call (pair p
// and K or V: copy 2p or 2p+1) form one flat order of vectors, and a
// persistent grid (kCopyCtasPerSm CTAs per SM) cuts it into equal contiguous
// shares, one per CTA: no CTA waits on a partial second wave, and a share
// may run across the end of one copy into the next.  Each thread keeps
// kUnroll vectors in flight.  The kernel is HBM-bound (every distinct byte
// read once and written once).
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.h"
#include "ptx.cuh"

namespace pa {

namespace {

constexpr int kCopyThreads = 256;
constexpr int kUnroll = 4;
constexpr int kCopyCtasPerSm = 8;

__global__ void __launch_bounds__(kCopyThreads, kCopyCtasPerSm)
copy_blocks_kernel(const uint4* src_k, const uint4* src_v, uint4* dst_k, uint4* dst_v,
                   const int32_t* __restrict__ pairs, int64_t vecs_per_block, int64_t total,
                   int64_t src_num_blocks, int64_t dst_num_blocks, int32_t* status) {
  // The pairs or the source blocks may come from the kernel launched just
  // before; a kernel launched after this one waits for all of it.
  griddep_wait();
  griddep_launch_dependents();
  const int64_t per = (total + gridDim.x - 1) / gridDim.x;
  const int64_t lo = blockIdx.x * per;
  const int64_t hi = lo + per < total ? lo + per : total;
  // The share [lo, hi) covers the end of one copy, whole copies, the start
  // of another: walk it copy by copy, each piece a contiguous range.
  for (int64_t c = lo / vecs_per_block; c * vecs_per_block < hi; ++c) {
    const int64_t base = c * vecs_per_block;
    const int64_t a = lo > base ? lo - base : 0;
    const int64_t b = hi < base + vecs_per_block ? hi - base : vecs_per_block;
    const int64_t pair = c >> 1;
    const int64_t s = __ldg(pairs + 2 * pair);
    const int64_t d = __ldg(pairs + 2 * pair + 1);
    if (s < 0 || s >= src_num_blocks || d < 0 || d >= dst_num_blocks) {
      // reported by the CTA whose share holds the pair's first vector
      if (a == 0 && !(c & 1) && threadIdx.x == 0) set_status(status, -7 /* PA_ERR_BAD_BLOCK */);
      continue;
    }
    const uint4* src = ((c & 1) ? src_v : src_k) + s * vecs_per_block;
    uint4* dst = ((c & 1) ? dst_v : dst_k) + d * vecs_per_block;
    for (int64_t i = a + threadIdx.x; i < b; i += kCopyThreads * kUnroll) {
      uint4 r[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t j = i + u * kCopyThreads;
        if (j < b) r[u] = src[j];
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t j = i + u * kCopyThreads;
        if (j < b) dst[j] = r[u];
      }
    }
  }
}

}  // namespace

cudaError_t launch_copy_blocks(const void* src_k, const void* src_v, void* dst_k, void* dst_v,
                               const int32_t* pairs, int num_pairs, int64_t block_bytes,
                               int64_t src_num_blocks, int64_t dst_num_blocks, int32_t* status,
                               cudaStream_t stream) {
  const int64_t vecs = block_bytes / 16;
  const int64_t total = static_cast<int64_t>(num_pairs) * 2 * vecs;
  if (total <= 0) return cudaErrorInvalidValue;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return cudaGetLastError();
  // persistent grid, never more CTAs than there are vectors for each to copy
  int64_t grid = static_cast<int64_t>(sms) * kCopyCtasPerSm;
  const int64_t most = (total + kCopyThreads - 1) / kCopyThreads;
  if (grid > most) grid = most;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kCopyThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t err = cudaLaunchKernelEx(
      &cfg, copy_blocks_kernel, static_cast<const uint4*>(src_k), static_cast<const uint4*>(src_v),
      static_cast<uint4*>(dst_k), static_cast<uint4*>(dst_v), pairs, vecs, total, src_num_blocks,
      dst_num_blocks, status);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace pa
