// copy_blocks: whole-block copies between two pools (or within one): the
// device side of copy-on-write ("The KV Cache and PagedAttention", section
// "Shared, Copied on Write": a text that must change a block it shares
// first receives a duplicate of it) and of moving blocks out of a pool and back
// (section "When Memory Runs Out").
//
// A block of one pool tensor is one contiguous run of H * B * D elements, so
// a copy is a plain stream of 16-byte vectors.  Each CTA copies one piece of
// one (pair, K-or-V) block with every thread keeping kUnroll vectors in
// flight; the grid covers all pieces of all pairs at once.  The kernel is
// HBM-bound (every byte read once and written once).  A persistent grid
// (one equal share of all copies per CTA) measured slower than this one on
// bursts of 448 copies of 160 KB (23.8 against 21.4 microseconds): its
// shares cross copy boundaries, and the extra index work per piece costs
// more than the partial last wave it saves.
//
// Two other forms measured slower on the same bursts: a CTA per run of
// pairs with one source, reading it once and writing every destination
// (29.5 microseconds: too few CTAs left writing), and the run's CTAs each
// taking one slice of the source for all destinations (23.5).
// PA_COPY_STREAMING_STORE=1 writes with st.global.cs (evict-first); it
// measured no different, nor did 8 vectors in flight (21.2 us), 512 threads
// (21.9) or 128 threads of 8 vectors (21.3); 64 KB pieces were slower
// (23.3-25.0).  Moving the pieces through the bulk-copy unit instead (one
// warp per piece: bulk loads into shared memory, each chunk written out by
// a bulk store as soon as it lands; pieces of 16, 32 or 64 KB in 1 to 8
// chunks) measured the same 21.1-21.3 microseconds: the bursts are bound by
// the memory system's writes, not by how the copies are issued.
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.h"
#include "ptx.cuh"

namespace pa {

namespace {

#ifndef PA_COPY_THREADS
#define PA_COPY_THREADS 256
#endif
#ifndef PA_COPY_UNROLL
#define PA_COPY_UNROLL 4
#endif
#ifndef PA_COPY_ROUNDS
#define PA_COPY_ROUNDS 2
#endif
constexpr int kCopyThreads = PA_COPY_THREADS;
constexpr int kUnroll = PA_COPY_UNROLL;  // 16-byte vectors in flight per thread
constexpr int64_t kVecsPerCta = kCopyThreads * kUnroll * PA_COPY_ROUNDS;  // 32 KB per CTA

#ifndef PA_COPY_STREAMING_STORE
#define PA_COPY_STREAMING_STORE 0
#endif

__device__ __forceinline__ void store_vec(uint4* p, uint4 v) {
#if PA_COPY_STREAMING_STORE
  __stcs(p, v);
#else
  *p = v;
#endif
}

__global__ void __launch_bounds__(kCopyThreads)
copy_blocks_kernel(const uint4* src_k, const uint4* src_v, uint4* dst_k, uint4* dst_v,
                   const int32_t* __restrict__ pairs, int64_t vecs_per_block, int ctas_per_copy,
                   int64_t src_num_blocks, int64_t dst_num_blocks, int32_t* status) {
  // The pairs or the source blocks may come from the kernel launched just
  // before; a kernel launched after this one waits for all of it.
  griddep_wait();
  griddep_launch_dependents();
  const int64_t copy = blockIdx.x / ctas_per_copy;  // (pair, K or V)
  const int piece = static_cast<int>(blockIdx.x - copy * ctas_per_copy);
  const int64_t pair = copy >> 1;
  const bool is_v = copy & 1;
  const int64_t s = __ldg(pairs + 2 * pair);
  const int64_t d = __ldg(pairs + 2 * pair + 1);
  if (s < 0 || s >= src_num_blocks || d < 0 || d >= dst_num_blocks) {
    if (piece == 0 && !is_v && threadIdx.x == 0) set_status(status, -7 /* PA_ERR_BAD_BLOCK */);
    return;
  }
  const uint4* src = (is_v ? src_v : src_k) + s * vecs_per_block;
  uint4* dst = (is_v ? dst_v : dst_k) + d * vecs_per_block;
  const int64_t per = (vecs_per_block + ctas_per_copy - 1) / ctas_per_copy;
  const int64_t lo = piece * per;
  const int64_t hi = lo + per < vecs_per_block ? lo + per : vecs_per_block;
  for (int64_t i = lo + threadIdx.x; i < hi; i += kCopyThreads * kUnroll) {
    uint4 r[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t j = i + u * kCopyThreads;
      if (j < hi) r[u] = src[j];
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t j = i + u * kCopyThreads;
      if (j < hi) store_vec(dst + j, r[u]);
    }
  }
}

}  // namespace

cudaError_t launch_copy_blocks(const void* src_k, const void* src_v, void* dst_k, void* dst_v,
                               const int32_t* pairs, int num_pairs, int64_t block_bytes,
                               int64_t src_num_blocks, int64_t dst_num_blocks, int32_t* status,
                               cudaStream_t stream) {
  const int64_t vecs = block_bytes / 16;
  const int ctas_per_copy = static_cast<int>((vecs + kVecsPerCta - 1) / kVecsPerCta);
  const int64_t grid = static_cast<int64_t>(num_pairs) * 2 * ctas_per_copy;
  if (grid <= 0 || grid > 0x7fffffff) return cudaErrorInvalidValue;
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
      static_cast<uint4*>(dst_k), static_cast<uint4*>(dst_v), pairs, vecs, ctas_per_copy,
      src_num_blocks, dst_num_blocks, status);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace pa
