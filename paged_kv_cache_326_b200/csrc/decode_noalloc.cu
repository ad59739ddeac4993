// pa_paged_attn_decode_noalloc: paged decode attention for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc, or cannot hand this library a buffer
// of their own: a host framework that owns every device allocation and gives
// out no scratch, a fixed device-memory budget set before serving starts, or a
// latency-bound loop where an allocation (which may synchronise the device)
// is not allowed.  This entry point runs the same kernels as
// pa_paged_attn_decode, but its scratch is a file-scope device array that the
// library carries with it, so the caller passes only inputs and outputs.
#include <cuda.h>  // CUcontext and CUresult, for the two driver entry points below
#include <cuda_runtime.h>

#include <cstdint>
#include <map>
#include <mutex>
#include <utility>

#include "kernels.h"
#include "pagedattn.h"

namespace {

// 16 MiB of scratch, zero at load, kept by every GPU that loads the library
// until the process exits.  Enough for, e.g., 256 texts x 40 heads x 128.
constexpr size_t kScratchBytes = size_t{16} << 20;
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current context (0 if there is none or
// the driver cannot say).  A device reset ends the primary context; the one
// the runtime makes next has a new id, and the module holding
// g_decode_scratch is loaded again into it, possibly at another address.
unsigned long long current_context_id() {
  static std::once_flag once;
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(f);
    f = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &f, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(f);
    cudaGetLastError();
  });
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of g_decode_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, never a device address, so it is
// resolved with cudaGetSymbolAddress: once per (device, context), the first
// time a call runs there.  The lookup itself makes the device's primary
// context current if no runtime call has yet.
int scratch_address(void** out) {
  static std::mutex mu;
  static std::map<std::pair<int, unsigned long long>, void*> addr;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return PA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(mu);
  const unsigned long long ctx = current_context_id();
  if (ctx != 0) {
    const auto it = addr.find({dev, ctx});
    if (it != addr.end()) {
      *out = it->second;
      return PA_OK;
    }
  }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) {
    cudaGetLastError();
    return PA_ERR_CUDA;
  }
  // cache it under the context the lookup ran in (made current by it if
  // there was none); without a context id, look it up on every call
  const unsigned long long ctx_now = ctx != 0 ? ctx : current_context_id();
  if (ctx_now != 0) addr[{dev, ctx_now}] = p;
  *out = p;
  return PA_OK;
}

}  // namespace

extern "C" int pa_paged_attn_decode_noalloc(void* out, const void* q, const void* k_cache,
                                            const void* v_cache, const int32_t* block_tables,
                                            const int32_t* context_lens, float scale,
                                            int num_seqs, int num_heads, int head_dim,
                                            int block_size, int max_blocks_per_seq,
                                            int64_t num_blocks, pa_dtype dt, int32_t* d_status,
                                            pa_stream_t stream) {
  if (num_seqs == 0) return PA_OK;
  // only the 16-bit kernels run here
  const size_t need =
      pa::decode_workspace_bytes(num_seqs, num_heads, num_heads, head_dim, block_size,
                                 max_blocks_per_seq, pa::option_decode_warps(), false);
  if (need == 0) return PA_ERR_INVALID;
  if (need > kScratchBytes) return PA_ERR_TOO_LARGE;
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc != PA_OK) return rc;
  return pa_paged_attn_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale,
                              num_seqs, num_heads, head_dim, block_size, max_blocks_per_seq,
                              num_blocks, dt, scratch, kScratchBytes, d_status, stream);
}
