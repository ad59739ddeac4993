// C ABI of libpagedattn.so (declared and documented in include/pagedattn.h):
// argument checks, then the launchers in kv_cache_write.cu and
// paged_attn_decode.cu.  Nothing here allocates device memory.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "kernels.h"
#include "pagedattn.h"

namespace {

std::atomic<int64_t> g_wait_limit_ns{1000000000};
std::atomic<int64_t> g_decode_warps{0};
std::atomic<int64_t> g_gqa_kernel{0};
std::atomic<int64_t> g_prefill_kernel{0};
std::atomic<int64_t> g_prefix_key_bits{64};
std::atomic<int64_t> g_fp8_kernel{0};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool shape_ok(int num_heads, int head_dim, int block_size) {
  return num_heads >= 1 && num_heads <= 1024 && (head_dim == 64 || head_dim == 128) &&
         (block_size == 4 || block_size == 8 || block_size == 16 || block_size == 32);
}

// Memory the current device can read and write at this address: its own
// device memory, managed memory, or pinned host memory mapped at the same
// address (unified addressing).
bool device_accessible(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (a.type == cudaMemoryTypeDevice) return a.device == dev;
  if (a.type == cudaMemoryTypeManaged) return true;
  if (a.type == cudaMemoryTypeHost) return a.devicePointer == p;
  return false;
}

// A usable per-tensor scale of the 8-bit cache: finite and positive.
bool scale_ok(float s) { return s > 0.f && s <= 3.402823466e38f; }

int from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return PA_OK;
  if (e == cudaErrorInvalidValue) return PA_ERR_INVALID;
  return PA_ERR_CUDA;
}

}  // namespace

namespace pa {
int64_t option_decode_warps() { return g_decode_warps.load(); }
int64_t option_gqa_kernel() { return g_gqa_kernel.load(); }
int64_t option_prefill_kernel() { return g_prefill_kernel.load(); }
int64_t option_prefix_key_bits() { return g_prefix_key_bits.load(); }
int64_t option_fp8_kernel() { return g_fp8_kernel.load(); }
}  // namespace pa

namespace {

// Checks shared by the shared-prefix entry points, then the launch.
int shared_common(void* out, const void* q, const void* k_cache, const void* v_cache,
                  const int32_t* prefix_tables, const int32_t* prefix_lens,
                  int max_prefix_blocks, const int32_t* tail_tables, const int32_t* tail_lens,
                  int max_tail_blocks, float scale, int num_groups, int group_size, int num_heads,
                  int num_kv_heads, int head_dim, int block_size, int64_t num_blocks,
                  pa_dtype dt, void* workspace, size_t workspace_bytes, int32_t* d_status,
                  pa_stream_t stream) {
  if (num_groups == 0) return PA_OK;
  if (num_groups < 0 || group_size < 1 || group_size > 1024 ||
      static_cast<int64_t>(num_groups) * group_size > 4096 || max_prefix_blocks < 1 ||
      max_tail_blocks < 1 || num_blocks <= 0 || num_heads < 1 || num_kv_heads < 1 ||
      num_heads % num_kv_heads || !shape_ok(num_kv_heads, head_dim, block_size) ||
      block_size < 8 || (dt != PA_F16 && dt != PA_BF16))
    return PA_ERR_INVALID;
  if (!out || !q || !k_cache || !v_cache || !prefix_tables || !prefix_lens || !tail_tables ||
      !tail_lens || !workspace)
    return PA_ERR_INVALID;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return PA_ERR_INVALID;
  if (!pa::mma_decode_pool_ok(num_kv_heads, block_size, num_blocks)) return PA_ERR_INVALID;
  pa::SharedPrefixArgs a;
  a.out = out;
  a.q = q;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.prefix_tables = prefix_tables;
  a.prefix_lens = prefix_lens;
  a.max_prefix_blocks = max_prefix_blocks;
  a.tail_tables = tail_tables;
  a.tail_lens = tail_lens;
  a.max_tail_blocks = max_tail_blocks;
  a.scale = scale;
  a.num_groups = num_groups;
  a.group_size = group_size;
  a.num_heads = num_heads;
  a.num_kv_heads = num_kv_heads;
  a.head_dim = head_dim;
  a.block_size = block_size;
  a.num_blocks = num_blocks;
  a.is_bf16 = dt == PA_BF16;
  a.workspace = workspace;
  a.workspace_bytes = workspace_bytes;
  a.status = d_status;
  a.wait_limit_ns = g_wait_limit_ns.load();
  a.forced_warps = g_decode_warps.load();
  return from_cuda(
      pa::launch_paged_attn_decode_shared(a, reinterpret_cast<cudaStream_t>(stream)));
}

}  // namespace

extern "C" {

const char* pa_status_string(int code) {
  switch (code) {
    case PA_OK: return "ok";
    case PA_ERR_INVALID: return "invalid argument";
    case PA_ERR_CUDA: return "CUDA runtime error";
    case PA_ERR_OUT_OF_BLOCKS: return "out of blocks";
    case PA_ERR_NO_SEQ: return "unknown sequence";
    case PA_ERR_EXISTS: return "sequence exists";
    case PA_ERR_TABLE_FULL: return "block table longer than max_blocks_per_seq";
    case PA_ERR_BAD_BLOCK: return "block table entry outside the pool";
    case PA_ERR_BAD_LEN: return "context length outside [0, max_blocks_per_seq*block_size]";
    case PA_ERR_BAD_SLOT: return "slot outside the pool";
    case PA_ERR_TIMEOUT: return "bounded wait gave up";
    case PA_ERR_CORRUPT: return "block manager counts inconsistent";
    case PA_ERR_TOO_LARGE: return "sizes need more scratch than the no-allocation entry point holds";
    default: return "unknown status";
  }
}

int pa_set_option(int key, int64_t value) {
  switch (key) {
    case PA_OPT_WAIT_LIMIT_NS: g_wait_limit_ns = value; return PA_OK;
    case PA_OPT_DECODE_WARPS:
      if (value < 0 || value > (int64_t{1} << 20)) return PA_ERR_INVALID;
      g_decode_warps = value;
      return PA_OK;
    case PA_OPT_GQA_KERNEL:
      if (value < 0 || value > 2) return PA_ERR_INVALID;
      g_gqa_kernel = value;
      return PA_OK;
    case PA_OPT_PREFILL_KERNEL:
      if (value < 0 || value > 2) return PA_ERR_INVALID;
      g_prefill_kernel = value;
      return PA_OK;
    case PA_OPT_FP8_KERNEL:
      if (value < 0 || value > 2) return PA_ERR_INVALID;
      g_fp8_kernel = value;
      return PA_OK;
    case PA_OPT_PREFIX_KEY_BITS:
      if (value < 1 || value > 64) return PA_ERR_INVALID;
      g_prefix_key_bits = value;
      return PA_OK;
    default: return PA_ERR_INVALID;
  }
}

int pa_kv_cache_write(const void* k, const void* v, void* k_cache, void* v_cache,
                      const int64_t* slot_mapping, int num_tokens, int num_heads, int head_dim,
                      int block_size, int64_t num_blocks, pa_dtype dt, int32_t* d_status,
                      pa_stream_t stream) {
  if (num_tokens < 0 || !shape_ok(num_heads, head_dim, block_size) || num_blocks <= 0 ||
      (dt != PA_F16 && dt != PA_BF16))
    return PA_ERR_INVALID;
  if (num_tokens == 0) return PA_OK;
  if (!k || !v || !k_cache || !v_cache || !slot_mapping) return PA_ERR_INVALID;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_INVALID;
  return from_cuda(pa::launch_kv_cache_write(k, v, k_cache, v_cache, slot_mapping, num_tokens,
                                             num_heads, head_dim, block_size, num_blocks,
                                             d_status, reinterpret_cast<cudaStream_t>(stream)));
}

size_t pa_paged_attn_decode_workspace_size(int num_seqs, int num_heads, int head_dim,
                                           int block_size, int max_blocks_per_seq) {
  return pa::decode_workspace_bytes(num_seqs, num_heads, num_heads, head_dim, block_size,
                                    max_blocks_per_seq, g_decode_warps.load());
}

size_t pa_paged_attn_decode_gqa_workspace_size(int num_seqs, int num_heads, int num_kv_heads,
                                               int head_dim, int block_size,
                                               int max_blocks_per_seq) {
  return pa::decode_workspace_bytes(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                    max_blocks_per_seq, g_decode_warps.load());
}

}  // extern "C"

namespace {

// Checks shared by the decode entry points, then the launch.
int decode_common(void* out, const void* q, const void* k_cache, const void* v_cache,
                  const int32_t* block_tables, const int32_t* context_lens, float scale,
                  int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
                  int max_blocks_per_seq, int64_t num_blocks, pa_dtype dt, void* workspace,
                  size_t workspace_bytes, int32_t* d_status, pa_stream_t stream,
                  const void* k_new, const void* v_new, const int64_t* slot_mapping,
                  bool fp8 = false, float k_scale = 1.f, float v_scale = 1.f) {
  if (num_seqs == 0) return PA_OK;
  if (fp8 && !(scale_ok(k_scale) && scale_ok(v_scale))) return PA_ERR_INVALID;
  if (!pa::decode_sizes_supported(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                  max_blocks_per_seq) ||
      num_blocks <= 0 || (dt != PA_F16 && dt != PA_BF16))
    return PA_ERR_INVALID;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !workspace)
    return PA_ERR_INVALID;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return PA_ERR_INVALID;
  if (slot_mapping && (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new)))
    return PA_ERR_INVALID;
  pa::DecodeArgs a;
  a.out = out;
  a.q = q;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.scale = scale;
  a.num_seqs = num_seqs;
  a.num_heads = num_heads;
  a.num_kv_heads = num_kv_heads;
  a.head_dim = head_dim;
  a.block_size = block_size;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.num_blocks = num_blocks;
  a.is_bf16 = dt == PA_BF16;
  a.workspace = workspace;
  a.workspace_bytes = workspace_bytes;
  a.status = d_status;
  a.wait_limit_ns = g_wait_limit_ns.load();
  a.forced_warps = g_decode_warps.load();
  a.k_new = k_new;
  a.v_new = v_new;
  a.slot_mapping = slot_mapping;
  a.fp8 = fp8;
  a.k_scale = k_scale;
  a.v_scale = v_scale;
  return from_cuda(pa::launch_paged_attn_decode(a, reinterpret_cast<cudaStream_t>(stream)));
}

}  // namespace

extern "C" {

int pa_paged_attn_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                         const int32_t* block_tables, const int32_t* context_lens, float scale,
                         int num_seqs, int num_heads, int head_dim, int block_size,
                         int max_blocks_per_seq, int64_t num_blocks, pa_dtype dt,
                         void* workspace, size_t workspace_bytes, int32_t* d_status,
                         pa_stream_t stream) {
  return decode_common(out, q, k_cache, v_cache, block_tables, context_lens, scale, num_seqs,
                       num_heads, num_heads, head_dim, block_size, max_blocks_per_seq, num_blocks,
                       dt, workspace, workspace_bytes, d_status, stream, nullptr, nullptr, nullptr);
}

int pa_kv_cache_write_fp8(const void* k, const void* v, void* k_cache, void* v_cache,
                          const int64_t* slot_mapping, float k_scale, float v_scale,
                          int num_tokens, int num_heads, int head_dim, int block_size,
                          int64_t num_blocks, pa_dtype dt, int32_t* d_status, pa_stream_t stream) {
  if (num_tokens < 0 || !shape_ok(num_heads, head_dim, block_size) || num_blocks <= 0 ||
      (dt != PA_F16 && dt != PA_BF16) || !scale_ok(k_scale) || !scale_ok(v_scale))
    return PA_ERR_INVALID;
  if (num_tokens == 0) return PA_OK;
  if (!k || !v || !k_cache || !v_cache || !slot_mapping) return PA_ERR_INVALID;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_INVALID;
  return from_cuda(pa::launch_kv_cache_write_fp8(
      k, v, k_cache, v_cache, slot_mapping, k_scale, v_scale, num_tokens, num_heads, head_dim,
      block_size, num_blocks, dt == PA_BF16, d_status, reinterpret_cast<cudaStream_t>(stream)));
}

int pa_paged_attn_decode_fp8(void* out, const void* q, const void* k_cache, const void* v_cache,
                             const int32_t* block_tables, const int32_t* context_lens,
                             float scale, float k_scale, float v_scale, int num_seqs,
                             int num_heads, int head_dim, int block_size, int max_blocks_per_seq,
                             int64_t num_blocks, pa_dtype dt, void* workspace,
                             size_t workspace_bytes, int32_t* d_status, pa_stream_t stream) {
  return decode_common(out, q, k_cache, v_cache, block_tables, context_lens, scale, num_seqs,
                       num_heads, num_heads, head_dim, block_size, max_blocks_per_seq, num_blocks,
                       dt, workspace, workspace_bytes, d_status, stream, nullptr, nullptr, nullptr,
                       true, k_scale, v_scale);
}

int pa_paged_attn_decode_fp8_gqa(void* out, const void* q, const void* k_cache,
                                 const void* v_cache, const int32_t* block_tables,
                                 const int32_t* context_lens, float scale, float k_scale,
                                 float v_scale, int num_seqs, int num_heads, int num_kv_heads,
                                 int head_dim, int block_size, int max_blocks_per_seq,
                                 int64_t num_blocks, pa_dtype dt, void* workspace,
                                 size_t workspace_bytes, int32_t* d_status, pa_stream_t stream) {
  return decode_common(out, q, k_cache, v_cache, block_tables, context_lens, scale, num_seqs,
                       num_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                       num_blocks, dt, workspace, workspace_bytes, d_status, stream, nullptr,
                       nullptr, nullptr, true, k_scale, v_scale);
}

int pa_prefill(void* out, const void* q, const void* k, const void* v, void* k_cache,
               void* v_cache, const int64_t* slot_mapping, const int32_t* cu_seqlens,
               int num_seqs, int num_tokens, int max_seqlen, float scale, int num_heads,
               int num_kv_heads, int head_dim, int block_size, int64_t num_blocks, pa_dtype dt,
               int32_t* d_status, pa_stream_t stream) {
  if (num_seqs < 0 || num_seqs > 65535 || num_tokens < 0 || max_seqlen < 0 ||
      num_heads < 1 || num_heads > 65535 || num_kv_heads < 1 || num_heads % num_kv_heads ||
      (head_dim != 64 && head_dim != 128) || (dt != PA_F16 && dt != PA_BF16))
    return PA_ERR_INVALID;
  if (num_seqs == 0 || num_tokens == 0) return PA_OK;
  if (!out || !q || !k || !v || !cu_seqlens) return PA_ERR_INVALID;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k) || !aligned16(v)) return PA_ERR_INVALID;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool tc = g_prefill_kernel.load() != 1;
  if (k_cache) {  // store the prompts' keys and values in their blocks
    if (!v_cache || !slot_mapping || !shape_ok(num_kv_heads, head_dim, block_size) ||
        num_blocks <= 0 || !aligned16(k_cache) || !aligned16(v_cache))
      return PA_ERR_INVALID;
    // the tcgen05 kernel stores them itself, alongside the attention; the
    // warp-level kernel after a separate cache write
    if (!tc) {
      const int rc = from_cuda(pa::launch_kv_cache_write(k, v, k_cache, v_cache, slot_mapping,
                                                         num_tokens, num_kv_heads, head_dim,
                                                         block_size, num_blocks, d_status, st));
      if (rc != PA_OK) return rc;
    }
  }
  pa::PrefillArgs a;
  a.out = out;
  a.q = q;
  a.k = k;
  a.v = v;
  a.cu_seqlens = cu_seqlens;
  a.num_seqs = num_seqs;
  a.num_tokens = num_tokens;
  a.max_seqlen = max_seqlen;
  a.num_heads = num_heads;
  a.num_kv_heads = num_kv_heads;
  a.head_dim = head_dim;
  a.scale = scale;
  a.is_bf16 = dt == PA_BF16;
  a.status = d_status;
  a.wait_limit_ns = g_wait_limit_ns.load();
  if (tc && k_cache) {
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.block_size = block_size;
    a.num_blocks = num_blocks;
    a.slot_mapping = slot_mapping;
  }
  return from_cuda(tc ? pa::launch_prefill_tc(a, st) : pa::launch_prefill(a, st));
}

int pa_prefill_with_prefix(void* out, const void* q, const void* k, const void* v,
                           void* k_cache, void* v_cache, const int64_t* slot_mapping,
                           const int32_t* cu_seqlens, const int32_t* block_tables,
                           const int32_t* cached_lens, int num_seqs, int num_tokens,
                           int max_seqlen, int max_blocks_per_seq, float scale, int num_heads,
                           int num_kv_heads, int head_dim, int block_size, int64_t num_blocks,
                           pa_dtype dt, int32_t* d_status, pa_stream_t stream) {
  if (num_seqs < 0 || num_seqs > 65535 || num_tokens < 0 || max_seqlen < 0 ||
      max_blocks_per_seq < 1 || num_heads < 1 || num_heads > 65535 || num_kv_heads < 1 ||
      num_heads % num_kv_heads || (head_dim != 64 && head_dim != 128) ||
      (dt != PA_F16 && dt != PA_BF16) || g_prefill_kernel.load() == 1 ||
      !pa::prefill_tc_paged_ok(block_size, num_blocks))
    return PA_ERR_INVALID;
  if (num_seqs == 0 || num_tokens == 0) return PA_OK;
  if (!out || !q || !k || !v || !cu_seqlens || !k_cache || !v_cache || !block_tables ||
      !cached_lens)
    return PA_ERR_INVALID;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k) || !aligned16(v) ||
      !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_INVALID;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (slot_mapping && !shape_ok(num_kv_heads, head_dim, block_size)) return PA_ERR_INVALID;
  pa::PrefillArgs a;
  a.out = out;
  a.q = q;
  a.k = k;
  a.v = v;
  a.cu_seqlens = cu_seqlens;
  a.num_seqs = num_seqs;
  a.num_tokens = num_tokens;
  a.max_seqlen = max_seqlen;
  a.num_heads = num_heads;
  a.num_kv_heads = num_kv_heads;
  a.head_dim = head_dim;
  a.scale = scale;
  a.is_bf16 = dt == PA_BF16;
  a.status = d_status;
  a.wait_limit_ns = g_wait_limit_ns.load();
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.block_size = block_size;
  a.num_blocks = num_blocks;
  a.block_tables = block_tables;
  a.cached_lens = cached_lens;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.slot_mapping = slot_mapping;  // the kernel stores the new tokens' keys and values
  return from_cuda(pa::launch_prefill_tc(a, st));
}

int pa_read_probe(const void* buf, size_t bytes, uint32_t* d_sink, int sink_words,
                  pa_stream_t stream) {
  if (!buf || !d_sink || bytes == 0 || (bytes & 15u) || sink_words < 1 || !aligned16(buf))
    return PA_ERR_INVALID;
  return from_cuda(pa::launch_read_probe(buf, static_cast<int64_t>(bytes), d_sink, sink_words,
                                         reinterpret_cast<cudaStream_t>(stream)));
}

int pa_write_probe(void* buf, size_t bytes, pa_stream_t stream) {
  if (!buf || bytes == 0 || (bytes & 15u) || !aligned16(buf)) return PA_ERR_INVALID;
  return from_cuda(pa::launch_write_probe(buf, static_cast<int64_t>(bytes),
                                          reinterpret_cast<cudaStream_t>(stream)));
}

int pa_exp2_probe(const float* d_x, float* d_y, int64_t n, int method, pa_stream_t stream) {
  if (n < 0 || (method != 0 && method != 1) || (n > 0 && (!d_x || !d_y))) return PA_ERR_INVALID;
  return from_cuda(pa::launch_exp2_probe(d_x, d_y, n, method,
                                         reinterpret_cast<cudaStream_t>(stream)));
}

int pa_copy_blocks(const void* src_k, const void* src_v, int64_t src_num_blocks, void* dst_k,
                   void* dst_v, int64_t dst_num_blocks, const int32_t* block_pairs,
                   int num_pairs, int num_heads, int head_dim, int block_size, pa_dtype dt,
                   int32_t* d_status, pa_stream_t stream) {
  if (num_pairs < 0 || !shape_ok(num_heads, head_dim, block_size) || src_num_blocks <= 0 ||
      dst_num_blocks <= 0 || (dt != PA_F16 && dt != PA_BF16 && dt != PA_E4M3))
    return PA_ERR_INVALID;
  if (num_pairs == 0) return PA_OK;
  if (!src_k || !src_v || !dst_k || !dst_v || !block_pairs) return PA_ERR_INVALID;
  if (!aligned16(src_k) || !aligned16(src_v) || !aligned16(dst_k) || !aligned16(dst_v) ||
      (reinterpret_cast<uintptr_t>(block_pairs) & 3u) != 0)
    return PA_ERR_INVALID;
  if (!device_accessible(src_k) || !device_accessible(src_v) || !device_accessible(dst_k) ||
      !device_accessible(dst_v) || !device_accessible(block_pairs))
    return PA_ERR_INVALID;
  const int64_t block_bytes =
      static_cast<int64_t>(num_heads) * block_size * head_dim * (dt == PA_E4M3 ? 1 : 2);
  return from_cuda(pa::launch_copy_blocks(src_k, src_v, dst_k, dst_v, block_pairs, num_pairs,
                                          block_bytes, src_num_blocks, dst_num_blocks, d_status,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

int pa_paged_attn_decode_gqa(void* out, const void* q, const void* k_cache, const void* v_cache,
                             const int32_t* block_tables, const int32_t* context_lens,
                             float scale, int num_seqs, int num_heads, int num_kv_heads,
                             int head_dim, int block_size, int max_blocks_per_seq,
                             int64_t num_blocks, pa_dtype dt, void* workspace,
                             size_t workspace_bytes, int32_t* d_status, pa_stream_t stream) {
  return decode_common(out, q, k_cache, v_cache, block_tables, context_lens, scale, num_seqs,
                       num_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                       num_blocks, dt, workspace, workspace_bytes, d_status, stream, nullptr,
                       nullptr, nullptr);
}

int pa_decode_step(void* out, const void* q, const void* k, const void* v, void* k_cache,
                   void* v_cache, const int64_t* slot_mapping, const int32_t* block_tables,
                   const int32_t* context_lens, float scale, int num_seqs, int num_heads,
                   int head_dim, int block_size, int max_blocks_per_seq, int64_t num_blocks,
                   pa_dtype dt, void* workspace, size_t workspace_bytes, int32_t* d_status,
                   pa_stream_t stream) {
  if (num_seqs != 0 && !slot_mapping) return PA_ERR_INVALID;
  return decode_common(out, q, k_cache, v_cache, block_tables, context_lens, scale, num_seqs,
                       num_heads, num_heads, head_dim, block_size, max_blocks_per_seq, num_blocks,
                       dt, workspace, workspace_bytes, d_status, stream, k, v, slot_mapping);
}

int pa_decode_step_fp8(void* out, const void* q, const void* k, const void* v, void* k_cache,
                       void* v_cache, const int64_t* slot_mapping, const int32_t* block_tables,
                       const int32_t* context_lens, float scale, float k_scale, float v_scale,
                       int num_seqs, int num_heads, int head_dim, int block_size,
                       int max_blocks_per_seq, int64_t num_blocks, pa_dtype dt, void* workspace,
                       size_t workspace_bytes, int32_t* d_status, pa_stream_t stream) {
  if (num_seqs != 0 && !slot_mapping) return PA_ERR_INVALID;
  return decode_common(out, q, k_cache, v_cache, block_tables, context_lens, scale, num_seqs,
                       num_heads, num_heads, head_dim, block_size, max_blocks_per_seq, num_blocks,
                       dt, workspace, workspace_bytes, d_status, stream, k, v, slot_mapping, true,
                       k_scale, v_scale);
}

size_t pa_paged_attn_decode_shared_workspace_size(int num_groups, int group_size, int num_heads,
                                                  int head_dim, int block_size,
                                                  int max_prefix_blocks, int max_tail_blocks) {
  if (max_prefix_blocks < 1 || max_tail_blocks < 1) return 0;
  return pa::shared_prefix_workspace_bytes(num_groups, group_size, num_heads, num_heads,
                                           head_dim, block_size, max_prefix_blocks,
                                           max_tail_blocks, g_decode_warps.load());
}

size_t pa_paged_attn_decode_shared_gqa_workspace_size(int num_groups, int group_size,
                                                      int num_heads, int num_kv_heads,
                                                      int head_dim, int block_size,
                                                      int max_prefix_blocks, int max_tail_blocks) {
  if (max_prefix_blocks < 1 || max_tail_blocks < 1 || num_kv_heads < 1 ||
      num_heads % num_kv_heads)
    return 0;
  return pa::shared_prefix_workspace_bytes(num_groups, group_size, num_heads, num_kv_heads,
                                           head_dim, block_size, max_prefix_blocks,
                                           max_tail_blocks, g_decode_warps.load());
}

int pa_paged_attn_decode_shared(void* out, const void* q, const void* k_cache,
                                const void* v_cache, const int32_t* prefix_tables,
                                const int32_t* prefix_lens, int max_prefix_blocks,
                                const int32_t* tail_tables, const int32_t* tail_lens,
                                int max_tail_blocks, float scale, int num_groups, int group_size,
                                int num_heads, int head_dim, int block_size, int64_t num_blocks,
                                pa_dtype dt, void* workspace, size_t workspace_bytes,
                                int32_t* d_status, pa_stream_t stream) {
  return shared_common(out, q, k_cache, v_cache, prefix_tables, prefix_lens, max_prefix_blocks,
                       tail_tables, tail_lens, max_tail_blocks, scale, num_groups, group_size,
                       num_heads, num_heads, head_dim, block_size, num_blocks, dt, workspace,
                       workspace_bytes, d_status, stream);
}

int pa_paged_attn_decode_shared_gqa(void* out, const void* q, const void* k_cache,
                                    const void* v_cache, const int32_t* prefix_tables,
                                    const int32_t* prefix_lens, int max_prefix_blocks,
                                    const int32_t* tail_tables, const int32_t* tail_lens,
                                    int max_tail_blocks, float scale, int num_groups,
                                    int group_size, int num_heads, int num_kv_heads,
                                    int head_dim, int block_size, int64_t num_blocks, pa_dtype dt,
                                    void* workspace, size_t workspace_bytes, int32_t* d_status,
                                    pa_stream_t stream) {
  return shared_common(out, q, k_cache, v_cache, prefix_tables, prefix_lens, max_prefix_blocks,
                       tail_tables, tail_lens, max_tail_blocks, scale, num_groups, group_size,
                       num_heads, num_kv_heads, head_dim, block_size, num_blocks, dt, workspace,
                       workspace_bytes, d_status, stream);
}

}  // extern "C"
