// Internal launcher declarations shared by the C-ABI layer and the kernels.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace pa {

// The 8-bit cache's write: codes of k / k_scale and v / v_scale (E4M3, round
// to nearest even, saturating); k, v are fp16 (bf16 if `bf16`).
cudaError_t launch_kv_cache_write_fp8(const void* k, const void* v, void* k_cache, void* v_cache,
                                      const int64_t* slot_mapping, float k_scale, float v_scale,
                                      int num_tokens, int num_heads, int head_dim, int block_size,
                                      int64_t num_blocks, bool bf16, int32_t* status,
                                      cudaStream_t stream);

// A tiled TMA map of a 16-bit (fp16 or bf16) tensor of `rank` dimensions
// (innermost first; strides in bytes of dimensions 1..rank-1), boxes of
// `box` elements, 128-byte swizzle, zero fill out of bounds.  False if the
// CUDA driver's encoder refuses it.
bool encode_swizzled_map(CUtensorMap* map, const void* base, bool bf16, int rank,
                         const uint64_t* dims, const uint64_t* strides_bytes,
                         const uint32_t* box);
// The same for any element type the driver names (one-byte codes among them).
bool encode_tiled_map(CUtensorMap* map, const void* base, CUtensorMapDataType type, int rank,
                      const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box);
// The same without swizzle: a box lands in shared memory as a plain
// row-major array (inner box of at most 256 elements).
bool encode_plain_map(CUtensorMap* map, const void* base, CUtensorMapDataType type, int rank,
                      const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box);

cudaError_t launch_kv_cache_write(const void* k, const void* v, void* k_cache, void* v_cache,
                                  const int64_t* slot_mapping, int num_tokens, int num_heads,
                                  int head_dim, int block_size, int64_t num_blocks,
                                  int32_t* status, cudaStream_t stream);

// Whole-block copies: for each (src, dst) in pairs[num_pairs][2], block dst of
// the destination K and V pools receives block src of the source pools
// (block_bytes each).  Ids outside their pool: PA_ERR_BAD_BLOCK, skipped.
cudaError_t launch_copy_blocks(const void* src_k, const void* src_v, void* dst_k, void* dst_v,
                               const int32_t* pairs, int num_pairs, int64_t block_bytes,
                               int64_t src_num_blocks, int64_t dst_num_blocks, int32_t* status,
                               cudaStream_t stream);

// Prompt phase: causal attention within each packed prompt (prefill.cu).
struct PrefillArgs {
  void* out;
  const void* q;
  const void* k;
  const void* v;
  const int32_t* cu_seqlens;
  int num_seqs;
  int num_tokens;
  int max_seqlen;
  int num_heads;
  int num_kv_heads;
  int head_dim;
  float scale;
  int is_bf16;
  int32_t* status;
  int64_t wait_limit_ns = 1000000000;
  // tcgen05 kernel only.  The paged cache: with cached_lens, prompt s's first
  // cached_lens[s] tokens are read from it through block_tables (q, k, v and
  // out then hold the other tokens); with slot_mapping, the new tokens' keys
  // and values are stored in it by the kernel itself.
  void* k_cache = nullptr;
  void* v_cache = nullptr;
  int block_size = 0;
  int64_t num_blocks = 0;
  const int32_t* block_tables = nullptr;
  const int32_t* cached_lens = nullptr;
  int max_blocks_per_seq = 0;
  const int64_t* slot_mapping = nullptr;
};
// Warp-level tensor cores (mma.sync, prefill.cu) and 5th-generation tensor
// cores (tcgen05 with TMEM accumulators, prefill_tc.cu).
cudaError_t launch_prefill(const PrefillArgs& a, cudaStream_t stream);
cudaError_t launch_prefill_tc(const PrefillArgs& a, cudaStream_t stream);
// Block sizes and pool sizes for which the tcgen05 kernel reads and writes
// the paged cache itself.
bool prefill_tc_paged_ok(int block_size, int64_t num_blocks);
// Current PA_OPT_PREFILL_KERNEL setting (0 automatic = tcgen05, 1 mma.sync, 2 tcgen05).
int64_t option_prefill_kernel();

// Read-only streaming probe: reads `bytes` (a multiple of 16) of `buf` once;
// one word per CTA lands in sink[0 .. sink_words).
cudaError_t launch_read_probe(const void* buf, int64_t bytes, uint32_t* sink, int sink_words,
                              cudaStream_t stream);
// Write-only streaming probe: writes `bytes` (a multiple of 16) of `buf`.
cudaError_t launch_write_probe(void* buf, int64_t bytes, cudaStream_t stream);
// y = 2^x elementwise: method 0 the FMA-pipe polynomial of the softmax
// kernels (exp2poly.cuh), 1 the exponential unit (ex2.approx).
cudaError_t launch_exp2_probe(const float* x, float* y, int64_t n, int method,
                              cudaStream_t stream);

struct DecodeArgs {
  void* out;
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_tables;
  const int32_t* context_lens;
  float scale;
  int num_seqs;
  int num_heads;     // query heads
  int num_kv_heads;  // key/value heads of the pool (== num_heads: multi-head)
  int head_dim;
  int block_size;
  int max_blocks_per_seq;
  int64_t num_blocks;
  int is_bf16;
  void* workspace;
  size_t workspace_bytes;
  int32_t* status;
  int64_t wait_limit_ns;
  int64_t forced_warps;  // 0 = fill the device
  // 8-bit (E4M3) cache with per-tensor scales (pa_paged_attn_decode_fp8).
  bool fp8 = false;
  float k_scale = 1.f;
  float v_scale = 1.f;
  // Fused decode step (pa_decode_step) only; all null otherwise.
  const void* k_new = nullptr;
  const void* v_new = nullptr;
  const int64_t* slot_mapping = nullptr;
  // One pass of the shared-prefix decode: partial records only, no merge
  // (and, on the grouped-query kernel, queries taken from a group's texts).
  bool cascade = false;
  // With cascade: the kernel launched just before this one (on the same
  // stream, also a cascade pass) triggers its dependents early and writes
  // nothing this pass reads; this pass then waits for it only at its exit.
  bool cascade_overlap = false;
};

bool decode_sizes_supported(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                            int block_size, int max_blocks_per_seq);

// Size of the decode workspace for these sizes on the current device, or 0
// if the sizes are unsupported: the most any decode kernel these sizes may
// run needs (without the 8-bit kernel when with_fp8 is false).
size_t decode_workspace_bytes(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                              int block_size, int max_blocks_per_seq, int64_t forced_warps,
                              bool with_fp8 = true);

// Current PA_OPT_DECODE_WARPS setting.
int64_t option_decode_warps();
// Current PA_OPT_GQA_KERNEL setting (0 automatic, 1 CUDA cores, 2 tensor cores).
int64_t option_gqa_kernel();
// Current PA_OPT_FP8_KERNEL setting (0 automatic, 1 CUDA cores, 2 tensor cores).
int64_t option_fp8_kernel();

// Tensor-core decode over an 8-bit cache (paged_attn_decode_mma_fp8.cu):
// fp16 queries, head_dim 128, multi-head or grouped-query pools, blocks of
// 8, 16 or 32, a pool that fits 32-bit TMA row coordinates.
bool mma_fp8_decode_ok(const DecodeArgs& a);
size_t mma_fp8_workspace_bytes(int num_seqs, int num_heads, int num_kv_heads, int block_size,
                               int max_blocks_per_seq, int64_t forced_warps);
cudaError_t launch_paged_attn_decode_mma_fp8(const DecodeArgs& a, cudaStream_t stream);

// Tensor-core grouped-query decode (paged_attn_decode_mma.cu): whether the
// head layout and block size suit it, whether the pool fits its 32-bit TMA
// row coordinates, its workspace size, and the launch.
bool mma_decode_shape_ok(int num_heads, int num_kv_heads, int head_dim, int block_size);
bool mma_decode_pool_ok(int num_kv_heads, int block_size, int64_t num_blocks);
size_t mma_decode_workspace_bytes(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                  int block_size, int max_blocks_per_seq, int64_t forced_warps);
cudaError_t launch_paged_attn_decode_mma(const DecodeArgs& a, cudaStream_t stream);

// A decode launch's split of query heads: per key/value head nsub work
// subsets of gs query heads (or, in the shared-prefix pass, of gs
// (text, query head) columns), vheads virtual heads in all.  Records of a
// unit hold gs columns.
struct DecodeLayout {
  int nsub;
  int gs;
  int vheads;
};
DecodeLayout mma_decode_layout(int num_heads, int num_kv_heads);
DecodeLayout mma_fp8_layout(int num_heads, int num_kv_heads);
DecodeLayout mma_cascade_layout(int num_heads, int num_kv_heads, int group_size);
// The layout launch_paged_attn_decode uses for these arguments.
DecodeLayout decode_layout(const DecodeArgs& a);

// The shared-prefix pass of the grouped-query kernel (a.cascade set):
// a.num_seqs groups of `group_size` texts; the columns of a key/value head
// are the group's (text, query head) pairs.  Partial records only, no
// merge.
bool mma_cascade_ok(int num_heads, int num_kv_heads, int group_size, int head_dim,
                    int block_size);
size_t mma_cascade_workspace_bytes(int num_groups, int group_size, int num_heads,
                                   int num_kv_heads, int head_dim, int block_size,
                                   int max_blocks_per_seq, int64_t forced_warps);
cudaError_t launch_paged_attn_decode_mma_cascade(const DecodeArgs& a, int group_size,
                                                 cudaStream_t stream);

// Shared-prefix decode (shared_prefix.cu): the prefix pass, the tail pass,
// then the merge of both passes' records.
struct SharedPrefixArgs {
  void* out;
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* prefix_tables;
  const int32_t* prefix_lens;
  int max_prefix_blocks;
  const int32_t* tail_tables;
  const int32_t* tail_lens;
  int max_tail_blocks;
  float scale;
  int num_groups;
  int group_size;
  int num_heads;
  int num_kv_heads;
  int head_dim;
  int block_size;
  int64_t num_blocks;
  int is_bf16;
  void* workspace;
  size_t workspace_bytes;
  int32_t* status;
  int64_t wait_limit_ns;
  int64_t forced_warps;
};
size_t shared_prefix_workspace_bytes(int num_groups, int group_size, int num_heads,
                                     int num_kv_heads, int head_dim, int block_size,
                                     int max_prefix_blocks, int max_tail_blocks,
                                     int64_t forced_warps);
cudaError_t launch_paged_attn_decode_shared(const SharedPrefixArgs& a, cudaStream_t stream);

// Launches the decode kernel and the split reduce on `stream`.
// Returns cudaErrorInvalidValue for unsupported sizes or a short workspace.
cudaError_t launch_paged_attn_decode(const DecodeArgs& a, cudaStream_t stream);

}  // namespace pa
