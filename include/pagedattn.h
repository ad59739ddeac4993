/*
 * pagedattn.h — C ABI of libpagedattn.so: paged decode attention, the KV-cache
 * write, and a host-side block manager, for NVIDIA B200 (sm_100a).
 *
 * The method is PagedAttention as described in "The KV Cache and
 * PagedAttention" (sections "Like Pages of Memory", "The Block Table",
 * "Shared, Copied on Write") and "KV cache" ("How it works"): each text's keys
 * and values are cut into fixed-size blocks that may sit anywhere in a pool;
 * a per-text block table maps logical to physical blocks; in each generation
 * step the new token's key and value go to their slot and its query
 * attends over every stored key of its text, the new one included.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Every pointer to tensor data is a DEVICE pointer owned by the caller,
 *    except the block manager's arguments, which are HOST pointers.  The
 *    library never allocates or frees device memory; the only device memory
 *    it keeps is the static scratch of pa_paged_attn_decode_noalloc.
 *  - Tensors are dense and row-major ("contiguous").  Element types are
 *    IEEE fp16 or bfloat16 (pa_dtype), 2 bytes each.
 *  - Pool layout: k_cache and v_cache are each
 *        [num_blocks][num_heads][block_size][head_dim]
 *    so the keys of one (block, head) pair are one contiguous
 *    block_size*head_dim*2-byte tile.  Slot s is place s % block_size of
 *    physical block s / block_size.
 *  - Device calls are asynchronous on `stream` (NULL = the legacy default
 *    stream).  A non-zero return means nothing was launched, except
 *    PA_ERR_CUDA after a launch, which reports cudaGetLastError().
 *  - Data errors that only the GPU can see (a table entry outside the pool, a
 *    context length past the table, a slot past the pool, a wait that gave
 *    up) are recorded in *d_status, a caller-owned device int32 that should be
 *    zero before the call: the first error code seen is stored there (later
 *    ones do not overwrite it).  d_status may be NULL.  No call traps,
 *    asserts or aborts on bad data; offending reads and writes are skipped.
 *  - Support: head_dim in {64, 128}; block_size in {4, 8, 16, 32};
 *    num_seqs <= 4096; num_heads <= 1024.
 */
#ifndef PAGEDATTN_H
#define PAGEDATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;                       /* same type as cudaStream_t */
typedef struct CUstream_st* pa_stream_t;

/* Element types.  PA_E4M3 (8-bit cache codes) only where a call says so:
 * pa_copy_blocks's pools; the 8-bit entry points take their fp16/bf16
 * tensors' type as dt and the cache as raw codes. */
typedef enum { PA_F16 = 0, PA_BF16 = 1, PA_E4M3 = 2 } pa_dtype;

enum {
  PA_OK = 0,
  PA_ERR_INVALID = -1,        /* bad argument (null pointer, unsupported size, workspace too small) */
  PA_ERR_CUDA = -2,           /* a CUDA runtime call failed */
  PA_ERR_OUT_OF_BLOCKS = -3,  /* block manager: pool exhausted; state unchanged */
  PA_ERR_NO_SEQ = -4,         /* block manager: unknown sequence id */
  PA_ERR_EXISTS = -5,         /* block manager: sequence id already present */
  PA_ERR_TABLE_FULL = -6,     /* block manager: a table does not fit max_blocks_per_seq */
  PA_ERR_BAD_BLOCK = -7,      /* device: block table entry outside [0, num_blocks) */
  PA_ERR_BAD_LEN = -8,        /* device: context length < 0 or > max_blocks_per_seq*block_size */
  PA_ERR_BAD_SLOT = -9,       /* device: slot >= num_blocks*block_size */
  PA_ERR_TIMEOUT = -10,       /* device: a bounded wait on a shared-memory barrier gave up */
  PA_ERR_CORRUPT = -11,       /* block manager: internal counts inconsistent */
  PA_ERR_TOO_LARGE = -12      /* sizes need more scratch than pa_paged_attn_decode_noalloc holds */
};

/* Human-readable name of a status code.  Never NULL. */
const char* pa_status_string(int code);

/*
 * pa_kv_cache_write — store each new token's key and value in its slot.
 *
 * Definition: "KV cache", section "How it works" (each generated token's
 * key and value join the cache) and "The KV Cache and PagedAttention",
 * section "One Token at a Time" (a step computes keys and values for the new
 * token alone and keeps the older ones).  For t < num_tokens with slot_mapping[t]
 * >= 0:  k_cache[slot/B][h][slot%B][:] = k[t][h][:]  (and v likewise), for
 * every head h.  A pure copy: the stored bits equal the input bits.
 *
 *   k, v           [num_tokens][num_heads][head_dim]  dt, device, read
 *   k_cache,v_cache pool, layout above, device, written at the given slots only
 *   slot_mapping   [num_tokens] int64, device; a negative slot skips the token
 *   num_blocks     pool size in blocks (bounds check: slot < num_blocks*B,
 *                  else PA_ERR_BAD_SLOT in *d_status and the token is skipped)
 *   d_status       nullable device int32 (see conventions)
 * Two tokens with the same slot race; the pages never produce that.
 * num_tokens == 0 is a no-op.  Returns PA_OK or PA_ERR_INVALID / PA_ERR_CUDA.
 */
int pa_kv_cache_write(const void* k, const void* v, void* k_cache, void* v_cache,
                      const int64_t* slot_mapping, int num_tokens, int num_heads, int head_dim,
                      int block_size, int64_t num_blocks, pa_dtype dt, int32_t* d_status,
                      pa_stream_t stream);

/*
 * pa_paged_attn_decode_workspace_size — bytes of device scratch that
 * pa_paged_attn_decode needs for these sizes on the CURRENT device (it
 * depends on the device's SM count).  Host only; allocates nothing.
 * Returns 0 for unsupported sizes.
 */
size_t pa_paged_attn_decode_workspace_size(int num_seqs, int num_heads, int head_dim,
                                           int block_size, int max_blocks_per_seq);

/*
 * pa_paged_attn_decode — decode-phase attention through block tables.
 *
 * Definition: "KV cache", section "How it works": the new token's query is
 * scored against every key in the cache, its own among them, and the
 * resulting weights blend the cached values; "The KV Cache and
 * PagedAttention", section "The Block Table": the kernel looks up each
 * logical block's physical block in the table and reads its keys and values
 * from there.  For text s with L = context_lens[s] tokens
 * and every head h:
 *     z_t = scale * sum_d q[s][h][d] * K_t[d],   t < L,
 *     out[s][h][:] = sum_t softmax(z)_t * V_t[:],
 * where token t lives in physical block block_tables[s][t / B], place t % B.
 * Arithmetic: fp32 products and sums, online (running-max) softmax, result
 * rounded to dt (round to nearest even).  L == 0 gives zeros.
 *
 *   out            [num_seqs][num_heads][head_dim] dt, device, written
 *   q              [num_seqs][num_heads][head_dim] dt, device
 *   k_cache,v_cache pool (layout above), device; only rows t < L are read
 *   block_tables   [num_seqs][max_blocks_per_seq] int32, device; entries at or
 *                  past ceil(L/B) are ignored
 *   context_lens   [num_seqs] int32, device; counts the token written this
 *                  step (call pa_kv_cache_write first, same stream)
 *   scale          usually 1/sqrt(head_dim)
 *   num_blocks     pool size in blocks (bounds check of table entries)
 *   workspace      device scratch of at least
 *                  pa_paged_attn_decode_workspace_size(...) bytes, 256-byte
 *                  aligned; no initial contents needed (its grain counter is
 *                  tagged with a per-call epoch, and the call's last kernel
 *                  zeroes it, so a call replayed from a captured CUDA graph
 *                  starts clean too); must not be shared by calls that may
 *                  run at the same time
 *   d_status       nullable device int32 (see conventions)
 * Work is split over all SMs in 16-token (head_dim 128) or 32-token
 * (head_dim 64) chunks: static runs, then grains from a shared counter; a
 * (text, head) whose chunks span several work units is merged with a
 * log-sum-exp reduction by a second kernel on the same stream.  Both use
 * programmatic dependent launch.  For fixed inputs, sizes and device the
 * result is bitwise reproducible (which warp takes a grain does not change
 * how it is computed or merged).
 * Returns PA_OK or PA_ERR_INVALID / PA_ERR_CUDA.
 */
int pa_paged_attn_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                         const int32_t* block_tables, const int32_t* context_lens, float scale,
                         int num_seqs, int num_heads, int head_dim, int block_size,
                         int max_blocks_per_seq, int64_t num_blocks, pa_dtype dt,
                         void* workspace, size_t workspace_bytes, int32_t* d_status,
                         pa_stream_t stream);

/*
 * pa_decode_step — one whole decode step of one layer in one launch (plus the
 * merge): the cache write of pa_kv_cache_write for one new token per text,
 * then the attention of pa_paged_attn_decode.  A B200 fusion of the pages'
 * two steps ("KV cache", section "How it works": the new token's key and
 * value join the cache and take part in its own attention).
 *
 *   k, v           [num_seqs][num_heads][head_dim] dt: each text's new token
 *   slot_mapping   [num_seqs] int64: its slot (negative: not stored)
 *   other arguments as for pa_paged_attn_decode (same workspace size).
 *
 * Result: the pool afterwards and `out` are exactly those of
 * pa_kv_cache_write(k, v, ..., slot_mapping, num_tokens = num_seqs) followed
 * by pa_paged_attn_decode, provided slot_mapping[s] is the slot of position
 * context_lens[s] - 1 of text s (what the block manager's append_slot
 * returns) and no text reads another text's new slot (written blocks are
 * private after copy-on-write).  The attention takes position
 * context_lens[s] - 1 from k[s], v[s] directly, so the launch never waits on
 * its own write.  Returns PA_OK or PA_ERR_INVALID / PA_ERR_CUDA.
 */
int pa_decode_step(void* out, const void* q, const void* k, const void* v, void* k_cache,
                   void* v_cache, const int64_t* slot_mapping, const int32_t* block_tables,
                   const int32_t* context_lens, float scale, int num_seqs, int num_heads,
                   int head_dim, int block_size, int max_blocks_per_seq, int64_t num_blocks,
                   pa_dtype dt, void* workspace, size_t workspace_bytes, int32_t* d_status,
                   pa_stream_t stream);

/*
 * pa_decode_step_fp8 — pa_decode_step over 8-bit caches: the quantizing
 * write of pa_kv_cache_write_fp8 for one new token per text, then the
 * attention of pa_paged_attn_decode_fp8, in one launch (plus the merge)
 * ("The KV Cache and PagedAttention", section "What Came After": one byte a
 * number; "KV cache", section "How it works": the new token's key and value
 * join the cache and take part in its own attention).
 *
 *   k, v           [num_seqs][num_heads][head_dim] dt (fp16 or bf16): each
 *                  text's new token; stored as the codes of k / k_scale and
 *                  v / v_scale
 *   k_cache,v_cache 8-bit pools [num_blocks][num_heads][block_size][head_dim]
 *   k_scale, v_scale finite and > 0 (else PA_ERR_INVALID)
 *   other arguments as for pa_decode_step (workspace as for
 *                  pa_paged_attn_decode_fp8).  Multi-head only.
 *
 * Result: the pool afterwards and `out` are exactly those of
 * pa_kv_cache_write_fp8 followed by pa_paged_attn_decode_fp8 on the same
 * kernel, under the conditions of pa_decode_step.  The attention quantizes
 * position context_lens[s] - 1 from k[s], v[s] itself, with the write's
 * arithmetic, so the launch never waits on its own write.  With fp16
 * queries, head_dim 128 and blocks of 8, 16 or 32 it runs on the tensor-core
 * 8-bit kernel (PA_OPT_FP8_KERNEL picks the kernel), else on the CUDA cores.
 * Returns PA_OK or PA_ERR_INVALID / PA_ERR_CUDA.
 */
int pa_decode_step_fp8(void* out, const void* q, const void* k, const void* v, void* k_cache,
                       void* v_cache, const int64_t* slot_mapping, const int32_t* block_tables,
                       const int32_t* context_lens, float scale, float k_scale, float v_scale,
                       int num_seqs, int num_heads, int head_dim, int block_size,
                       int max_blocks_per_seq, int64_t num_blocks, pa_dtype dt, void* workspace,
                       size_t workspace_bytes, int32_t* d_status, pa_stream_t stream);

/*
 * pa_paged_attn_decode_shared_workspace_size — device scratch bytes that
 * pa_paged_attn_decode_shared needs for these sizes on the current device.
 * Host only.  Returns 0 for unsupported sizes.
 */
size_t pa_paged_attn_decode_shared_workspace_size(int num_groups, int group_size, int num_heads,
                                                  int head_dim, int block_size,
                                                  int max_prefix_blocks, int max_tail_blocks);

/*
 * pa_paged_attn_decode_shared — pa_paged_attn_decode for groups of texts that
 * share the leading blocks of one prompt ("The KV Cache and PagedAttention",
 * section "Shared, Copied on Write": the samples of one prompt point at the
 * same physical blocks).  Texts come in num_groups groups of group_size
 * consecutive texts (text t is in group t / group_size).  Text t attends over
 * its group's PREFIX (prefix_lens[g] tokens in the blocks of
 * prefix_tables[g]) followed by its own TAIL (tail_lens[t] tokens in the
 * blocks of tail_tables[t]):
 *     out[t][h][:] = sum over prefix and tail tokens of softmax(z) * V,
 * the same result as pa_paged_attn_decode over the joined table (up to
 * rounding).  Each shared key and value is read once per group, not once per
 * text: the group's queries run together on the tensor cores (a group of
 * more than 16 texts in subsets of at most 16, the smallest number of equal
 * subsets, each reading the prefix once), the tails on the multi-head
 * kernel, and a log-sum-exp merge joins the two.
 *
 *   out, q         [num_groups * group_size][num_heads][head_dim] dt, device
 *   k_cache,v_cache multi-head pool (layout above), device
 *   prefix_tables  [num_groups][max_prefix_blocks] int32, device
 *   prefix_lens    [num_groups] int32, device (0 allowed)
 *   tail_tables    [num_groups * group_size][max_tail_blocks] int32, device
 *   tail_lens      [num_groups * group_size] int32, device (0 allowed)
 *   group_size     1 .. 1024 (num_groups * group_size <= 4096); block_size
 *                  8, 16 or 32
 *   workspace      at least pa_paged_attn_decode_shared_workspace_size(...)
 *                  bytes, 256-byte aligned, not shared with concurrent calls
 * A text with no tokens at all gets zeros.  pa_split_shared_prefix builds the
 * four tables from ordinary block tables.  Data errors as for
 * pa_paged_attn_decode.  Bitwise reproducible for fixed inputs and device.
 * Returns PA_OK or PA_ERR_INVALID / PA_ERR_CUDA.
 */
int pa_paged_attn_decode_shared(void* out, const void* q, const void* k_cache,
                                const void* v_cache, const int32_t* prefix_tables,
                                const int32_t* prefix_lens, int max_prefix_blocks,
                                const int32_t* tail_tables, const int32_t* tail_lens,
                                int max_tail_blocks, float scale, int num_groups, int group_size,
                                int num_heads, int head_dim, int block_size, int64_t num_blocks,
                                pa_dtype dt, void* workspace, size_t workspace_bytes,
                                int32_t* d_status, pa_stream_t stream);

/*
 * pa_paged_attn_decode_shared_gqa_workspace_size — as
 * pa_paged_attn_decode_shared_workspace_size, for pools of num_kv_heads
 * key/value heads (num_heads a multiple of it; else 0).
 */
size_t pa_paged_attn_decode_shared_gqa_workspace_size(int num_groups, int group_size,
                                                      int num_heads, int num_kv_heads,
                                                      int head_dim, int block_size,
                                                      int max_prefix_blocks, int max_tail_blocks);

/*
 * pa_paged_attn_decode_shared_gqa — pa_paged_attn_decode_shared over a pool
 * of num_kv_heads key/value heads shared by num_heads query heads ("The KV
 * Cache and PagedAttention", section "What Came After": heads that share a
 * key/value set; section "Shared, Copied on Write": samples that share a
 * prompt's blocks): query head h reads key/value head
 * h / (num_heads / num_kv_heads).  The prefix pass takes, per key/value
 * head, the group's (text, query head) pairs as its tensor-core columns, in
 * subsets of at most 16, so each shared key and value is read once per
 * subset; the tails run on the grouped-query decode.
 *   k_cache,v_cache [num_blocks][num_kv_heads][block_size][head_dim] dt
 *   workspace      pa_paged_attn_decode_shared_gqa_workspace_size(...) bytes
 * Other arguments and errors as for pa_paged_attn_decode_shared.
 */
int pa_paged_attn_decode_shared_gqa(void* out, const void* q, const void* k_cache,
                                    const void* v_cache, const int32_t* prefix_tables,
                                    const int32_t* prefix_lens, int max_prefix_blocks,
                                    const int32_t* tail_tables, const int32_t* tail_lens,
                                    int max_tail_blocks, float scale, int num_groups,
                                    int group_size, int num_heads, int num_kv_heads,
                                    int head_dim, int block_size, int64_t num_blocks, pa_dtype dt,
                                    void* workspace, size_t workspace_bytes, int32_t* d_status,
                                    pa_stream_t stream);

/*
 * pa_split_shared_prefix — host only: cut ordinary block tables (as
 * pa_bm_export writes them) of num_seqs = groups * group_size texts into the
 * inputs of pa_paged_attn_decode_shared.  A group's prefix is its longest run
 * of leading table entries that all its texts hold at the same index and have
 * filled completely (at most max_prefix_blocks); each text's tail is the rest
 * of its table.  Unused entries are -1.  All pointers are HOST pointers.
 * PA_ERR_TABLE_FULL if a tail needs more than max_tail_blocks blocks,
 * PA_ERR_INVALID for bad sizes or a length outside the table; nothing is
 * written on error.
 */
int pa_split_shared_prefix(const int32_t* block_tables, const int32_t* context_lens, int num_seqs,
                           int max_blocks_per_seq, int block_size, int group_size,
                           int32_t* prefix_tables, int max_prefix_blocks, int32_t* prefix_lens,
                           int32_t* tail_tables, int max_tail_blocks, int32_t* tail_lens);

/*
 * pa_paged_attn_decode_gqa_workspace_size — as
 * pa_paged_attn_decode_workspace_size, for pa_paged_attn_decode_gqa with
 * num_kv_heads key/value heads.  Returns 0 for unsupported sizes (including
 * num_heads not a multiple of num_kv_heads).
 */
size_t pa_paged_attn_decode_gqa_workspace_size(int num_seqs, int num_heads, int num_kv_heads,
                                               int head_dim, int block_size,
                                               int max_blocks_per_seq);

/*
 * pa_paged_attn_decode_gqa — pa_paged_attn_decode for a pool holding fewer
 * key/value heads than there are query heads (grouped-query attention; one
 * key/value head is multi-query attention): "The KV Cache and
 * PagedAttention", section "What Came After" (groups of query heads use
 * common stored keys and values, so the cache is smaller).  With
 * G = num_heads / num_kv_heads, query head h reads key/value head h / G:
 *     z_t = scale * sum_d q[s][h][d] * K_t[h / G][d],
 *     out[s][h][:] = sum_t softmax(z)_t * V_t[h / G][:].
 *
 *   q, out         [num_seqs][num_heads][head_dim] dt, device
 *   k_cache,v_cache [num_blocks][num_kv_heads][block_size][head_dim] dt
 *   workspace      pa_paged_attn_decode_gqa_workspace_size(...) bytes
 *   other arguments, arithmetic, errors as for pa_paged_attn_decode.
 * num_kv_heads == num_heads is exactly pa_paged_attn_decode.  Each key/value
 * row is read from HBM once per (text, key/value head) and used by all the
 * query heads that share it (up to 16 per read; larger groups are split into
 * equal subsets that each read the rows).  The tensor-core kernel (see
 * PA_OPT_GQA_KERNEL) copies whole 16-token (32 at head_dim 64) runs of a
 * block, so rows past L in a text's last block are read and ignored; they
 * lie inside the pool, and their contents (NaN included) do not affect out.
 * num_heads must be a multiple of num_kv_heads (else PA_ERR_INVALID).
 */
int pa_paged_attn_decode_gqa(void* out, const void* q, const void* k_cache, const void* v_cache,
                             const int32_t* block_tables, const int32_t* context_lens,
                             float scale, int num_seqs, int num_heads, int num_kv_heads,
                             int head_dim, int block_size, int max_blocks_per_seq,
                             int64_t num_blocks, pa_dtype dt, void* workspace,
                             size_t workspace_bytes, int32_t* d_status, pa_stream_t stream);

/*
 * 8-bit KV cache ("The KV Cache and PagedAttention", section "What Came
 * After": one byte per cached number instead of two, so about twice the
 * tokens fit).  The pages fix no format; this library's reading:
 *  - each cached number is an E4M3 code (1 sign, 4 exponent bits with bias
 *    7, 3 mantissa bits; finite values only, largest 448; S.1111.111 is NaN);
 *  - one fp32 scale per cache tensor: code c of the key cache stands for
 *    value(c) * k_scale, of the value cache value(c) * v_scale;
 *  - the pools are laid out as the 16-bit ones, one byte per number:
 *    [num_blocks][num_heads][block_size][head_dim] uint8 codes.
 * Scales must be finite and positive (else PA_ERR_INVALID).
 */

/*
 * pa_kv_cache_write_fp8 — pa_kv_cache_write into 8-bit caches: element x of
 * k[t] (v[t]) is stored as the E4M3 code of the fp32 quotient x / k_scale
 * (x / v_scale), IEEE division, rounded to the nearest code with ties to the
 * even one, magnitudes past 448 saturating to +-448, NaN to NaN.
 *   k, v           [num_tokens][num_heads][head_dim] dt (fp16 or bf16)
 *   k_cache,v_cache 8-bit pools (above); other arguments and errors as for
 *                  pa_kv_cache_write.
 */
int pa_kv_cache_write_fp8(const void* k, const void* v, void* k_cache, void* v_cache,
                          const int64_t* slot_mapping, float k_scale, float v_scale,
                          int num_tokens, int num_heads, int head_dim, int block_size,
                          int64_t num_blocks, pa_dtype dt, int32_t* d_status, pa_stream_t stream);

/*
 * pa_paged_attn_decode_fp8 — pa_paged_attn_decode over 8-bit caches:
 *     z_t = scale * sum_d q[s][h][d] * value(K_t[d]) * k_scale,
 *     out[s][h][:] = sum_t softmax(z)_t * value(V_t[:]) * v_scale.
 * Codes are widened exactly; arithmetic as for pa_paged_attn_decode (fp32).
 *   q, out         [num_seqs][num_heads][head_dim] dt (fp16 or bf16)
 *   k_cache,v_cache 8-bit pools; the workspace is
 *                  pa_paged_attn_decode_workspace_size(...) bytes (the same
 *                  sizes as the 16-bit call).  Multi-head; grouped-query
 *                  pools go through pa_paged_attn_decode_fp8_gqa.  Other
 *                  arguments and errors as for pa_paged_attn_decode.
 * Each chunk of work is 4096/head_dim tokens (32 at head_dim 128), so every
 * copy still moves 4 KB of keys and 4 KB of values.  With fp16 queries,
 * head_dim 128 and blocks of 8, 16 or 32 the products run on the tensor
 * cores (PA_OPT_FP8_KERNEL picks the kernel): the codes are widened exactly
 * to fp16 and multiplied with fp32 accumulation.
 */
int pa_paged_attn_decode_fp8(void* out, const void* q, const void* k_cache, const void* v_cache,
                             const int32_t* block_tables, const int32_t* context_lens,
                             float scale, float k_scale, float v_scale, int num_seqs,
                             int num_heads, int head_dim, int block_size, int max_blocks_per_seq,
                             int64_t num_blocks, pa_dtype dt, void* workspace,
                             size_t workspace_bytes, int32_t* d_status, pa_stream_t stream);

/*
 * pa_paged_attn_decode_fp8_gqa — pa_paged_attn_decode_fp8 over 8-bit pools
 * of num_kv_heads heads shared by num_heads query heads ("The KV Cache and
 * PagedAttention", section "What Came After": heads that share a key/value
 * set, and one byte a number, side by side): query head h reads key/value
 * head h / (num_heads / num_kv_heads), with the formula of
 * pa_paged_attn_decode_fp8.
 *   k_cache,v_cache [num_blocks][num_kv_heads][block_size][head_dim] uint8
 *                  codes (written by pa_kv_cache_write_fp8 with num_heads =
 *                  num_kv_heads)
 *   workspace      pa_paged_attn_decode_gqa_workspace_size(...) bytes
 * With fp16 queries, head_dim 128 and blocks of 8, 16 or 32 it runs on the
 * tensor cores (PA_OPT_FP8_KERNEL picks the kernel): the query heads of a
 * key/value head are the columns of the product tile, up to 8 per pass
 * (larger groups in the fewest equal subsets of at most 8), so every code
 * read serves them all.  Otherwise it runs on the CUDA cores, each unit of
 * work carrying up to 4 query heads of one group (the largest of 4, 2, 1
 * that divides the group).  num_heads must be a multiple of num_kv_heads
 * (else PA_ERR_INVALID); other arguments and errors as for
 * pa_paged_attn_decode_fp8.
 */
int pa_paged_attn_decode_fp8_gqa(void* out, const void* q, const void* k_cache,
                                 const void* v_cache, const int32_t* block_tables,
                                 const int32_t* context_lens, float scale, float k_scale,
                                 float v_scale, int num_seqs, int num_heads, int num_kv_heads,
                                 int head_dim, int block_size, int max_blocks_per_seq,
                                 int64_t num_blocks, pa_dtype dt, void* workspace,
                                 size_t workspace_bytes, int32_t* d_status, pa_stream_t stream);

/*
 * pa_prefill — the prompt phase: every prompt's tokens attend causally over
 * the prompt's own keys and values, which are also stored in their blocks
 * ("The KV Cache and PagedAttention", section "One Token at a Time": the
 * prompt is processed all at once, and its keys and values are what later
 * steps reuse; "KV cache", section "How it works": position t attends over
 * positions 0..t).  Prompts are packed: prompt s is rows cu_seqlens[s] ..
 * cu_seqlens[s+1]-1 of q, k, v and out.  For prompt s, query head h and
 * position t (query head h reads key/value head h / (num_heads/num_kv_heads)):
 *     out[t][h] = sum_{u <= t in prompt s} softmax_u(scale * q[t][h] . k[u]) v[u].
 * Arithmetic: products on the tensor cores with fp32 sums, online softmax in
 * fp32; for bf16 the softmax weights enter the weighted sum of values as two
 * bf16 values (about 16 significant bits).  Every wait is bounded
 * (PA_OPT_WAIT_LIMIT_NS); one that gives up records PA_ERR_TIMEOUT.
 *
 *   out, q         [num_tokens][num_heads][head_dim] dt, device
 *   k, v           [num_tokens][num_kv_heads][head_dim] dt, device
 *   cu_seqlens     [num_seqs + 1] int32, device: 0 = cu[0] <= cu[1] <= ... <=
 *                  cu[num_seqs] = num_tokens (a prompt outside [0,
 *                  num_tokens] is skipped with PA_ERR_BAD_LEN in *d_status)
 *   max_seqlen     at least the longest prompt (a longer one is reported as
 *                  PA_ERR_BAD_LEN and its tail positions are not computed)
 *   k_cache, v_cache, slot_mapping, block_size, num_blocks
 *                  the pool and each token's slot, as for pa_kv_cache_write;
 *                  k_cache NULL skips the store (attention only)
 * On the tcgen05 kernel (the default) the store is done inside the
 * attention launch, by warps of its own that copy the prompts' key and
 * value rows to their slots while the others compute; on the warp-level
 * kernel a separate cache write runs first.  Either way the pool holds the
 * bits of pa_kv_cache_write afterwards (tokens of a prompt longer than
 * max_seqlen past max_seqlen are neither computed nor, on the tcgen05
 * kernel, stored).
 * Support: head_dim 64 or 128; num_seqs <= 65535.  Returns PA_OK or
 * PA_ERR_INVALID / PA_ERR_CUDA.
 */
int pa_prefill(void* out, const void* q, const void* k, const void* v, void* k_cache,
               void* v_cache, const int64_t* slot_mapping, const int32_t* cu_seqlens,
               int num_seqs, int num_tokens, int max_seqlen, float scale, int num_heads,
               int num_kv_heads, int head_dim, int block_size, int64_t num_blocks, pa_dtype dt,
               int32_t* d_status, pa_stream_t stream);

/*
 * pa_prefill_with_prefix — the prompt phase of prompts whose first tokens are
 * already in the cache ("The KV Cache and PagedAttention", section "What Came
 * After": a prompt that begins like an earlier one reuses the earlier one's
 * blocks, which saves the time spent on the prompt; pa_bm_add_seq_tokens
 * reports how many leading tokens were taken over).
 *
 * Prompt s has cached_lens[s] tokens stored in the pool, in the blocks
 * block_tables[s][0 .. cached_lens[s] / block_size - 1] (a multiple of
 * block_size); rows cu_seqlens[s] .. cu_seqlens[s+1]-1 of q, k, v and out are
 * its other tokens, at positions cached_lens[s] + i.  With K the stored keys
 * followed by the new ones (V likewise), row a + i is
 *     out[a+i][h] = sum_{u <= cached_lens[s] + i} softmax_u(scale * q[a+i][h] . K[u]) V[u],
 * which equals the rows of pa_prefill over the whole prompt that belong to
 * the new tokens (up to rounding).  The stored keys and values are read
 * through the table by the tensor-core kernel; nothing is recomputed for
 * them.  With slot_mapping non-NULL the new tokens' keys and values are
 * stored at their slots as pa_prefill does.
 *
 *   out, q, k, v   the new tokens only, as for pa_prefill
 *   k_cache, v_cache the pool (layout above), device; read through the
 *                  tables, written at slot_mapping
 *   slot_mapping   [num_tokens] int64, device, or NULL (no store)
 *   block_tables   [num_seqs][max_blocks_per_seq] int32, device
 *   cached_lens    [num_seqs] int32, device: 0 <= cached_lens[s] <=
 *                  max_blocks_per_seq * block_size, a multiple of block_size
 *                  (else PA_ERR_BAD_LEN in *d_status and prompt s is skipped);
 *                  a table entry outside [0, num_blocks) is PA_ERR_BAD_BLOCK
 *                  and its rows read as zeros
 * Support: the tcgen05 kernel only (PA_OPT_PREFILL_KERNEL 0 or 2), head_dim
 * 64 or 128, block_size 8, 16 or 32.  Returns PA_OK or PA_ERR_INVALID /
 * PA_ERR_CUDA.
 */
int pa_prefill_with_prefix(void* out, const void* q, const void* k, const void* v,
                           void* k_cache, void* v_cache, const int64_t* slot_mapping,
                           const int32_t* cu_seqlens, const int32_t* block_tables,
                           const int32_t* cached_lens, int num_seqs, int num_tokens,
                           int max_seqlen, int max_blocks_per_seq, float scale, int num_heads,
                           int num_kv_heads, int head_dim, int block_size, int64_t num_blocks,
                           pa_dtype dt, int32_t* d_status, pa_stream_t stream);

/*
 * pa_copy_blocks — copy whole blocks from one pool to another, or within one
 * pool: the device side of copy-on-write ("The KV Cache and
 * PagedAttention", section "Shared, Copied on Write": a text that must
 * change a block it shares first has that block duplicated into a free one,
 * then changes the duplicate, and the original's count falls by one;
 * pa_bm_append_slot returns the pair) and of moving blocks out of the pool
 * and back (section "When Memory Runs Out": blocks set aside in CPU memory).
 *
 *   src_k, src_v   [src_num_blocks][num_heads][block_size][head_dim] dt
 *                  (PA_F16, PA_BF16, or PA_E4M3 for 8-bit pools)
 *   dst_k, dst_v   [dst_num_blocks][num_heads][block_size][head_dim] dt; may
 *                  be src_k, src_v (copy-on-write)
 *   block_pairs    [num_pairs][2] int32: (source block, destination block)
 * For every pair, destination block dst of both pools receives source block
 * src: every head and place, bit for bit (a pure copy).  Every pair reads
 * the sources as they were before the call, so no block may be the
 * destination of two pairs, nor a destination and a source in one call (the
 * block manager's pairs never are); otherwise the result is unspecified.
 * Pools and block_pairs may be device memory of the current device, managed
 * memory, or pinned host memory mapped at the same address (e.g. a CPU
 * pool for blocks moved out); anything else is PA_ERR_INVALID, checked on the
 * host before launch.  A block id outside its pool is recorded as
 * PA_ERR_BAD_BLOCK in *d_status and that pair is skipped.  num_pairs == 0 is
 * a no-op.  Launched with programmatic dependent launch: it waits for the
 * kernel before it on the stream, and the next kernel waits for it.
 * Returns PA_OK or PA_ERR_INVALID / PA_ERR_CUDA.
 */
int pa_copy_blocks(const void* src_k, const void* src_v, int64_t src_num_blocks, void* dst_k,
                   void* dst_v, int64_t dst_num_blocks, const int32_t* block_pairs,
                   int num_pairs, int num_heads, int head_dim, int block_size, pa_dtype dt,
                   int32_t* d_status, pa_stream_t stream);

/*
 * pa_read_probe — a diagnostic with no counterpart in the pages: read `bytes`
 * (a multiple of 16) of device buffer `buf` once with a read-only streaming
 * kernel (a persistent grid, four 16-byte loads in flight per thread), to
 * measure the GPU's HBM read ceiling beside the decode kernels.  The loads
 * are folded with XOR into one word per CTA in d_sink (device, sink_words
 * words; 4 x the SM count is enough).  Returns PA_OK or PA_ERR_INVALID /
 * PA_ERR_CUDA.
 */
int pa_read_probe(const void* buf, size_t bytes, uint32_t* d_sink, int sink_words,
                  pa_stream_t stream);

/*
 * pa_write_probe — a diagnostic with no counterpart in the pages: write
 * `bytes` (a multiple of 16) of device buffer `buf` once with a write-only
 * streaming kernel (a persistent grid, four 16-byte streaming stores per
 * thread per round; the contents become an index pattern), to measure the
 * write ceiling that block copies (pa_copy_blocks) are compared with.
 * Returns PA_OK or PA_ERR_INVALID / PA_ERR_CUDA.
 */
int pa_write_probe(void* buf, size_t bytes, pa_stream_t stream);

/*
 * pa_exp2_probe — a diagnostic with no counterpart in the pages: d_y[i] =
 * 2^d_x[i] for i < n (device float arrays): method 0 an FMA-pipe polynomial
 * (range reduction to [-1/2, 1/2], degree-5 minimax polynomial, exponent
 * insertion; inputs below -125 give 2^-125), method 1 the exponential unit
 * (ex2.approx.ftz), which the softmax kernels use.  The polynomial was
 * built to take part of the prompt phase's exponentials and measured
 * slower there; this entry point lets a test hold it to its error bound on
 * the GPU itself.  Returns PA_OK or PA_ERR_INVALID /
 * PA_ERR_CUDA.
 */
int pa_exp2_probe(const float* d_x, float* d_y, int64_t n, int method, pa_stream_t stream);

/*
 * pa_paged_attn_decode_noalloc — pa_paged_attn_decode without a caller
 * workspace, for callers that cannot allocate device memory (a host framework
 * that owns every device allocation, a fixed memory budget, a loop where an
 * allocation and the device synchronisation it may bring are not allowed).
 * The pages have no counterpart: this is a deployment convenience.
 *
 * Same arguments, computation, result and errors as pa_paged_attn_decode,
 * minus workspace/workspace_bytes.  Its scratch is a static device array of
 * 16 MiB inside the library; every GPU that loads the library holds it until
 * the process exits.  Only the 16-bit kernels run here, so the limit applies
 * to what they need: sizes whose 16-bit scratch need exceeds 16 MiB are
 * rejected with PA_ERR_TOO_LARGE before anything is launched.  That need can
 * be below pa_paged_attn_decode_workspace_size, which also covers the 8-bit
 * kernels: 256 texts x 40 heads x 128 (blocks of 16, 128 per text) on a
 * 148-SM B200 needs less than 16 MiB here but more from that query.  The
 * call allocates and frees nothing.
 *
 * The first call on each device looks up the array's device address (a host
 * runtime call, cudaGetSymbolAddress); make that first call before any
 * stream capture.  The address is kept per device and context: after a
 * device reset (cudaDeviceReset), the first call in the new context looks it
 * up again.  All calls share the one array and leave their contents in
 * it (nothing in it needs to start at zero): calls that may overlap on the
 * GPU, on any streams, race and must be serialised by the caller.
 */
int pa_paged_attn_decode_noalloc(void* out, const void* q, const void* k_cache,
                                 const void* v_cache, const int32_t* block_tables,
                                 const int32_t* context_lens, float scale, int num_seqs,
                                 int num_heads, int head_dim, int block_size,
                                 int max_blocks_per_seq, int64_t num_blocks, pa_dtype dt,
                                 int32_t* d_status, pa_stream_t stream);

/*
 * Tuning and test options (process-wide, not thread-safe; set before use).
 *   PA_OPT_WAIT_LIMIT_NS  bound on each shared-memory barrier wait in the
 *                         decode kernel, in ns (default 1e9).  A negative
 *                         value makes every wait give up at once, which
 *                         exercises the PA_ERR_TIMEOUT path: the kernel then
 *                         drains its copies in flight (bounded by 1 s) and
 *                         returns with *d_status = PA_ERR_TIMEOUT.
 *   PA_OPT_DECODE_WARPS   number of working warps of the decode kernel
 *                         (0 = all SMs, the default).  1 gives a single-pass
 *                         run in which no text is split.
 *   PA_OPT_GQA_KERNEL     which kernel pa_paged_attn_decode_gqa runs when
 *                         num_heads > num_kv_heads: 0 (default) the
 *                         tensor-core kernel where it applies (block_size 8,
 *                         16 or 32 and num_blocks * num_kv_heads * block_size
 *                         < 2^31), else the CUDA-core one; 1 always the
 *                         CUDA-core kernel; 2 always the tensor-core kernel
 *                         (PA_ERR_INVALID where it does not apply).  Both
 *                         compute the same function with fp32 sums; the
 *                         tensor-core kernel carries the softmax weights into
 *                         the weighted sum of values as the sum of two dt
 *                         values (about 16 significant bits).
 *   PA_OPT_PREFILL_KERNEL which kernel pa_prefill runs: 0 (default) or 2 the
 *                         5th-generation tensor cores (tcgen05, accumulators
 *                         in tensor memory, 128 queries per CTA); 1 the
 *                         warp-level tensor cores (mma.sync).  Same function.
 *   PA_OPT_FP8_KERNEL     which kernel pa_paged_attn_decode_fp8 runs: 0
 *                         (default) the tensor-core kernel where it applies
 *                         (fp16 queries, head_dim 128, block_size 8, 16 or
 *                         32, num_blocks * num_heads * block_size < 2^31),
 *                         else the CUDA-core one; 1 always the CUDA-core
 *                         kernel; 2 always the tensor-core kernel
 *                         (PA_ERR_INVALID where it does not apply).  Both
 *                         widen the codes exactly and sum in fp32; the
 *                         tensor-core kernel carries the softmax weights into
 *                         the weighted sum of values as the sum of two fp16
 *                         values.
 *   PA_OPT_PREFIX_KEY_BITS bits of the chained prefix hash that block
 *                         managers created after the call use as their
 *                         lookup key, 1..64 (default 64).  Fewer bits make
 *                         different prefixes share keys; a test uses that to
 *                         exercise the checks that keep such prefixes from
 *                         sharing blocks.
 * Returns PA_OK or PA_ERR_INVALID for an unknown key or value.
 */
enum { PA_OPT_WAIT_LIMIT_NS = 1, PA_OPT_DECODE_WARPS = 2, PA_OPT_GQA_KERNEL = 3,
       PA_OPT_PREFILL_KERNEL = 4, PA_OPT_PREFIX_KEY_BITS = 5, PA_OPT_FP8_KERNEL = 6 };
int pa_set_option(int key, int64_t value);

/* ------------------------------------------------------------------------ */
/* Host block manager ("The KV Cache and PagedAttention", sections "The     */
/* Block Table", "Shared, Copied on Write", "When Memory Runs Out").  Pure  */
/* host code; all pointers are host pointers; not thread-safe per handle.   */
/* ------------------------------------------------------------------------ */
typedef struct pa_bm pa_bm;

/* A pool of num_blocks blocks of block_size tokens.  The free list starts in
 * block order (shuffle_seed == 0) or in a seeded random order; blocks are
 * taken from its front and returned to its back.  NULL on bad arguments. */
pa_bm* pa_bm_create(int64_t num_blocks, int block_size, uint64_t shuffle_seed);
void pa_bm_destroy(pa_bm* bm);

/* New text whose first num_tokens tokens (the prompt) are stored at once:
 * ceil(num_tokens / B) fresh blocks.  All or nothing. */
int pa_bm_add_seq(pa_bm* bm, int64_t seq_id, int num_tokens);

/* child shares every block of parent; each block's count rises by one. */
int pa_bm_fork(pa_bm* bm, int64_t parent, int64_t child);

/* Room for the text's next token.  A fresh block is taken only when the last
 * block is full (blocks are allocated one at a time, as earlier ones fill).  If the
 * last block is partial and shared, it is copied first: *cow_src and *cow_dst
 * receive the pair (the caller copies the block's rows on the device before
 * writing), the original's count drops by one; otherwise both are -1.
 * *slot receives the token's slot.  All or nothing. */
int pa_bm_append_slot(pa_bm* bm, int64_t seq_id, int64_t* slot, int32_t* cow_src,
                      int32_t* cow_dst);

/* The text is done: each block's count drops by one; blocks that reach zero
 * return to the free list, in table order. */
int pa_bm_free_seq(pa_bm* bm, int64_t seq_id);

int64_t pa_bm_num_free(const pa_bm* bm);
/* Reference count of a block, or PA_ERR_INVALID for an id outside the pool. */
int pa_bm_refcount(const pa_bm* bm, int32_t block);
/* Tokens stored for the text, or a negative status. */
int64_t pa_bm_num_tokens(const pa_bm* bm, int64_t seq_id);

/* Writes block_tables[n][max_blocks_per_seq] (int32, -1 past each text's last
 * block) and context_lens[n] (token counts) into caller host buffers, in the
 * order of seq_ids.  PA_ERR_TABLE_FULL if a table is longer than
 * max_blocks_per_seq; nothing is written on error. */
int pa_bm_export(const pa_bm* bm, const int64_t* seq_ids, int n, int32_t* block_tables,
                 int max_blocks_per_seq, int32_t* context_lens);

/* Prefix reuse ("The KV Cache and PagedAttention", section "What Came After":
 * each full block is identified by a hash of its tokens chained with the
 * hash of all tokens before it; a text that begins like an earlier one takes
 * over the earlier text's blocks).
 *
 * pa_bm_add_seq_tokens adds a text from its prompt's token ids (host array of
 * num_tokens int32).  It walks the prompt's full blocks in order and takes
 * over cached blocks with the same chained hash up to the first miss (each
 * count rises by one; a cached block waiting in the free list leaves it).
 * The rest are fresh blocks from the front of the free list, as in
 * pa_bm_add_seq.  The new full blocks are then cached; a partial last block
 * never is.  *num_cached_tokens (nullable) receives the number of leading
 * tokens whose blocks were taken over (a multiple of block_size): their keys
 * and values are already in the pool.  The caller stores the rest (a
 * negative slot skips the first tokens in pa_kv_cache_write and pa_prefill).
 *
 * A cached block whose count falls to zero stays cached while it waits in
 * the free list.  When the free list hands it out again it is evicted: its
 * hash is dropped.  Blocks added by pa_bm_add_seq or filled by appends are
 * not cached.  The chained hash is a 64-bit SplitMix64-style mix, used as
 * the lookup key.  A key match alone is not a hit: the cached block's own
 * token ids must equal the prompt's, and a second 64-bit hash of the whole
 * prefix (FNV-1a over the token ids' bytes), kept per cached block, must
 * match too.  Two different prefixes could share a block only if both
 * 64-bit hashes collided while the last block's ids agree.  A key already
 * held by a block whose check fails stays with that block; the new block
 * is then not cached.  All or nothing.
 * pa_bm_num_cached_blocks counts the hashes currently held. */
int pa_bm_add_seq_tokens(pa_bm* bm, int64_t seq_id, const int32_t* tokens, int num_tokens,
                         int* num_cached_tokens);
int64_t pa_bm_num_cached_blocks(const pa_bm* bm);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDATTN_H */
