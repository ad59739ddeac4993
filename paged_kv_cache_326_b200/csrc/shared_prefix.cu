// Decode attention for groups of texts that share the blocks of one prompt
// ("The KV Cache and PagedAttention", section "Shared, Copied on Write":
// several samples of one prompt point at the same physical blocks until one
// of them writes).  Each text's tokens are the group's shared PREFIX followed
// by its own TAIL; attention over their union is computed in two passes whose
// partial results are merged:
//
//   prefix pass  the grouped-query (tensor-core) kernel, one virtual text per
//                group: the group's texts' queries for head h are the columns
//                of one tile, so each shared key and value is read from HBM
//                once for the whole group instead of once per text;
//   tail pass    the multi-head (CUDA-core) kernel over each text's private
//                blocks;
//   merge        for text t and head h, the partial records (m, l, o) of both
//                passes combine as
//                    out = sum_i 2^(m_i - M) o_i / sum_i 2^(m_i - M) l_i,
//                    M = max_i m_i,
//                which is the softmax over prefix and tail together (up to
//                rounding: the log-sum-exp merge is exact algebra).
//
// Both passes run with their `cascade` flag set: every work unit leaves a
// record, none writes an output, so the merge sees every partial.  The prefix
// pass triggers its dependents as soon as its inputs are ready, so the tail
// pass (which reads nothing the prefix pass writes) fills SMs as prefix CTAs
// finish; the tail pass waits for the prefix grid on its way out, so the
// merge, which waits for the tail grid, sees both passes' records.
#include <cuda_runtime.h>

#include <cstdint>

#include "decode_common.cuh"
#include "kernels.h"

namespace pa {

namespace {

// Units u_lo .. u_lo + n - 1 of one launch that cover (text s, head h), from
// that launch's header (work split, then the chunk prefix over texts).
__device__ __forceinline__ void unit_range(const int32_t* header, int s, int h, int H, int& u_lo,
                                           int& n) {
  const int32_t* prefix = header + kHeaderInts;
  const int seg0 = prefix[s];
  const int ns = (prefix[s + 1] - seg0) / H;
  if (ns == 0) {
    u_lo = 0;
    n = 0;
    return;
  }
  WorkSplit sp;
  sp.total = header[0];
  sp.q = header[1];
  sp.grain = header[2];
  sp.W = header[3];
  sp.dyn_base = sp.W * sp.q;
  const int a = seg0 + h * ns;
  u_lo = sp.unit_of(a);
  n = sp.unit_of(a + ns - 1) - u_lo + 1;
}

// One warp per (text t, query head h): the prefix pass's records for
// column c = j G + h % G of key/value head h / G of group t / gs (text j of
// the group, G query heads per key/value head; the prefix pass ran the
// columns in subsets of gs_p as virtual heads kvh * nsub_p + c / gs_p), then
// the tail pass's records for text t and query head h (column h % G % gs_t
// of virtual head kvh * nsub_t + (h % G) / gs_t), merged in that fixed order
// (so the result does not depend on which warp produced a record).  Every
// lane reads the same records, so the running maximum is warp-uniform.
template <typename T, int D>
__global__ void __launch_bounds__(256)
shared_prefix_merge_kernel(T* __restrict__ out, const int32_t* __restrict__ hdr_p,
                           const float* __restrict__ rec_p, const int32_t* __restrict__ hdr_t,
                           const float* __restrict__ rec_t, unsigned long long* __restrict__ grab_p,
                           unsigned long long* __restrict__ grab_t, int num_groups, int gs, int H,
                           int G, DecodeLayout lp, DecodeLayout lt) {
  griddep_wait();
  // Both passes are done with their grain counters: zero them for the next call
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    *grab_p = 0ull;
    *grab_t = 0ull;
  }
  constexpr int PER = D / 32;
  constexpr int RS = D + 4;  // floats per record
  const int lane = threadIdx.x & 31;
  const int item = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int S = num_groups * gs;
  if (item >= S * H) return;
  const int t = item / H;
  const int h = item - t * H;
  const int g = t / gs;
  const int j = t - g * gs;
  const int kvh = h / G, qq = h - kvh * G;
  const int c = j * G + qq;                      // column in the prefix pass
  const int vh_p = kvh * lp.nsub + c / lp.gs, col_p = c % lp.gs;
  const int vh_t = kvh * lt.nsub + qq / lt.gs, col_t = qq % lt.gs;
  int pu, pn, tu, tn;
  unit_range(hdr_p, g, vh_p, lp.vheads, pu, pn);
  unit_range(hdr_t, t, vh_t, lt.vheads, tu, tn);
  const int64_t seg_p = static_cast<int64_t>(g) * lp.vheads + vh_p;
  const int64_t seg_t = static_cast<int64_t>(t) * lt.vheads + vh_t;
  const int n = pn + tn;
  auto rec = [&](int i) -> const float* {
    return i < pn ? rec_p + ((pu + i + seg_p) * lp.gs + col_p) * RS
                  : rec_t + ((tu + (i - pn) + seg_t) * lt.gs + col_t) * RS;
  };

  // One pass over the records, four loads in flight at a time; the running
  // maximum rises batch by batch (a single batch in the usual case: a prefix
  // and a tail each covered by one or two units).
  float M = -INFINITY;
  float L = 0.f;
  float acc[PER];
#pragma unroll
  for (int k = 0; k < PER; ++k) acc[k] = 0.f;
  for (int i0 = 0; i0 < n; i0 += 4) {
    float mv[4], lv[4], o[4][PER];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float* r = rec(min(i0 + u, n - 1));
      mv[u] = __ldcg(r);
      lv[u] = __ldcg(r + 1);
      if constexpr (PER == 4) {
        const float4 v = __ldcg(reinterpret_cast<const float4*>(r + 4 + lane * PER));
        o[u][0] = v.x;
        o[u][1] = v.y;
        o[u][2] = v.z;
        o[u][3] = v.w;
      } else {
        const float2 v = __ldcg(reinterpret_cast<const float2*>(r + 4 + lane * PER));
        o[u][0] = v.x;
        o[u][1] = v.y;
      }
    }
    float Mb = M;
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (i0 + u < n) Mb = fmaxf(Mb, mv[u]);
    if (Mb != M) {  // rescale what is summed so far (nothing, in the first batch)
      const float a = M == -INFINITY ? 0.f : fast_exp2(M - Mb);
      L *= a;
#pragma unroll
      for (int k = 0; k < PER; ++k) acc[k] *= a;
      M = Mb;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (i0 + u < n) {
        // a record of skipped (bad) blocks only carries m = -inf: weight 0
        const float f = mv[u] == -INFINITY ? 0.f : fast_exp2(mv[u] - M);
        L = fmaf(f, lv[u], L);
#pragma unroll
        for (int k = 0; k < PER; ++k) acc[k] = fmaf(f, o[u][k], acc[k]);
      }
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  T* orow = out + (static_cast<int64_t>(t) * H + h) * D + lane * PER;
  if constexpr (PER == 4) {
    uint2 v;
    v.x = Elem<T>::from_float2(acc[0] * inv, acc[1] * inv);
    v.y = Elem<T>::from_float2(acc[2] * inv, acc[3] * inv);
    *reinterpret_cast<uint2*>(orow) = v;
  } else {
    *reinterpret_cast<uint32_t*>(orow) = Elem<T>::from_float2(acc[0] * inv, acc[1] * inv);
  }
}

template <typename T, int D>
cudaError_t launch_shared_merge(const SharedPrefixArgs& a, const char* ws_p, int S_p,
                                const char* ws_t, int S_t, DecodeLayout lt,
                                cudaStream_t stream) {
  const int64_t items = static_cast<int64_t>(a.num_groups) * a.group_size * a.num_heads;
  const int per_cta = 8;  // warps, one per (text, head)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((items + per_cta - 1) / per_cta));
  cfg.blockDim = dim3(per_cta * 32);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(
      &cfg, shared_prefix_merge_kernel<T, D>, static_cast<T*>(a.out),
      reinterpret_cast<const int32_t*>(ws_p),
      reinterpret_cast<const float*>(ws_p + header_bytes(S_p) + kGrabBytes),
      reinterpret_cast<const int32_t*>(ws_t),
      reinterpret_cast<const float*>(ws_t + header_bytes(S_t) + kGrabBytes),
      reinterpret_cast<unsigned long long*>(const_cast<char*>(ws_p) + header_bytes(S_p)),
      reinterpret_cast<unsigned long long*>(const_cast<char*>(ws_t) + header_bytes(S_t)),
      a.num_groups, a.group_size, a.num_heads, a.num_heads / a.num_kv_heads,
      mma_cascade_layout(a.num_heads, a.num_kv_heads, a.group_size), lt);
}

// The two passes' workspaces, one after the other (256-byte aligned).
size_t prefix_part_bytes(int num_groups, int group_size, int num_heads, int num_kv_heads,
                         int head_dim, int block_size, int max_prefix_blocks,
                         int64_t forced_warps) {
  return align_up(mma_cascade_workspace_bytes(num_groups, group_size, num_heads, num_kv_heads,
                                              head_dim,
                                              block_size, max_prefix_blocks, forced_warps),
                  256);
}

DecodeArgs pass_args(const SharedPrefixArgs& a) {
  DecodeArgs d;
  d.out = a.out;
  d.q = a.q;
  d.k_cache = a.k_cache;
  d.v_cache = a.v_cache;
  d.scale = a.scale;
  d.num_heads = a.num_heads;
  d.num_kv_heads = a.num_kv_heads;
  d.head_dim = a.head_dim;
  d.block_size = a.block_size;
  d.num_blocks = a.num_blocks;
  d.is_bf16 = a.is_bf16;
  d.status = a.status;
  d.wait_limit_ns = a.wait_limit_ns;
  d.forced_warps = a.forced_warps;
  d.cascade = true;
  return d;
}

}  // namespace

size_t shared_prefix_workspace_bytes(int num_groups, int group_size, int num_heads,
                                     int num_kv_heads, int head_dim, int block_size,
                                     int max_prefix_blocks, int max_tail_blocks,
                                     int64_t forced_warps) {
  if (num_groups < 1 || group_size < 1 ||
      static_cast<int64_t>(num_groups) * group_size > kMaxSeqs)
    return 0;
  const size_t p = prefix_part_bytes(num_groups, group_size, num_heads, num_kv_heads, head_dim,
                                     block_size, max_prefix_blocks, forced_warps);
  const size_t t = decode_workspace_bytes(num_groups * group_size, num_heads, num_kv_heads,
                                          head_dim, block_size, max_tail_blocks, forced_warps);
  if (p == 0 || t == 0) return 0;
  return p + t;
}

cudaError_t launch_paged_attn_decode_shared(const SharedPrefixArgs& a, cudaStream_t stream) {
  const int S = a.num_groups * a.group_size;
  const size_t p_bytes = prefix_part_bytes(a.num_groups, a.group_size, a.num_heads,
                                           a.num_kv_heads, a.head_dim, a.block_size,
                                           a.max_prefix_blocks, a.forced_warps);
  const size_t t_bytes = decode_workspace_bytes(S, a.num_heads, a.num_kv_heads, a.head_dim,
                                                a.block_size, a.max_tail_blocks, a.forced_warps);
  if (p_bytes == 0 || t_bytes == 0 || a.workspace_bytes < p_bytes + t_bytes)
    return cudaErrorInvalidValue;
  char* ws_p = static_cast<char*>(a.workspace);
  char* ws_t = ws_p + p_bytes;

  DecodeArgs pp = pass_args(a);  // prefix pass: one virtual text per group
  pp.block_tables = a.prefix_tables;
  pp.context_lens = a.prefix_lens;
  pp.num_seqs = a.num_groups;
  pp.max_blocks_per_seq = a.max_prefix_blocks;
  pp.workspace = ws_p;
  pp.workspace_bytes = p_bytes;
  cudaError_t err = launch_paged_attn_decode_mma_cascade(pp, a.group_size, stream);
  if (err != cudaSuccess) return err;

  DecodeArgs tp = pass_args(a);  // tail pass: every text's own blocks
  tp.block_tables = a.tail_tables;
  tp.context_lens = a.tail_lens;
  tp.num_seqs = S;
  tp.max_blocks_per_seq = a.max_tail_blocks;
  tp.workspace = ws_t;
  tp.workspace_bytes = t_bytes;
  tp.cascade_overlap = true;
  err = launch_paged_attn_decode(tp, stream);
  if (err != cudaSuccess) return err;

  const DecodeLayout lt = decode_layout(tp);  // the tail pass's split of query heads
  if (a.head_dim == 128)
    err = a.is_bf16
              ? launch_shared_merge<__nv_bfloat16, 128>(a, ws_p, a.num_groups, ws_t, S, lt, stream)
              : launch_shared_merge<__half, 128>(a, ws_p, a.num_groups, ws_t, S, lt, stream);
  else
    err = a.is_bf16
              ? launch_shared_merge<__nv_bfloat16, 64>(a, ws_p, a.num_groups, ws_t, S, lt, stream)
              : launch_shared_merge<__half, 64>(a, ws_p, a.num_groups, ws_t, S, lt, stream);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace pa
