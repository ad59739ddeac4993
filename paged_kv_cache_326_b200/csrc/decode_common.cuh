// Pieces shared by the decode kernels (CUDA-core and tensor-core): launch
// parameters, the work split and its scheduler, the prologue, the cache write
// of the one-launch step, the log-sum-exp merge kernel, and the host-side
// launch planning.
//
// Work is laid out as one flat order of CHUNKS (CH consecutive tokens of one
// (text, virtual head)): text-major, then head, then chunk.  Each working
// warp first streams a static run of that order, then takes GRAINS of the
// rest from a shared counter (warps given equal bytes finish up to a third
// apart on B200, since SMs do not get equal shares of HBM bandwidth).  Runs
// and grains are the work UNITS; a (text, head) split across units yields one
// partial result per unit, merged by split_reduce_kernel.
#pragma once
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <map>
#include <mutex>
#include <tuple>
#include <utility>

#include "dtype.cuh"
#include "fp8.cuh"
#include "ptx.cuh"

namespace pa {

constexpr int kMaxSeqs = 4096;
constexpr int kDrainLimitNs = 1000000000;

#ifndef PA_STATIC_PERMILLE
#define PA_STATIC_PERMILLE 700
#endif
#ifndef PA_MIN_GRAIN
#define PA_MIN_GRAIN 16
#endif
// Each warp's static run is about kStaticPermille per mille of an even share;
// the rest goes out in grains of at least kMinGrain chunks, about
// kGrainsPerWarp per warp.  (Longer static runs, 850 or 930 per mille, or
// grains of at least 32 chunks measured slower on the batch-64 multi-head
// step and on the grouped-query steps, 16- and 8-bit: fewer partials to
// merge, but a longer tail of warps finishing late.)
constexpr int kStaticPermille = PA_STATIC_PERMILLE;
constexpr int kGrainsPerWarp = 12;
constexpr int kMinGrain = PA_MIN_GRAIN;

__host__ __device__ constexpr int chunk_tokens(int D) { return 2048 / D; }

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Workspace: a header (the work split, then prefix[S+1]), the grain counter,
// then the partial records (GS heads x (m, l, pad, pad, o[D]) fp32 per unit
// and (text, virtual head)).  CTA 0 of the decode kernel writes the header;
// the merge kernel reads it.
constexpr int kHeaderInts = 8;  // total, q, grain, W, 4 spare
inline size_t header_bytes(int num_seqs) {
  return align_up(sizeof(int32_t) * (kHeaderInts + num_seqs + 1), 256);
}
constexpr size_t kGrabBytes = 256;
// The grain counter holds the call's epoch in bits 30-63 and the chunks
// handed out below them.  A stale epoch (an earlier call's, or never set)
// reads as zero, so the workspace never needs clearing before a call; the
// merge kernel also resets the counter to zero once the decode grid is done,
// so a call replayed with the same epoch (a captured CUDA graph) starts from
// zero too.
constexpr unsigned long long kGrabMask = (1ull << 30) - 1;
constexpr unsigned long long kEpochMask = (1ull << 34) - 1;

// Units a launch with `warps` working warps can create (static runs plus at
// most kGrainsPerWarp grains per warp).
inline int64_t max_units(int64_t warps) { return warps * (kGrainsPerWarp + 1) + 1; }
inline size_t records_bytes(int64_t records, int D, int gs) {
  return static_cast<size_t>(records) * gs * (D + 4) * sizeof(float);
}

struct DecodeParams {
  void* out;
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_tables;
  const int32_t* context_lens;
  float qk_scale_log2;  // scale * log2(e) (* the keys' scale for an 8-bit cache)
  float v_scale;        // the values' scale for an 8-bit cache, else 1
  float k_scale;        // the keys' scale for an 8-bit cache, else 1
  int num_seqs;
  int num_heads;      // virtual heads: key/value heads x subsets (the flat order's heads)
  int num_q_heads;    // query heads of q and out
  int num_kv_heads;   // key/value heads of the pool
  int nsub;           // subsets per key/value head
  int gs;             // query heads per subset
  int max_blocks_per_seq;
  int64_t num_blocks;
  int num_work_warps;
  const void* k_new;              // one-launch step only: the new token's k, v
  const void* v_new;
  const int64_t* slot_mapping;    // one-launch step only: their slots
  int32_t* header;                // work split + prefix, for the merge kernel
  unsigned long long* grab;       // grain counter
  unsigned long long epoch;       // 34-bit, never 0
  float* records;
  int32_t* status;
  int64_t wait_limit_ns;
  // Shared-prefix (cascade) passes: every unit leaves a partial record, even
  // for a (text, head) it covers whole, and no output is written (a third
  // kernel merges the records of both passes).  In the grouped-query kernel
  // the gs query heads of virtual text s and head h are then the same head h
  // of texts s * gs .. s * gs + gs - 1 (q laid out [texts][heads][D]).
  // 2: as 1, for a pass whose predecessor on the stream is the other pass
  // (it waits for that grid at its exit instead of its start).
  int cascade = 0;
};

// The work split of one launch; every CTA computes the same one.
struct WorkSplit {
  int total = 0;     // chunks in the flat order
  int W = 1;         // working warps
  int q = 0;         // static run of each warp (units 0..W-1)
  int dyn_base = 0;  // first chunk handed out in grains (units W, W+1, ...)
  int dyn = 0;       // chunks handed out in grains
  int grain = 1;     // chunks per grain

  __host__ __device__ int unit_of(int c) const {
    return c < dyn_base ? c / q : W + (c - dyn_base) / grain;
  }
};

__device__ __forceinline__ WorkSplit make_split(int total, int W) {
  WorkSplit sp;
  sp.total = total;
  sp.W = W;
  int q = W == 1 ? total
                 : static_cast<int>(static_cast<long long>(total) * kStaticPermille / 1000 / W);
  if (q < 32 && W > 1) q = 0;
  sp.q = q;
  sp.dyn_base = W * q;
  sp.dyn = total - sp.dyn_base;
  sp.grain = max(kMinGrain, (sp.dyn + kGrainsPerWarp * W - 1) / (kGrainsPerWarp * W));
  return sp;
}

// Prologue, run by every thread of the CTA: prefix[s] = H * (chunks of the
// texts before s) in shared memory (block-wide scan of the context lengths,
// clamped to the table with PA_ERR_BAD_LEN), the header (CTA 0), and zeros
// for the outputs of texts with no tokens (spread over the CTAs).
template <typename T, int D, int CH, int NTHREADS>
__device__ __forceinline__ WorkSplit decode_prologue(const DecodeParams& p, int32_t* prefix, int32_t* warp_tot,
                                     int cap) {
  const int S = p.num_seqs, H = p.num_heads;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (S + NTHREADS - 1) / NTHREADS;
  const int s0 = min(S, tid * per), s1 = min(S, s0 + per);
  int local = 0;
  for (int s = s0; s < s1; ++s) {
    int L = __ldg(p.context_lens + s);
    if (L < 0 || L > cap) {
      if (blockIdx.x == 0) set_status(p.status, -8 /* PA_ERR_BAD_LEN */);
      L = min(max(L, 0), cap);
    }
    local += (L + CH - 1) / CH;
  }
  int incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  int before = 0;
  for (int w = 0; w < warp; ++w) before += warp_tot[w];
  int run = before + incl - local;
  for (int s = s0; s < s1; ++s) {
    const int L = min(max(__ldg(p.context_lens + s), 0), cap);
    prefix[s] = run * H;
    run += (L + CH - 1) / CH;
  }
  if (tid == NTHREADS - 1) prefix[S] = run * H;
  __syncthreads();

  const WorkSplit sp = make_split(prefix[S], p.num_work_warps);
  if (blockIdx.x == 0) {
    if (tid == 0) {
      p.header[0] = sp.total;
      p.header[1] = sp.q;
      p.header[2] = sp.grain;
      p.header[3] = sp.W;
    }
    for (int i = tid; i <= S; i += NTHREADS) p.header[kHeaderInts + i] = prefix[i];
  }
  const int Hq = p.num_q_heads;
  for (int s = p.cascade ? S : blockIdx.x; s < S; s += gridDim.x) {
    if (prefix[s + 1] == prefix[s]) {
      uint4* o = reinterpret_cast<uint4*>(static_cast<T*>(p.out) + static_cast<int64_t>(s) * Hq * D);
      for (int i = tid; i < Hq * D / 8; i += NTHREADS) o[i] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  return sp;
}

// Per-lane look-ahead entry: where one chunk of a window lives.
template <int NB>
struct Lookahead {
  int s, h, j, len;  // len is the raw context length (clamped at use)
  int blk[NB];
};

// One warp's view of the work: its units (static run, then grains) cut into
// windows of at most 32 chunks, and the per-lane look-ahead of a window.  A
// unit's last two windows are balanced, so only the very last window of all
// the work can be shorter than a copy ring.
template <int CH, int B, int NB>
struct Scheduler {
  // copies of the launch parameters it needs (kept by value so no reference
  // to the kernel's parameter space is taken)
  unsigned long long* grab;
  const int32_t* context_lens;
  const int32_t* block_tables;
  int S, H, max_blocks;
  const int32_t* prefix;
  WorkSplit sp;
  int w, lane, step;
  unsigned long long e34;
  bool static_taken = false, exhausted = false, pend_live = false;
  unsigned long long pend = 0;  // lane 0: counter value of the next grain
  int u_start = 0, u_count = 0, u_id = -1, u_off = 0;

  __device__ __forceinline__ Scheduler(const DecodeParams& p, const int32_t* prefix_,
                                       const WorkSplit& sp_, int w_, int lane_)
      : grab(p.grab), context_lens(p.context_lens), block_tables(p.block_tables),
        S(p.num_seqs), H(p.num_heads), max_blocks(p.max_blocks_per_seq), prefix(prefix_),
        sp(sp_), w(w_), lane(lane_) {
    step = 1;
    while (step * 2 <= S) step *= 2;
    e34 = p.epoch & kEpochMask;
  }

  // Chunk offset of the grain whose counter value is `old` (lane 0).  A
  // stale epoch is replaced by compare-and-swap.
  __device__ __forceinline__ int grab_resolve(unsigned long long old) {
    const unsigned long long g = static_cast<unsigned long long>(sp.grain);
    if ((old >> 30) == e34) return static_cast<int>(old & kGrabMask);
    unsigned long long seen = old + g;
    while (true) {
      if ((seen >> 30) == e34) {
        const unsigned long long o2 = atomicAdd(grab, g);
        if ((o2 >> 30) == e34) return static_cast<int>(o2 & kGrabMask);
        seen = o2 + g;
        continue;
      }
      const unsigned long long prev = atomicCAS(grab, seen, (e34 << 30) | g);
      if (prev == seen) return 0;
      seen = prev;
    }
  }

  __device__ __forceinline__ void grab_issue() {
    if (lane == 0) pend = atomicAdd(grab, static_cast<unsigned long long>(sp.grain));
    pend_live = true;
  }

  __device__ __forceinline__ void next_unit() {
    if (!static_taken) {
      static_taken = true;
      if (sp.q > 0) {
        u_start = w * sp.q;
        u_count = sp.q;
        u_id = w;
        u_off = 0;
        if (sp.dyn > 0) grab_issue();
        return;
      }
    }
    if (sp.dyn <= 0) {
      exhausted = true;
      return;
    }
    if (!pend_live) grab_issue();
    int off = 0;
    if (lane == 0) off = grab_resolve(pend);
    off = __shfl_sync(0xffffffffu, off, 0);
    pend_live = false;
    if (off >= sp.dyn) {
      exhausted = true;
      return;
    }
    u_start = sp.dyn_base + off;
    u_count = min(sp.grain, sp.dyn - off);
    u_id = sp.W + off / sp.grain;
    u_off = 0;
    grab_issue();  // the next grain, resolved when this one runs out
  }

  // Next window of this warp's work: start chunk, count (0 = no more), unit.
  __device__ __forceinline__ void next_window(int& ws, int& wc, int& wu) {
    if (!exhausted && u_off >= u_count) next_unit();
    if (exhausted) {
      ws = 0;
      wc = 0;
      wu = -1;
      return;
    }
    const int rem = u_count - u_off;
    const int n = rem <= 32 ? rem : (rem < 64 ? rem / 2 : 32);
    ws = u_start + u_off;
    wc = n;
    wu = u_id;
    u_off += n;
  }

  // Where each chunk of a window lives, one chunk per lane.  Reads only
  // shared memory before issuing its global loads, whose results are not
  // used until the copy issue reaches this window.
  __device__ __forceinline__ Lookahead<NB> lookahead(int ws, int wc) const {
    Lookahead<NB> e;
    if (wc <= 0) {
      e.s = e.h = e.j = e.len = 0;
#pragma unroll
      for (int k = 0; k < NB; ++k) e.blk[k] = -1;
      return e;
    }
    const int c = ws + min(lane, wc - 1);
    int s = 0;
    for (int st = step; st > 0; st >>= 1)
      if (s + st < S && prefix[s + st] <= c) s += st;
    const int seg0 = prefix[s];
    const int ns = (prefix[s + 1] - seg0) / H;
    const int within = c - seg0;
    const int h = within / ns;
    const int j = within - h * ns;
    e.s = s;
    e.h = h;
    e.j = j;
    e.len = __ldg(context_lens + s);
    const int32_t* row = block_tables + static_cast<int64_t>(s) * max_blocks;
#pragma unroll
    for (int k = 0; k < NB; ++k) {
      const int idx = (j * CH) / B + k;
      e.blk[k] = idx < max_blocks ? __ldg(row + idx) : -1;
    }
    return e;
  }
};

// The one-launch step's cache write: 16-byte vectors of the new k, v
// ([S][Hkv][D]) spread over the working warps (warp w of W), stored at their
// slots.  No read in the same launch touches these slots.
template <int D, int B>
__device__ __forceinline__ void fused_cache_write(const DecodeParams& p, int w, int W, int lane) {
  const int Hkv = p.num_kv_heads;
  const int vpr = D / 8;
  const int64_t per_text = static_cast<int64_t>(Hkv) * vpr;
  const int64_t nvec = per_text * p.num_seqs;
  const int64_t num_slots = p.num_blocks * B;
  uint4* kcw = static_cast<uint4*>(const_cast<void*>(p.k_cache));
  uint4* vcw = static_cast<uint4*>(const_cast<void*>(p.v_cache));
  for (int64_t i = static_cast<int64_t>(w) * 32 + lane; i < nvec; i += static_cast<int64_t>(W) * 32) {
    const int64_t s = i / per_text;
    const int64_t r = i - s * per_text;
    const int64_t slot = __ldg(p.slot_mapping + s);
    if (slot < 0) continue;
    if (slot >= num_slots) {
      if (r == 0) set_status(p.status, -9 /* PA_ERR_BAD_SLOT */);
      continue;
    }
    const int64_t h = r / vpr, c = r - (r / vpr) * vpr;
    const int64_t blk = slot / B, place = slot - blk * B;
    const int64_t dst = ((blk * Hkv + h) * B + place) * vpr + c;
    kcw[dst] = __ldg(static_cast<const uint4*>(p.k_new) + i);
    vcw[dst] = __ldg(static_cast<const uint4*>(p.v_new) + i);
  }
}

// fused_cache_write for an 8-bit cache: each lane takes 8 numbers of a new
// row and stores their codes (e4m3x8_quantize with the keys' or the values'
// scale, as the 8-bit cache write does).
template <typename T, int D, int B>
__device__ __forceinline__ void fused_cache_write_f8(const DecodeParams& p, int w, int W,
                                                     int lane) {
  const int Hkv = p.num_kv_heads;
  const int vpr = D / 8;
  const int64_t per_text = static_cast<int64_t>(Hkv) * vpr;
  const int64_t nvec = per_text * p.num_seqs;
  const int64_t num_slots = p.num_blocks * B;
  uint2* kcw = static_cast<uint2*>(const_cast<void*>(p.k_cache));
  uint2* vcw = static_cast<uint2*>(const_cast<void*>(p.v_cache));
  for (int64_t i = static_cast<int64_t>(w) * 32 + lane; i < nvec; i += static_cast<int64_t>(W) * 32) {
    const int64_t s = i / per_text;
    const int64_t r = i - s * per_text;
    const int64_t slot = __ldg(p.slot_mapping + s);
    if (slot < 0) continue;
    if (slot >= num_slots) {
      if (r == 0) set_status(p.status, -9 /* PA_ERR_BAD_SLOT */);
      continue;
    }
    const int64_t h = r / vpr, c = r - (r / vpr) * vpr;
    const int64_t blk = slot / B, place = slot - blk * B;
    const int64_t dst = ((blk * Hkv + h) * B + place) * vpr + c;
    float x[8];
    unpack8<T>(__ldg(static_cast<const uint4*>(p.k_new) + i), x);
    kcw[dst] = e4m3x8_quantize(x, p.k_scale);
    unpack8<T>(__ldg(static_cast<const uint4*>(p.v_new) + i), x);
    vcw[dst] = e4m3x8_quantize(x, p.v_scale);
  }
}

// Merge the partials of one (text, head) from units w_lo..w_hi (records
// `rec_stride` floats apart): with M = max_i m_i and f_i = 2^(m_i - M),
//     out = (sum_i f_i o_i) / (sum_i f_i l_i),
// which equals the softmax-weighted sum over all the text's tokens (up to
// rounding).  Partials are read in unit order, so the result does not depend
// on which warp produced them.
template <typename T, int D>
__device__ __forceinline__ void merge_partials(const float* records, int64_t rec_stride,
                                               T* out_row, int64_t sh, int w_lo, int w_hi,
                                               int lane) {
  constexpr int PER = D / 32;
  const int n = w_hi - w_lo + 1;
  // running max over the partials, one partial per lane
  float M = -INFINITY;
  for (int i = lane; i < n; i += 32) M = fmaxf(M, __ldcg(records + (w_lo + i + sh) * rec_stride));
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  float L = 0.f;
  float acc[PER];
#pragma unroll
  for (int k = 0; k < PER; ++k) acc[k] = 0.f;
  for (int i0 = 0; i0 < n; i0 += 32) {
    // weight f_i = 2^(m_i - M) of partial i0 + lane, and its share of the sum
    float f = 0.f, lf = 0.f;
    if (i0 + lane < n) {
      const float* rec = records + (w_lo + i0 + lane + sh) * rec_stride;
      f = M == -INFINITY ? 0.f : fast_exp2(__ldcg(rec) - M);
      lf = f * __ldcg(rec + 1);
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) lf += __shfl_xor_sync(0xffffffffu, lf, off);
    L += lf;
    // outputs: eight partials' loads in flight at a time
    const int cnt = min(32, n - i0);
    for (int b = 0; b < cnt; b += 8) {
      float o[8][PER];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float* rec =
            records + (w_lo + i0 + min(b + u, cnt - 1) + sh) * rec_stride + 4 + lane * PER;
        if constexpr (PER == 4) {
          const float4 v = __ldcg(reinterpret_cast<const float4*>(rec));
          o[u][0] = v.x;
          o[u][1] = v.y;
          o[u][2] = v.z;
          o[u][3] = v.w;
        } else {
          const float2 v = __ldcg(reinterpret_cast<const float2*>(rec));
          o[u][0] = v.x;
          o[u][1] = v.y;
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float fu = __shfl_sync(0xffffffffu, f, min(b + u, 31));
        if (b + u < cnt) {
#pragma unroll
          for (int k = 0; k < PER; ++k) acc[k] = fmaf(fu, o[u][k], acc[k]);
        }
      }
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  T* o = out_row + lane * PER;
  if constexpr (PER == 4) {
    uint2 v;
    v.x = Elem<T>::from_float2(acc[0] * inv, acc[1] * inv);
    v.y = Elem<T>::from_float2(acc[2] * inv, acc[3] * inv);
    *reinterpret_cast<uint2*>(o) = v;
  } else {
    *reinterpret_cast<uint32_t*>(o) = Elem<T>::from_float2(acc[0] * inv, acc[1] * inv);
  }
}

// Merge kernel: for every (text, virtual head) whose chunks fell into several
// work units, combine the units' partials (log-sum-exp) for each of its gs
// query heads; the decode kernel has already written every other output.
// Launched right after the decode kernel with programmatic dependent launch:
// its CTAs become resident early and griddepcontrol.wait holds them until the
// decode kernel's writes are visible.  One warp per (text, virtual head,
// query head of the subset).
template <typename T, int D>
__global__ void __launch_bounds__(256)
split_reduce_kernel(T* __restrict__ out, const int32_t* __restrict__ header,
                    const float* __restrict__ records, unsigned long long* __restrict__ grab,
                    int num_seqs, int num_vheads, int num_q_heads, int nsub, int gs) {
  griddep_wait();
  // The decode grid is done with its grain counter: zero it for the next call
  if (blockIdx.x == 0 && threadIdx.x == 0) *grab = 0ull;
  const int lane = threadIdx.x & 31;
  const int item = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (item >= num_seqs * num_vheads * gs) return;
  const int seg = item / gs;
  const int g = item - seg * gs;
  const int s = seg / num_vheads;
  const int vh = seg - s * num_vheads;
  WorkSplit sp;
  sp.total = header[0];
  sp.q = header[1];
  sp.grain = header[2];
  sp.W = header[3];
  sp.dyn_base = sp.W * sp.q;
  const int32_t* prefix = header + kHeaderInts;
  const int seg0 = prefix[s];
  const int ns = (prefix[s + 1] - seg0) / num_vheads;
  if (ns == 0) return;  // zero-filled by the decode kernel
  const int a = seg0 + vh * ns;
  const int u_lo = sp.unit_of(a);
  const int u_hi = sp.unit_of(a + ns - 1);
  if (u_lo == u_hi) return;  // finished in place by the decode kernel
  const int group = num_q_heads / (num_vheads / nsub);  // query heads per key/value head
  const int qh = (vh / nsub) * group + (vh % nsub) * gs + g;
  merge_partials<T, D>(records + g * (D + 4), static_cast<int64_t>(gs) * (D + 4),
                       out + (static_cast<int64_t>(s) * num_q_heads + qh) * D, seg, u_lo, u_hi,
                       lane);
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

inline int device_sm_count() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return sms;
}

// A fresh 34-bit epoch per launch (never 0, so a zeroed workspace holds no
// live counts).
inline unsigned long long next_epoch() {
  static std::atomic<unsigned long long> counter{0};
  unsigned long long e;
  do {
    e = (counter.fetch_add(1) + 1) & kEpochMask;
  } while (e == 0);
  return e;
}

// Resident CTAs per SM of `kernel` with `smem` dynamic shared memory and
// `threads` per CTA, cached per (device, kernel, smem).  The kernel's dynamic
// shared-memory limit is raised once per (device, kernel) to `smem_max`, the
// most any call can need, so a smaller call never lowers it below what a
// larger one uses.
inline int resident_ctas(const void* kernel, size_t smem, size_t smem_max, int threads) {
  static std::mutex mu;
  static std::map<std::tuple<int, const void*, size_t>, int> cache;
  static std::map<std::pair<int, const void*>, bool> raised;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_tuple(dev, kernel, smem);
  const auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  const auto rkey = std::make_pair(dev, kernel);
  if (!raised.count(rkey)) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem_max)) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    raised[rkey] = true;
  }
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, threads, smem) != cudaSuccess) {
    cudaGetLastError();
    occ = 0;
  }
  cache[key] = occ;
  return occ;
}

// How query heads map onto work: a key/value head's G query heads are split
// into nsub subsets of gs; the flat order runs over Hkv * nsub "virtual
// heads".  Multi-head attention is G = gs = nsub = 1.
struct HeadLayout {
  int group = 1, gs = 1, nsub = 1, vheads = 0;
};

struct Plan {
  int grid = 0;
  int work_warps = 0;
  size_t smem = 0;
};

// Persistent grid: every SM filled with resident CTAs, but never more warps
// than there can be chunks.
inline Plan plan_decode(const void* kernel, size_t smem, size_t smem_max, int warps_per_cta,
                        int CH, int B, int num_seqs, int num_vheads, int max_blocks_per_seq,
                        int64_t forced_warps) {
  Plan pl;
  pl.smem = smem;
  const int occ = resident_ctas(kernel, smem, smem_max, warps_per_cta * 32);
  const int sms = device_sm_count();
  if (occ <= 0 || sms <= 0) return pl;
  const int64_t cap = static_cast<int64_t>(max_blocks_per_seq) * B;
  const int64_t chunks_max = static_cast<int64_t>(num_seqs) * num_vheads * ((cap + CH - 1) / CH);
  int64_t warps = static_cast<int64_t>(sms) * occ * warps_per_cta;
  const int64_t useful = ((chunks_max + warps_per_cta - 1) / warps_per_cta) * warps_per_cta;
  if (warps > useful) warps = useful;
  if (forced_warps > 0) warps = forced_warps;
  if (warps < 1) warps = 1;
  pl.work_warps = static_cast<int>(warps);
  pl.grid = static_cast<int>((warps + warps_per_cta - 1) / warps_per_cta);
  return pl;
}

// Launch the merge kernel after a decode launch (programmatic dependent
// launch on the same stream).
template <typename T, int D>
cudaError_t launch_merge(const DecodeParams& p, int gs, cudaStream_t stream) {
  const int64_t items = static_cast<int64_t>(p.num_seqs) * p.num_heads * gs;
  const int per_cta = 8;  // warps, one per (text, virtual head, query head of the subset)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((items + per_cta - 1) / per_cta));
  cfg.blockDim = dim3(per_cta * 32);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, split_reduce_kernel<T, D>, static_cast<T*>(p.out),
                            static_cast<const int32_t*>(p.header),
                            static_cast<const float*>(p.records), p.grab, p.num_seqs,
                            p.num_heads, p.num_q_heads, p.nsub, gs);
}

}  // namespace pa
