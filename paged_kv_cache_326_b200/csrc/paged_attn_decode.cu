// paged_attn_decode: decode-phase attention through block tables, and the
// log-sum-exp merge of partial results (split_reduce_kernel).
//
// What it computes ("KV cache", section "How it works"; "The KV Cache and
// PagedAttention", section "The Block Table"): for text s and head h, the new
// query q[s][h] attends over the L_s stored keys, the new one included; token
// t lives in physical block block_tables[s][t / B] at place t % B:
//     out[s][h] = sum_t softmax_t(scale * q . K_t) * V_t.
//
// How (B200 design, not the pages' A100 kernel):
//  * The work is HBM-bound (about one flop per byte), so no tensor cores: each
//    (text, head) is a GEMV over its keys and another over its values.
//  * The unit of work is a CHUNK: CH consecutive tokens of one (text, head)
//    (CH = 16 at head_dim 128, 32 at head_dim 64, so a chunk's keys are 4 KB
//    and keys + values 8 KB).  All chunks of all (text, head) pairs are laid
//    out in one flat order (text-major, then head, then chunk).  A persistent
//    grid fills every SM; each warp first streams a static run of that order
//    (about 70% of an even share), then takes grains of the rest from a
//    shared counter.  Measured on B200, warps given equal bytes finish up to a
//    third apart (SMs do not get equal shares of HBM bandwidth); the grains
//    absorb that, so long and short texts alike keep all 148 SMs busy to the
//    end.
//  * A (text, head) whose chunks fall into several work units yields one
//    partial result per unit (running max m, sum l, unnormalised output o),
//    merged by split_reduce_kernel (log-sum-exp).  The merge is a second,
//    tiny kernel rather than an in-kernel "last arriver" step because the
//    GPU-scope atomics and fences that step needs stall the whole SM's
//    streaming (measured: 12% to 27% slower per launch), while kernel order
//    needs none.  A (text, head) that falls inside one unit is finished in
//    place.
//  * Each warp is its own pipeline: lane 0 issues bulk (TMA) copies of the
//    chunk's key rows and value rows, straight from their physical blocks,
//    into a ring of STAGES shared-memory stages, each with an mbarrier that
//    counts the bytes landed; all 32 lanes consume.  The issue runs STAGES
//    chunks ahead and crosses (text, head) and unit boundaries, so the copy
//    engine never idles at a boundary.  Only valid rows are copied: the
//    unfilled tail of a text's last block is never read from HBM.
//  * Block-table entries and context lengths are fetched one chunk per lane
//    for a whole window of up to 32 chunks, a window ahead of use, and handed
//    to the issuing lane with shuffles, so no table lookup sits on the
//    critical path.
//  * Dot products: a key row of head_dim elements is read by D/8 lanes as
//    16-byte vectors and reduced with shuffles; the softmax is the online
//    (running-max) form in fp32, in base 2 with log2(e) folded into the scale.
//  * Every wait is bounded; a wait that gives up records PA_ERR_TIMEOUT,
//    drains the copies in flight (bounded too) and returns.
//  * Both kernels launch with programmatic dependent launch, so their CTAs
//    are resident while the kernel before them finishes; griddepcontrol.wait
//    holds every read until that kernel's writes are visible.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <map>
#include <mutex>
#include <tuple>
#include <utility>

#include "dtype.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace pa {

namespace {

#ifndef PA_DECODE_WARPS
#define PA_DECODE_WARPS 4
#endif
#ifndef PA_DECODE_STAGES
#define PA_DECODE_STAGES 3
#endif
constexpr int kDecodeWarps = PA_DECODE_WARPS;    // warps per CTA
constexpr int kDecodeStages = PA_DECODE_STAGES;  // ring depth per warp
constexpr int kMaxSeqs = 4096;
// Work split: each warp first streams a static run of about kStaticPermille
// per mille of an even share; the rest is handed out in grains from a shared
// counter, at least kMinGrain chunks each and about kGrainsPerWarp per warp.
#ifndef PA_STATIC_PERMILLE
#define PA_STATIC_PERMILLE 700
#endif
#ifndef PA_MIN_GRAIN
#define PA_MIN_GRAIN 16
#endif
constexpr int kStaticPermille = PA_STATIC_PERMILLE;
constexpr int kGrainsPerWarp = 12;
constexpr int kMinGrain = PA_MIN_GRAIN;
constexpr int kDrainLimitNs = 1000000000;
__host__ __device__ constexpr int chunk_tokens(int D) { return 2048 / D; }
// One stage: K rows (4 KB), V rows (4 KB), the unit's GS query rows, a flag.
__host__ __device__ constexpr int stage_bytes(int D, int gs) { return 2 * 4096 + gs * 2 * D + 128; }
__host__ __device__ constexpr int warp_area_bytes(int D, int stages, int gs) {
  return stages * stage_bytes(D, gs) + 128;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Workspace: a header (the work split, then prefix[S+1]), the grain counter,
// then the partial records.  The header is written by CTA 0 of the decode
// kernel and read by the merge kernel.
constexpr int kHeaderInts = 8;  // total, q, grain, W, 4 spare
size_t header_bytes(int num_seqs) {
  return align_up(sizeof(int32_t) * (kHeaderInts + num_seqs + 1), 256);
}
constexpr size_t kGrabBytes = 256;
// The grain counter holds the call's epoch above bit 30; a stale epoch (an
// earlier call's, or never set) reads as zero, so the workspace never needs
// clearing.
constexpr unsigned long long kGrabMask = (1ull << 30) - 1;
constexpr unsigned long long kEpochMask = (1ull << 40) - 1;

struct DecodeParams {
  void* out;
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_tables;
  const int32_t* context_lens;
  float qk_scale_log2;
  int num_seqs;
  int num_heads;      // virtual heads: key/value heads x subsets (the flat order's heads)
  int num_q_heads;    // query heads of q and out
  int num_kv_heads;   // key/value heads of the pool
  int nsub;           // subsets per key/value head (GS query heads each)
  int max_blocks_per_seq;
  int64_t num_blocks;
  int num_work_warps;
  const void* k_new;              // fused step only: the new token's k, v [S][H][D]
  const void* v_new;
  const int64_t* slot_mapping;    // fused step only: their slots
  int32_t* header;                // work split + prefix, for the merge kernel
  unsigned long long* grab;       // grain counter
  unsigned long long epoch;       // 40-bit, never 0
  float* records;
  int32_t* status;
  int64_t wait_limit_ns;
};

// Per-lane look-ahead entry: where flat chunk (run start + position) lives.
template <int NB>
struct Lookahead {
  int s, h, j, len;  // len is the raw context length (clamped at use)
  int blk[NB];
};

// Count one more stored partial of a (text, head) in this call; returns the
// count including this one.
// Merge the partials of one (text, head), stored by units w_lo..w_hi: with
// M = max_i m_i and f_i = 2^(m_i - M),
//     out = (sum_i f_i o_i) / (sum_i f_i l_i),
// which equals the softmax-weighted sum over all the text's tokens (up to
// rounding).  Partials are read in warp order, so the result does not depend
// on which warp merges.  Reads go through L2 (other SMs wrote them).
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
        const float* rec = records + (w_lo + i0 + min(b + u, cnt - 1) + sh) * rec_stride + 4 + lane * PER;
        if constexpr (PER == 4) {
          const float4 v = __ldcg(reinterpret_cast<const float4*>(rec));
          o[u][0] = v.x; o[u][1] = v.y; o[u][2] = v.z; o[u][3] = v.w;
        } else {
          const float2 v = __ldcg(reinterpret_cast<const float2*>(rec));
          o[u][0] = v.x; o[u][1] = v.y;
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

}  // namespace

// FUSED: also store each text's new key/value at its slot, and take the
// text's last position (the new token) from the inputs instead of the pool,
// so nothing in this launch waits on its own write.
// GS: query heads per work unit (1 = multi-head attention).  With grouped-
// query attention the GS query heads of a unit share one key/value head, so
// every K/V row copied is used GS times from registers.
template <typename T, int D, int B, int WARPS, int STAGES, bool FUSED, int GS>
__global__ void __launch_bounds__(WARPS * 32, 2)
paged_decode_kernel(const DecodeParams p) {
  constexpr int CH = chunk_tokens(D);        // tokens per chunk
  constexpr int LPT = D / 8;                 // lanes per token row (16-byte vectors)
  constexpr int TPI = 32 / LPT;              // token rows per warp-wide load
  constexpr int ITERS = CH / TPI;            // loads per chunk (8)
  constexpr int NB = CH >= B ? CH / B : 1;   // physical blocks a chunk touches
  constexpr int TILE = CH * D;               // elements of K (or V) per chunk
  constexpr int STRIDE = stage_bytes(D, GS);
  constexpr int AREA = warp_area_bytes(D, STAGES, GS);
  static_assert(CH % TPI == 0 && (CH % B == 0 || B % CH == 0), "shape");

  extern __shared__ __align__(128) uint8_t smem[];
  int32_t* prefix = reinterpret_cast<int32_t*>(smem + WARPS * AREA);
  __shared__ int32_t warp_tot[WARPS];

  const int S = p.num_seqs;
  const int H = p.num_heads;  // virtual heads in the flat order
  const int Hq = p.num_q_heads, Hkv = p.num_kv_heads, NSUB = p.nsub;
  const int G = Hq / Hkv;       // query heads per key/value head
  // virtual head -> its key/value head and its first query head
  auto kv_head = [&](int vh) { return vh / NSUB; };
  auto q_head0 = [&](int vh) { return (vh / NSUB) * G + (vh % NSUB) * GS; };
  const int cap = p.max_blocks_per_seq * B;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;

  // Inputs may come from the kernel launched just before (the cache write).
  griddep_wait();

  // ---- prologue: prefix[s] = H * (chunks of texts before s), block-wide scan
  {
    const int nthr = WARPS * 32;
    const int per = (S + nthr - 1) / nthr;
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
      int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int before = 0;
    for (int w = 0; w < warp; ++w) before += warp_tot[w];
    int run = before + incl - local;
    for (int s = s0; s < s1; ++s) {
      int L = min(max(__ldg(p.context_lens + s), 0), cap);
      prefix[s] = run * H;
      run += (L + CH - 1) / CH;
    }
    if (tid == nthr - 1) prefix[S] = run * H;
    __syncthreads();
  }
  const int total = prefix[S];
  const int W = p.num_work_warps;
  // Static runs of q chunks (units 0..W-1), then grains of `grain` chunks (units
  // W, W+1, ...) covering the rest of the flat order.
  int q = W == 1 ? total : static_cast<int>(static_cast<long long>(total) * kStaticPermille / 1000 / W);
  if (q < 32 && W > 1) q = 0;
  const int dyn_base = W * q;
  const int dyn = total - dyn_base;
  const int grain = max(kMinGrain, (dyn + kGrainsPerWarp * W - 1) / (kGrainsPerWarp * W));
  if (blockIdx.x == 0) {
    if (tid == 0) {
      p.header[0] = total;
      p.header[1] = q;
      p.header[2] = grain;
      p.header[3] = W;
    }
    for (int i = tid; i <= S; i += WARPS * 32) p.header[kHeaderInts + i] = prefix[i];
  }
  // Texts with no tokens get zeros (spread over the CTAs).
  for (int s = blockIdx.x; s < S; s += gridDim.x) {
    if (prefix[s + 1] == prefix[s]) {
      uint4* o = reinterpret_cast<uint4*>(static_cast<T*>(p.out) + static_cast<int64_t>(s) * Hq * D);
      for (int i = tid; i < Hq * D / 8; i += WARPS * 32) o[i] = make_uint4(0u, 0u, 0u, 0u);
    }
  }

  const int w = blockIdx.x * WARPS + warp;
  // Fused step: the cache write, 16-byte vectors spread over the working
  // warps (as in kv_cache_write_kernel).  No read in this launch touches
  // these slots, so each warp does its share whenever it has a moment: right
  // after issuing its first copies, while it waits for them.
  auto fused_write = [&]() {
    if constexpr (FUSED) {
      const int vpr = D / 8;
      const int64_t per_text = static_cast<int64_t>(Hkv) * vpr;
      const int64_t nvec = per_text * S;
      const int64_t num_slots = p.num_blocks * B;
      uint4* kcw = static_cast<uint4*>(const_cast<void*>(p.k_cache));
      uint4* vcw = static_cast<uint4*>(const_cast<void*>(p.v_cache));
      for (int64_t i = static_cast<int64_t>(w) * 32 + lane; i < nvec;
           i += static_cast<int64_t>(W) * 32) {
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
  };
  if (w >= W) return;
  if (total == 0) {
    fused_write();
    return;
  }

  uint8_t* area = smem + warp * AREA;
  uint64_t* bars = reinterpret_cast<uint64_t*>(area + STAGES * STRIDE);
  if (lane == 0) {
#pragma unroll
    for (int st = 0; st < STAGES; ++st) mbar_init(&bars[st], 1);
    fence_barrier_init();
  }
  __syncwarp();

  const uint64_t policy = l2_evict_first_policy();
  const T* __restrict__ kc = static_cast<const T*>(p.k_cache);
  const T* __restrict__ vc = static_cast<const T*>(p.v_cache);
  const T* __restrict__ qg = static_cast<const T*>(p.q);

  int step = 1;
  while (step * 2 <= S) step *= 2;

  // ---- work units and their windows ----------------------------------
  // A unit is a run of consecutive flat chunks: first this warp's static run,
  // then grains taken from the shared counter.  Units are cut into windows of
  // at most 32 chunks (one chunk per lane for the look-ahead); a unit's last
  // two windows are balanced, so only the very last window of all the work
  // can be shorter than the copy ring.
  const unsigned long long e34 = p.epoch & ((1ull << 34) - 1);
  // Chunk offset of the grain whose counter value is `old` (lane 0).  The
  // counter carries this call's epoch above bit 30; a stale epoch (left by an
  // earlier call, or never set) is replaced by compare-and-swap, so the
  // workspace never needs clearing.
  auto grab_resolve = [&](unsigned long long old) -> int {
    if ((old >> 30) == e34) return static_cast<int>(old & kGrabMask);
    unsigned long long seen = old + static_cast<unsigned long long>(grain);
    while (true) {
      if ((seen >> 30) == e34) {
        const unsigned long long o2 = atomicAdd(p.grab, static_cast<unsigned long long>(grain));
        if ((o2 >> 30) == e34) return static_cast<int>(o2 & kGrabMask);
        seen = o2 + static_cast<unsigned long long>(grain);
        continue;
      }
      const unsigned long long prev =
          atomicCAS(p.grab, seen, (e34 << 30) | static_cast<unsigned long long>(grain));
      if (prev == seen) return 0;
      seen = prev;
    }
  };
  bool static_taken = false, exhausted = false, pend_live = false;
  unsigned long long pend = 0;  // lane 0: counter value of the next grain
  int u_start = 0, u_count = 0, u_id = -1, u_off = 0;
  auto grab_issue = [&]() {
    if (lane == 0) pend = atomicAdd(p.grab, static_cast<unsigned long long>(grain));
    pend_live = true;
  };
  auto next_unit = [&]() {
    if (!static_taken) {
      static_taken = true;
      if (q > 0) {
        u_start = w * q;
        u_count = q;
        u_id = w;
        u_off = 0;
        if (dyn > 0) grab_issue();
        return;
      }
    }
    if (dyn <= 0) {
      exhausted = true;
      return;
    }
    if (!pend_live) grab_issue();
    int off = 0;
    if (lane == 0) off = grab_resolve(pend);
    off = __shfl_sync(0xffffffffu, off, 0);
    pend_live = false;
    if (off >= dyn) {
      exhausted = true;
      return;
    }
    u_start = dyn_base + off;
    u_count = min(grain, dyn - off);
    u_id = W + off / grain;
    u_off = 0;
    grab_issue();  // the next grain, resolved when this one runs out
  };
  // Next window of this warp's work: start chunk, count (0 = no more), unit.
  auto next_window = [&](int& ws, int& wc, int& wu) {
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
  };

  // Where each chunk of a window lives, one chunk per lane.  Reads only
  // shared memory before issuing its global loads, whose results are not
  // used until the copy issue reaches this window.
  auto lookahead = [&](int ws, int wc) {
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
    e.len = __ldg(p.context_lens + s);
    const int32_t* row = p.block_tables + static_cast<int64_t>(s) * p.max_blocks_per_seq;
#pragma unroll
    for (int k = 0; k < NB; ++k) {
      const int idx = (j * CH) / B + k;
      e.blk[k] = idx < p.max_blocks_per_seq ? __ldg(row + idx) : -1;
    }
    return e;
  };

  int ws0, wc0, wu0, ws1, wc1, wu1;
  next_window(ws0, wc0, wu0);
  next_window(ws1, wc1, wu1);
  Lookahead<NB> win0 = lookahead(ws0, wc0);
  Lookahead<NB> win1 = lookahead(ws1, wc1);
  int i0 = 0;       // consumer's index in window 0
  int issued = 0;   // chunks whose copies were issued (stage = issued % STAGES)

  // Issue the copies of the chunk `k` places after the start of window 0 into
  // the next stage (lane 0 copies, every lane takes part in the shuffles).
  auto issue = [&](int k) {
    bool hi;
    int src;
    if (k < wc0) {
      hi = false;
      src = k;
    } else if (k - wc0 < wc1) {
      hi = true;
      src = k - wc0;
    } else {
      return;  // no more work
    }
    const bool unit_start = src == 0 && (hi ? wu1 != wu0 : issued == 0);
    const int s = __shfl_sync(0xffffffffu, hi ? win1.s : win0.s, src);
    const int h = __shfl_sync(0xffffffffu, hi ? win1.h : win0.h, src);
    const int j = __shfl_sync(0xffffffffu, hi ? win1.j : win0.j, src);
    const int len_raw = __shfl_sync(0xffffffffu, hi ? win1.len : win0.len, src);
    int blk[NB];
#pragma unroll
    for (int k = 0; k < NB; ++k) blk[k] = __shfl_sync(0xffffffffu, hi ? win1.blk[k] : win0.blk[k], src);
    const int st = issued % STAGES;
    ++issued;
    if (lane == 0) {
      uint8_t* stage = area + st * STRIDE;
      T* sK = reinterpret_cast<T*>(stage);
      T* sV = sK + TILE;
      T* sQ = sV + TILE;
      int32_t* flag = reinterpret_cast<int32_t*>(stage + 2 * 4096 + GS * 2 * D);
      const int len = min(max(len_raw, 0), cap);
      const int nvalid = min(CH, len - j * CH);
      const bool first = unit_start || j == 0;
      // rows of this chunk that each touched block supplies
      bool bad = false;
#pragma unroll
      for (int k = 0; k < NB; ++k) {
        const int rows = (CH >= B) ? min(B, nvalid - k * B) : nvalid;
        if (rows > 0 && (blk[k] < 0 || blk[k] >= p.num_blocks)) bad = true;
      }
      if (bad) set_status(p.status, -7 /* PA_ERR_BAD_BLOCK */);
      fence_proxy_async_smem();
      *flag = bad ? 1 : 0;
      const uint32_t qbytes = first ? GS * D * 2 : 0;
      const uint32_t kvbytes = bad ? 0 : 2u * nvalid * D * 2;
      mbar_arrive_expect_tx(&bars[st], qbytes + kvbytes);
      if (first)
        bulk_copy_g2s(sQ, qg + (static_cast<int64_t>(s) * Hq + q_head0(h)) * D, GS * D * 2, &bars[st],
                      policy);
      if (!bad) {
        // Fused step: the chunk holding the text's last position takes that
        // row from the new k/v instead of the pool.
        const bool new_row = FUSED && j * CH + nvalid == len;
        const int pool_rows = nvalid - (new_row ? 1 : 0);
        if constexpr (CH >= B) {
#pragma unroll
          for (int k = 0; k < NB; ++k) {
            const int rows = min(B, pool_rows - k * B);
            if (rows > 0) {
              const int64_t off = (static_cast<int64_t>(blk[k]) * Hkv + kv_head(h)) * B * D;
              bulk_copy_g2s(sK + k * B * D, kc + off, rows * D * 2, &bars[st], policy);
              bulk_copy_g2s(sV + k * B * D, vc + off, rows * D * 2, &bars[st], policy);
            }
          }
        } else {
          const int row0 = (j * CH) % B;
          const int64_t off = ((static_cast<int64_t>(blk[0]) * Hkv + kv_head(h)) * B + row0) * D;
          if (pool_rows > 0) {
            bulk_copy_g2s(sK, kc + off, pool_rows * D * 2, &bars[st], policy);
            bulk_copy_g2s(sV, vc + off, pool_rows * D * 2, &bars[st], policy);
          }
        }
        if (new_row) {
          const int64_t src_off = (static_cast<int64_t>(s) * Hkv + kv_head(h)) * D;
          bulk_copy_g2s(sK + pool_rows * D, static_cast<const T*>(p.k_new) + src_off, D * 2,
                        &bars[st], policy);
          bulk_copy_g2s(sV + pool_rows * D, static_cast<const T*>(p.v_new) + src_off, D * 2,
                        &bars[st], policy);
        }
      }
    }
  };

#pragma unroll
  for (int k = 0; k < STAGES; ++k) issue(k);
  fused_write();

  const int dchunk = lane % LPT;
  const int tsub = lane / LPT;
  // Per query head of this unit (GS of them share every K/V row read).
  float qf[GS][8];
  float acc[GS][8];
  float m[GS], lsum[GS];
  int piece_j0 = 0;
  int prev_unit = -1;

  for (int pos = 0; wc0 > 0; ++pos) {
    const int s = __shfl_sync(0xffffffffu, win0.s, i0);
    const int h = __shfl_sync(0xffffffffu, win0.h, i0);
    const int j = __shfl_sync(0xffffffffu, win0.j, i0);
    const int len = min(max(__shfl_sync(0xffffffffu, win0.len, i0), 0), cap);
    const int st = pos % STAGES;
    const uint32_t parity = (pos / STAGES) & 1;

    if (!mbar_wait_bounded(&bars[st], parity, p.wait_limit_ns)) {
      set_status(p.status, -10 /* PA_ERR_TIMEOUT */);
      for (int d = pos; d < issued; ++d)
        mbar_wait_bounded(&bars[d % STAGES], (d / STAGES) & 1, kDrainLimitNs);
      return;
    }

    const uint8_t* stage = area + st * STRIDE;
    const T* sK = reinterpret_cast<const T*>(stage);
    const T* sV = sK + TILE;
    const T* sQ = sV + TILE;
    const int bad = *reinterpret_cast<const int32_t*>(stage + 2 * 4096 + GS * 2 * D);

    if (j == 0 || wu0 != prev_unit) {
      piece_j0 = j;
#pragma unroll
      for (int g = 0; g < GS; ++g) {
        float qraw[8];
        unpack8<T>(*reinterpret_cast<const uint4*>(sQ + g * D + dchunk * 8), qraw);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          qf[g][k] = qraw[k] * p.qk_scale_log2;
          acc[g][k] = 0.f;
        }
        m[g] = -INFINITY;
        lsum[g] = 0.f;
      }
    }
    const int nvalid = bad ? 0 : min(CH, len - j * CH);

    // scores (base-2 logits) of this lane's token rows, for every head
    float sc[GS][ITERS];
#pragma unroll
    for (int it = 0; it < ITERS; ++it) {
      float kf[8];
      unpack8<T>(*reinterpret_cast<const uint4*>(sK + (it * TPI + tsub) * D + dchunk * 8), kf);
#pragma unroll
      for (int g = 0; g < GS; ++g) {
        float d0 = qf[g][0] * kf[0];
#pragma unroll
        for (int k = 1; k < 8; ++k) d0 = fmaf(qf[g][k], kf[k], d0);
        sc[g][it] = d0;
      }
    }
#pragma unroll
    for (int g = 0; g < GS; ++g)
#pragma unroll
      for (int it = 0; it < ITERS; ++it) {
#pragma unroll
        for (int off = LPT / 2; off >= 1; off >>= 1)
          sc[g][it] += __shfl_xor_sync(0xffffffffu, sc[g][it], off);
      }
    if (nvalid < CH) {
#pragma unroll
      for (int it = 0; it < ITERS; ++it)
        if (it * TPI + tsub >= nvalid) {
#pragma unroll
          for (int g = 0; g < GS; ++g) sc[g][it] = -INFINITY;
        }
    }
#pragma unroll
    for (int g = 0; g < GS; ++g) {
      float cm = sc[g][0];
#pragma unroll
      for (int it = 1; it < ITERS; ++it) cm = fmaxf(cm, sc[g][it]);
#pragma unroll
      for (int off = LPT; off < 32; off <<= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, off));
      const float m_new = fmaxf(m[g], cm);
      if (m_new != -INFINITY) {
        const float alpha = fast_exp2(m[g] - m_new);
        float psum = 0.f;
#pragma unroll
        for (int it = 0; it < ITERS; ++it) {
          sc[g][it] = fast_exp2(sc[g][it] - m_new);
          psum += sc[g][it];
        }
        lsum[g] = fmaf(lsum[g], alpha, psum);
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[g][k] *= alpha;
        m[g] = m_new;
      } else {
#pragma unroll
        for (int it = 0; it < ITERS; ++it) sc[g][it] = 0.f;
      }
    }
    if (nvalid == CH) {
#pragma unroll
      for (int it = 0; it < ITERS; ++it) {
        float vf[8];
        unpack8<T>(*reinterpret_cast<const uint4*>(sV + (it * TPI + tsub) * D + dchunk * 8), vf);
#pragma unroll
        for (int g = 0; g < GS; ++g)
#pragma unroll
          for (int k = 0; k < 8; ++k) acc[g][k] = fmaf(sc[g][it], vf[k], acc[g][k]);
      }
    } else {
#pragma unroll
      for (int it = 0; it < ITERS; ++it) {
        if (it * TPI + tsub < nvalid) {
          float vf[8];
          unpack8<T>(*reinterpret_cast<const uint4*>(sV + (it * TPI + tsub) * D + dchunk * 8), vf);
#pragma unroll
          for (int g = 0; g < GS; ++g)
#pragma unroll
            for (int k = 0; k < 8; ++k) acc[g][k] = fmaf(sc[g][it], vf[k], acc[g][k]);
        }
      }
    }

    // This stage is consumed: refill it before the epilogue, whose global
    // stores must not leave the copy engine idle.
    __syncwarp();
    issue(i0 + STAGES);

    const int ns = (len + CH - 1) / CH;
    const bool unit_ends = i0 + 1 == wc0 && (wc1 == 0 || wu1 != wu0);
    if (unit_ends || j == ns - 1) {
      const int64_t sh = static_cast<int64_t>(s) * H + h;          // (text, virtual head)
      const int64_t qrow = static_cast<int64_t>(s) * Hq + q_head0(h);  // first query head
      const bool whole = piece_j0 == 0 && j == ns - 1;
      float* recs = p.records + (static_cast<int64_t>(wu0) + sh) * (GS * (D + 4));
#pragma unroll
      for (int g = 0; g < GS; ++g) {
        float l_all = lsum[g];
        float o[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) o[k] = acc[g][k];
#pragma unroll
        for (int off = LPT; off < 32; off <<= 1) {
          l_all += __shfl_xor_sync(0xffffffffu, l_all, off);
#pragma unroll
          for (int k = 0; k < 8; ++k) o[k] += __shfl_xor_sync(0xffffffffu, o[k], off);
        }
        if (whole) {
          if (tsub == 0) {
            const float inv = l_all > 0.f ? 1.f / l_all : 0.f;
#pragma unroll
            for (int k = 0; k < 8; ++k) o[k] *= inv;
            *reinterpret_cast<uint4*>(static_cast<T*>(p.out) + (qrow + g) * D + dchunk * 8) =
                pack8<T>(o);
          }
        } else {
          float* rec = recs + g * (D + 4);
          if (lane == 0) {
            rec[0] = m[g];
            rec[1] = l_all;
          }
          if (tsub == 0) {
            float4* dst = reinterpret_cast<float4*>(rec + 4 + dchunk * 8);
            dst[0] = make_float4(o[0], o[1], o[2], o[3]);
            dst[1] = make_float4(o[4], o[5], o[6], o[7]);
          }
        }
      }
    }

    prev_unit = wu0;
    if (++i0 == wc0) {  // window 0 done: the next one moves up
      ws0 = ws1;
      wc0 = wc1;
      wu0 = wu1;
      win0 = win1;
      next_window(ws1, wc1, wu1);
      win1 = lookahead(ws1, wc1);
      i0 = 0;
    }
  }
}

// Merge kernel: for every (text, head) whose chunks fell into several work
// units, combine the units' partials (log-sum-exp); the decode kernel has
// already written every other output.  Launched right after the decode
// kernel with programmatic dependent launch: its CTAs become resident early
// and griddepcontrol.wait holds them until the decode kernel's writes are
// visible.  One warp per (text, head).
template <typename T, int D, int GS>
__global__ void __launch_bounds__(256)
split_reduce_kernel(T* __restrict__ out, const int32_t* __restrict__ header,
                    const float* __restrict__ records, int num_seqs, int num_vheads,
                    int num_q_heads, int nsub) {
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int seg = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (seg >= num_seqs * num_vheads) return;
  const int s = seg / num_vheads;
  const int vh = seg - s * num_vheads;
  const int q = header[1], grain = header[2], W = header[3];
  const int32_t* prefix = header + kHeaderInts;
  const int seg0 = prefix[s];
  const int ns = (prefix[s + 1] - seg0) / num_vheads;
  if (ns == 0) return;  // zero-filled by the decode kernel
  const int dyn_base = W * q;
  auto unit_of = [&](int c) { return c < dyn_base ? c / q : W + (c - dyn_base) / grain; };
  const int a = seg0 + vh * ns;
  const int u_lo = unit_of(a);
  const int u_hi = unit_of(a + ns - 1);
  if (u_lo == u_hi) return;  // finished in place by the decode kernel
  const int group = num_q_heads / (num_vheads / nsub);  // query heads per key/value head
  const int qh0 = (vh / nsub) * group + (vh % nsub) * GS;
#pragma unroll 1
  for (int g = 0; g < GS; ++g)
    merge_partials<T, D>(records + g * (D + 4), GS * (D + 4),
                         out + (static_cast<int64_t>(s) * num_q_heads + qh0 + g) * D, seg, u_lo,
                         u_hi, lane);
}

namespace {

int device_sm_count() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return sms;
}

size_t decode_smem_bytes(int D, int num_seqs, int gs) {
  return static_cast<size_t>(kDecodeWarps) * warp_area_bytes(D, kDecodeStages, gs) +
         align_up(sizeof(int32_t) * (num_seqs + 1), 16);
}

// How query heads map onto work: a key/value head's G query heads are split
// into nsub subsets of GS (GS in {4, 2, 1}, the largest that divides G); the
// flat order runs over Hkv * nsub "virtual heads".  Multi-head attention is
// G = GS = nsub = 1.
struct HeadLayout {
  int group = 1, gs = 1, nsub = 1, vheads = 0;
};
HeadLayout head_layout(int num_heads, int num_kv_heads) {
  HeadLayout l;
  if (num_kv_heads < 1 || num_heads < 1 || num_heads % num_kv_heads) return l;
  l.group = num_heads / num_kv_heads;
  l.gs = l.group % 4 == 0 ? 4 : (l.group % 2 == 0 ? 2 : 1);
  l.nsub = l.group / l.gs;
  l.vheads = num_kv_heads * l.nsub;
  return l;
}

// Resident CTAs per SM of `kernel` with `smem` dynamic shared memory, cached
// per (device, kernel, smem).  The kernel's dynamic shared-memory limit is
// raised once per (device, kernel) to the most any call can need, so a call
// with fewer texts never lowers it below what a larger one uses.
int resident_ctas(const void* kernel, size_t smem, int head_dim, int gs) {
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
    const size_t most = decode_smem_bytes(head_dim, kMaxSeqs, gs);
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(most)) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    raised[rkey] = true;
  }
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, kDecodeWarps * 32, smem) !=
      cudaSuccess) {
    cudaGetLastError();
    occ = 0;
  }
  cache[key] = occ;
  return occ;
}

// A fresh 40-bit epoch per launch (never 0, so a zeroed workspace holds no
// live counts).
unsigned long long next_epoch() {
  static std::atomic<unsigned long long> counter{0};
  unsigned long long e;
  do {
    e = (counter.fetch_add(1) + 1) & kEpochMask;
  } while (e == 0);
  return e;
}

struct Plan {
  int grid = 0;
  int work_warps = 0;
  size_t smem = 0;
};

// Persistent grid: every SM filled with resident CTAs, but never more warps
// than there can be chunks.
Plan plan_decode(const void* kernel, int D, int B, int num_seqs, int num_heads,
                 int max_blocks_per_seq, int64_t forced_warps, int gs) {
  Plan pl;
  pl.smem = decode_smem_bytes(D, num_seqs, gs);
  const int occ = resident_ctas(kernel, pl.smem, D, gs);
  const int sms = device_sm_count();
  if (occ <= 0 || sms <= 0) return pl;
  const int CH = chunk_tokens(D);
  const int64_t cap = static_cast<int64_t>(max_blocks_per_seq) * B;
  const int64_t chunks_max = static_cast<int64_t>(num_seqs) * num_heads * ((cap + CH - 1) / CH);
  int64_t warps = static_cast<int64_t>(sms) * occ * kDecodeWarps;
  const int64_t useful = ((chunks_max + kDecodeWarps - 1) / kDecodeWarps) * kDecodeWarps;
  if (warps > useful) warps = useful;
  if (forced_warps > 0) warps = forced_warps;
  if (warps < 1) warps = 1;
  pl.work_warps = static_cast<int>(warps);
  pl.grid = static_cast<int>((warps + kDecodeWarps - 1) / kDecodeWarps);
  return pl;
}

// Units (static runs plus grains) a launch with `warps` working warps can
// create: grains number at most kGrainsPerWarp per warp.
int64_t max_units(int64_t warps) { return warps * (kGrainsPerWarp + 1) + 1; }

size_t records_bytes(int64_t records, int D, int gs) {
  return static_cast<size_t>(records) * gs * (D + 4) * sizeof(float);
}

template <typename T, int D, int B, bool FUSED, int GS>
const void* decode_kernel_ptr() {
  return reinterpret_cast<const void*>(
      &paged_decode_kernel<T, D, B, kDecodeWarps, kDecodeStages, FUSED, GS>);
}

template <typename T, int D, int B, bool FUSED, int GS>
cudaError_t launch_typed(const DecodeArgs& a, const HeadLayout& hl, cudaStream_t stream) {
  const Plan pl = plan_decode(decode_kernel_ptr<T, D, B, FUSED, GS>(), D, B, a.num_seqs,
                              hl.vheads, a.max_blocks_per_seq, a.forced_warps, GS);
  if (pl.grid <= 0) return cudaErrorInvalidConfiguration;
  const int64_t segs = static_cast<int64_t>(a.num_seqs) * hl.vheads;
  const size_t need = header_bytes(a.num_seqs) + kGrabBytes +
                      records_bytes(max_units(pl.work_warps) + segs, D, GS);
  if (a.workspace_bytes < need) return cudaErrorInvalidValue;
  DecodeParams p;
  p.out = a.out;
  p.q = a.q;
  p.k_cache = a.k_cache;
  p.v_cache = a.v_cache;
  p.block_tables = a.block_tables;
  p.context_lens = a.context_lens;
  p.qk_scale_log2 = a.scale * 1.4426950408889634f;  // log2(e)
  p.num_seqs = a.num_seqs;
  p.num_heads = hl.vheads;
  p.num_q_heads = a.num_heads;
  p.num_kv_heads = a.num_kv_heads;
  p.nsub = hl.nsub;
  p.max_blocks_per_seq = a.max_blocks_per_seq;
  p.num_blocks = a.num_blocks;
  p.num_work_warps = pl.work_warps;
  char* ws = static_cast<char*>(a.workspace);
  p.header = reinterpret_cast<int32_t*>(ws);
  p.grab = reinterpret_cast<unsigned long long*>(ws + header_bytes(a.num_seqs));
  p.epoch = next_epoch();
  p.records = reinterpret_cast<float*>(ws + header_bytes(a.num_seqs) + kGrabBytes);
  p.status = a.status;
  p.wait_limit_ns = a.wait_limit_ns;
  p.k_new = a.k_new;
  p.v_new = a.v_new;
  p.slot_mapping = a.slot_mapping;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.grid);
  cfg.blockDim = dim3(kDecodeWarps * 32);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t err = cudaLaunchKernelEx(
      &cfg, paged_decode_kernel<T, D, B, kDecodeWarps, kDecodeStages, FUSED, GS>, p);
  if (err != cudaSuccess) return err;
  const int per_cta = 8;  // warps, one per (text, virtual head)
  cfg.gridDim = dim3(static_cast<unsigned>((segs + per_cta - 1) / per_cta));
  cfg.blockDim = dim3(per_cta * 32);
  cfg.dynamicSmemBytes = 0;
  err = cudaLaunchKernelEx(&cfg, split_reduce_kernel<T, D, GS>, static_cast<T*>(a.out),
                           static_cast<const int32_t*>(p.header),
                           static_cast<const float*>(p.records), a.num_seqs, hl.vheads,
                           a.num_heads, hl.nsub);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

template <typename T, int D, bool FUSED, int GS>
cudaError_t dispatch_block(const DecodeArgs& a, const HeadLayout& hl, cudaStream_t stream) {
  switch (a.block_size) {
    case 4: return launch_typed<T, D, 4, FUSED, GS>(a, hl, stream);
    case 8: return launch_typed<T, D, 8, FUSED, GS>(a, hl, stream);
    case 16: return launch_typed<T, D, 16, FUSED, GS>(a, hl, stream);
    case 32: return launch_typed<T, D, 32, FUSED, GS>(a, hl, stream);
    default: return cudaErrorInvalidValue;
  }
}

template <typename T, bool FUSED, int GS>
cudaError_t dispatch_dim(const DecodeArgs& a, const HeadLayout& hl, cudaStream_t stream) {
  switch (a.head_dim) {
    case 64: return dispatch_block<T, 64, FUSED, GS>(a, hl, stream);
    case 128: return dispatch_block<T, 128, FUSED, GS>(a, hl, stream);
    default: return cudaErrorInvalidValue;
  }
}

template <typename T>
cudaError_t dispatch_heads(const DecodeArgs& a, const HeadLayout& hl, cudaStream_t stream) {
  if (a.slot_mapping)  // fused decode step: multi-head only
    return hl.gs == 1 ? dispatch_dim<T, true, 1>(a, hl, stream) : cudaErrorInvalidValue;
  switch (hl.gs) {
    case 1: return dispatch_dim<T, false, 1>(a, hl, stream);
    case 2: return dispatch_dim<T, false, 2>(a, hl, stream);
    case 4: return dispatch_dim<T, false, 4>(a, hl, stream);
    default: return cudaErrorInvalidValue;
  }
}

template <int D, bool FUSED, int GS>
const void* kernel_for(int block_size, bool bf16) {
  switch (block_size) {
    case 4: return bf16 ? decode_kernel_ptr<__nv_bfloat16, D, 4, FUSED, GS>() : decode_kernel_ptr<__half, D, 4, FUSED, GS>();
    case 8: return bf16 ? decode_kernel_ptr<__nv_bfloat16, D, 8, FUSED, GS>() : decode_kernel_ptr<__half, D, 8, FUSED, GS>();
    case 16: return bf16 ? decode_kernel_ptr<__nv_bfloat16, D, 16, FUSED, GS>() : decode_kernel_ptr<__half, D, 16, FUSED, GS>();
    case 32: return bf16 ? decode_kernel_ptr<__nv_bfloat16, D, 32, FUSED, GS>() : decode_kernel_ptr<__half, D, 32, FUSED, GS>();
    default: return nullptr;
  }
}

template <int D>
const void* kernel_for_variant(int block_size, bool bf16, bool fused, int gs) {
  if (fused) return gs == 1 ? kernel_for<D, true, 1>(block_size, bf16) : nullptr;
  switch (gs) {
    case 1: return kernel_for<D, false, 1>(block_size, bf16);
    case 2: return kernel_for<D, false, 2>(block_size, bf16);
    case 4: return kernel_for<D, false, 4>(block_size, bf16);
    default: return nullptr;
  }
}

}  // namespace

bool decode_sizes_supported(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                            int block_size, int max_blocks_per_seq) {
  if (num_seqs < 1 || num_seqs > kMaxSeqs || num_heads < 1 || num_heads > 1024) return false;
  const HeadLayout hl = head_layout(num_heads, num_kv_heads);
  if (hl.vheads < 1 || hl.vheads > 1024) return false;
  if (head_dim != 64 && head_dim != 128) return false;
  if (block_size != 4 && block_size != 8 && block_size != 16 && block_size != 32) return false;
  if (max_blocks_per_seq < 1) return false;
  const int64_t CH = chunk_tokens(head_dim);
  const int64_t cap = static_cast<int64_t>(max_blocks_per_seq) * block_size;
  const int64_t chunks = static_cast<int64_t>(num_seqs) * hl.vheads * ((cap + CH - 1) / CH);
  return chunks < (int64_t{1} << 30) && cap < (int64_t{1} << 30);
}

size_t decode_workspace_bytes(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                              int block_size, int max_blocks_per_seq, int64_t forced_warps) {
  if (!decode_sizes_supported(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                              max_blocks_per_seq))
    return 0;
  const HeadLayout hl = head_layout(num_heads, num_kv_heads);
  int64_t warps = 0;
  for (int variant = 0; variant < 4; ++variant) {
    const bool bf16 = variant & 1, fused = variant & 2;
    if (fused && hl.gs != 1) continue;
    const void* k = head_dim == 128 ? kernel_for_variant<128>(block_size, bf16, fused, hl.gs)
                                    : kernel_for_variant<64>(block_size, bf16, fused, hl.gs);
    const Plan pl = plan_decode(k, head_dim, block_size, num_seqs, hl.vheads, max_blocks_per_seq,
                                forced_warps, hl.gs);
    if (pl.grid <= 0) return 0;
    if (pl.work_warps > warps) warps = pl.work_warps;
  }
  const int64_t segs = static_cast<int64_t>(num_seqs) * hl.vheads;
  return header_bytes(num_seqs) + kGrabBytes + records_bytes(max_units(warps) + segs, head_dim, hl.gs);
}

cudaError_t launch_paged_attn_decode(const DecodeArgs& a, cudaStream_t stream) {
  if (!decode_sizes_supported(a.num_seqs, a.num_heads, a.num_kv_heads, a.head_dim, a.block_size,
                              a.max_blocks_per_seq))
    return cudaErrorInvalidValue;
  const HeadLayout hl = head_layout(a.num_heads, a.num_kv_heads);
  return a.is_bf16 ? dispatch_heads<__nv_bfloat16>(a, hl, stream)
                   : dispatch_heads<__half>(a, hl, stream);
}

}  // namespace pa
