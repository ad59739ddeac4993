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

#include <cstdint>
#include <type_traits>

#include "decode_common.cuh"
#include "fp8.cuh"
#include "kernels.h"

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
// The 8-bit kernel is bound by instruction latency more than by copies in
// flight: two stages let three CTAs (12 warps) share an SM with the same
// bytes in flight as two CTAs of three stages.
#ifndef PA_DECODE_STAGES_F8
#define PA_DECODE_STAGES_F8 2
#endif
constexpr int kDecodeStagesF8 = PA_DECODE_STAGES_F8;
// Blocks of 8 or fewer rows: a chunk takes two or more copies of K and of V,
// and two stages, three CTAs an SM, beat three stages, two CTAs (skewed
// lengths, bf16: 414 against 474 us at blocks of 8); at blocks of 16 and up
// three stages stay (the batch-64 step: 238 against 246 us).
#ifndef PA_DECODE_STAGES_SMALL_B
#define PA_DECODE_STAGES_SMALL_B 2
#endif
constexpr int kDecodeStagesSmallB = PA_DECODE_STAGES_SMALL_B;
__host__ __device__ constexpr int decode_stages(bool f8, int B) {
  return f8 ? kDecodeStagesF8 : B <= 8 ? kDecodeStagesSmallB : kDecodeStages;
}
// One stage: K rows (4 KB), V rows (4 KB), the unit's GS query rows, a flag.
__host__ __device__ constexpr int stage_bytes(int D, int gs) { return 2 * 4096 + gs * 2 * D + 128; }
__host__ __device__ constexpr int warp_area_bytes(int D, int stages, int gs) {
  return stages * stage_bytes(D, gs) + 128;
}

}  // namespace

// FUSED: also store each text's new key/value at its slot, and take the
// text's last position (the new token) from the inputs instead of the pool,
// so nothing in this launch waits on its own write.
// GS: query heads per work unit (1 = multi-head attention).  With grouped-
// query attention the GS query heads of a unit share one key/value head, so
// every K/V row copied is used GS times from registers.
// F8: the cache holds 8-bit E4M3 codes (one byte per number, per-tensor
// scales) instead of T; a chunk is then twice the tokens for the same 4 KB,
// and each lane dequantizes 16 codes per 16-byte vector in registers.
template <typename T, int D, int B, int WARPS, int STAGES, bool FUSED, int GS, bool F8>
__global__ void __launch_bounds__(WARPS * 32, 2)
paged_decode_kernel(const DecodeParams p) {
  constexpr int EB = F8 ? 1 : 2;             // cache bytes per number
  constexpr int CH = 4096 / (D * EB);        // tokens per chunk (4 KB of keys)
  constexpr int VEC = 16 / EB;               // numbers per 16-byte vector
  constexpr int LPT = D / VEC;               // lanes per token row
  constexpr int TPI = 32 / LPT;              // token rows per warp-wide load
  constexpr int ITERS = CH / TPI;            // loads per chunk (8)
  constexpr int NB = CH >= B ? CH / B : 1;   // physical blocks a chunk touches
  constexpr int ROWB = D * EB;               // bytes per cache row
  constexpr int STRIDE = stage_bytes(D, GS);
  constexpr int AREA = warp_area_bytes(D, STAGES, GS);
  static_assert(CH % TPI == 0 && (CH % B == 0 || B % CH == 0), "shape");
  // one 16-byte vector of cache numbers -> VEC floats
  auto load_vec = [](const uint8_t* src, float (&f)[VEC]) {
    const uint4 v = *reinterpret_cast<const uint4*>(src);
    if constexpr (F8) {
      unpack16_e4m3(v, f);
    } else {
      unpack8<T>(v, f);
    }
  };

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
  // The tail pass of a shared-prefix decode reads nothing the pass before it
  // writes: it starts at once and waits for that pass only on its way out,
  // so that the merge launched after it sees both passes' records.
  const bool wait_at_exit = p.cascade == 2;
  if (!wait_at_exit) griddep_wait();

  const WorkSplit sp = decode_prologue<T, D, CH, WARPS * 32>(p, prefix, warp_tot, cap);
  const int total = sp.total;
  const int W = sp.W;

  const int w = blockIdx.x * WARPS + warp;
  // One-launch step: the cache write.  No read in this launch touches these
  // slots, so each warp does its share whenever it has a moment: right after
  // issuing its first copies, while it waits for them.
  auto fused_write = [&]() {
    if constexpr (FUSED && F8) fused_cache_write_f8<T, D, B>(p, w, W, lane);
    else if constexpr (FUSED) fused_cache_write<D, B>(p, w, W, lane);
  };
  if (w >= W) {
    if (wait_at_exit) griddep_wait();
    return;
  }
  if (total == 0) {
    fused_write();
    if (wait_at_exit) griddep_wait();
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
  const uint8_t* __restrict__ kc = static_cast<const uint8_t*>(p.k_cache);
  const uint8_t* __restrict__ vc = static_cast<const uint8_t*>(p.v_cache);
  const T* __restrict__ qg = static_cast<const T*>(p.q);

  Scheduler<CH, B, NB> sched(p, prefix, sp, w, lane);
  auto next_window = [&](int& ws, int& wc, int& wu) { sched.next_window(ws, wc, wu); };
  auto lookahead = [&](int ws, int wc) { return sched.lookahead(ws, wc); };

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
      uint8_t* sK = stage;
      uint8_t* sV = stage + 4096;
      T* sQ = reinterpret_cast<T*>(stage + 8192);
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
      // Fused step: the chunk holding the text's last position takes that
      // row from the new k/v instead of the pool (copied here for a 16-bit
      // cache; for an 8-bit cache the consumer writes its codes).
      const bool new_row = FUSED && j * CH + nvalid == len;
      const int pool_rows = nvalid - (new_row ? 1 : 0);
      const uint32_t qbytes = first ? GS * D * 2 : 0;
      const uint32_t kvbytes = bad ? 0 : 2u * (F8 ? pool_rows : nvalid) * ROWB;
      mbar_arrive_expect_tx(&bars[st], qbytes + kvbytes);
      if (first)
        bulk_copy_g2s(sQ, qg + (static_cast<int64_t>(s) * Hq + q_head0(h)) * D, GS * D * 2, &bars[st],
                      policy);
      if (!bad) {
        if constexpr (CH >= B) {
#pragma unroll
          for (int k = 0; k < NB; ++k) {
            const int rows = min(B, pool_rows - k * B);
            if (rows > 0) {
              const int64_t off = (static_cast<int64_t>(blk[k]) * Hkv + kv_head(h)) * B * ROWB;
              bulk_copy_g2s(sK + k * B * ROWB, kc + off, rows * ROWB, &bars[st], policy);
              bulk_copy_g2s(sV + k * B * ROWB, vc + off, rows * ROWB, &bars[st], policy);
            }
          }
        } else {
          const int row0 = (j * CH) % B;
          const int64_t off = ((static_cast<int64_t>(blk[0]) * Hkv + kv_head(h)) * B + row0) * ROWB;
          if (pool_rows > 0) {
            bulk_copy_g2s(sK, kc + off, pool_rows * ROWB, &bars[st], policy);
            bulk_copy_g2s(sV, vc + off, pool_rows * ROWB, &bars[st], policy);
          }
        }
        if (!F8 && new_row) {
          const int64_t src_off = (static_cast<int64_t>(s) * Hkv + kv_head(h)) * D;
          bulk_copy_g2s(sK + pool_rows * ROWB, static_cast<const T*>(p.k_new) + src_off, ROWB,
                        &bars[st], policy);
          bulk_copy_g2s(sV + pool_rows * ROWB, static_cast<const T*>(p.v_new) + src_off, ROWB,
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
  // An 8-bit cache with fp16 queries keeps the query as raw fp16 pairs and
  // forms the scores with fp16 x fp16 -> fp32 FMAs straight from the widened
  // codes (exact products; the scale is applied to the sum).
  constexpr bool MIXED = F8 && std::is_same<T, __half>::value;
  float qf[GS][VEC];
  uint32_t qh[GS][MIXED ? VEC / 2 : 1];
  float acc[GS][VEC];
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
      if (wait_at_exit) griddep_wait();
      return;
    }

    const uint8_t* stage = area + st * STRIDE;
    const uint8_t* sK = stage;
    const uint8_t* sV = stage + 4096;
    const T* sQ = reinterpret_cast<const T*>(stage + 8192);
    const int bad = *reinterpret_cast<const int32_t*>(stage + 2 * 4096 + GS * 2 * D);

    if (j == 0 || wu0 != prev_unit) {
      piece_j0 = j;
#pragma unroll
      for (int g = 0; g < GS; ++g) {
#pragma unroll
        for (int h8 = 0; h8 < VEC / 8; ++h8) {
          const uint4 qv = *reinterpret_cast<const uint4*>(sQ + g * D + dchunk * VEC + h8 * 8);
          if constexpr (MIXED) {
            qh[g][h8 * 4 + 0] = qv.x;
            qh[g][h8 * 4 + 1] = qv.y;
            qh[g][h8 * 4 + 2] = qv.z;
            qh[g][h8 * 4 + 3] = qv.w;
          } else {
            float qraw[8];
            unpack8<T>(qv, qraw);
#pragma unroll
            for (int k = 0; k < 8; ++k) qf[g][h8 * 8 + k] = qraw[k] * p.qk_scale_log2;
          }
#pragma unroll
          for (int k = 0; k < 8; ++k) acc[g][h8 * 8 + k] = 0.f;
        }
        m[g] = -INFINITY;
        lsum[g] = 0.f;
      }
    }
    const int nvalid = bad ? 0 : min(CH, len - j * CH);
    if constexpr (F8 && FUSED) {
      // The one-launch step's new row over an 8-bit cache: its codes (the
      // cache write's quantization) take the stage row after the pool rows,
      // which the copies left empty.  The refill of this stage is ordered
      // after these writes by the proxy fence its issue begins with.
      if (nvalid > 0 && j * CH + nvalid == len) {
        const int64_t src = (static_cast<int64_t>(s) * Hkv + kv_head(h)) * D;
        uint8_t* rk = const_cast<uint8_t*>(sK) + (nvalid - 1) * ROWB;
        uint8_t* rv = const_cast<uint8_t*>(sV) + (nvalid - 1) * ROWB;
        for (int c = lane; c < D / 8; c += 32) {
          float x[8];
          unpack8<T>(__ldg(reinterpret_cast<const uint4*>(static_cast<const T*>(p.k_new) + src) + c), x);
          *reinterpret_cast<uint2*>(rk + c * 8) = e4m3x8_quantize(x, p.k_scale);
          unpack8<T>(__ldg(reinterpret_cast<const uint4*>(static_cast<const T*>(p.v_new) + src) + c), x);
          *reinterpret_cast<uint2*>(rv + c * 8) = e4m3x8_quantize(x, p.v_scale);
        }
        __syncwarp();
      }
    }

    // scores (base-2 logits) of this lane's token rows, for every head
    float sc[GS][ITERS];
#pragma unroll
    for (int it = 0; it < ITERS; ++it) {
      if constexpr (MIXED) {
        const uint4 kv = *reinterpret_cast<const uint4*>(sK + (it * TPI + tsub) * ROWB + dchunk * 16);
        const uint32_t kw[4] = {kv.x, kv.y, kv.z, kv.w};
        uint32_t kh[VEC / 2];
#pragma unroll
        for (int i = 0; i < 4; ++i) e4m3x4_to_half2x2(kw[i], kh[2 * i], kh[2 * i + 1]);
#pragma unroll
        for (int g = 0; g < GS; ++g) {
          float d0 = 0.f, d1 = 0.f;
#pragma unroll
          for (int i = 0; i < VEC / 2; i += 2) {
            d0 = dot2_f16_f32(qh[g][i], kh[i], d0);
            d1 = dot2_f16_f32(qh[g][i + 1], kh[i + 1], d1);
          }
          sc[g][it] = (d0 + d1) * p.qk_scale_log2;
        }
      } else {
        float kf[VEC];
        load_vec(sK + (it * TPI + tsub) * ROWB + dchunk * 16, kf);
#pragma unroll
        for (int g = 0; g < GS; ++g) {
          float d0 = qf[g][0] * kf[0];
#pragma unroll
          for (int k = 1; k < VEC; ++k) d0 = fmaf(qf[g][k], kf[k], d0);
          sc[g][it] = d0;
        }
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
        for (int k = 0; k < VEC; ++k) acc[g][k] *= alpha;
        m[g] = m_new;
      } else {
#pragma unroll
        for (int it = 0; it < ITERS; ++it) sc[g][it] = 0.f;
      }
    }
    // acc += p * v for one token row (packed fp32 FMAs on the 8-bit cache)
    auto accumulate = [&](int it) {
      float vf[VEC];
      load_vec(sV + (it * TPI + tsub) * ROWB + dchunk * 16, vf);
#pragma unroll
      for (int g = 0; g < GS; ++g) {
        if constexpr (F8) {
          const float2 p2 = make_float2(sc[g][it], sc[g][it]);
#pragma unroll
          for (int k = 0; k < VEC; k += 2) {
            const float2 r = __ffma2_rn(p2, make_float2(vf[k], vf[k + 1]),
                                        make_float2(acc[g][k], acc[g][k + 1]));
            acc[g][k] = r.x;
            acc[g][k + 1] = r.y;
          }
        } else {
#pragma unroll
          for (int k = 0; k < VEC; ++k) acc[g][k] = fmaf(sc[g][it], vf[k], acc[g][k]);
        }
      }
    };
    if (nvalid == CH) {
#pragma unroll
      for (int it = 0; it < ITERS; ++it) accumulate(it);
    } else {
#pragma unroll
      for (int it = 0; it < ITERS; ++it)
        if (it * TPI + tsub < nvalid) accumulate(it);
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
      const bool whole = piece_j0 == 0 && j == ns - 1 && !p.cascade;
      float* recs = p.records + (static_cast<int64_t>(wu0) + sh) * (GS * (D + 4));
#pragma unroll
      for (int g = 0; g < GS; ++g) {
        float l_all = lsum[g];
        float o[VEC];
#pragma unroll
        for (int k = 0; k < VEC; ++k) o[k] = acc[g][k];
#pragma unroll
        for (int off = LPT; off < 32; off <<= 1) {
          l_all += __shfl_xor_sync(0xffffffffu, l_all, off);
#pragma unroll
          for (int k = 0; k < VEC; ++k) o[k] += __shfl_xor_sync(0xffffffffu, o[k], off);
        }
        if (whole) {
          if (tsub == 0) {
            // v_scale (1 for a T cache) turns sums of codes into values
            const float inv = l_all > 0.f ? p.v_scale / l_all : 0.f;
#pragma unroll
            for (int h8 = 0; h8 < VEC / 8; ++h8) {
              float o8[8];
#pragma unroll
              for (int k = 0; k < 8; ++k) o8[k] = o[h8 * 8 + k] * inv;
              *reinterpret_cast<uint4*>(static_cast<T*>(p.out) + (qrow + g) * D + dchunk * VEC +
                                        h8 * 8) = pack8<T>(o8);
            }
          }
        } else {
          float* rec = recs + g * (D + 4);
          if (lane == 0) {
            rec[0] = m[g];
            rec[1] = l_all;
          }
          if (tsub == 0) {
            float4* dst = reinterpret_cast<float4*>(rec + 4 + dchunk * VEC);
#pragma unroll
            for (int k4 = 0; k4 < VEC / 4; ++k4)
              dst[k4] = make_float4(o[4 * k4] * p.v_scale, o[4 * k4 + 1] * p.v_scale,
                                    o[4 * k4 + 2] * p.v_scale, o[4 * k4 + 3] * p.v_scale);
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
  if (wait_at_exit) griddep_wait();
}

namespace {

size_t decode_smem_bytes(int D, int num_seqs, int gs, bool fp8, int B) {
  return static_cast<size_t>(kDecodeWarps) * warp_area_bytes(D, decode_stages(fp8, B), gs) +
         align_up(sizeof(int32_t) * (num_seqs + 1), 16);
}

// CUDA-core kernel: a key/value head's G query heads are split into nsub
// subsets of GS (GS in {4, 2, 1}, the largest that divides G).
HeadLayout head_layout(int num_heads, int num_kv_heads) {
  HeadLayout l;
  if (num_kv_heads < 1 || num_heads < 1 || num_heads % num_kv_heads) return l;
  l.group = num_heads / num_kv_heads;
  l.gs = l.group % 4 == 0 ? 4 : (l.group % 2 == 0 ? 2 : 1);
  l.nsub = l.group / l.gs;
  l.vheads = num_kv_heads * l.nsub;
  return l;
}

// Persistent grid for one decode kernel variant.
Plan plan_variant(const void* kernel, int D, int B, int num_seqs, int vheads,
                  int max_blocks_per_seq, int64_t forced_warps, int gs, bool fp8) {
  return plan_decode(kernel, decode_smem_bytes(D, num_seqs, gs, fp8, B),
                     decode_smem_bytes(D, kMaxSeqs, gs, fp8, B),
                     kDecodeWarps, fp8 ? 4096 / D : chunk_tokens(D), B, num_seqs, vheads,
                     max_blocks_per_seq, forced_warps);
}

template <typename T, int D, int B, bool FUSED, int GS, bool F8>
const void* decode_kernel_ptr() {
  return reinterpret_cast<const void*>(
      &paged_decode_kernel<T, D, B, kDecodeWarps, decode_stages(F8, B), FUSED, GS, F8>);
}

template <typename T, int D, int B, bool FUSED, int GS, bool F8>
cudaError_t launch_typed(const DecodeArgs& a, const HeadLayout& hl, cudaStream_t stream) {
  const Plan pl = plan_variant(decode_kernel_ptr<T, D, B, FUSED, GS, F8>(), D, B, a.num_seqs,
                               hl.vheads, a.max_blocks_per_seq, a.forced_warps, GS, F8);
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
  // log2(e), and for an 8-bit cache the keys' scale, folded into the
  // query; the values' scale multiplies the output
  p.qk_scale_log2 = a.scale * 1.4426950408889634f * (F8 ? a.k_scale : 1.f);
  p.v_scale = F8 ? a.v_scale : 1.f;
  p.k_scale = F8 ? a.k_scale : 1.f;
  p.num_seqs = a.num_seqs;
  p.num_heads = hl.vheads;
  p.num_q_heads = a.num_heads;
  p.num_kv_heads = a.num_kv_heads;
  p.nsub = hl.nsub;
  p.gs = GS;
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
  p.cascade = a.cascade ? (a.cascade_overlap ? 2 : 1) : 0;
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
      &cfg, paged_decode_kernel<T, D, B, kDecodeWarps, decode_stages(F8, B), FUSED, GS, F8>, p);
  if (err != cudaSuccess) return err;
  if (p.cascade) return cudaGetLastError();  // the caller merges
  err = launch_merge<T, D>(p, GS, stream);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

template <typename T, int D, bool FUSED, int GS, bool F8>
cudaError_t dispatch_block(const DecodeArgs& a, const HeadLayout& hl, cudaStream_t stream) {
  switch (a.block_size) {
    case 4: return launch_typed<T, D, 4, FUSED, GS, F8>(a, hl, stream);
    case 8: return launch_typed<T, D, 8, FUSED, GS, F8>(a, hl, stream);
    case 16: return launch_typed<T, D, 16, FUSED, GS, F8>(a, hl, stream);
    case 32: return launch_typed<T, D, 32, FUSED, GS, F8>(a, hl, stream);
    default: return cudaErrorInvalidValue;
  }
}

template <typename T, bool FUSED, int GS, bool F8>
cudaError_t dispatch_dim(const DecodeArgs& a, const HeadLayout& hl, cudaStream_t stream) {
  switch (a.head_dim) {
    case 64: return dispatch_block<T, 64, FUSED, GS, F8>(a, hl, stream);
    case 128: return dispatch_block<T, 128, FUSED, GS, F8>(a, hl, stream);
    default: return cudaErrorInvalidValue;
  }
}

template <typename T>
cudaError_t dispatch_heads(const DecodeArgs& a, const HeadLayout& hl, cudaStream_t stream) {
  if (a.fp8) {  // 8-bit cache; query heads per unit as for 16-bit
    if (a.slot_mapping)  // one-launch step: multi-head only
      return hl.gs == 1 ? dispatch_dim<T, true, 1, true>(a, hl, stream) : cudaErrorInvalidValue;
    switch (hl.gs) {
      case 1: return dispatch_dim<T, false, 1, true>(a, hl, stream);
      case 2: return dispatch_dim<T, false, 2, true>(a, hl, stream);
      case 4: return dispatch_dim<T, false, 4, true>(a, hl, stream);
      default: return cudaErrorInvalidValue;
    }
  }
  if (a.slot_mapping)  // fused decode step: multi-head only
    return hl.gs == 1 ? dispatch_dim<T, true, 1, false>(a, hl, stream) : cudaErrorInvalidValue;
  switch (hl.gs) {
    case 1: return dispatch_dim<T, false, 1, false>(a, hl, stream);
    case 2: return dispatch_dim<T, false, 2, false>(a, hl, stream);
    case 4: return dispatch_dim<T, false, 4, false>(a, hl, stream);
    default: return cudaErrorInvalidValue;
  }
}

template <int D, bool FUSED, int GS, bool F8>
const void* kernel_for(int block_size, bool bf16) {
  switch (block_size) {
    case 4: return bf16 ? decode_kernel_ptr<__nv_bfloat16, D, 4, FUSED, GS, F8>() : decode_kernel_ptr<__half, D, 4, FUSED, GS, F8>();
    case 8: return bf16 ? decode_kernel_ptr<__nv_bfloat16, D, 8, FUSED, GS, F8>() : decode_kernel_ptr<__half, D, 8, FUSED, GS, F8>();
    case 16: return bf16 ? decode_kernel_ptr<__nv_bfloat16, D, 16, FUSED, GS, F8>() : decode_kernel_ptr<__half, D, 16, FUSED, GS, F8>();
    case 32: return bf16 ? decode_kernel_ptr<__nv_bfloat16, D, 32, FUSED, GS, F8>() : decode_kernel_ptr<__half, D, 32, FUSED, GS, F8>();
    default: return nullptr;
  }
}

template <int D>
const void* kernel_for_variant(int block_size, bool bf16, bool fused, int gs, bool fp8) {
  if (fp8) {
    if (fused) return gs == 1 ? kernel_for<D, true, 1, true>(block_size, bf16) : nullptr;
    switch (gs) {
      case 1: return kernel_for<D, false, 1, true>(block_size, bf16);
      case 2: return kernel_for<D, false, 2, true>(block_size, bf16);
      case 4: return kernel_for<D, false, 4, true>(block_size, bf16);
      default: return nullptr;
    }
  }
  if (fused) return gs == 1 ? kernel_for<D, true, 1, false>(block_size, bf16) : nullptr;
  switch (gs) {
    case 1: return kernel_for<D, false, 1, false>(block_size, bf16);
    case 2: return kernel_for<D, false, 2, false>(block_size, bf16);
    case 4: return kernel_for<D, false, 4, false>(block_size, bf16);
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
                              int block_size, int max_blocks_per_seq, int64_t forced_warps,
                              bool with_fp8) {
  if (!decode_sizes_supported(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                              max_blocks_per_seq))
    return 0;
  const HeadLayout hl = head_layout(num_heads, num_kv_heads);
  int64_t warps = 0;
  // every kernel these sizes may run: fp16 / bf16, two calls / one launch,
  // 16-bit / 8-bit cache
  for (int variant = 0; variant < 8; ++variant) {
    const bool bf16 = variant & 1, fused = variant & 2, fp8 = variant & 4;
    if (fused && hl.gs != 1) continue;
    if (fp8 && !with_fp8) continue;
    const void* k = head_dim == 128 ? kernel_for_variant<128>(block_size, bf16, fused, hl.gs, fp8)
                                    : kernel_for_variant<64>(block_size, bf16, fused, hl.gs, fp8);
    const Plan pl = plan_variant(k, head_dim, block_size, num_seqs, hl.vheads, max_blocks_per_seq,
                                 forced_warps, hl.gs, fp8);
    if (pl.grid <= 0) return 0;
    if (pl.work_warps > warps) warps = pl.work_warps;
  }
  const int64_t segs = static_cast<int64_t>(num_seqs) * hl.vheads;
  size_t bytes =
      header_bytes(num_seqs) + kGrabBytes + records_bytes(max_units(warps) + segs, head_dim, hl.gs);
  // The 8-bit cache may run on the tensor-core kernel: size for it too.
  if (with_fp8 && head_dim == 128 && (block_size == 8 || block_size == 16 || block_size == 32)) {
    const size_t f8 = mma_fp8_workspace_bytes(num_seqs, num_heads, num_kv_heads, block_size,
                                              max_blocks_per_seq, forced_warps);
    if (f8 == 0) return 0;
    if (f8 > bytes) bytes = f8;
  }
  // Grouped-query shapes may run on either kernel: size for both.
  if (mma_decode_shape_ok(num_heads, num_kv_heads, head_dim, block_size)) {
    const size_t mma = mma_decode_workspace_bytes(num_seqs, num_heads, num_kv_heads, head_dim,
                                                  block_size, max_blocks_per_seq, forced_warps);
    if (mma == 0) return 0;
    if (mma > bytes) bytes = mma;
  }
  return bytes;
}

DecodeLayout decode_layout(const DecodeArgs& a) {
  // the same choice of kernel as launch_paged_attn_decode below
  if (a.fp8 && mma_fp8_decode_ok(a) && option_fp8_kernel() != 1)
    return mma_fp8_layout(a.num_heads, a.num_kv_heads);
  const int64_t mode = option_gqa_kernel();
  const bool mma_ok = !a.slot_mapping && !a.fp8 &&
                      mma_decode_shape_ok(a.num_heads, a.num_kv_heads, a.head_dim, a.block_size) &&
                      mma_decode_pool_ok(a.num_kv_heads, a.block_size, a.num_blocks);
  if (mma_ok && mode != 1) return mma_decode_layout(a.num_heads, a.num_kv_heads);
  const HeadLayout hl = head_layout(a.num_heads, a.num_kv_heads);
  return DecodeLayout{hl.nsub, hl.gs, hl.vheads};
}

cudaError_t launch_paged_attn_decode(const DecodeArgs& a, cudaStream_t stream) {
  if (!decode_sizes_supported(a.num_seqs, a.num_heads, a.num_kv_heads, a.head_dim, a.block_size,
                              a.max_blocks_per_seq))
    return cudaErrorInvalidValue;
  // 8-bit cache: tensor cores unless PA_OPT_FP8_KERNEL asks for the CUDA
  // cores (or the query type, shape or pool does not suit them).
  if (a.fp8) {
    const int64_t f8mode = option_fp8_kernel();
    const bool f8_ok = mma_fp8_decode_ok(a);
    if (f8mode == 2 && !f8_ok) return cudaErrorInvalidValue;
    if (f8_ok && f8mode != 1) return launch_paged_attn_decode_mma_fp8(a, stream);
  }
  // Grouped-query attention: tensor cores unless PA_OPT_GQA_KERNEL asks for
  // the CUDA cores (or the shape or pool does not suit them).
  const int64_t mode = option_gqa_kernel();
  const bool mma_ok = !a.slot_mapping && !a.fp8 &&
                      mma_decode_shape_ok(a.num_heads, a.num_kv_heads, a.head_dim, a.block_size) &&
                      mma_decode_pool_ok(a.num_kv_heads, a.block_size, a.num_blocks);
  if (mode == 2 && !mma_ok) return cudaErrorInvalidValue;
  if (mma_ok && mode != 1) return launch_paged_attn_decode_mma(a, stream);
  const HeadLayout hl = head_layout(a.num_heads, a.num_kv_heads);
  return a.is_bf16 ? dispatch_heads<__nv_bfloat16>(a, hl, stream)
                   : dispatch_heads<__half>(a, hl, stream);
}

}  // namespace pa
