// paged_attn_decode_mma: grouped-query decode attention on the tensor cores.
//
// What it computes ("The KV Cache and PagedAttention", sections "The Block
// Table" and "What Came After"): for text s and query head h, the new query
// attends over the text's L_s stored keys and values of key/value head h / G
// (G query heads share one key/value head); token t lives in physical block
// block_tables[s][t / B] at place t % B:
//     out[s][h] = sum_t softmax_t(scale * q[s][h] . K_t[h / G]) * V_t[h / G].
//
// Why tensor cores here: with G query heads per key/value head every key and
// value row is used G times, so the arithmetic per HBM byte is G times that
// of multi-head decode (8 flops per byte at G = 8).  On the CUDA cores that
// work, with its conversions and shuffles, takes longer than streaming the
// bytes; as a pair of small matrix products it costs the tensor cores almost
// nothing, and the kernel is again bound by HBM.  The products are the
// warp-level mma.sync m16n8k16 (fp16 or bf16 in, fp32 accumulate): the tiles
// are one warp's 16-token chunk against at most 16 query heads, too small for
// the CTA-wide tcgen05 shapes, whose accumulators and 128-row tiles would
// need many warps' chunks gathered per step and add a TMEM round trip to
// every chunk without raising a bound that is not the tensor pipe's.
//
// Per chunk of CH tokens (16 at head_dim 128, 32 at head_dim 64) and the GS
// query heads of one work unit (GS <= 16, padded to 8 or 16 columns):
//   * S^T = K Q^T: tokens are the 16 rows of the product and query heads its
//     columns, so a group of 8 heads fills a column tile exactly.  K comes
//     from shared memory through ldmatrix; Q^T stays in registers for the
//     whole (text, head) run.
//   * online softmax in base 2 per column (head): a running max m and sum l
//     per head; m is raised (a reduction over the 8 lanes that hold a head's
//     tokens, and a rescale) only when a score passes it by more than 2^8,
//     which one warp vote detects.
//   * O^T += V^T P^T: head_dim is the row dimension; V^T is read with the
//     transposing ldmatrix; P^T is the S^T accumulator transposed in
//     registers (movmatrix), 8x8 at a time, as the sum of two input-type
//     values (about 16 significant bits; both parts go through the product).
// Keys and values reach shared memory by 2-D tiled TMA loads with the
// 128-byte swizzle (each 128-byte row's 16-byte pieces permuted by the row
// index), so the 8 rows an ldmatrix reads at once lie in distinct banks.
// Everything else is shared with the CUDA-core kernel: the flat chunk order,
// static runs then grains, partial records and the log-sum-exp merge kernel,
// bounded waits, programmatic dependent launch.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "decode_common.cuh"
#include "kernels.h"
#include "mma_ptx.cuh"

namespace pa {

#ifndef PA_DECODE_SPLIT_P_F16
#define PA_DECODE_SPLIT_P_F16 0
#endif
// 1: fp16 weights also enter the value products as P_hi + P_lo
constexpr bool kSplitPF16 = PA_DECODE_SPLIT_P_F16 != 0;

namespace {

#ifndef PA_MMA_WARPS
#define PA_MMA_WARPS 4
#endif
#ifndef PA_MMA_STAGES
#define PA_MMA_STAGES 2
#endif
constexpr int kMmaWarps = PA_MMA_WARPS;    // warps per CTA
constexpr int kMmaStages = PA_MMA_STAGES;  // ring depth per warp

// One stage: the K tile (CH rows x head_dim, 4 KB), the V tile (4 KB), then
// the unit's query rows (8 * NT rows x head_dim).  Every tile starts on a
// 1024-byte boundary, where the 128-byte swizzle pattern starts.
__host__ __device__ constexpr int mma_stage_bytes(int D, int nt) { return 8192 + 8 * nt * D * 2; }
__host__ __device__ constexpr int mma_warp_bytes(int D, int stages, int nt) {
  return stages * mma_stage_bytes(D, nt) + 1024;  // + barriers and flags
}

// Address of element (t, d) (d a multiple of 8) of a swizzled tile of CH rows:
// head_dim is split into 64-element halves, each CH rows of 128 bytes, and
// 16-byte piece c of row t sits at piece c ^ (t % 8).
template <int CH>
__device__ __forceinline__ uint32_t swz(uint32_t tile, int t, int d) {
  return tile + (d >> 6) * (CH * 128) + t * 128 + ((((d & 63) >> 3) ^ (t & 7)) << 4);
}

template <typename T, int D, int B, int WARPS, int STAGES, int NT>
__global__ void __launch_bounds__(WARPS * 32, 2)
paged_decode_mma_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v) {
  constexpr int CH = chunk_tokens(D);         // tokens per chunk
  constexpr int NB = CH >= B ? CH / B : 1;    // physical blocks a chunk touches
  constexpr int R = CH >= B ? B : CH;         // rows per TMA box
  constexpr int HALVES = D / 64;              // 64-element (128-byte) column boxes
  constexpr int TM = CH / 16;                 // 16-token tiles per chunk
  constexpr int KD = D / 16;                  // 16-wide head_dim steps
  constexpr int STRIDE = mma_stage_bytes(D, NT);
  constexpr int AREA = mma_warp_bytes(D, STAGES, NT);
  constexpr uint32_t BOX_BYTES = 64 * R * 2;
  static_assert(CH % 16 == 0 && (CH % B == 0 || B % CH == 0) && B >= 8, "shape");
  static_assert(STRIDE % 1024 == 0 && AREA % 1024 == 0, "swizzle alignment");

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // The swizzle is a function of the shared-memory address: align by hand.
  uint8_t* smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
  int32_t* prefix = reinterpret_cast<int32_t*>(smem + WARPS * AREA);
  __shared__ int32_t warp_tot[WARPS];

  const int Hq = p.num_q_heads, Hkv = p.num_kv_heads, NSUB = p.nsub, GS = p.gs;
  const int G = Hq / Hkv;
  // virtual head -> key/value head and first query head (one subset per
  // key/value head, the usual case, needs no division)
  auto kv_head = [&](int vh) { return NSUB == 1 ? vh : vh / NSUB; };
  auto q_head0 = [&](int vh) { return NSUB == 1 ? vh * G : (vh / NSUB) * G + (vh % NSUB) * GS; };
  const int cap = p.max_blocks_per_seq * B;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;

  if (lane == 0) {
    prefetch_tensor_map(&tm_k);
    prefetch_tensor_map(&tm_v);
  }
  // Inputs may come from the kernel launched just before (the cache write).
  griddep_wait();
  // A shared-prefix pass lets the tail pass after it start on SMs it leaves.
  if (p.cascade) griddep_launch_dependents();

  const WorkSplit sp = decode_prologue<T, D, CH, WARPS * 32>(p, prefix, warp_tot, cap);
  const int W = sp.W;
  const int w = blockIdx.x * WARPS + warp;
  if (w >= W || sp.total == 0) return;

  uint8_t* area = smem + warp * AREA;
  uint64_t* bars = reinterpret_cast<uint64_t*>(area + STAGES * STRIDE);
  int32_t* flags = reinterpret_cast<int32_t*>(bars + STAGES);
  // Query rows past GS are never copied; give them zeros once.
  for (int st = 0; st < STAGES; ++st) {
    uint4* qz = reinterpret_cast<uint4*>(area + st * STRIDE + 8192);
    for (int i = lane; i < 8 * NT * D * 2 / 16; i += 32) qz[i] = make_uint4(0u, 0u, 0u, 0u);
  }
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
#pragma unroll
    for (int st = 0; st < STAGES; ++st) mbar_init(&bars[st], 1);
    fence_barrier_init();
  }
  __syncwarp();

  const uint64_t policy = l2_evict_first_policy();
  const T* __restrict__ qg = static_cast<const T*>(p.q);

  Scheduler<CH, B, NB> sched(p, prefix, sp, w, lane);
  int ws0, wc0, wu0, ws1, wc1, wu1;
  sched.next_window(ws0, wc0, wu0);
  sched.next_window(ws1, wc1, wu1);
  Lookahead<NB> win0 = sched.lookahead(ws0, wc0);
  Lookahead<NB> win1 = sched.lookahead(ws1, wc1);
  int i0 = 0;      // consumer's index in window 0
  int issued = 0;  // chunks whose copies were issued (stage = issued % STAGES)

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
    for (int b = 0; b < NB; ++b) blk[b] = __shfl_sync(0xffffffffu, hi ? win1.blk[b] : win0.blk[b], src);
    const int st = issued % STAGES;
    ++issued;
    if (lane == 0) {
      uint8_t* stage = area + st * STRIDE;
      uint8_t* sK = stage;
      uint8_t* sV = stage + 4096;
      uint8_t* sQ = stage + 8192;
      const int len = min(max(len_raw, 0), cap);
      const int nvalid = min(CH, len - j * CH);
      const bool first = unit_start || j == 0;
      bool bad = false;
      int boxes = 0;
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const int rows = (CH >= B) ? min(B, nvalid - b * B) : nvalid;
        if (rows > 0) {
          ++boxes;
          if (blk[b] < 0 || blk[b] >= p.num_blocks) bad = true;
        }
      }
      if (bad) set_status(p.status, -7 /* PA_ERR_BAD_BLOCK */);
      flags[st] = bad ? 1 : 0;
      fence_proxy_async_smem();
      const uint32_t qbytes = first ? GS * D * 2 : 0;
      const uint32_t kvbytes = bad ? 0 : 2u * HALVES * boxes * BOX_BYTES;
      mbar_arrive_expect_tx(&bars[st], qbytes + kvbytes);
      if (first) {
        if (!p.cascade) {
          bulk_copy_g2s(sQ, qg + (static_cast<int64_t>(s) * Hq + q_head0(h)) * D, GS * D * 2,
                        &bars[st], policy);
        } else {
          // Shared-prefix pass: the columns of group s's key/value head
          // kv_head(h) are its (text, query head) pairs, text-major, in
          // NSUB subsets of GS; this unit has subset h % NSUB.  Column c is
          // text c / G of the group and query head kv_head(h) * G + c % G.
          const int sub = NSUB == 1 ? 0 : h % NSUB;
          const int64_t text0 = static_cast<int64_t>(s) * (GS * NSUB / G);
          for (int g = 0; g < GS; ++g) {
            const int c = sub * GS + g;
            const int64_t text = text0 + c / G;
            const int qh = kv_head(h) * G + c % G;
            bulk_copy_g2s(sQ + g * D * 2, qg + (text * Hq + qh) * D, D * 2, &bars[st], policy);
          }
        }
      }
      if (!bad) {
        const int kvh = kv_head(h);
        const int row0 = CH >= B ? 0 : (j * CH) % B;
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          const int rows = (CH >= B) ? min(B, nvalid - b * B) : nvalid;
          if (rows > 0) {
            const int y = (blk[b] * Hkv + kvh) * B + row0;
#pragma unroll
            for (int hf = 0; hf < HALVES; ++hf) {
              tma_load_2d(sK + hf * CH * 128 + b * R * 128, &tm_k, hf * 64, y, &bars[st], policy);
              tma_load_2d(sV + hf * CH * 128 + b * R * 128, &tm_v, hf * 64, y, &bars[st], policy);
            }
          }
        }
      }
    }
  };

#pragma unroll
  for (int k = 0; k < STAGES; ++k) issue(k);

  // Per-lane fragments.  Column (head) c of a tile is held by lanes with
  // lane % 4 == c / 2; row r by lanes with lane / 4 == r % 8.
  uint32_t qf[KD][NT][2];  // Q^T operand, per 16-wide head_dim step
  float o[KD][NT][4];      // O^T accumulators: rows head_dim, columns heads
  float m[NT][2], l[NT][2];
  int piece_j0 = 0;
  int prev_unit = -1;
  const float scale = p.qk_scale_log2;

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

    const uint32_t sK = smem_addr(area + st * STRIDE);
    const uint32_t sV = sK + 4096;
    const uint32_t sQ = sK + 8192;
    const int bad = flags[st];

    if (j == 0 || wu0 != prev_unit) {
      piece_j0 = j;
      // Q^T fragments: lane gives row (head) nt*8 + lane % 8 at column
      // (head_dim) ks*16 + (lane / 8) * 8, covering steps ks and ks + 1.
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int ks = 0; ks < KD; ks += 2) {
          uint32_t r[4];
          ldsm_x4(sQ + ((nt * 8 + (lane & 7)) * D + ks * 16 + (lane >> 3) * 8) * 2, r);
          qf[ks][nt][0] = r[0];
          qf[ks][nt][1] = r[1];
          qf[ks + 1][nt][0] = r[2];
          qf[ks + 1][nt][1] = r[3];
        }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          m[nt][e] = -INFINITY;
          l[nt][e] = 0.f;
        }
#pragma unroll
        for (int md = 0; md < KD; ++md)
#pragma unroll
          for (int c = 0; c < 4; ++c) o[md][nt][c] = 0.f;
      }
    }
    const int nvalid = bad ? 0 : min(CH, len - j * CH);

    // ---- S^T = K Q^T (rows: tokens, columns: heads) ----
    // With one token tile the head_dim steps alternate between two
    // accumulators, halving the chain of dependent products.
    constexpr int ACC = TM == 1 ? 2 : 1;
    float sa[ACC][TM][NT][4];
#pragma unroll
    for (int x = 0; x < ACC; ++x)
#pragma unroll
      for (int mt = 0; mt < TM; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int c = 0; c < 4; ++c) sa[x][mt][nt][c] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KD; ++ks)
#pragma unroll
      for (int mt = 0; mt < TM; ++mt) {
        uint32_t a[4];
        ldsm_x4(swz<CH>(sK, mt * 16 + ((lane >> 3) & 1) * 8 + (lane & 7), ks * 16 + (lane >> 4) * 8),
                a);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          mma_16816<T>(sa[ks % ACC][mt][nt], a, qf[ks][nt][0], qf[ks][nt][1]);
      }

    // ---- online softmax per head (base 2) ----
    // Scores become base-2 logits; tokens past nvalid get -inf.
    const int r0 = lane >> 2;  // token row of c0, c1 (c2, c3: r0 + 8)
    float sc[TM][NT][4];
#pragma unroll
    for (int mt = 0; mt < TM; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int t = mt * 16 + r0 + (c >> 1) * 8;
          float v = sa[0][mt][nt][c];
          if constexpr (ACC == 2) v += sa[1][mt][nt][c];
          sc[mt][nt][c] = t < nvalid ? v * scale : -INFINITY;
        }
    // The running max m of a head is only raised when a score passes it by
    // more than kSlack: weights 2^(s - m) then stay below 2^kSlack, and the
    // usual case (no score that high) needs one warp vote instead of a
    // reduction across lanes and a rescale of the accumulators.  Any m gives
    // the same softmax; m, l and o stay consistent with each other.
    constexpr float kSlack = 8.f;
    float cm[NT][2];
    bool raise = false;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float x = -INFINITY;
#pragma unroll
        for (int mt = 0; mt < TM; ++mt) x = fmaxf(x, fmaxf(sc[mt][nt][e], sc[mt][nt][2 + e]));
        cm[nt][e] = x;
        raise |= x > m[nt][e] + kSlack;
      }
    if (__any_sync(0xffffffffu, raise)) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float x = cm[nt][e];
          x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 4));
          x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 8));
          x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 16));
          const float m_new = fmaxf(m[nt][e], x);
          // m_new == m (incl. both -inf) leaves everything as it is
          const float alpha = m_new == m[nt][e] ? 1.f : fast_exp2(m[nt][e] - m_new);
          l[nt][e] *= alpha;
#pragma unroll
          for (int md = 0; md < KD; ++md) {
            o[md][nt][e] *= alpha;
            o[md][nt][2 + e] *= alpha;
          }
          m[nt][e] = m_new;
        }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        // m == -inf: every score so far is -inf, every weight 0
        const float mm = m[nt][e] == -INFINITY ? 0.f : m[nt][e];
        float psum = 0.f;
#pragma unroll
        for (int mt = 0; mt < TM; ++mt) {
          sc[mt][nt][e] = fast_exp2(sc[mt][nt][e] - mm);
          sc[mt][nt][2 + e] = fast_exp2(sc[mt][nt][2 + e] - mm);
          psum += sc[mt][nt][e] + sc[mt][nt][2 + e];
        }
        l[nt][e] += psum;
      }

    // ---- O^T += V^T P^T ----
    // P^T operand of token tile mt: rows 0-7 and 8-15 of S^T, each an 8x8
    // block transposed in registers.  For bf16 the weights are kept as the
    // sum of two bf16 values, P = P_hi + P_lo (P_hi = P rounded, P_lo = the
    // rest rounded), about 16 significant bits, and both parts are applied:
    // one bf16 value alone (8 bits) can cost more than the fp32 contract's
    // error where the weighted values nearly cancel.  fp16 weights (11 bits)
    // enter once (PA_DECODE_SPLIT_P_F16=1 splits them too).
    constexpr bool SPLIT = std::is_same<T, __nv_bfloat16>::value || kSplitPF16;
    uint32_t pb[TM][NT][2], pl[TM][NT][SPLIT ? 2 : 1];
#pragma unroll
    for (int mt = 0; mt < TM; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const float x0 = sc[mt][nt][2 * r], x1 = sc[mt][nt][2 * r + 1];
          const uint32_t hi = Elem<T>::from_float2(x0, x1);
          const float2 back = Elem<T>::to_float2(hi);
          pb[mt][nt][r] = movmatrix_trans(hi);
          if constexpr (SPLIT)
            pl[mt][nt][r] = movmatrix_trans(Elem<T>::from_float2(x0 - back.x, x1 - back.y));
        }
    // Tokens past nvalid hold whatever the pool has there (possibly NaN);
    // their weights are zero, but 0 * NaN is not, so zero those V elements.
    const int tq = (lane & 3) * 2;
#pragma unroll
    for (int mt = 0; mt < TM; ++mt) {
      const bool tail = nvalid < (mt + 1) * 16;  // warp-uniform
      uint32_t mask_lo = 0xffffffffu, mask_hi = 0xffffffffu;
      if (tail) {
        const int t0 = mt * 16 + tq;
        mask_lo = (t0 < nvalid ? 0x0000ffffu : 0u) | (t0 + 1 < nvalid ? 0xffff0000u : 0u);
        mask_hi = (t0 + 8 < nvalid ? 0x0000ffffu : 0u) | (t0 + 9 < nvalid ? 0xffff0000u : 0u);
      }
#pragma unroll
      for (int md = 0; md < KD; ++md) {
        uint32_t a[4];
        ldsm_x4_trans(swz<CH>(sV, mt * 16 + (lane >> 4) * 8 + (lane & 7), md * 16 + ((lane >> 3) & 1) * 8),
                      a);
        if (tail) {
          a[0] &= mask_lo;
          a[1] &= mask_lo;
          a[2] &= mask_hi;
          a[3] &= mask_hi;
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          mma_16816<T>(o[md][nt], a, pb[mt][nt][0], pb[mt][nt][1]);
          if constexpr (SPLIT) mma_16816<T>(o[md][nt], a, pl[mt][nt][0], pl[mt][nt][1]);
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
      const int64_t sh = static_cast<int64_t>(s) * p.num_heads + h;  // (text, virtual head)
      const int64_t qrow = static_cast<int64_t>(s) * Hq + q_head0(h);  // first query head
      const bool whole = piece_j0 == 0 && j == ns - 1 && !p.cascade;
      float lt[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float v = l[nt][e];
          v += __shfl_xor_sync(0xffffffffu, v, 4);
          v += __shfl_xor_sync(0xffffffffu, v, 8);
          v += __shfl_xor_sync(0xffffffffu, v, 16);
          lt[nt][e] = v;
        }
      if (whole) {
        // Normalise, then transpose 8x8 blocks so that each lane holds two
        // consecutive head_dim entries of one head: row lane / 4.
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const float i0v = lt[nt][0] > 0.f ? 1.f / lt[nt][0] : 0.f;
          const float i1v = lt[nt][1] > 0.f ? 1.f / lt[nt][1] : 0.f;
          const int g = nt * 8 + r0;
          T* orow = static_cast<T*>(p.out) + (qrow + g) * D;
#pragma unroll
          for (int md = 0; md < KD; ++md) {
            const uint32_t lo =
                movmatrix_trans(Elem<T>::from_float2(o[md][nt][0] * i0v, o[md][nt][1] * i1v));
            const uint32_t hi =
                movmatrix_trans(Elem<T>::from_float2(o[md][nt][2] * i0v, o[md][nt][3] * i1v));
            if (g < GS) {
              *reinterpret_cast<uint32_t*>(orow + md * 16 + tq) = lo;
              *reinterpret_cast<uint32_t*>(orow + md * 16 + 8 + tq) = hi;
            }
          }
        }
      } else {
        float* recs = p.records + (static_cast<int64_t>(wu0) + sh) * (GS * (D + 4));
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int g = nt * 8 + tq + e;
            if (g < GS) {
              float* rec = recs + g * (D + 4);
              if (r0 == 0) {
                rec[0] = m[nt][e];
                rec[1] = lt[nt][e];
              }
#pragma unroll
              for (int md = 0; md < KD; ++md) {
                rec[4 + md * 16 + r0] = o[md][nt][e];
                rec[4 + md * 16 + 8 + r0] = o[md][nt][2 + e];
              }
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
      sched.next_window(ws1, wc1, wu1);
      win1 = sched.lookahead(ws1, wc1);
      i0 = 0;
    }
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

size_t mma_smem_bytes(int D, int num_seqs, int nt) {
  return 1024 /* alignment slack */ +
         static_cast<size_t>(kMmaWarps) * mma_warp_bytes(D, kMmaStages, nt) +
         align_up(sizeof(int32_t) * (num_seqs + 1), 16);
}

// A key/value head's G query heads are split into nsub subsets of gs <= 16
// (the fewest subsets whose size divides G); columns are padded to 8 or 16.
HeadLayout mma_head_layout(int num_heads, int num_kv_heads) {
  HeadLayout l;
  if (num_kv_heads < 1 || num_heads < 1 || num_heads % num_kv_heads) return l;
  l.group = num_heads / num_kv_heads;
  int nsub = (l.group + 15) / 16;
  while (l.group % nsub) ++nsub;
  l.nsub = nsub;
  l.gs = l.group / nsub;
  l.vheads = num_kv_heads * nsub;
  return l;
}

int column_tiles(int gs) { return gs > 8 ? 2 : 1; }

// The pool [num_blocks][Hkv][B][D] seen as a 2-D tensor of num_blocks*Hkv*B
// rows of D elements; boxes of 64 elements (128 bytes) x `rows` rows with the
// 128-byte swizzle.
bool encode_pool_map(CUtensorMap* map, const void* pool, bool bf16, int64_t rows, int D,
                     int box_rows) {
  const uint64_t dims[2] = {static_cast<uint64_t>(D), static_cast<uint64_t>(rows)};
  const uint64_t strides[1] = {static_cast<uint64_t>(D) * 2};
  const uint32_t box[2] = {64u, static_cast<uint32_t>(box_rows)};
  return encode_swizzled_map(map, pool, bf16, 2, dims, strides, box);
}

template <typename T, int D, int B, int NT>
const void* mma_kernel_ptr() {
  return reinterpret_cast<const void*>(
      &paged_decode_mma_kernel<T, D, B, kMmaWarps, kMmaStages, NT>);
}

Plan plan_mma(const void* kernel, int D, int B, int num_seqs, int vheads, int max_blocks_per_seq,
              int64_t forced_warps, int nt) {
  return plan_decode(kernel, mma_smem_bytes(D, num_seqs, nt), mma_smem_bytes(D, kMaxSeqs, nt),
                     kMmaWarps, chunk_tokens(D), B, num_seqs, vheads, max_blocks_per_seq,
                     forced_warps);
}

template <typename T, int D, int B, int NT>
cudaError_t launch_mma_typed(const DecodeArgs& a, const HeadLayout& hl, cudaStream_t stream) {
  const Plan pl = plan_mma(mma_kernel_ptr<T, D, B, NT>(), D, B, a.num_seqs, hl.vheads,
                           a.max_blocks_per_seq, a.forced_warps, NT);
  if (pl.grid <= 0) return cudaErrorInvalidConfiguration;
  const int64_t segs = static_cast<int64_t>(a.num_seqs) * hl.vheads;
  const size_t need = header_bytes(a.num_seqs) + kGrabBytes +
                      records_bytes(max_units(pl.work_warps) + segs, D, hl.gs);
  if (a.workspace_bytes < need) return cudaErrorInvalidValue;
  constexpr int CH = chunk_tokens(D);
  const int64_t rows = a.num_blocks * a.num_kv_heads * B;
  CUtensorMap tm_k, tm_v;
  if (!encode_pool_map(&tm_k, a.k_cache, a.is_bf16, rows, D, CH >= B ? B : CH) ||
      !encode_pool_map(&tm_v, a.v_cache, a.is_bf16, rows, D, CH >= B ? B : CH))
    return cudaErrorInvalidValue;
  DecodeParams p;
  p.out = a.out;
  p.q = a.q;
  p.k_cache = a.k_cache;
  p.v_cache = a.v_cache;
  p.block_tables = a.block_tables;
  p.context_lens = a.context_lens;
  p.qk_scale_log2 = a.scale * 1.4426950408889634f;  // log2(e)
  p.v_scale = 1.f;
  p.num_seqs = a.num_seqs;
  p.num_heads = hl.vheads;
  p.num_q_heads = a.num_heads;
  p.num_kv_heads = a.num_kv_heads;
  p.nsub = hl.nsub;
  p.gs = hl.gs;
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
  p.k_new = nullptr;
  p.v_new = nullptr;
  p.slot_mapping = nullptr;
  p.cascade = a.cascade ? 1 : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.grid);
  cfg.blockDim = dim3(kMmaWarps * 32);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t err = cudaLaunchKernelEx(
      &cfg, paged_decode_mma_kernel<T, D, B, kMmaWarps, kMmaStages, NT>, p, tm_k, tm_v);
  if (err != cudaSuccess) return err;
  if (p.cascade) return cudaGetLastError();  // the caller merges
  err = launch_merge<T, D>(p, hl.gs, stream);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

template <typename T, int D, int NT>
cudaError_t mma_dispatch_block(const DecodeArgs& a, const HeadLayout& hl, cudaStream_t stream) {
  switch (a.block_size) {
    case 8: return launch_mma_typed<T, D, 8, NT>(a, hl, stream);
    case 16: return launch_mma_typed<T, D, 16, NT>(a, hl, stream);
    case 32: return launch_mma_typed<T, D, 32, NT>(a, hl, stream);
    default: return cudaErrorInvalidValue;
  }
}

template <typename T>
cudaError_t mma_dispatch(const DecodeArgs& a, const HeadLayout& hl, cudaStream_t stream) {
  const int nt = column_tiles(hl.gs);
  if (a.head_dim == 128)
    return nt == 1 ? mma_dispatch_block<T, 128, 1>(a, hl, stream)
                   : mma_dispatch_block<T, 128, 2>(a, hl, stream);
  if (a.head_dim == 64)
    return nt == 1 ? mma_dispatch_block<T, 64, 1>(a, hl, stream)
                   : mma_dispatch_block<T, 64, 2>(a, hl, stream);
  return cudaErrorInvalidValue;
}

template <int D, int NT>
const void* mma_kernel_for(int block_size, bool bf16) {
  switch (block_size) {
    case 8: return bf16 ? mma_kernel_ptr<__nv_bfloat16, D, 8, NT>() : mma_kernel_ptr<__half, D, 8, NT>();
    case 16: return bf16 ? mma_kernel_ptr<__nv_bfloat16, D, 16, NT>() : mma_kernel_ptr<__half, D, 16, NT>();
    case 32: return bf16 ? mma_kernel_ptr<__nv_bfloat16, D, 32, NT>() : mma_kernel_ptr<__half, D, 32, NT>();
    default: return nullptr;
  }
}

}  // namespace

bool mma_decode_shape_ok(int num_heads, int num_kv_heads, int head_dim, int block_size) {
  if (num_kv_heads < 1 || num_heads < 1 || num_heads % num_kv_heads) return false;
  if (num_heads == num_kv_heads) return false;  // multi-head: the CUDA-core kernel
  if (head_dim != 64 && head_dim != 128) return false;
  return block_size == 8 || block_size == 16 || block_size == 32;
}

bool mma_decode_pool_ok(int num_kv_heads, int block_size, int64_t num_blocks) {
  // TMA row coordinates are 32-bit.
  return num_blocks > 0 && num_blocks * num_kv_heads * block_size < (int64_t{1} << 31);
}

namespace {

size_t mma_workspace_for(int num_seqs, const HeadLayout& hl, int head_dim, int block_size,
                         int max_blocks_per_seq, int64_t forced_warps) {
  if (hl.vheads < 1) return 0;
  const int nt = column_tiles(hl.gs);
  int64_t warps = 0;
  for (int bf16 = 0; bf16 < 2; ++bf16) {
    const void* k = head_dim == 128
                        ? (nt == 1 ? mma_kernel_for<128, 1>(block_size, bf16)
                                   : mma_kernel_for<128, 2>(block_size, bf16))
                        : (nt == 1 ? mma_kernel_for<64, 1>(block_size, bf16)
                                   : mma_kernel_for<64, 2>(block_size, bf16));
    if (!k) return 0;
    const Plan pl = plan_mma(k, head_dim, block_size, num_seqs, hl.vheads, max_blocks_per_seq,
                             forced_warps, nt);
    if (pl.grid <= 0) return 0;
    if (pl.work_warps > warps) warps = pl.work_warps;
  }
  const int64_t segs = static_cast<int64_t>(num_seqs) * hl.vheads;
  return header_bytes(num_seqs) + kGrabBytes +
         records_bytes(max_units(warps) + segs, head_dim, hl.gs);
}

// The shared-prefix pass: one virtual text per group, one subset of
// `group_size` query columns (the group's texts) per head.
// Shared-prefix pass: the columns of a key/value head are the group's
// (text, query head) pairs, group_size * G of them; more than 16 are split
// into nsub subsets of gs <= 16 (the smallest count that divides them), one
// virtual head per (key/value head, subset), each reading the prefix once.
HeadLayout cascade_head_layout(int num_heads, int num_kv_heads, int group_size) {
  HeadLayout l;
  if (num_kv_heads < 1 || num_heads < 1 || num_heads % num_kv_heads || group_size < 1) return l;
  l.group = num_heads / num_kv_heads;
  const int cols = group_size * l.group;
  int nsub = (cols + 15) / 16;
  while (cols % nsub) ++nsub;
  l.nsub = nsub;
  l.gs = cols / nsub;
  l.vheads = num_kv_heads * nsub;
  return l;
}

}  // namespace

size_t mma_decode_workspace_bytes(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                  int block_size, int max_blocks_per_seq, int64_t forced_warps) {
  return mma_workspace_for(num_seqs, mma_head_layout(num_heads, num_kv_heads), head_dim,
                           block_size, max_blocks_per_seq, forced_warps);
}

bool mma_cascade_ok(int num_heads, int num_kv_heads, int group_size, int head_dim,
                    int block_size) {
  return num_heads >= 1 && num_kv_heads >= 1 && num_heads % num_kv_heads == 0 &&
         group_size >= 1 && group_size <= 1024 &&
         (head_dim == 64 || head_dim == 128) &&
         (block_size == 8 || block_size == 16 || block_size == 32);
}

size_t mma_cascade_workspace_bytes(int num_groups, int group_size, int num_heads,
                                   int num_kv_heads, int head_dim, int block_size,
                                   int max_blocks_per_seq, int64_t forced_warps) {
  if (!mma_cascade_ok(num_heads, num_kv_heads, group_size, head_dim, block_size)) return 0;
  return mma_workspace_for(num_groups, cascade_head_layout(num_heads, num_kv_heads, group_size),
                           head_dim, block_size, max_blocks_per_seq, forced_warps);
}

DecodeLayout mma_decode_layout(int num_heads, int num_kv_heads) {
  const HeadLayout l = mma_head_layout(num_heads, num_kv_heads);
  return DecodeLayout{l.nsub, l.gs, l.vheads};
}

DecodeLayout mma_cascade_layout(int num_heads, int num_kv_heads, int group_size) {
  const HeadLayout l = cascade_head_layout(num_heads, num_kv_heads, group_size);
  return DecodeLayout{l.nsub, l.gs, l.vheads};
}

cudaError_t launch_paged_attn_decode_mma_cascade(const DecodeArgs& a, int group_size,
                                                 cudaStream_t stream) {
  if (!a.cascade || a.slot_mapping || a.fp8 ||
      !mma_cascade_ok(a.num_heads, a.num_kv_heads, group_size, a.head_dim, a.block_size) ||
      !mma_decode_pool_ok(a.num_kv_heads, a.block_size, a.num_blocks))
    return cudaErrorInvalidValue;
  const HeadLayout hl = cascade_head_layout(a.num_heads, a.num_kv_heads, group_size);
  return a.is_bf16 ? mma_dispatch<__nv_bfloat16>(a, hl, stream)
                   : mma_dispatch<__half>(a, hl, stream);
}

cudaError_t launch_paged_attn_decode_mma(const DecodeArgs& a, cudaStream_t stream) {
  if (!mma_decode_shape_ok(a.num_heads, a.num_kv_heads, a.head_dim, a.block_size) ||
      !mma_decode_pool_ok(a.num_kv_heads, a.block_size, a.num_blocks) || a.slot_mapping)
    return cudaErrorInvalidValue;
  const HeadLayout hl = mma_head_layout(a.num_heads, a.num_kv_heads);
  return a.is_bf16 ? mma_dispatch<__nv_bfloat16>(a, hl, stream)
                   : mma_dispatch<__half>(a, hl, stream);
}

}  // namespace pa
