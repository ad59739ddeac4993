// paged_attn_decode_mma_fp8: decode attention over an 8-bit (E4M3) cache on
// the warp-level tensor cores, for fp16 queries and head_dim 128.
//
// What it computes ("The KV Cache and PagedAttention", sections "The Block
// Table" and "What Came After": one byte per stored number): for text s and
// head h, with Kc_t and Vc_t the values of token t's codes,
//     out[s][h] = v_scale * sum_t softmax_t(scale * k_scale * q . Kc_t) Vc_t,
// token t in physical block block_tables[s][t / B], place t % B.
//
// Why tensor cores for multi-head decode: per byte of cache the 8-bit path
// has twice the numbers of the 16-bit one to widen and multiply.  On the CUDA
// cores (lanes splitting a key row, shuffle-reduced dot products, fp32 FMAs
// per number) that work, not HBM, set the pace.  Here every product runs as
// mma.sync m16n8k16 (fp16 in, fp32 accumulate) on codes widened exactly to
// fp16 by cvt.rn.f16x2.e4m3x2; only the conversions stay on the CUDA cores.
// Multi-head: the single query is copied into all eight columns of the
// tile, so every lane's accumulators hold finished scores and outputs: no
// cross-lane reduction of dot products and no transpose of the scores.
// Grouped-query pools ("What Came After": heads that share a key/value set):
// the columns are the query heads of one key/value head (up to 8 per pass;
// a group of G in the fewest equal subsets of at most 8, a subset of gs < 8
// repeating its heads over the spare columns), so one read of the codes
// serves the whole subset; each lane then holds two columns' scores, keeps
// a running max and sum per column, and fetches its column's weights for
// the value products from the lane that computed them.
//
// A chunk is 32 tokens (4 KB of key codes, 4 KB of value codes), fetched by
// 2-D tiled TMA with the 128-byte swizzle (16-byte piece k of row r stored at
// piece k ^ (r % 8)).  Lane (g, c) = (lane / 4, lane % 4):
//   * S^T = K Q^T (rows: tokens, K dimension: head_dim).  A sum over head_dim
//     may visit the dimensions in any order if the query visits them in the
//     same one: the lane owns dimensions [32c, 32c + 32) of its two token
//     rows g, g + 8 (per 16-token tile), loaded as two 16-byte pieces each,
//     and step kk of the product takes dimensions 32c + 4kk .. + 3; the
//     lane's query fragment is the same 32 dimensions.  Rows g and g + 8
//     share a swizzle, and eight lanes of a load phase hit eight distinct
//     pieces, so the loads are free of bank conflicts.
//   * Online softmax in base 2 with a lazy running max (raised only when a
//     score passes it by more than 2^8); each lane holds the scores of tokens
//     g, g + 8, 16 + g, 24 + g.
//   * O^T += V^T P^T (rows: head_dim, K dimension: tokens).  The tokens may
//     be summed in any order too: K positions 2c, 2c + 1, 2c + 8, 2c + 9 of a
//     16-token tile take tokens 2c, 2c + 8, 2c + 1, 2c + 9, so a lane's P pair
//     comes whole from the lane that holds both scores (one shuffle per
//     pair), and the lane's four value rows fall into eight distinct pieces
//     per load phase.  The lane owns output dimensions [16g, 16g + 16): one
//     16-byte piece of each of its rows, bytes of two rows interleaved by
//     prmt into code pairs for cvt.  P enters rounded to fp16 (11
//     significant bits, as in the CUDA-core kernels; PA_DECODE_SPLIT_P_F16=1
//     applies P_hi + P_lo, about 22 bits, at twice the value products).
// Everything else (the flat chunk order, static runs then grains, partial
// records and the log-sum-exp merge, bounded waits, programmatic dependent
// launch) is shared with the other decode kernels.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "decode_common.cuh"
#include "fp8.cuh"
#include "kernels.h"
#include "mma_ptx.cuh"

namespace pa {

#ifndef PA_DECODE_SPLIT_P_F16
#define PA_DECODE_SPLIT_P_F16 0
#endif
// 1: the weights enter the value products as P_hi + P_lo
constexpr bool kSplitPF16 = PA_DECODE_SPLIT_P_F16 != 0;

namespace {

#ifndef PA_F8MMA_WARPS
#define PA_F8MMA_WARPS 4
#endif
#ifndef PA_F8MMA_STAGES
#define PA_F8MMA_STAGES 3
#endif
#ifndef PA_F8MMA_STAGES_GQA
#define PA_F8MMA_STAGES_GQA 2
#endif
#ifndef PA_F8MMA_WARPS_GQA
#define PA_F8MMA_WARPS_GQA 2
#endif
constexpr int kF8Warps = PA_F8MMA_WARPS;    // warps per CTA
// The grouped-query kernel's warps per CTA.  On the Llama-2-70B-shaped 8-bit
// step: 2 warps a CTA with the query rows read from global memory (12 warps
// an SM) 87.4 us; with the query rows in the stages (21 KB a warp), 4 warps
// a CTA (8 an SM) 89.0-89.3, 2 (10) 88.8, 3 (9) 93.4, 5 (register-capped)
// 99.0, 6 (one CTA) 109.4; 4 warps with the rows from global memory 90.2.
constexpr int kF8WarpsGqa = PA_F8MMA_WARPS_GQA;
__host__ __device__ constexpr int f8_warps(bool gqa) { return gqa ? kF8WarpsGqa : kF8Warps; }
// Ring depth per warp.  Multi-head: 3 stages, 2 CTAs (8 warps) an SM, 136.2
// us on the batch-64 step against 142.4 for 2 stages, 3 CTAs (12 warps) on
// the same box; grouped-query: 2 (3 measured the same).
constexpr int kF8Stages = PA_F8MMA_STAGES;
constexpr int kF8StagesGqa = PA_F8MMA_STAGES_GQA;
__host__ __device__ constexpr int f8_stages(bool gqa) { return gqa ? kF8StagesGqa : kF8Stages; }
constexpr int kF8D = 128;                   // head_dim
constexpr int kF8CH = 32;                   // tokens per chunk: 4 KB of key codes

// One warp's area: the stages' K and V tiles (4 KB each, every tile on a
// 1024-byte boundary), then the stages' query rows (qrows of 256 B each),
// barriers and flags; rounded up to 1024 bytes.
__host__ __device__ constexpr int f8_warp_bytes(int stages, int qrows) {
  return (stages * 8192 + stages * 256 * qrows + stages * 12 + 1023) / 1024 * 1024;
}
#ifndef PA_F8_GQA_Q_GLOBAL
#define PA_F8_GQA_Q_GLOBAL 1
#endif
// Grouped-query: 1 loads a unit's query rows from global memory straight
// into registers at the unit's first chunk (the stages then hold no query
// rows); 0 brings them with the chunk's copies, up to 8 rows per stage.
constexpr bool kF8GqaQGlobal = PA_F8_GQA_Q_GLOBAL != 0;
// Query rows a stage holds: one (multi-head), or up to the tile's eight
// columns (grouped-query), or none.
__host__ __device__ constexpr int f8_qrows(bool gqa) {
  return gqa ? (kF8GqaQGlobal ? 0 : 8) : 1;
}

__device__ __forceinline__ uint4 lds128(const uint8_t* p) {
  return *reinterpret_cast<const uint4*>(p);
}

}  // namespace

template <int B, int WARPS, int STAGES, bool GQA>
__global__ void __launch_bounds__(WARPS * 32, 3)
paged_decode_mma_fp8_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v) {
  constexpr int D = kF8D;
  constexpr int CH = kF8CH;
  constexpr int NB = CH >= B ? CH / B : 1;  // physical blocks a chunk touches
  constexpr int R = CH >= B ? B : CH;       // rows per TMA box
  constexpr uint32_t BOX_BYTES = R * 128;
  constexpr int QR = f8_qrows(GQA);
  constexpr bool QG = GQA && kF8GqaQGlobal;  // query rows from global memory
  constexpr int AREA = f8_warp_bytes(STAGES, QR);
  static_assert(B >= 8 && CH % B == 0, "block sizes 8, 16, 32");

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // The swizzle is a function of the shared-memory address: align by hand.
  uint8_t* smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
  int32_t* prefix = reinterpret_cast<int32_t*>(smem + WARPS * AREA);
  __shared__ int32_t warp_tot[WARPS];

  const int Hq = p.num_q_heads, Hkv = p.num_kv_heads;
  // Grouped-query: virtual head vh is subset vh % nsub of key/value head
  // vh / nsub, query heads q_head0(vh) .. + GS - 1 (GS <= 8), one per
  // column of the tile; multi-head: the head itself in every column.
  const int NSUB = p.nsub, GS = GQA ? p.gs : 1;
  const int G = Hq / Hkv;
  auto kv_head = [&](int vh) { return !GQA ? vh : NSUB == 1 ? vh : vh / NSUB; };
  auto q_head0 = [&](int vh) {
    return !GQA ? vh : NSUB == 1 ? vh * G : (vh / NSUB) * G + (vh % NSUB) * GS;
  };
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

  const WorkSplit sp = decode_prologue<__half, D, CH, WARPS * 32>(p, prefix, warp_tot, cap);
  const int W = sp.W;
  const int w = blockIdx.x * WARPS + warp;
  if (w >= W) return;
  // One-launch step (multi-head pools): the cache write of every text's new
  // row, each warp a share, as in the CUDA-core kernel.
  const bool fused = !GQA && p.slot_mapping != nullptr;
  if (sp.total == 0) {
    if (fused) fused_cache_write_f8<__half, D, B>(p, w, W, lane);
    return;
  }

  uint8_t* tiles = smem + warp * AREA;
  uint8_t* qbuf = tiles + STAGES * 8192;
  uint64_t* bars = reinterpret_cast<uint64_t*>(qbuf + STAGES * 256 * QR);
  int32_t* flags = reinterpret_cast<int32_t*>(bars + STAGES);
  if (lane == 0) {
#pragma unroll
    for (int st = 0; st < STAGES; ++st) mbar_init(&bars[st], 1);
    fence_barrier_init();
  }
  __syncwarp();

  const uint64_t policy = l2_evict_first_policy();
  const __half* __restrict__ qg = static_cast<const __half*>(p.q);

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
      uint8_t* sK = tiles + st * 8192;
      uint8_t* sV = sK + 4096;
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
      const uint32_t qbytes = first && !QG ? GS * D * 2 : 0;
      const uint32_t kvbytes = bad ? 0 : 2u * boxes * BOX_BYTES;
      mbar_arrive_expect_tx(&bars[st], qbytes + kvbytes);
      if (first && !QG)  // the unit's query rows (contiguous: GS heads in a row)
        bulk_copy_g2s(qbuf + st * 256 * QR, qg + (static_cast<int64_t>(s) * Hq + q_head0(h)) * D,
                      GS * D * 2, &bars[st], policy);
      if (!bad) {
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          const int rows = (CH >= B) ? min(B, nvalid - b * B) : nvalid;
          if (rows > 0) {
            const int y = (blk[b] * Hkv + kv_head(h)) * B;
            tma_load_2d(sK + b * BOX_BYTES, &tm_k, 0, y, &bars[st], policy);
            tma_load_2d(sV + b * BOX_BYTES, &tm_v, 0, y, &bars[st], policy);
          }
        }
      }
    }
  };

#pragma unroll
  for (int k = 0; k < STAGES; ++k) issue(k);
  // (the write while the first copies are in flight)
  if (fused) fused_cache_write_f8<__half, D, B>(p, w, W, lane);

  const int g = lane >> 2, c = lane & 3;
  uint32_t qh[16];   // query dimensions [32c, 32c + 32) of column g, as fp16 pairs
  // O^T: dimension 16g + 2md (+1 for entries 2, 3), column 2c (entries 0, 2)
  // and 2c + 1 (entries 1, 3); multi-head: all columns alike
  float o[8][4];
  float m = -INFINITY, l = 0.f;  // multi-head: running max (warp-uniform); this lane's share of the sum
  // grouped-query: the same for columns 2c and 2c + 1 (the max uniform over g)
  float mg[2] = {-INFINITY, -INFINITY}, lg[2] = {0.f, 0.f};
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

    const uint8_t* sK = tiles + st * 8192;
    const uint8_t* sV = sK + 4096;
    const int bad = flags[st];

    if (j == 0 || wu0 != prev_unit) {
      piece_j0 = j;
      const uint8_t* qrow = qbuf + st * 256 * QR + (GQA ? (g % GS) * 256 : 0) + c * 64;
      const uint4* qrow_g = reinterpret_cast<const uint4*>(
          qg + (static_cast<int64_t>(s) * Hq + q_head0(h) + g % GS) * D + c * 32);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 x = QG ? __ldg(qrow_g + i) : lds128(qrow + 16 * i);
        qh[4 * i + 0] = x.x;
        qh[4 * i + 1] = x.y;
        qh[4 * i + 2] = x.z;
        qh[4 * i + 3] = x.w;
      }
      m = -INFINITY;
      l = 0.f;
      mg[0] = mg[1] = -INFINITY;
      lg[0] = lg[1] = 0.f;
#pragma unroll
      for (int md = 0; md < 8; ++md)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[md][e] = 0.f;
    }
    const int nvalid = bad ? 0 : min(CH, len - j * CH);
    if (fused && nvalid > 0 && j * CH + nvalid == len) {
      // The chunk holding the text's last position takes that row from the
      // new k, v: its codes (the cache write's quantization) replace stage
      // row nvalid - 1, which the copies brought from the pool (possibly
      // while another warp was writing the same codes there).  Lanes 0-15
      // write the K row, 16-31 the V row, 8 codes each, at the swizzled
      // place of their 16-byte piece.
      const int r = nvalid - 1, part = lane & 15;
      const bool isv = lane >= 16;
      const __half* src = static_cast<const __half*>(isv ? p.v_new : p.k_new) +
                          (static_cast<int64_t>(s) * Hkv + h) * D + 8 * part;
      float x[8];
      unpack8<__half>(__ldg(reinterpret_cast<const uint4*>(src)), x);
      uint8_t* row = const_cast<uint8_t*>(isv ? sV : sK) + r * 128;
      *reinterpret_cast<uint2*>(row + (((part >> 1) ^ (r & 7)) << 4) + (part & 1) * 8) =
          e4m3x8_quantize(x, isv ? p.v_scale : p.k_scale);
      fence_proxy_async_smem();  // before this stage's refill by the copy engine
      __syncwarp();
    }

    // ---- S^T = K Q^T: two 16-token tiles, two accumulators each ----
    float sa[2][2][4];
#pragma unroll
    for (int x = 0; x < 2; ++x)
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sa[x][mt][e] = 0.f;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      // rows mt*16 + g and + 8 (both swizzled by g); pieces 2c, 2c + 1
      const uint8_t* r0 = sK + (mt * 16 + g) * 128;
      const uint8_t* r1 = r0 + 8 * 128;
      const uint4 k00 = lds128(r0 + (((2 * c) ^ g) << 4));
      const uint4 k01 = lds128(r0 + (((2 * c + 1) ^ g) << 4));
      const uint4 k10 = lds128(r1 + (((2 * c) ^ g) << 4));
      const uint4 k11 = lds128(r1 + (((2 * c + 1) ^ g) << 4));
      const uint32_t w0[8] = {k00.x, k00.y, k00.z, k00.w, k01.x, k01.y, k01.z, k01.w};
      const uint32_t w1[8] = {k10.x, k10.y, k10.z, k10.w, k11.x, k11.y, k11.z, k11.w};
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        uint32_t a[4];
        e4m3x4_to_half2x2(w0[kk], a[0], a[2]);  // row g: dims 32c + 4kk + {0,1}, {2,3}
        e4m3x4_to_half2x2(w1[kk], a[1], a[3]);  // row g + 8
        mma_16816<__half>(sa[kk & 1][mt], a, qh[2 * kk], qh[2 * kk + 1]);
      }
    }

    // ---- online softmax (base 2): tokens g, g + 8, 16 + g, 24 + g ----
    constexpr float kSlack = 8.f;
    // P pairs (token g, token g + 8) of each 16-token tile in fp16 (and the
    // rest, when split); grouped-query: [column 2c + j][tile]
    uint32_t ph[2][2], pl[2][2] = {{0u, 0u}, {0u, 0u}};
    if constexpr (GQA) {
      float sc[2][4];
#pragma unroll
      for (int jc = 0; jc < 2; ++jc) {
        sc[jc][0] = (sa[0][0][jc] + sa[1][0][jc]) * scale;
        sc[jc][1] = (sa[0][0][2 + jc] + sa[1][0][2 + jc]) * scale;
        sc[jc][2] = (sa[0][1][jc] + sa[1][1][jc]) * scale;
        sc[jc][3] = (sa[0][1][2 + jc] + sa[1][1][2 + jc]) * scale;
      }
      if (nvalid < CH) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if ((i >> 1) * 16 + (i & 1) * 8 + g >= nvalid) sc[0][i] = sc[1][i] = -INFINITY;
      }
      float cm[2];
#pragma unroll
      for (int jc = 0; jc < 2; ++jc)
        cm[jc] = fmaxf(fmaxf(sc[jc][0], sc[jc][1]), fmaxf(sc[jc][2], sc[jc][3]));
      if (__any_sync(0xffffffffu, cm[0] > mg[0] + kSlack || cm[1] > mg[1] + kSlack)) {
        float alpha[2];
#pragma unroll
        for (int jc = 0; jc < 2; ++jc) {
          float x = cm[jc];  // the column's max over the warp's tokens (lanes of one c)
          x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 4));
          x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 8));
          x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 16));
          const float m_new = fmaxf(mg[jc], x);
          alpha[jc] = m_new == mg[jc] ? 1.f : fast_exp2(mg[jc] - m_new);
          lg[jc] *= alpha[jc];
          mg[jc] = m_new;
        }
#pragma unroll
        for (int md = 0; md < 8; ++md)
#pragma unroll
          for (int e = 0; e < 4; ++e) o[md][e] *= alpha[e & 1];
      }
#pragma unroll
      for (int jc = 0; jc < 2; ++jc) {
        const float mm = mg[jc] == -INFINITY ? 0.f : mg[jc];
        float pr[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) pr[i] = fast_exp2(sc[jc][i] - mm);
        lg[jc] += (pr[0] + pr[1]) + (pr[2] + pr[3]);
#pragma unroll
        for (int kt = 0; kt < 2; ++kt) {
          ph[jc][kt] = Elem<__half>::from_float2(pr[2 * kt], pr[2 * kt + 1]);
          if constexpr (kSplitPF16) {
            const float2 back = Elem<__half>::to_float2(ph[jc][kt]);
            pl[jc][kt] = Elem<__half>::from_float2(pr[2 * kt] - back.x, pr[2 * kt + 1] - back.y);
          }
        }
      }
    } else {
    float sc[4];
    sc[0] = (sa[0][0][0] + sa[1][0][0]) * scale;
    sc[1] = (sa[0][0][2] + sa[1][0][2]) * scale;
    sc[2] = (sa[0][1][0] + sa[1][1][0]) * scale;
    sc[3] = (sa[0][1][2] + sa[1][1][2]) * scale;
    if (nvalid < CH) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if ((i >> 1) * 16 + (i & 1) * 8 + g >= nvalid) sc[i] = -INFINITY;
    }
    const float cm = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
    if (__any_sync(0xffffffffu, cm > m + kSlack)) {
      float x = cm;
      x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 4));
      x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 8));
      x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 16));
      const float m_new = fmaxf(m, x);
      // m_new == m (incl. both -inf) leaves everything as it is
      const float alpha = m_new == m ? 1.f : fast_exp2(m - m_new);
      l *= alpha;
#pragma unroll
      for (int md = 0; md < 8; ++md)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[md][e] *= alpha;
      m = m_new;
    }
    const float mm = m == -INFINITY ? 0.f : m;
    float pr[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) pr[i] = fast_exp2(sc[i] - mm);
    l += (pr[0] + pr[1]) + (pr[2] + pr[3]);
#pragma unroll
    for (int kt = 0; kt < 2; ++kt) {
      ph[0][kt] = Elem<__half>::from_float2(pr[2 * kt], pr[2 * kt + 1]);
      if constexpr (kSplitPF16) {
        const float2 back = Elem<__half>::to_float2(ph[0][kt]);
        pl[0][kt] = Elem<__half>::from_float2(pr[2 * kt] - back.x, pr[2 * kt + 1] - back.y);
      }
    }
    }

    // ---- O^T += V^T P^T ----
#pragma unroll
    for (int kt = 0; kt < 2; ++kt) {
      // K positions 2c, 2c+1 <- tokens 2c, 2c+8 (held together by lane g = 2c);
      // K positions 2c+8, 2c+9 <- tokens 2c+1, 2c+9 (lane g = 2c + 1).
      // Grouped-query: this lane's column g is column 2(g/2) + (g%2) of the
      // lane (2c or 2c + 1, g/2); both of its columns come over, one is kept.
      uint32_t b0h, b1h, b0l = 0u, b1l = 0u;
      if constexpr (GQA) {
        const int src0 = (2 * c) * 4 + (g >> 1), src1 = (2 * c + 1) * 4 + (g >> 1);
        const bool odd = g & 1;
        uint32_t x0 = __shfl_sync(0xffffffffu, ph[0][kt], src0);
        uint32_t x1 = __shfl_sync(0xffffffffu, ph[1][kt], src0);
        b0h = odd ? x1 : x0;
        x0 = __shfl_sync(0xffffffffu, ph[0][kt], src1);
        x1 = __shfl_sync(0xffffffffu, ph[1][kt], src1);
        b1h = odd ? x1 : x0;
        if constexpr (kSplitPF16) {
          x0 = __shfl_sync(0xffffffffu, pl[0][kt], src0);
          x1 = __shfl_sync(0xffffffffu, pl[1][kt], src0);
          b0l = odd ? x1 : x0;
          x0 = __shfl_sync(0xffffffffu, pl[0][kt], src1);
          x1 = __shfl_sync(0xffffffffu, pl[1][kt], src1);
          b1l = odd ? x1 : x0;
        }
      } else {
        b0h = __shfl_sync(0xffffffffu, ph[0][kt], (2 * c) * 4);
        b1h = __shfl_sync(0xffffffffu, ph[0][kt], (2 * c + 1) * 4);
        if constexpr (kSplitPF16) {
          b0l = __shfl_sync(0xffffffffu, pl[0][kt], (2 * c) * 4);
          b1l = __shfl_sync(0xffffffffu, pl[0][kt], (2 * c + 1) * 4);
        }
      }
      const int t0 = kt * 16 + 2 * c;
      uint4 v0 = lds128(sV + t0 * 128 + ((g ^ (2 * c)) << 4));
      uint4 v1 = lds128(sV + (t0 + 8) * 128 + ((g ^ (2 * c)) << 4));
      uint4 v2 = lds128(sV + (t0 + 1) * 128 + ((g ^ (2 * c + 1)) << 4));
      uint4 v3 = lds128(sV + (t0 + 9) * 128 + ((g ^ (2 * c + 1)) << 4));
      // Rows past nvalid hold whatever the pool or an earlier chunk left there
      // (possibly NaN codes); their weights are zero, but 0 * NaN is not.
      if (nvalid < (kt + 1) * 16) {
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
        if (t0 >= nvalid) v0 = z;
        if (t0 + 8 >= nvalid) v1 = z;
        if (t0 + 1 >= nvalid) v2 = z;
        if (t0 + 9 >= nvalid) v3 = z;
      }
      const uint32_t x0[4] = {v0.x, v0.y, v0.z, v0.w}, x1[4] = {v1.x, v1.y, v1.z, v1.w};
      const uint32_t x2[4] = {v2.x, v2.y, v2.z, v2.w}, x3[4] = {v3.x, v3.y, v3.z, v3.w};
#pragma unroll
      for (int wd = 0; wd < 4; ++wd) {
        // bytes 4wd, 4wd+1 (dimensions 16g + 4wd, + 1: tile 2wd) and
        // 4wd+2, 4wd+3 (tile 2wd + 1), each pair from two token rows
        uint32_t a[4];
        e4m3x4_to_half2x2(__byte_perm(x0[wd], x1[wd], 0x5140), a[0], a[1]);
        e4m3x4_to_half2x2(__byte_perm(x2[wd], x3[wd], 0x5140), a[2], a[3]);
        mma_16816<__half>(o[2 * wd], a, b0h, b1h);
        if constexpr (kSplitPF16) mma_16816<__half>(o[2 * wd], a, b0l, b1l);
        e4m3x4_to_half2x2(__byte_perm(x0[wd], x1[wd], 0x7362), a[0], a[1]);
        e4m3x4_to_half2x2(__byte_perm(x2[wd], x3[wd], 0x7362), a[2], a[3]);
        mma_16816<__half>(o[2 * wd + 1], a, b0h, b1h);
        if constexpr (kSplitPF16) mma_16816<__half>(o[2 * wd + 1], a, b0l, b1l);
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
      const bool whole = piece_j0 == 0 && j == ns - 1 && !p.cascade;
      if constexpr (GQA) {
        float lt[2];
#pragma unroll
        for (int jc = 0; jc < 2; ++jc) {
          lt[jc] = lg[jc];
          lt[jc] += __shfl_xor_sync(0xffffffffu, lt[jc], 4);
          lt[jc] += __shfl_xor_sync(0xffffffffu, lt[jc], 8);
          lt[jc] += __shfl_xor_sync(0xffffffffu, lt[jc], 16);
        }
        const int qh0 = q_head0(h);
        float* recs = p.records + (static_cast<int64_t>(wu0) + sh) * (GS * (D + 4));
#pragma unroll
        for (int jc = 0; jc < 2; ++jc) {
          const int col = 2 * c + jc;  // query head qh0 + col
          if (col >= GS) continue;
          if (whole) {
            const float inv = lt[jc] > 0.f ? p.v_scale / lt[jc] : 0.f;
            float f[8];
            __half* orow =
                static_cast<__half*>(p.out) + (static_cast<int64_t>(s) * Hq + qh0 + col) * D + 16 * g;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                f[2 * i] = o[4 * half + i][jc] * inv;
                f[2 * i + 1] = o[4 * half + i][2 + jc] * inv;
              }
              *reinterpret_cast<uint4*>(orow + 8 * half) = pack8<__half>(f);
            }
          } else {
            float* rec = recs + col * (D + 4);
            if (g == 0) {
              rec[0] = mg[jc];
              rec[1] = lt[jc];
            }
            float4* dst = reinterpret_cast<float4*>(rec + 4 + 16 * g);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_float4(o[2 * i][jc] * p.v_scale, o[2 * i][2 + jc] * p.v_scale,
                                   o[2 * i + 1][jc] * p.v_scale, o[2 * i + 1][2 + jc] * p.v_scale);
          }
        }
      } else {
      float lt = l;
      lt += __shfl_xor_sync(0xffffffffu, lt, 4);
      lt += __shfl_xor_sync(0xffffffffu, lt, 8);
      lt += __shfl_xor_sync(0xffffffffu, lt, 16);
      if (whole) {
        if (c == 0) {
          // v_scale turns sums of codes into values
          const float inv = lt > 0.f ? p.v_scale / lt : 0.f;
          float f[8];
          __half* orow = static_cast<__half*>(p.out) + sh * D + 16 * g;
#pragma unroll
          for (int half = 0; half < 2; ++half) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              f[2 * i] = o[4 * half + i][0] * inv;
              f[2 * i + 1] = o[4 * half + i][2] * inv;
            }
            *reinterpret_cast<uint4*>(orow + 8 * half) = pack8<__half>(f);
          }
        }
      } else {
        float* rec = p.records + (static_cast<int64_t>(wu0) + sh) * (D + 4);
        if (lane == 0) {
          rec[0] = m;
          rec[1] = lt;
        }
        if (c == 0) {
          float4* dst = reinterpret_cast<float4*>(rec + 4 + 16 * g);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_float4(o[2 * i][0] * p.v_scale, o[2 * i][2] * p.v_scale,
                                 o[2 * i + 1][0] * p.v_scale, o[2 * i + 1][2] * p.v_scale);
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

namespace {

size_t f8_smem_bytes(int num_seqs, bool gqa) {
  return 1024 /* alignment slack */ +
         static_cast<size_t>(f8_warps(gqa)) * f8_warp_bytes(f8_stages(gqa), f8_qrows(gqa)) +
         align_up(sizeof(int32_t) * (num_seqs + 1), 16);
}

template <int B, bool GQA>
const void* f8_kernel_ptr() {
  return reinterpret_cast<const void*>(
      &paged_decode_mma_fp8_kernel<B, f8_warps(GQA), f8_stages(GQA), GQA>);
}

template <bool GQA>
const void* f8_kernel_for(int block_size) {
  switch (block_size) {
    case 8: return f8_kernel_ptr<8, GQA>();
    case 16: return f8_kernel_ptr<16, GQA>();
    case 32: return f8_kernel_ptr<32, GQA>();
    default: return nullptr;
  }
}

Plan plan_f8(const void* kernel, bool gqa, int B, int num_seqs, int vheads,
             int max_blocks_per_seq, int64_t forced_warps) {
  return plan_decode(kernel, f8_smem_bytes(num_seqs, gqa), f8_smem_bytes(kMaxSeqs, gqa),
                     f8_warps(gqa), kF8CH, B, num_seqs, vheads, max_blocks_per_seq, forced_warps);
}

// The 8-bit pool [num_blocks][H][B][128] seen as a 2-D tensor of
// num_blocks*H*B rows of 128 one-byte codes; boxes of 128 x `rows`, 128-byte
// swizzle.
bool encode_code_map(CUtensorMap* map, const void* pool, int64_t rows, int box_rows) {
  const uint64_t dims[2] = {static_cast<uint64_t>(kF8D), static_cast<uint64_t>(rows)};
  const uint64_t strides[1] = {static_cast<uint64_t>(kF8D)};
  const uint32_t box[2] = {static_cast<uint32_t>(kF8D), static_cast<uint32_t>(box_rows)};
  return encode_tiled_map(map, pool, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, dims, strides, box);
}

template <int B, bool GQA>
cudaError_t launch_f8_typed(const DecodeArgs& a, const DecodeLayout& hl, cudaStream_t stream) {
  const Plan pl = plan_f8(f8_kernel_ptr<B, GQA>(), GQA, B, a.num_seqs, hl.vheads,
                          a.max_blocks_per_seq, a.forced_warps);
  if (pl.grid <= 0) return cudaErrorInvalidConfiguration;
  const int64_t segs = static_cast<int64_t>(a.num_seqs) * hl.vheads;
  const size_t need = header_bytes(a.num_seqs) + kGrabBytes +
                      records_bytes(max_units(pl.work_warps) + segs, kF8D, hl.gs);
  if (a.workspace_bytes < need) return cudaErrorInvalidValue;
  const int64_t rows = a.num_blocks * a.num_kv_heads * B;
  CUtensorMap tm_k, tm_v;
  constexpr int R = kF8CH >= B ? B : kF8CH;
  if (!encode_code_map(&tm_k, a.k_cache, rows, R) || !encode_code_map(&tm_v, a.v_cache, rows, R))
    return cudaErrorInvalidValue;
  DecodeParams p;
  p.out = a.out;
  p.q = a.q;
  p.k_cache = a.k_cache;
  p.v_cache = a.v_cache;
  p.block_tables = a.block_tables;
  p.context_lens = a.context_lens;
  // log2(e) and the keys' scale folded into the score scale; the values'
  // scale multiplies the output
  p.qk_scale_log2 = a.scale * 1.4426950408889634f * a.k_scale;
  p.v_scale = a.v_scale;
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
  // one-launch step: the new rows and their slots (null otherwise)
  p.k_new = a.k_new;
  p.v_new = a.v_new;
  p.slot_mapping = a.slot_mapping;
  p.k_scale = a.k_scale;
  p.cascade = 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.grid);
  cfg.blockDim = dim3(f8_warps(GQA) * 32);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t err = cudaLaunchKernelEx(
      &cfg, paged_decode_mma_fp8_kernel<B, f8_warps(GQA), f8_stages(GQA), GQA>, p, tm_k, tm_v);
  if (err != cudaSuccess) return err;
  err = launch_merge<__half, kF8D>(p, hl.gs, stream);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace

// Grouped-query pools: a key/value head's G query heads in nsub equal
// subsets of gs <= 8 (the smallest count that divides G), one subset per
// pass over the key/value head's codes, a query head per tile column.
DecodeLayout mma_fp8_layout(int num_heads, int num_kv_heads) {
  const int G = num_kv_heads > 0 ? num_heads / num_kv_heads : 1;
  int nsub = (G + 7) / 8;
  while (G % nsub) ++nsub;
  return DecodeLayout{nsub, G / nsub, num_kv_heads * nsub};
}

bool mma_fp8_decode_ok(const DecodeArgs& a) {
  // (the one-launch step, with slot_mapping, on multi-head pools only)
  return a.fp8 && !a.is_bf16 && !a.cascade && a.head_dim == kF8D &&
         (!a.slot_mapping || a.num_heads == a.num_kv_heads) &&
         a.num_kv_heads >= 1 && a.num_heads % a.num_kv_heads == 0 &&
         (a.block_size == 8 || a.block_size == 16 || a.block_size == 32) &&
         mma_decode_pool_ok(a.num_kv_heads, a.block_size, a.num_blocks);
}

size_t mma_fp8_workspace_bytes(int num_seqs, int num_heads, int num_kv_heads, int block_size,
                               int max_blocks_per_seq, int64_t forced_warps) {
  if (num_kv_heads < 1 || num_heads % num_kv_heads) return 0;
  const DecodeLayout hl = mma_fp8_layout(num_heads, num_kv_heads);
  const bool gqa = num_heads != num_kv_heads;
  const void* k = gqa ? f8_kernel_for<true>(block_size) : f8_kernel_for<false>(block_size);
  if (!k) return 0;
  const Plan pl = plan_f8(k, gqa, block_size, num_seqs, hl.vheads, max_blocks_per_seq,
                          forced_warps);
  if (pl.grid <= 0) return 0;
  const int64_t segs = static_cast<int64_t>(num_seqs) * hl.vheads;
  return header_bytes(num_seqs) + kGrabBytes +
         records_bytes(max_units(pl.work_warps) + segs, kF8D, hl.gs);
}

cudaError_t launch_paged_attn_decode_mma_fp8(const DecodeArgs& a, cudaStream_t stream) {
  if (!mma_fp8_decode_ok(a)) return cudaErrorInvalidValue;
  const DecodeLayout hl = mma_fp8_layout(a.num_heads, a.num_kv_heads);
  if (a.num_heads == a.num_kv_heads) {
    switch (a.block_size) {
      case 8: return launch_f8_typed<8, false>(a, hl, stream);
      case 16: return launch_f8_typed<16, false>(a, hl, stream);
      case 32: return launch_f8_typed<32, false>(a, hl, stream);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (a.block_size) {
    case 8: return launch_f8_typed<8, true>(a, hl, stream);
    case 16: return launch_f8_typed<16, true>(a, hl, stream);
    case 32: return launch_f8_typed<32, true>(a, hl, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace pa
