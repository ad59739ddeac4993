// prefill_tc: the prompt phase on the 5th-generation tensor cores (tcgen05).
//
// What it computes is prefill.cu's function ("The KV Cache and
// PagedAttention", section "One Token at a Time"; "KV cache", section "How it
// works"): for prompt s, query head h and position t,
//     out[t][h] = sum_{u <= t} softmax_u(scale * q[t][h] . k[u]) v[u],
// query head h reading key/value head h / (Hq / Hkv).  With a stored prefix
// (section "What Came After": a prompt that begins like an earlier one reuses
// the earlier one's blocks and skips their compute), prompt s's first
// cached_lens[s] tokens are not in q, k, v: their keys and values are read
// from the paged cache through block_tables[s], and the new rows are the
// positions after them.
//
// How (FlashAttention-4's arrangement on sm_100a, with two threads a row):
// one CTA takes two tiles of 128 queries of one (prompt, head), 256
// consecutive queries, and runs twenty warps with separate jobs:
//   * warp 17 loads: Q of both tiles once, then each block of 128 keys of K
//     and of V, each into a ring of its own of 2 slots: a K slot refills once
//     both tiles' S have read it, a step before the block's V slot frees,
//     which gives the loads about two steps of lead.  Tiled TMA with the
//     128-byte swizzle: the new tokens from q, k, v (the [T][H][D] tensors
//     seen as (D, H, T); boxes 64 x 1 x rows), the stored prefix from the
//     cache pools (seen as (D, B, H, N); one box of 64 x B rows per physical
//     block, found in the block table);
//   * warp 16 (lane 0 issuing, the whole warp running the loop) issues the
//     tensor-core products, tcgen05.mma kind::f16, accumulating in tensor
//     memory (TMEM): S_t = Q_t K^T (both operands K-major in shared memory)
//     and O_t += P_t V (P_t from TMEM, V MN-major in shared memory), in the
//     order S0, S1, then per block PV0, S0', PV1, S1': while one tile's
//     softmax runs, the tensor pipe works on the other tile's products;
//   * warps 0-15, four warpgroups: the softmax, warpgroups 2t and 2t+1 for
//     tile t, two threads per query row (warps w and w + 4 read the same 32
//     TMEM lanes): one takes the block's keys 0-63, the other keys 64-127.
//     Each reads its 64 scores from TMEM, the pair exchange their maxima
//     through shared memory at a named barrier of the tile's 256 threads
//     (which also carries a vote on failure), and each computes its 64
//     weights.  Base 2; the running max is raised only when a score passes
//     it by more than 2^8, which then rescales the row of O in TMEM (each
//     thread its half of head_dim).  Two scores per packed fp32 instruction,
//     maxima three at a time.  P (and for bf16 the rest P - P_hi, so P enters
//     as about 16 significant bits) goes back into the S columns it was
//     computed from, as packed 16-bit pairs.
//   * After its last block each pair adds up its partial row sums (the same
//     barrier), and each thread divides its half of the row of O by the sum
//     and stores it.
//   * warps 18 and 19 store the new tokens' keys and values in the cache
//     (when asked to): the CTAs of a key/value head's first query head copy
//     the prompt's rows of k and v to their slots, a bulk copy into a
//     staging row of shared memory and a bulk copy out of it per row, each
//     CTA a share of the tokens in proportion to its attention work, while
//     the other warps compute; the attention is bound by the tensor and
//     exponential units and leaves HBM mostly idle.  (Storing from the K/V
//     tiles in shared memory measured slower: the stores held the ring's
//     slots; so did plain 16-byte loads and stores from registers.)
// Why two threads a row: the exponential unit does 4 exp2 a clock per SM
// sub-partition, so a block's 2 x 128 x 128 weights take as long as its
// products; with one thread a row each tile's softmax ran twice as long as
// the other tile's products, and the tensor pipe waited.  Making the two
// tiles take turns on the exponential unit (tile 1's weights of a block
// after tile 0's, tile 0's of the next after tile 1's, through a pair of
// barriers) measured slower: 670 against 712 TFLOP/s for the attention
// alone.
// Order of the CTAs: the hardware hands them out x fastest, then y, then
// z; the grid is (head, pair, prompt), so each prompt's pairs of all heads
// go heaviest first (0.7% faster than each (prompt, head)'s pairs in turn;
// the heaviest pairs of the whole launch first lost 2.5%: a head's keys and
// values no longer stay in L2 between its pairs).
// Barriers: per ring slot, for K and for V, full (TMA bytes) and empty (the
// last product that reads it); per tile S ready, P ready (256 arrivals) and
// O done.  TMEM per tile: S (and P over it) 128 columns, O head_dim; 512 for
// the two tiles, one CTA per SM.
// Every wait is bounded: a wait that gives up records PA_ERR_TIMEOUT and
// raises a CTA-wide abort flag; each role then drains what it issued
// (bounded), TMEM is freed and the CTA returns.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>
#include <set>
#include <type_traits>

#include "dtype.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "tcgen05.cuh"

namespace pa {

namespace {

constexpr int kTcBM = 128;      // queries per tile (MMA M)
constexpr int kTcBN = 128;      // keys per block (MMA N of S, K of P V)
constexpr int kTcHalf = kTcBN / 2;  // keys per softmax thread and block
constexpr int kTcTiles = 2;     // query tiles per CTA
constexpr int kTcStages = 2;    // slots of each of the K and V rings (32 KB each)
// Warpgroups 0-3: the softmax; warpgroup 4: the MMA warp, the load warp and
// the two store warps.  The launch gives every thread 96 registers (640 x 96 of
// the SM's 65,536).  A build option splits them unevenly (warpgroup 4 lowers
// to kTcRegsLow, the softmax warpgroups raise to kTcRegsHigh, with
// 4 x 128 x high + 128 x low <= 640 x 96); with the softmax reading its
// scores 32 at a time no split is needed (none spills at 96), and the split
// tried (104 / 56) spilled in warpgroup 4.
constexpr int kTcThreads = 640;
constexpr int kTcSoftmaxWarps = 16;
constexpr int kMmaWarp = 16, kLoadWarp = 17, kStoreWarp0 = 18;  // warps 18, 19 store
#ifndef PA_TC_REGS_HIGH
#define PA_TC_REGS_HIGH 96
#endif
#ifndef PA_TC_REGS_LOW
#define PA_TC_REGS_LOW 96
#endif
constexpr uint32_t kTcRegsLaunch = 96, kTcRegsHigh = PA_TC_REGS_HIGH, kTcRegsLow = PA_TC_REGS_LOW;
static_assert(4 * 128 * kTcRegsHigh + 128 * kTcRegsLow <= kTcThreads * kTcRegsLaunch,
              "register split");
// TMEM columns of a tile: S from kColS (kTcBN of them), P written over S
// (see the softmax), O from kColO.
constexpr uint32_t kColS = 0, kColO = 128;
constexpr uint32_t kTileCols = 256, kTmemCols = 512;
constexpr int64_t kTcDrainNs = 1000000000;

#ifndef PA_TC_PREFETCH
#define PA_TC_PREFETCH 2
#endif
// When the softmax's second read of keys 0-31 is issued: 1 before the
// exchange of maxima, 2 right after it (before keys 32-63's weights; 705
// against 697 TFLOP/s for the attention alone), 0 after keys 32-63's
// weights (fewest registers live).
constexpr int kTcPrefetch = PA_TC_PREFETCH;
#ifndef PA_TC_STORE_BLOCKS
#define PA_TC_STORE_BLOCKS 1
#endif
// 1: the store warps move a block's rows of k and v with one tiled load and
// one bulk store each where the slots allow (else row by row)
constexpr bool kTcStoreBlocks = PA_TC_STORE_BLOCKS != 0;
#ifndef PA_TC_MAX_ONE_WAIT
#define PA_TC_MAX_ONE_WAIT 0
#endif
// 1: the max pass issues both of its TMEM loads under one wait
constexpr bool kTcMaxOneWait = PA_TC_MAX_ONE_WAIT != 0;

// max(a, b, c) in one instruction (three-input max.f32 of sm_100)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Named barrier `id` over `count` threads that also ORs a flag across them:
// every participant learns whether any of them raised it.
__device__ __forceinline__ bool bar_any(uint32_t id, uint32_t count, bool flag) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, %2, %3, q;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(flag ? 1u : 0u), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

template <int D>
struct TcLayout {
  static constexpr int HALVES = D / 64;           // 64-element (128-byte) column blocks
  static constexpr int Q_BYTES = kTcBM * D * 2;   // one tile of Q: 32 KB at head_dim 128
  static constexpr int KV_BYTES = kTcBN * D * 2;  // one block of K (or V): 32 KB at D = 128
  static constexpr int STAGE = 2 * KV_BYTES;      // K slot i, then V slot i
  // shared memory asked for (+ 1 KB to align by hand): the head_dim-128
  // amount at every head_dim, so one CTA holds an SM (its 512 TMEM
  // columns), and the store warps' staging (one 256-byte row per thread)
  static constexpr int SMEM = 1024 + kTcTiles * (kTcBM * 128 * 2) +
                              kTcStages * (2 * kTcBN * 128 * 2) + 64 * 128 * 2;
};

struct TcParams {
  void* out;
  const int32_t* cu_seqlens;
  int num_tokens;
  int max_seqlen;
  int Hq;
  int Hkv;
  float scale_log2;
  int32_t* status;
  int64_t wait_limit_ns;
  // The paged cache (block size B, num_blocks blocks): a stored prefix is
  // read from it through block_tables / cached_lens (null: none), and the
  // new tokens' keys and values k, v are written to it at slot_mapping
  // (null: not).
  int B;
  const void* k;
  const void* v;
  void* k_cache;
  void* v_cache;
  const int64_t* slot_mapping;
  int64_t num_blocks;
  const int32_t* block_tables;
  const int32_t* cached_lens;
  int max_blocks;
  int B_shift;  // log2(B): block sizes are powers of two
  // 1: the store warps move whole blocks (tm_ks / tm_vs are encoded)
  int store_blocks;
};

template <typename T, int D>
__global__ void __launch_bounds__(kTcThreads, 1)
prefill_tc_kernel(const TcParams p, const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const __grid_constant__ CUtensorMap tm_kc, const __grid_constant__ CUtensorMap tm_vc,
                  const __grid_constant__ CUtensorMap tm_ks, const __grid_constant__ CUtensorMap tm_vs) {
  using LY = TcLayout<D>;
  constexpr bool BF16 = std::is_same<T, __nv_bfloat16>::value;
  constexpr uint32_t IDESC_S = tc::idesc_f16(kTcBM, kTcBN, BF16, false);
  constexpr uint32_t IDESC_O = tc::idesc_f16(kTcBM, D, BF16, true);
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 128-byte swizzle patterns repeat every 1024 bytes of shared address: align by hand
  uint8_t* smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
  uint8_t* sQ = smem;                               // tile t at t * Q_BYTES
  uint8_t* sKV = smem + kTcTiles * LY::Q_BYTES;     // K slot i at i * STAGE, V slot i after it
  // per ring slot, separately for K (index 0) and V (index 1): full (TMA
  // bytes) and empty (the last product that reads it)
  __shared__ uint64_t bar_q, bar_full[2][kTcStages], bar_empty[2][kTcStages];
  __shared__ uint64_t bar_s[kTcTiles], bar_p[kTcTiles], bar_o[kTcTiles], bar_st;
  __shared__ uint64_t bar_stw[2];  // the store warps' own barriers (whole-block stores)
  // the two halves of a row trade partial maxima (two buffers, alternating
  // by block) and, at the end, partial sums
  __shared__ float xmax[2][kTcTiles][2][kTcBM];
  __shared__ float xsum[kTcTiles][2][kTcBM];
  __shared__ uint32_t tmem_base;
  __shared__ volatile int abort_flag;

  griddep_wait();
  // (head h, pair index xp counted from the last pair, prompt s)
  const int h = blockIdx.x, xp = blockIdx.y, s = blockIdx.z;
  const int a = __ldg(p.cu_seqlens + s), b = __ldg(p.cu_seqlens + s + 1);
  if (a < 0 || b < a || b > p.num_tokens) {
    if (xp == 0 && h == 0 && threadIdx.x == 0) set_status(p.status, -8 /* PA_ERR_BAD_LEN */);
    return;
  }
  const int L = b - a;  // new tokens of this prompt
  if (L > p.max_seqlen && xp == 0 && h == 0 && threadIdx.x == 0)
    set_status(p.status, -8 /* PA_ERR_BAD_LEN: a prompt longer than max_seqlen */);
  // stored prefix: a whole number of blocks that the table holds
  const int cl = p.cached_lens ? __ldg(p.cached_lens + s) : 0;
  if (cl < 0 || cl % p.B || cl > p.max_blocks * p.B) {
    if (xp == 0 && h == 0 && threadIdx.x == 0) set_status(p.status, -8 /* PA_ERR_BAD_LEN */);
    return;
  }
  const int npre = (cl + kTcBN - 1) / kTcBN;        // key blocks of the stored prefix
  const int pair = gridDim.y - 1 - xp;               // heaviest pairs of tiles first
  const int q0 = pair * kTcTiles * kTcBM;            // first new row of tile 0
  if (q0 >= L) return;                               // the whole CTA leaves: nothing allocated
  const int kvh = h / (p.Hq / p.Hkv);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // key blocks each tile needs: the prefix's, then the new keys up to its
  // last row; tile 1 may be empty
  int nkb_t[kTcTiles];
#pragma unroll
  for (int t = 0; t < kTcTiles; ++t) {
    const int lo = q0 + t * kTcBM;
    const int hi = min(L, lo + kTcBM);
    nkb_t[t] = lo < L ? npre + (hi + kTcBN - 1) / kTcBN : 0;
  }
  const int nkb = nkb_t[kTcTiles - 1] > 0 ? nkb_t[kTcTiles - 1] : nkb_t[0];

  if (tid == 0) {
    abort_flag = 0;
    mbar_init(&bar_q, 1);
#pragma unroll
    for (int w = 0; w < 2; ++w)
#pragma unroll
      for (int i = 0; i < kTcStages; ++i) {
        mbar_init(&bar_full[w][i], 1);
        mbar_init(&bar_empty[w][i], 1);
      }
#pragma unroll
    for (int t = 0; t < kTcTiles; ++t) {
      mbar_init(&bar_s[t], 1);
      mbar_init(&bar_p[t], 2 * kTcBM);  // both threads of every row
      mbar_init(&bar_o[t], 1);
    }
    mbar_init(&bar_st, 64);  // the store warps' 64 threads
    mbar_init(&bar_stw[0], 32);
    mbar_init(&bar_stw[1], 32);
    fence_barrier_init();
  }
  if (warp == 0) tc::alloc(&tmem_base, kTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_base;
  const int64_t lim = p.wait_limit_ns;
  auto give_up = [&]() {
    set_status(p.status, -10 /* PA_ERR_TIMEOUT */);
    abort_flag = 1;
  };
  // a bounded wait that also ends once the CTA has given up
  auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (abort_flag) return false;
    if (!mbar_wait_bounded(bar, parity, lim)) {
      give_up();
      return false;
    }
    return true;
  };
  // a wait whose outcome the whole warp shares
  auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
    return !__any_sync(0xffffffffu, !wait(bar, parity));
  };

  if (warp >= kTcSoftmaxWarps) {
  // warpgroup 4 (lowers its registers, if split, then) runs its roles
  if constexpr (kTcRegsLow != kTcRegsLaunch) tc::regs_lower<kTcRegsLow>();
  if (warp == kLoadWarp) {
    // ---------------- loads (lane 0) ----------------
    if (lane == 0) {
      tc::prefetch_map(&tm_q);
      tc::prefetch_map(&tm_k);
      tc::prefetch_map(&tm_v);
      if (p.cached_lens) {
        tc::prefetch_map(&tm_kc);
        tc::prefetch_map(&tm_vc);
      }
      const int nq = nkb_t[1] > 0 ? 2 : 1;
      mbar_arrive_expect_tx(&bar_q, nq * LY::Q_BYTES);
      for (int t = 0; t < nq; ++t)
#pragma unroll
        for (int hf = 0; hf < LY::HALVES; ++hf)
          tc::tma_load_3d(sQ + t * LY::Q_BYTES + hf * (kTcBM * 128), &tm_q, hf * 64, h,
                          a + q0 + t * kTcBM, &bar_q);
      // Key block jj: the stored prefix's block jj (jj < npre), else block
      // jj - npre of the new keys; K (w = 0) and V (w = 1) in their rings.
      const int32_t* table =
          p.cached_lens ? p.block_tables + static_cast<int64_t>(s) * p.max_blocks : nullptr;
      auto load_part = [&](int jj, int w) {
        const int st = jj % kTcStages;
        uint8_t* dst = sKV + st * LY::STAGE + w * LY::KV_BYTES;
        uint64_t* bar = &bar_full[w][st];
        mbar_arrive_expect_tx(bar, LY::KV_BYTES);
        if (jj < npre) {
          // one box of B rows per physical block; rows past the prefix (and
          // bad table entries) are read from block num_blocks, outside the
          // pool: zeros, so their scores are finite and their values add
          // nothing
          for (int r0 = 0; r0 < kTcBN; r0 += p.B) {
            const int pos = jj * kTcBN + r0;
            int blk = static_cast<int>(p.num_blocks);
            if (pos < cl) {
              const int e = __ldg(table + pos / p.B);
              if (e >= 0 && e < p.num_blocks) {
                blk = e;
              } else if (w == 0) {
                set_status(p.status, -7 /* PA_ERR_BAD_BLOCK */);
              }
            }
#pragma unroll
            for (int hf = 0; hf < LY::HALVES; ++hf)
              tc::tma_load_4d(dst + hf * (kTcBN * 128) + r0 * 128, w ? &tm_vc : &tm_kc,
                              hf * 64, 0, kvh, blk, bar);
          }
        } else {
          const int j = jj - npre;
#pragma unroll
          for (int hf = 0; hf < LY::HALVES; ++hf)
            tc::tma_load_3d(dst + hf * (kTcBN * 128), w ? &tm_v : &tm_k, hf * 64, kvh,
                            a + j * kTcBN, bar);
        }
      };
      int issued_w[2] = {0, 0};
      bool ok = true;
      for (int jj = 0; jj < nkb && ok; ++jj) {
        const int st = jj % kTcStages;
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          if (!ok) break;
          if (jj >= kTcStages && !(ok = wait(&bar_empty[w][st], ((jj / kTcStages) - 1) & 1)))
            break;
          load_part(jj, w);
          issued_w[w] = jj + 1;
        }
      }
      // drain: the copies in flight must land before this CTA's shared
      // memory goes
      mbar_wait_bounded(&bar_q, 0, kTcDrainNs);
#pragma unroll
      for (int w = 0; w < 2; ++w)
        for (int j = issued_w[w] > kTcStages ? issued_w[w] - kTcStages : 0; j < issued_w[w]; ++j)
          mbar_wait_bounded(&bar_full[w][j % kTcStages], (j / kTcStages) & 1, kTcDrainNs);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ---------------- tensor-core products ----------------
    // One issuer for both tiles, in the order PV0, S0', PV1, S1': the tiles'
    // softmaxes then alternate, each running while the tensor pipe has the
    // other tile's products.  (A warp per tile measured slower: the tiles
    // fell into step, their softmaxes contending for the exponential unit
    // while the pipe stood idle.)  The whole warp runs the loop; lane 0
    // alone issues each product and commit (the same lane throughout, so
    // its commits track its products).
    const uint32_t leader = lane == 0;
    // descriptors of the two Q tiles and of the K and V slots; a step along
    // K adds its byte offset >> 4 to the start-address field
    uint64_t dq[kTcTiles], dk[kTcStages], dv[kTcStages];
#pragma unroll
    for (int t = 0; t < kTcTiles; ++t) dq[t] = tc::smem_desc(smem_addr(sQ + t * LY::Q_BYTES), 16, 1024);
#pragma unroll
    for (int i = 0; i < kTcStages; ++i) {
      dk[i] = tc::smem_desc(smem_addr(sKV + i * LY::STAGE), 16, 1024);
      dv[i] = tc::smem_desc(smem_addr(sKV + i * LY::STAGE + LY::KV_BYTES), kTcBN * 128, 1024);
    }
    int s_done0 = 0, s_done1 = 0, o_done0 = 0, o_done1 = 0;
    int k_ready = 0, v_ready = 0;  // blocks whose K, V tiles are known to have landed
    auto issue_s = [&](int t, int j) -> bool {  // S_t = Q_t K_j^T
      // (the previous block's scores were read: its P is written, P V issued)
      if (j >= k_ready) {
        if (!wwait(&bar_full[0][j % kTcStages], (j / kTcStages) & 1)) return false;
        k_ready = j + 1;
      }
      tc::fence_after_sync();
      const uint64_t q = t ? dq[1] : dq[0];
      const uint64_t k = (j % kTcStages) ? dk[1] : dk[0];
      const uint32_t d = tmem + t * kTileCols + kColS;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks)
        tc::mma_ss_by(leader, d, q + ((((ks >> 2) * (kTcBM * 128)) + (ks & 3) * 32) >> 4),
                      k + ((((ks >> 2) * (kTcBN * 128)) + (ks & 3) * 32) >> 4), IDESC_S, ks > 0);
      tc::commit_by(leader, &bar_s[t]);
      if (t) ++s_done1; else ++s_done0;
      return true;
    };
    auto issue_pv = [&](int t, int j) -> bool {  // O_t += P_t V_j
      if (j >= v_ready) {
        if (!wwait(&bar_full[1][j % kTcStages], (j / kTcStages) & 1)) return false;
        v_ready = j + 1;
      }
      if (!wwait(&bar_p[t], j & 1)) return false;
      tc::fence_after_sync();
      const uint64_t v = (j % kTcStages) ? dv[1] : dv[0];
      const uint32_t base = tmem + t * kTileCols;
#pragma unroll
      for (int ks = 0; ks < kTcBN / 16; ++ks) {
        // 16 keys a product; their P columns (the softmax's layout: keys
        // 16g..16g+15 at 32 (g / 2) + 8 (g % 2) for fp16, at 16g (P_hi) and
        // 16g + 8 (P_lo) for bf16: each 32 keys' P within their own S columns)
        const uint64_t bv = v + ((ks * 2048) >> 4);
        if constexpr (BF16) {
          tc::mma_ts_by(leader, base + kColO, base + kColS + ks * 16, bv, IDESC_O, j > 0 || ks > 0);
          tc::mma_ts_by(leader, base + kColO, base + kColS + ks * 16 + 8, bv, IDESC_O, true);
        } else {
          tc::mma_ts_by(leader, base + kColO, base + kColS + (ks >> 1) * 32 + (ks & 1) * 8, bv,
                        IDESC_O, j > 0 || ks > 0);
        }
      }
      tc::commit_by(leader, &bar_o[t]);
      if (t) ++o_done1; else ++o_done0;
      return true;
    };
    // Slot releases: K of block j once both tiles' S_t(j) are issued, V of
    // block j once both tiles' P_t(j) V are (a commit tracks every product
    // issued before it).
    int k_empties = 0, v_empties = 0;
    bool ok = wwait(&bar_q, 0);
    if (ok && nkb_t[0] > 0) ok = issue_s(0, 0);
    if (ok && nkb_t[1] > 0) ok = issue_s(1, 0);
    if (ok && nkb > 0) {
      tc::commit_by(leader, &bar_empty[0][0]);
      k_empties = 1;
    }
    for (int j = 0; j < nkb && ok; ++j) {
#pragma unroll
      for (int t = 0; t < kTcTiles; ++t) {
        if (!ok || j >= nkb_t[t]) continue;
        ok = issue_pv(t, j);
        if (ok && j + 1 < nkb_t[t]) ok = issue_s(t, j + 1);
      }
      if (ok) {
        tc::commit_by(leader, &bar_empty[1][j % kTcStages]);
        v_empties = j + 1;
        if (j + 1 < nkb) {
          tc::commit_by(leader, &bar_empty[0][(j + 1) % kTcStages]);
          k_empties = j + 2;
        }
      }
    }
    // drain: every product issued must finish, and every commit arrive,
    // before TMEM and this CTA's shared memory are given up
    for (int j = k_empties > kTcStages ? k_empties - kTcStages : 0; j < k_empties; ++j)
      mbar_wait_bounded(&bar_empty[0][j % kTcStages], (j / kTcStages) & 1, kTcDrainNs);
    for (int j = v_empties > kTcStages ? v_empties - kTcStages : 0; j < v_empties; ++j)
      mbar_wait_bounded(&bar_empty[1][j % kTcStages], (j / kTcStages) & 1, kTcDrainNs);
    if (s_done0 > 0) mbar_wait_bounded(&bar_s[0], (s_done0 - 1) & 1, kTcDrainNs);
    if (o_done0 > 0) mbar_wait_bounded(&bar_o[0], (o_done0 - 1) & 1, kTcDrainNs);
    if (s_done1 > 0) mbar_wait_bounded(&bar_s[1], (s_done1 - 1) & 1, kTcDrainNs);
    if (o_done1 > 0) mbar_wait_bounded(&bar_o[1], (o_done1 - 1) & 1, kTcDrainNs);
    __syncwarp();
  } else if (p.slot_mapping && h % (p.Hq / p.Hkv) == 0) {
    // ---------------- the new tokens' keys and values to the cache ----------------
    // The CTAs of a key/value head's first query head store the prompt's
    // tokens (each token of the prompt and head once): K and V rows from k,
    // v to their slots, by warps 18 and 19 while the others compute (the
    // pool holds the bits of pa_kv_cache_write afterwards).  Pair p of
    // tiles has about 4p + 3 blocks of attention, so it takes that share of
    // the prompt's tokens: [L c_p / c_P, L c_{p+1} / c_P) with
    // c_p = 2p^2 + p (the sum of 4i + 3 over i < p) and P pairs.  A slot
    // outside the pool is recorded as PA_ERR_BAD_SLOT and that token
    // skipped; a negative one skips it.
    const int64_t npairs = (L + kTcTiles * kTcBM - 1) / (kTcTiles * kTcBM);
    const int64_t cP = 2 * npairs * npairs + npairs;
    auto cum = [](int64_t q) { return 2 * q * q + q; };
    const int tok0 = static_cast<int>(L * cum(pair) / cP);
    const int n_tok = static_cast<int>(L * cum(pair + 1) / cP) - tok0;
    const int64_t num_slots = p.num_blocks * p.B;
    const int lid = (warp - kStoreWarp0) * 32 + lane;
    const uint64_t read_pol = l2_evict_first_policy();
    constexpr uint32_t ROW = D * 2;
    if (p.store_blocks) {
      // Whole blocks (a block's K and V rows of this head take at most 8 KB):
      // the shares' bounds are rounded down to multiples of B, so each
      // share is a run of groups of B tokens that start a block when the
      // prompt's slots run in order.  Warp 18 takes the even groups, warp
      // 19 the odd ones, each through its own 8 KB of staging.  A group
      // whose B slots are one block's, in order, moves as two tiled loads
      // (B rows of k, of v, from the [T][Hkv][D] tensors) and two bulk
      // stores of B rows each: 4 copies for 2B rows.  Any other group (the
      // prompt's last, partial one; slots out of order, negative or outside
      // the pool) goes row by row as below.
      const int Bq = p.B;
      auto bound = [&](int64_t q) -> int {
        if (q >= npairs) return L;
        return static_cast<int>(L * cum(q) / cP) & ~(Bq - 1);
      };
      const int t_lo = bound(pair), t_hi = bound(pair + 1);
      const int ws = warp - kStoreWarp0;
      uint8_t* stg = sKV + kTcStages * LY::STAGE + ws * 8192;
      uint64_t* wb = &bar_stw[ws];
      uint32_t wph = 0;
      const int ng = (t_hi - t_lo + Bq - 1) / Bq;
      for (int gi = ws; gi < ng; gi += 2) {
        const int t0 = t_lo + gi * Bq;
        const int n = min(Bq, t_hi - t0);
        const int64_t sl = lane < n ? __ldg(p.slot_mapping + a + t0 + lane) : -1;
        const int64_t s0 = __shfl_sync(0xffffffffu, sl, 0);
        const bool whole = n == Bq && s0 >= 0 && s0 < num_slots && (s0 & (Bq - 1)) == 0 &&
                           __all_sync(0xffffffffu, lane >= n || sl == s0 + lane);
        uint8_t* dst[2] = {nullptr, nullptr};
        if (whole) {
          if (lane == 0) {
            mbar_arrive_expect_tx(wb, 2u * Bq * ROW);
            tc::tma_load_3d(stg, &tm_ks, 0, kvh, a + t0, wb);
            tc::tma_load_3d(stg + Bq * ROW, &tm_vs, 0, kvh, a + t0, wb);
          } else {
            mbar_arrive(wb);
          }
        } else {
          // rows r = lane, lane + 32 of the group: K rows 0..n-1, then V rows
          uint32_t bytes = 0;
          const uint8_t* src[2] = {nullptr, nullptr};
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int r = lane + 32 * u;
            if (r < 2 * n) {
              const int kv = r >= n;
              const int64_t row = a + t0 + (r - kv * n);
              const int64_t slot = __ldg(p.slot_mapping + row);
              if (slot >= num_slots) {
                if (!kv) set_status(p.status, -9 /* PA_ERR_BAD_SLOT */);
              } else if (slot >= 0) {
                const int64_t blk = slot >> p.B_shift, place = slot & (p.B - 1);
                dst[u] = static_cast<uint8_t*>(kv ? p.v_cache : p.k_cache) +
                         (((blk * p.Hkv + kvh) << p.B_shift) + place) * ROW;
                src[u] = static_cast<const uint8_t*>(kv ? p.v : p.k) + (row * p.Hkv + kvh) * ROW;
                bytes += ROW;
              }
            }
          }
          if (bytes) {
            mbar_arrive_expect_tx(wb, bytes);
#pragma unroll
            for (int u = 0; u < 2; ++u)
              if (src[u]) bulk_copy_g2s(stg + (lane + 32 * u) * ROW, src[u], ROW, wb, read_pol);
          } else {
            mbar_arrive(wb);
          }
        }
        // one outcome for the whole warp (its lanes time their waits apart)
        const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(wb, wph, lim));
        if (!ok) {
          give_up();
          mbar_wait_bounded(wb, wph, kTcDrainNs);  // the copies still in flight
          break;
        }
        wph ^= 1;
        if (whole) {
          if (lane == 0) {
            const int64_t off = ((s0 >> p.B_shift) * p.Hkv + kvh) * Bq * ROW;
            tc::bulk_store(static_cast<uint8_t*>(p.k_cache) + off, stg, Bq * ROW);
            tc::bulk_store(static_cast<uint8_t*>(p.v_cache) + off, stg + Bq * ROW, Bq * ROW);
          }
        } else {
#pragma unroll
          for (int u = 0; u < 2; ++u)
            if (dst[u]) tc::bulk_store(dst[u], stg + (lane + 32 * u) * ROW, ROW);
        }
        tc::bulk_commit();
        tc::bulk_wait_read_all();  // the staging is read: it can be refilled
        __syncwarp();
      }
      tc::bulk_wait_read_all();
    } else {
    // Batches of 64 rows (K rows, then V rows), one per thread: a bulk copy
    // brings the row into the staging area, a bulk copy takes it to its
    // slot; the staging row is reused once that copy has read it.
    uint8_t* stage_row = sKV + kTcStages * LY::STAGE + lid * ROW;
    const int rows = 2 * n_tok;
    uint32_t phase = 0;
    // (The reads' L2 priority, evict-first, normal or evict-last, and an
    // evict-first hint on the writes measured within 0.4% of each other; a
    // barrier per thread instead of one for the 64, or 96 staging rows,
    // measured slower.)
    for (int r0 = 0; r0 < rows; r0 += 64, phase ^= 1) {
      const int rr = r0 + lid;
      void* dst = nullptr;
      if (rr < rows) {
        const int kv = rr >= n_tok;
        const int64_t row = a + tok0 + (rr - kv * n_tok);
        const int64_t slot = __ldg(p.slot_mapping + row);
        if (slot >= num_slots) {
          if (!kv) set_status(p.status, -9 /* PA_ERR_BAD_SLOT */);
        } else if (slot >= 0) {
          const int64_t blk = slot >> p.B_shift, place = slot & (p.B - 1);
          dst = static_cast<uint8_t*>(kv ? p.v_cache : p.k_cache) +
                (((blk * p.Hkv + kvh) << p.B_shift) + place) * ROW;
          mbar_arrive_expect_tx(&bar_st, ROW);
          bulk_copy_g2s(stage_row, static_cast<const uint8_t*>(kv ? p.v : p.k) +
                                       (row * p.Hkv + kvh) * ROW,
                        ROW, &bar_st, read_pol);
        }
      }
      if (!dst) mbar_arrive(&bar_st);
      if (!mbar_wait_bounded(&bar_st, phase, lim)) {
        give_up();
        break;
      }
      if (dst) {
        tc::bulk_store(dst, stage_row, ROW);
        tc::bulk_commit();
        tc::bulk_wait_read_all();  // the row is read: the staging can be refilled
      }
    }
    tc::bulk_wait_read_all();
    }
  }
  } else {
    // ---------------- softmax: half of one query row ----------------
    // (the softmax warpgroups first raise their registers, if split)
    if constexpr (kTcRegsHigh != kTcRegsLaunch) tc::regs_raise<kTcRegsHigh>();
    const int t = warp >> 3;                     // tile of this pair of warpgroups
    const int hf = (warp >> 2) & 1;              // which half of each block's keys
    const int row = (warp & 3) * 32 + lane;      // row within the tile = TMEM lane
    const int qpos = q0 + t * kTcBM + row;       // new row within the prompt (position cl + qpos)
    const uint32_t rbase = tmem + t * kTileCols + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    // Named barrier of the exchange: the tile's 256 threads.  (One barrier
    // per pair of warps that share rows, 64 threads, measured 0.5% slower.)
    const uint32_t tile_bar = 1 + t;
    constexpr uint32_t kBarThreads = 2 * kTcBM;
    float m = -INFINITY, l = 0.f;
    bool failed = false;
    const int nk = nkb_t[t];
    for (int jj = 0; jj < nk; ++jj) {
      // tcgen05.ld/st are warp-collective: guards around them are warp-uniform
      failed = __any_sync(0xffffffffu, failed || !wait(&bar_s[t], jj & 1));
      // Keys of this block from `lim` on are hidden from this row: past the
      // stored prefix in its last block (rows read as zeros), or past the row
      // itself among the new keys.
      int lim;
      if (jj < npre) {
        lim = min(kTcBN, cl - jj * kTcBN);
      } else {
        lim = min(kTcBN, max(0, qpos - (jj - npre) * kTcBN + 1));
      }
      const int lim_h = lim - hf * kTcHalf;      // the same, counted within this half
      // Hidden keys exist only in a warp's diagonal block and in the
      // prefix's last block: only warps that have any mask.
      const bool mask = __any_sync(0xffffffffu, lim_h < kTcHalf);
      // this half's scores, 32 at a time (two passes over TMEM keep the
      // registers of four warpgroups within the SM's)
      auto load32 = [&](int i, uint32_t (&v)[32]) {
        tc::ld32(rbase + kColS + hf * kTcHalf + i * 32, v);
        tc::wait_ld();
        if (mask) {
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (i * 32 + c >= lim_h) v[c] = __float_as_uint(-INFINITY);
        }
      };
      float pm = -INFINITY;                      // their max (raw scores)
      uint32_t v1[32], v0[32];                   // the half's keys 32-63 and 0-31
      if (!failed) {
        tc::fence_after_sync();
        // four independent partial maxima of three-input maxima
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        auto max_of = [&](const uint32_t (&v)[32]) {
#pragma unroll
          for (int c = 0; c < 32; c += 8)
#pragma unroll
            for (int u = 0; u < 4; ++u)
              mx[u] = fmax3(mx[u], __uint_as_float(v[c + 2 * u]), __uint_as_float(v[c + 2 * u + 1]));
        };
        if constexpr (kTcMaxOneWait) {
          // both loads in flight, one wait
          tc::ld32(rbase + kColS + hf * kTcHalf, v0);
          tc::ld32(rbase + kColS + hf * kTcHalf + 32, v1);
          tc::wait_ld();
          if (mask) {
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              if (c >= lim_h) v0[c] = __float_as_uint(-INFINITY);
              if (32 + c >= lim_h) v1[c] = __float_as_uint(-INFINITY);
            }
          }
          max_of(v0);
          max_of(v1);
        } else {
          load32(0, v0);
          max_of(v0);
          load32(1, v1);  // kept for the weights
          max_of(v1);
        }
        pm = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
        xmax[jj & 1][t][hf][row] = pm;
        // keys 0-31 again, their load in flight across the exchange
        if constexpr (kTcPrefetch == 1) tc::ld32(rbase + kColS + hf * kTcHalf, v0);
      }
      // the pair's maxima meet here; every thread of the tile learns whether
      // any gave up, so all leave together
      if (bar_any(tile_bar, kBarThreads, failed)) {
        failed = true;
        break;
      }
      // base-2 logits: the scale (> 0) is applied in the exponent
      const float rmax = fmaxf(pm, xmax[jj & 1][t][hf ^ 1][row]) * p.scale_log2;
      // P_t and O_t are in use by the previous block's product until it is
      // done, which is known here: S is issued after it, and the S-ready
      // commit tracks every product the MMA warp issued before it.
      const bool raise = rmax > m + 8.f;
      const float m_new = raise ? rmax : m;
      const float alpha = raise && m != -INFINITY ? fast_exp2(m - m_new) : 1.f;
      if (jj > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
        // this thread's half of the row of O
#pragma unroll
        for (int c0 = hf * (D / 2); c0 < hf * (D / 2) + D / 2; c0 += 32) {
          uint32_t o[2][16];
#pragma unroll
          for (int i = 0; i < 2; ++i) tc::ld16(rbase + kColO + c0 + i * 16, o[i]);
          tc::wait_ld();
#pragma unroll
          for (int i = 0; i < 2; ++i) {
#pragma unroll
            for (int c = 0; c < 16; ++c)
              o[i][c] = __float_as_uint(__uint_as_float(o[i][c]) * alpha);
            tc::st16(rbase + kColO + c0 + i * 16, o[i]);
          }
        }
      }
      l *= alpha;
      m = m_new;
      const float mm = m == -INFINITY ? 0.f : m;
      const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
      const float2 nm2 = make_float2(-mm, -mm);
      float2 ls[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};  // partial sums
      // The weights 2^(scale * s - m), two per packed fma; hidden scores are
      // -inf: weight 0.  Keys 32-63 of the half first (still in registers),
      // then keys 0-31 (read again, the load in flight meanwhile).
      // P goes back over the S columns of its own 32 keys as packed 16-bit
      // pairs: keys 16g..16g+15 (g = 0..7 over the block) take columns
      // 32 (g / 2) + 8 (g % 2) .. +7 (fp16), or 16g..16g+7 for P_hi and
      // 16g+8..16g+15 for P_lo = P - P_hi (bf16).
      auto chunk = [&](uint32_t (&v)[32], int i) {  // keys 32i..32i+31 of the half
      uint32_t pk[16];  // fp16: the chunk's two groups of 8 columns, stored together
#pragma unroll
      for (int g = 2 * i; g < 2 * i + 2; ++g) {  // this half's groups of 16 keys
        uint32_t ph[8], pl[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          const float2 x = __ffma2_rn(make_float2(__uint_as_float(v[(g & 1) * 16 + e]),
                                                  __uint_as_float(v[(g & 1) * 16 + e + 1])),
                                      sc2, nm2);
          const float2 pw = make_float2(fast_exp2(x.x), fast_exp2(x.y));
          ls[(e >> 1) & 1] = __fadd2_rn(ls[(e >> 1) & 1], pw);
          ph[e / 2] = Elem<T>::from_float2(pw.x, pw.y);
          if constexpr (BF16) {
            const float2 back = Elem<T>::to_float2(ph[e / 2]);
            pl[e / 2] = Elem<T>::from_float2(pw.x - back.x, pw.y - back.y);
          }
        }
        if constexpr (BF16) {
          uint32_t w[16];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            w[c] = ph[c];
            w[8 + c] = pl[c];
          }
          tc::st16(rbase + kColS + (4 * hf + g) * 16, w);
        } else {
#pragma unroll
          for (int c = 0; c < 8; ++c) pk[(g & 1) * 8 + c] = ph[c];
          if (g & 1) tc::st16(rbase + kColS + hf * 64 + i * 32, pk);
        }
      }
      };
      if constexpr (kTcPrefetch == 2) tc::ld32(rbase + kColS + hf * kTcHalf, v0);
      chunk(v1, 1);
      if constexpr (kTcPrefetch == 0) tc::ld32(rbase + kColS + hf * kTcHalf, v0);
      tc::wait_ld();
      if (mask) {
#pragma unroll
        for (int c = 0; c < 32; ++c)
          if (c >= lim_h) v0[c] = __float_as_uint(-INFINITY);
      }
      chunk(v0, 0);
      l += (ls[0].x + ls[0].y) + (ls[1].x + ls[1].y);
      tc::wait_st();
      tc::fence_before_sync();
      mbar_arrive(&bar_p[t]);
    }
    if (nk > 0) {
      // ---- epilogue: out = O / l, each thread its half of head_dim ----
      failed = __any_sync(0xffffffffu, failed || !wait(&bar_o[t], (nk - 1) & 1));
      xsum[t][hf][row] = l;
      if (!bar_any(tile_bar, kBarThreads, failed)) {
        tc::fence_after_sync();
        const float lt = l + xsum[t][hf ^ 1][row];
        const bool store = qpos < L;
        const float inv = lt > 0.f ? 1.f / lt : 0.f;
        T* orow = static_cast<T*>(p.out) + (static_cast<int64_t>(a + qpos) * p.Hq + h) * D;
#pragma unroll
        for (int c0 = hf * (D / 2); c0 < hf * (D / 2) + D / 2; c0 += 32) {
          uint32_t o[2][16];
#pragma unroll
          for (int i = 0; i < 2; ++i) tc::ld16(rbase + kColO + c0 + i * 16, o[i]);
          tc::wait_ld();
          if (store) {
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              float f[8];
#pragma unroll
              for (int k = 0; k < 8; ++k) f[k] = __uint_as_float(o[i][k]) * inv;
              *reinterpret_cast<uint4*>(orow + c0 + i * 16) = pack8<T>(f);
#pragma unroll
              for (int k = 0; k < 8; ++k) f[k] = __uint_as_float(o[i][8 + k]) * inv;
              *reinterpret_cast<uint4*>(orow + c0 + i * 16 + 8) = pack8<T>(f);
            }
          }
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::dealloc(tmem, kTmemCols);
}

template <typename T, int D>
cudaError_t launch_prefill_tc_typed(const PrefillArgs& a, cudaStream_t stream) {
  using LY = TcLayout<D>;
  {
    static std::mutex mu;
    static std::set<int> raised;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaGetLastError();
    std::lock_guard<std::mutex> lock(mu);
    if (!raised.count(dev)) {
      // The register split inside the kernel draws on the launch's
      // allocation: it must have been compiled to the count the split
      // assumes, or the warpgroups that raise theirs would wait forever.
      cudaFuncAttributes fa;
      if (cudaFuncGetAttributes(&fa, prefill_tc_kernel<T, D>) != cudaSuccess)
        return cudaGetLastError();
      constexpr bool split = kTcRegsHigh != kTcRegsLaunch || kTcRegsLow != kTcRegsLaunch;
      if (split && 4 * 128 * kTcRegsHigh + 128 * kTcRegsLow >
                       static_cast<uint32_t>(fa.numRegs) * kTcThreads)
        return cudaErrorInvalidConfiguration;
      if (cudaFuncSetAttribute(prefill_tc_kernel<T, D>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, LY::SMEM) !=
          cudaSuccess)
        return cudaGetLastError();
      raised.insert(dev);
    }
  }
  const int tiles = (a.max_seqlen + kTcTiles * kTcBM - 1) / (kTcTiles * kTcBM);  // pairs
  if (tiles <= 0) return cudaSuccess;
  // q as (D, Hq, T), k and v as (D, Hkv, T); boxes 64 x 1 x rows
  CUtensorMap tq, tk, tv;
  const uint64_t rows = static_cast<uint64_t>(a.num_tokens);
  const uint64_t dq[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(a.num_heads), rows};
  const uint64_t dk[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(a.num_kv_heads), rows};
  const uint64_t sq[2] = {static_cast<uint64_t>(D) * 2,
                          static_cast<uint64_t>(a.num_heads) * D * 2};
  const uint64_t sk[2] = {static_cast<uint64_t>(D) * 2,
                          static_cast<uint64_t>(a.num_kv_heads) * D * 2};
  const uint32_t bq[3] = {64u, 1u, static_cast<uint32_t>(kTcBM)};  // one tile of Q
  const uint32_t bk[3] = {64u, 1u, static_cast<uint32_t>(kTcBN)};
  const bool bf16 = std::is_same<T, __nv_bfloat16>::value;
  if (!encode_swizzled_map(&tq, a.q, bf16, 3, dq, sq, bq) ||
      !encode_swizzled_map(&tk, a.k, bf16, 3, dk, sk, bk) ||
      !encode_swizzled_map(&tv, a.v, bf16, 3, dk, sk, bk))
    return cudaErrorInvalidValue;
  // the cache pools [N][Hkv][B][D] as (D, B, Hkv, N); one physical block of
  // one head per box of 64 x B (only when a stored prefix is read)
  CUtensorMap tkc = tk, tvc = tv;
  const bool paged = a.cached_lens != nullptr;
  if (paged) {
    const uint64_t dc[4] = {static_cast<uint64_t>(D), static_cast<uint64_t>(a.block_size),
                            static_cast<uint64_t>(a.num_kv_heads),
                            static_cast<uint64_t>(a.num_blocks)};
    const uint64_t sc[3] = {static_cast<uint64_t>(D) * 2,
                            static_cast<uint64_t>(a.block_size) * D * 2,
                            static_cast<uint64_t>(a.num_kv_heads) * a.block_size * D * 2};
    const uint32_t bc[4] = {64u, static_cast<uint32_t>(a.block_size), 1u, 1u};
    if (!encode_swizzled_map(&tkc, a.k_cache, bf16, 4, dc, sc, bc) ||
        !encode_swizzled_map(&tvc, a.v_cache, bf16, 4, dc, sc, bc))
      return cudaErrorInvalidValue;
  }
  // the new tokens' k and v as (D, Hkv, T) again, unswizzled boxes of D x 1
  // x B: one block's rows of one head, row-major, for whole-block stores
  CUtensorMap tks = tk, tvs = tv;
  const bool store_blocks = kTcStoreBlocks && a.slot_mapping && a.block_size <= 32 &&
                            2 * a.block_size * D * 2 <= 8192;
  if (store_blocks) {
    const uint32_t bs[3] = {static_cast<uint32_t>(D), 1u, static_cast<uint32_t>(a.block_size)};
    const CUtensorMapDataType ty =
        bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    if (!encode_plain_map(&tks, a.k, ty, 3, dk, sk, bs) ||
        !encode_plain_map(&tvs, a.v, ty, 3, dk, sk, bs))
      return cudaErrorInvalidValue;
  }
  TcParams p;
  p.store_blocks = store_blocks ? 1 : 0;
  p.out = a.out;
  p.cu_seqlens = a.cu_seqlens;
  p.num_tokens = a.num_tokens;
  p.max_seqlen = a.max_seqlen;
  p.Hq = a.num_heads;
  p.Hkv = a.num_kv_heads;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.status = a.status;
  p.wait_limit_ns = a.wait_limit_ns;
  p.B = paged ? a.block_size : 1;
  p.num_blocks = a.num_blocks;
  p.block_tables = a.block_tables;
  p.cached_lens = a.cached_lens;
  p.max_blocks = a.max_blocks_per_seq;
  p.k = a.k;
  p.v = a.v;
  p.k_cache = a.k_cache;
  p.v_cache = a.v_cache;
  p.slot_mapping = a.slot_mapping;
  if (a.slot_mapping) p.B = a.block_size;
  p.B_shift = 0;
  while ((1 << p.B_shift) < p.B) ++p.B_shift;
  cudaLaunchConfig_t cfg = {};
  if (tiles > 65535) return cudaErrorInvalidValue;  // prompts of up to 16.7 M tokens
  cfg.gridDim = dim3(a.num_heads, tiles, a.num_seqs);
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = LY::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t err =
      cudaLaunchKernelEx(&cfg, prefill_tc_kernel<T, D>, p, tq, tk, tv, tkc, tvc, tks, tvs);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace

bool prefill_tc_paged_ok(int block_size, int64_t num_blocks) {
  // boxes of B rows start on 1024-byte boundaries of the swizzled tiles;
  // block indices (num_blocks itself reads as zeros) fit the 32-bit
  // coordinates of the tensor map
  return (block_size == 8 || block_size == 16 || block_size == 32) && num_blocks > 0 &&
         num_blocks < (int64_t{1} << 31) - 1;
}

cudaError_t launch_prefill_tc(const PrefillArgs& a, cudaStream_t stream) {
  if (a.cached_lens &&
      (!a.k_cache || !a.v_cache || !prefill_tc_paged_ok(a.block_size, a.num_blocks) ||
       !a.block_tables || a.max_blocks_per_seq < 1))
    return cudaErrorInvalidValue;
  if (a.slot_mapping && (!a.k_cache || !a.v_cache || a.block_size < 1 ||
                         (a.block_size & (a.block_size - 1)) || a.num_blocks < 1))
    return cudaErrorInvalidValue;
  if (a.head_dim == 128)
    return a.is_bf16 ? launch_prefill_tc_typed<__nv_bfloat16, 128>(a, stream)
                     : launch_prefill_tc_typed<__half, 128>(a, stream);
  if (a.head_dim == 64)
    return a.is_bf16 ? launch_prefill_tc_typed<__nv_bfloat16, 64>(a, stream)
                     : launch_prefill_tc_typed<__half, 64>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace pa
