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
// How (FlashAttention-4's arrangement on sm_100a): one CTA takes two tiles of
// 128 queries of one (prompt, head), 256 consecutive queries, and runs twelve
// warps with separate jobs:
//   * warp 9 loads: Q of both tiles once, then each block of kTcBN keys
//     (128; 64 as a build option) of K and of V, each into a ring of its own
//     of 2 slots (3 for 64-key blocks): a K slot refills once both tiles' S
//     have read it, a step before the block's V slot frees, which gives the
//     loads about two steps of lead.  Tiled TMA with the 128-byte swizzle: the new
//     tokens from q, k, v (the [T][H][D] tensors seen as (D, H, T); boxes
//     64 x 1 x rows), the stored prefix from the cache pools (seen as
//     (D, B, H, N); one box of 64 x B rows per physical block, found in the
//     block table).  The CTA that holds a key block's own queries also
//     stores that block of the new keys and values in the cache: TMA stores
//     of the tiles already in shared memory, one box per physical block, when
//     the block's slots fill whole physical blocks in order (the usual case),
//     else row by row from the warp's lanes;
//   * warp 8 (lane 0 issuing, the whole warp running the loop) issues the
//     tensor-core products, tcgen05.mma kind::f16, accumulating in tensor
//     memory (TMEM): S_t = Q_t K^T (both operands K-major in shared memory)
//     and O_t += P_t V (P_t from TMEM, V MN-major in shared memory), in the
//     order S0, S1, then per block PV0, S0', PV1, S1': while one tile's
//     softmax runs, the tensor pipe works on the other tile's products;
//   * warps 0-3 and 4-7: the softmax of tile 0 and tile 1, one thread per
//     query row (its warp's 32 TMEM lanes), so the row max and sum stay in
//     the thread.  The row's scores are read from TMEM once (a build option
//     reads them twice, for the max and for the weights, 32 at a time, to
//     spare registers); then the max, then the weights.  Base 2; the running max is raised only
//     when a score passes it by more than 2^8, which then rescales that row
//     of O in TMEM.  Two scores per packed fp32 instruction, maxima three at
//     a time; a build option moves a share of the weights of unmasked blocks
//     to an FMA-pipe polynomial (exp2poly.cuh).  P (and for bf16 the rest
//     P - P_hi, so P enters as about 16 significant bits) goes back into the
//     S columns it was computed from, as packed 16-bit pairs.
//   * After its last block each softmax thread divides its row of O by its
//     sum and stores it.
// Barriers: per ring slot, for K and for V, full (TMA bytes) and empty (the
// last product that reads it); per tile S ready, P ready (128 arrivals) and
// O done.  TMEM per tile:
// S (and P over it) kTcBN columns, O head_dim, 256 in all; 512 for the two
// tiles, one CTA per SM.  Blocks of 128 keys halve the handoffs per product
// (every wait on a completed barrier still costs over a hundred cycles) and
// give S products of N = 128, which the tensor pipe runs at full rate.
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
#include "exp2poly.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "tcgen05.cuh"

namespace pa {

namespace {

constexpr int kTcBM = 128;      // queries per tile (MMA M)
#ifndef PA_TC_BN
#define PA_TC_BN 128
#endif
constexpr int kTcBN = PA_TC_BN;   // keys per block (MMA N of S, K of P V): 64 or 128
static_assert(kTcBN == 64 || kTcBN == 128, "blocks of 64 or 128 keys");
constexpr int kTcTiles = 2;     // query tiles per CTA
constexpr int kTcStages = kTcBN == 128 ? 2 : 3;  // K/V ring depth (64 KB or 32 KB a stage)
// 8 softmax warps (warpgroups 0 and 1), then warpgroup 2: the MMA warp, the
// load warp and two idle warps.  The launch gives every thread 168 registers
// (384 x 168 of the SM's 65,536); warpgroup 2 then lowers to kTcRegsLow and
// the softmax warpgroups raise to kTcRegsHigh:
// 2 x 128 x 208 + 128 x 80 = 63,488 <= 64,512 (the split at which neither
// side spills).
constexpr int kTcThreads = 384;
constexpr int kMmaWarp = 8, kLoadWarp = 9;
#ifndef PA_TC_REGS_HIGH
#define PA_TC_REGS_HIGH 208
#endif
#ifndef PA_TC_REGS_LOW
#define PA_TC_REGS_LOW 80
#endif
constexpr uint32_t kTcRegsHigh = PA_TC_REGS_HIGH, kTcRegsLow = PA_TC_REGS_LOW;
static_assert(2 * 128 * kTcRegsHigh + 128 * kTcRegsLow <= kTcThreads * 168, "register split");
// TMEM columns of a tile: S from kColS (kTcBN of them), P written over S
// (see the softmax), O from kColO.
constexpr uint32_t kColS = 0, kColO = 128;
constexpr uint32_t kTileCols = 256, kTmemCols = 512;
constexpr int64_t kTcDrainNs = 1000000000;
#ifndef PA_TC_POLY_PAIRS
#define PA_TC_POLY_PAIRS 0
#endif
// Of every four pairs of softmax weights in a block below the diagonal, this
// many are computed by the FMA-pipe polynomial (exp2poly.cuh), the rest by
// the exponential unit.
constexpr int kTcPolyPairs = PA_TC_POLY_PAIRS;
#ifndef PA_TC_PACKED
#define PA_TC_PACKED 1
#endif
// 1: the softmax's scores go through packed fp32 instructions two at a time
// and three-input maxima; 0: one score per instruction.
constexpr bool kTcPacked = PA_TC_PACKED != 0;

#ifndef PA_TC_ONE_LOAD
#define PA_TC_ONE_LOAD 1
#endif
// 1: the softmax reads a row's scores from TMEM once, all kTcBN of them into
// registers (568 against 548 TFLOP/s on the 16 x 2,048-token step); 0:
// twice (the max, then the weights 32 at a time).
constexpr bool kTcOneLoad = PA_TC_ONE_LOAD != 0;

// max(a, b, c) in one instruction (three-input max.f32 of sm_100)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

template <int D>
struct TcLayout {
  static constexpr int HALVES = D / 64;           // 64-element (128-byte) column blocks
  static constexpr int Q_BYTES = kTcBM * D * 2;   // one tile of Q: 32 KB at head_dim 128
  static constexpr int KV_BYTES = kTcBN * D * 2;  // one block of K (or V): 32 KB at D = 128
  static constexpr int STAGE = 2 * KV_BYTES;      // K block, then V block
  // shared memory asked for (+ 1 KB to align by hand): the head_dim-128
  // amount at every head_dim, so one CTA holds an SM (its 512 TMEM columns)
  static constexpr int SMEM = 1024 + kTcTiles * (kTcBM * 128 * 2) + kTcStages * (2 * kTcBN * 128 * 2);
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
  // read from it through block_tables / cached_lens (null: none), and the new
  // tokens' keys and values are written to it at slot_mapping (null: not).
  int B;
  int64_t num_blocks;
  const int32_t* block_tables;
  const int32_t* cached_lens;
  int max_blocks;
  const int64_t* slot_mapping;
  void* k_cache;
  void* v_cache;
};

template <typename T, int D>
__global__ void __launch_bounds__(kTcThreads, 1)
prefill_tc_kernel(const TcParams p, const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const __grid_constant__ CUtensorMap tm_kc, const __grid_constant__ CUtensorMap tm_vc) {
  using LY = TcLayout<D>;
  constexpr bool BF16 = std::is_same<T, __nv_bfloat16>::value;
  constexpr uint32_t IDESC_S = tc::idesc_f16(kTcBM, kTcBN, BF16, false);
  constexpr uint32_t IDESC_O = tc::idesc_f16(kTcBM, D, BF16, true);
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 128-byte swizzle patterns repeat every 1024 bytes of shared address: align by hand
  uint8_t* smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
  uint8_t* sQ = smem;                               // tile t at t * Q_BYTES
  uint8_t* sKV = smem + kTcTiles * LY::Q_BYTES;     // stage i at i * STAGE
  // per ring slot, separately for K (index 0) and V (index 1): full (TMA
  // bytes) and empty (the last product that reads it)
  __shared__ uint64_t bar_q, bar_full[2][kTcStages], bar_empty[2][kTcStages];
  __shared__ uint64_t bar_s[kTcTiles], bar_p[kTcTiles], bar_o[kTcTiles];
  __shared__ uint32_t tmem_base;
  __shared__ volatile int abort_flag;

  griddep_wait();
  const int s = blockIdx.z, h = blockIdx.y;
  const int a = __ldg(p.cu_seqlens + s), b = __ldg(p.cu_seqlens + s + 1);
  if (a < 0 || b < a || b > p.num_tokens) {
    if (blockIdx.x == 0 && h == 0 && threadIdx.x == 0) set_status(p.status, -8 /* PA_ERR_BAD_LEN */);
    return;
  }
  const int L = b - a;  // new tokens of this prompt
  if (L > p.max_seqlen && blockIdx.x == 0 && h == 0 && threadIdx.x == 0)
    set_status(p.status, -8 /* PA_ERR_BAD_LEN: a prompt longer than max_seqlen */);
  // stored prefix: a whole number of blocks that the table holds
  const int cl = p.cached_lens ? __ldg(p.cached_lens + s) : 0;
  if (cl < 0 || cl % p.B || cl > p.max_blocks * p.B) {
    if (blockIdx.x == 0 && h == 0 && threadIdx.x == 0) set_status(p.status, -8 /* PA_ERR_BAD_LEN */);
    return;
  }
  const int npre = (cl + kTcBN - 1) / kTcBN;        // key blocks of the stored prefix
  const int pair = gridDim.x - 1 - blockIdx.x;       // heaviest pairs of tiles first
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
      mbar_init(&bar_p[t], kTcBM);
      mbar_init(&bar_o[t], 1);
    }
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

  if (warp >= 8) {
  // warpgroup 2 lowers its registers, then runs its roles
  tc::regs_lower<kTcRegsLow>();
  if (warp == kLoadWarp) {
    // ---------------- loads (lane 0) and stores of the new keys ----------------
    if (lane == 0) {
      tc::prefetch_map(&tm_q);
      tc::prefetch_map(&tm_k);
      tc::prefetch_map(&tm_v);
      if (p.cached_lens || p.slot_mapping) {
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
    }
    // Key block jj: the stored prefix's block jj (jj < npre), else block
    // jj - npre of the new keys.  K and V have rings of their own (w = 0, 1),
    // so a K slot is refilled as soon as both tiles' S products have read
    // it, a step before the V slot of the same block frees.
    const int32_t* table = p.cached_lens ? p.block_tables + static_cast<int64_t>(s) * p.max_blocks
                                         : nullptr;
    auto load_part = [&](int jj, int w) {  // lane 0
      const int st = jj % kTcStages;
      uint8_t* dst = sKV + st * LY::STAGE + w * LY::KV_BYTES;
      uint64_t* bar = &bar_full[w][st];
      mbar_arrive_expect_tx(bar, LY::KV_BYTES);
      if (jj < npre) {
        // one box of B rows per physical block; rows past the prefix (and bad
        // table entries) are read from block num_blocks, outside the pool:
        // zeros, so their scores are finite and their values add nothing
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
            tc::tma_load_4d(dst + hf * (kTcBN * 128) + r0 * 128, w ? &tm_vc : &tm_kc, hf * 64, 0,
                            kvh, blk, bar);
        }
      } else {
        const int j = jj - npre;
#pragma unroll
        for (int hf = 0; hf < LY::HALVES; ++hf)
          tc::tma_load_3d(dst + hf * (kTcBN * 128), w ? &tm_v : &tm_k, hf * 64, kvh,
                          a + j * kTcBN, bar);
      }
    };
    // The new keys' blocks whose rows are this CTA's own queries go to the
    // cache from here (one query head per key/value head stores them).
    const bool stores = p.slot_mapping && h % (p.Hq / p.Hkv) == 0;
    const int own_lo = npre + q0 / kTcBN;
    const int64_t num_slots = p.num_blocks * p.B;
    // a wait whose outcome the whole warp shares (the stores use warp votes)
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return !__any_sync(0xffffffffu, !wait(bar, parity));
    };
    // store the K (w = 0) or V (w = 1) tile of block jj, once it has landed
    auto store_part = [&](int jj, int w) -> bool {  // whole warp
      const int st = jj % kTcStages;
      if (!wwait(&bar_full[w][st], (jj / kTcStages) & 1)) return false;
      const uint8_t* src = sKV + st * LY::STAGE + w * LY::KV_BYTES;
      const CUtensorMap* map = w ? &tm_vc : &tm_kc;
      T* cache = static_cast<T*>(w ? p.v_cache : p.k_cache);
      const int j = jj - npre;
      bool plain = false;
      for (int r0 = 0; r0 < kTcBN; r0 += p.B) {
        // lane r < B takes row r0 + r of the block: new token j*kTcBN + r0 + r
        const int pos = j * kTcBN + r0 + lane;
        int64_t slot = -2;  // no token
        if (lane < p.B && pos < L) slot = __ldg(p.slot_mapping + a + pos);
        const int64_t s0 = __shfl_sync(0xffffffffu, slot, 0);
        const bool in_order = lane >= p.B || slot == s0 + lane;
        if (__all_sync(0xffffffffu, in_order) && s0 >= 0 && s0 % p.B == 0 &&
            s0 + p.B <= num_slots) {
          // the B rows fill physical block s0 / B in order: one box per half
          if (lane == 0) {
            const int blk = static_cast<int>(s0 / p.B);
#pragma unroll
            for (int hf = 0; hf < LY::HALVES; ++hf)
              tc::tma_store_4d(map, src + hf * (kTcBN * 128) + r0 * 128, hf * 64, 0, kvh, blk);
            tc::bulk_commit();
          }
        } else if (lane < p.B && slot >= num_slots) {
          if (w == 0) set_status(p.status, -9 /* PA_ERR_BAD_SLOT */);
        } else if (lane < p.B && slot >= 0) {
          // row by row: undo the swizzle (16-byte piece c of row r sits at
          // piece c ^ (r % 8)) and write the row at its slot
          const int r = r0 + lane;
          const int64_t row = ((slot / p.B) * p.Hkv + kvh) * p.B + slot % p.B;
          uint4* dst = reinterpret_cast<uint4*>(cache + row * D);
#pragma unroll
          for (int hf = 0; hf < LY::HALVES; ++hf)
#pragma unroll
            for (int c = 0; c < 8; ++c)
              dst[hf * 8 + c] = *reinterpret_cast<const uint4*>(
                  src + hf * (kTcBN * 128) + r * 128 + ((c ^ (r & 7)) << 4));
          plain = true;
        }
      }
      // generic reads of the slot before the next TMA load writes it
      if (plain) fence_proxy_async_smem();
      __syncwarp();
      return true;
    };
    int issued_w[2] = {0, 0}, stored = own_lo;
    bool ok = true;
    for (int jj = 0; jj < nkb && ok; ++jj) {
      const int st = jj % kTcStages;
#pragma unroll
      for (int w = 0; w < 2 && ok; ++w) {
        if (jj >= kTcStages) {
          if (!(ok = wwait(&bar_empty[w][st], ((jj / kTcStages) - 1) & 1))) break;
          // the slot still holds block jj - kTcStages: store it if it is ours,
          // and let the stores finish reading it before it is refilled
          if (stores && jj - kTcStages >= own_lo) {
            if (!(ok = store_part(jj - kTcStages, w))) break;
            if (w == 1) stored = jj - kTcStages + 1;
            if (lane == 0) tc::bulk_wait_read_all();
            __syncwarp();
          }
        }
        if (lane == 0) load_part(jj, w);
        issued_w[w] = jj + 1;
      }
    }
    // our blocks still in the rings
    for (int jj = stored; stores && ok && jj < issued_w[1]; ++jj)
      ok = store_part(jj, 0) && store_part(jj, 1);
    if (lane == 0) {
      // drain: the stores must have read their tiles, and the copies in
      // flight landed, before this CTA's shared memory goes (the stores'
      // global writes complete with the grid, like any other store)
      tc::bulk_wait_read_all();
      mbar_wait_bounded(&bar_q, 0, kTcDrainNs);
#pragma unroll
      for (int w = 0; w < 2; ++w)
        for (int j = issued_w[w] > kTcStages ? issued_w[w] - kTcStages : 0; j < issued_w[w]; ++j)
          mbar_wait_bounded(&bar_full[w][j % kTcStages], (j / kTcStages) & 1, kTcDrainNs);
    }
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
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return !__any_sync(0xffffffffu, !wait(bar, parity));
    };
    // descriptors of the two Q tiles and of the K and V blocks of each stage;
    // a step along K adds its byte offset >> 4 to the start-address field
    uint64_t dq[kTcTiles], dk[kTcStages], dv[kTcStages];
#pragma unroll
    for (int t = 0; t < kTcTiles; ++t) dq[t] = tc::smem_desc(smem_addr(sQ + t * LY::Q_BYTES), 16, 1024);
#pragma unroll
    for (int i = 0; i < kTcStages; ++i) {
      dk[i] = tc::smem_desc(smem_addr(sKV + i * LY::STAGE), 16, 1024);
      dv[i] = tc::smem_desc(smem_addr(sKV + i * LY::STAGE + LY::KV_BYTES), kTcBN * 128, 1024);
    }
    // a stage's descriptor by a run-time index, without local memory
    auto sel = [](const uint64_t (&a)[kTcStages], int i) -> uint64_t {
      uint64_t r = a[0];
#pragma unroll
      for (int k = 1; k < kTcStages; ++k)
        if (i == k) r = a[k];
      return r;
    };
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
      const uint64_t k = sel(dk, j % kTcStages);
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
      const uint64_t v = sel(dv, j % kTcStages);
      const uint32_t base = tmem + t * kTileCols;
#pragma unroll
      for (int ks = 0; ks < kTcBN / 16; ++ks) {
        // 16 keys a product; their P columns (the softmax's layout)
        const uint64_t b = v + ((ks * 2048) >> 4);
        if constexpr (BF16) {
          tc::mma_ts_by(leader, base + kColO, base + kColS + ks * 16, b, IDESC_O, j > 0 || ks > 0);
          tc::mma_ts_by(leader, base + kColO, base + kColS + ks * 16 + 8, b, IDESC_O, true);
        } else {
          tc::mma_ts_by(leader, base + kColO, base + kColS + ks * 8, b, IDESC_O, j > 0 || ks > 0);
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
  }
  } else {
    // ---------------- softmax of one query row ----------------
    // (the softmax warpgroups first raise their registers)
    tc::regs_raise<kTcRegsHigh>();
    const int t = warp >> 2;                     // tile of this warpgroup
    const int row = tid & (kTcBM - 1);           // row within the tile = TMEM lane
    const int qpos = q0 + t * kTcBM + row;       // new row within the prompt (position cl + qpos)
    const uint32_t rbase = tmem + t * kTileCols + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    float m = -INFINITY, l = 0.f;
    bool failed = false;
    const int nk = nkb_t[t];
    for (int jj = 0; jj < nk; ++jj) {
      // tcgen05.ld/st are warp-collective: guards around them are warp-uniform
      failed = __any_sync(0xffffffffu, failed || !wait(&bar_s[t], jj & 1));
      if (failed) break;
      tc::fence_after_sync();
      // Keys of this block from `lim` on are hidden from this row: past the
      // stored prefix in its last block (rows read as zeros), or past the row
      // itself among the new keys.  `below`: no score of this warp's rows is
      // hidden, so part of the weights may come from the polynomial.
      int lim;
      bool below;
      if (jj < npre) {
        lim = min(kTcBN, cl - jj * kTcBN);
        below = jj * kTcBN + kTcBN <= cl;
      } else {
        const int j = jj - npre;
        lim = min(kTcBN, max(0, qpos - j * kTcBN + 1));
        below = j * kTcBN + kTcBN - 1 <= q0 + t * kTcBM + (warp & 3) * 32;
      }
      // Hidden keys exist only in a warp's diagonal block and in the prefix's
      // last block: the warps that have any take the masking path, the rest
      // (most blocks) the one without a compare per score.
      const bool masked = lim < kTcBN;
      float2 ls[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};  // partial sums
      auto block = [&](auto mask_tag) {
        constexpr bool MASK = decltype(mask_tag)::value;
        auto score = [&](uint32_t bits, int key) -> float {
          if constexpr (MASK) return key >= lim ? -INFINITY : __uint_as_float(bits);
          return __uint_as_float(bits);
        };
        // the row's scores, when they are read once
        uint32_t all[kTcOneLoad ? kTcBN / 32 : 1][32];
        // Pass 1, the row max: the scores 64 columns at a time (two loads in
        // flight, one wait), four independent partial maxima of three-input
        // maxima.
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        auto max_of = [&](const uint32_t (&v)[32], int key0) {
#pragma unroll
          for (int c = 0; c < 32; c += 8)
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int key = key0 + c + 2 * u;
              const float a = score(v[c + 2 * u], key), b = score(v[c + 2 * u + 1], key + 1);
              if constexpr (kTcPacked) {
                mx[u] = fmax3(mx[u], a, b);
              } else {
                mx[u] = fmaxf(fmaxf(mx[u], a), b);
              }
            }
        };
        if constexpr (kTcOneLoad) {
#pragma unroll
          for (int c = 0; c < kTcBN / 32; ++c) tc::ld32(rbase + kColS + c * 32, all[c]);
          tc::wait_ld();
#pragma unroll
          for (int c = 0; c < kTcBN / 32; ++c) max_of(all[c], c * 32);
        } else {
#pragma unroll
          for (int h = 0; h < kTcBN / 64; ++h) {
            uint32_t v[2][32];
            tc::ld32(rbase + kColS + h * 64, v[0]);
            tc::ld32(rbase + kColS + h * 64 + 32, v[1]);
            tc::wait_ld();
            max_of(v[0], h * 64);
            max_of(v[1], h * 64 + 32);
          }
        }
        // base-2 logits: the scale (> 0) is applied in the exponent
        const float rmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * p.scale_log2;
        // P_t and O_t are in use by the previous block's product until it is
        // done, which is known here: S is issued after it, and the S-ready
        // commit tracks every product the MMA warp issued before it.
        const bool raise = rmax > m + 8.f;
        const float m_new = raise ? rmax : m;
        const float alpha = raise && m != -INFINITY ? fast_exp2(m - m_new) : 1.f;
        if (jj > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 64) {
            uint32_t v[4][16];
#pragma unroll
            for (int i = 0; i < 4; ++i) tc::ld16(rbase + kColO + c0 + i * 16, v[i]);
            tc::wait_ld();
#pragma unroll
            for (int i = 0; i < 4; ++i) {
#pragma unroll
              for (int c = 0; c < 16; ++c)
                v[i][c] = __float_as_uint(__uint_as_float(v[i][c]) * alpha);
              tc::st16(rbase + kColO + c0 + i * 16, v[i]);
            }
          }
        }
        l *= alpha;
        m = m_new;
        const float mm = m == -INFINITY ? 0.f : m;
        const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
        const float2 nm2 = make_float2(-mm, -mm);
        // Pass 2, the weights 2^(scale * s - m), 32 keys at a time (read
        // again from TMEM, the next chunk's load in flight while this one is
        // computed, unless the scores were read once), two scores per packed
        // fma; hidden scores are -inf: weight 0.  Below the diagonal,
        // kTcPolyPairs of every four pairs of weights come from the FMA-pipe
        // polynomial and the rest from the exponential unit.
        // P goes back over S as packed 16-bit pairs: keys 16g..16g+15 take
        // columns 8g..8g+7 (fp16), or 16g..16g+7 for P_hi and 16g+8..16g+15
        // for P_lo = P - P_hi (bf16, so P enters with about 16 significant
        // bits).  Chunk c's P thus lands in columns that chunks 0..c were
        // read from, never in one still to be read.
        auto weights = [&](const uint32_t (&v)[32], int c) {
          uint32_t ph[16], pl[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const int key = c * 32 + e;
            const float a = score(v[e], key), b = score(v[e + 1], key + 1);
            const bool poly = below && ((e >> 1) & 3) >= 4 - kTcPolyPairs;
            float2 pw;
            if constexpr (kTcPacked) {
              const float2 x = __ffma2_rn(make_float2(a, b), sc2, nm2);
              pw = poly ? exp2_poly2(x) : make_float2(fast_exp2(x.x), fast_exp2(x.y));
              ls[(e >> 1) & 1] = __fadd2_rn(ls[(e >> 1) & 1], pw);
            } else {
              pw = make_float2(fast_exp2(fmaf(a, p.scale_log2, -mm)),
                               fast_exp2(fmaf(b, p.scale_log2, -mm)));
              ls[(e >> 1) & 1].x += pw.x + pw.y;
            }
            ph[e / 2] = Elem<T>::from_float2(pw.x, pw.y);
            if constexpr (BF16) {
              const float2 back = Elem<T>::to_float2(ph[e / 2]);
              pl[e / 2] = Elem<T>::from_float2(pw.x - back.x, pw.y - back.y);
            }
          }
          if constexpr (BF16) {
            uint32_t w[2][16];
#pragma unroll
            for (int g = 0; g < 2; ++g)
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                w[g][i] = ph[g * 8 + i];
                w[g][8 + i] = pl[g * 8 + i];
              }
            tc::st16(rbase + kColS + c * 32, w[0]);
            tc::st16(rbase + kColS + c * 32 + 16, w[1]);
          } else {
            tc::st16(rbase + kColS + c * 16, ph);
          }
        };
        if constexpr (kTcOneLoad) {
#pragma unroll
          for (int c = 0; c < kTcBN / 32; ++c) weights(all[c], c);
        } else {
          uint32_t v[2][32];
          tc::ld32(rbase + kColS, v[0]);
          tc::wait_ld();
#pragma unroll
          for (int c = 0; c < kTcBN / 32; ++c) {
            if (c + 1 < kTcBN / 32) tc::ld32(rbase + kColS + (c + 1) * 32, v[(c + 1) & 1]);
            weights(v[c & 1], c);
            if (c + 1 < kTcBN / 32) tc::wait_ld();
          }
        }
      };
      if (__any_sync(0xffffffffu, masked)) {
        block(std::true_type{});
      } else {
        block(std::false_type{});
      }
      l += (ls[0].x + ls[0].y) + (ls[1].x + ls[1].y);
      tc::wait_st();
      tc::fence_before_sync();
      mbar_arrive(&bar_p[t]);
    }
    if (!failed && nk > 0) {
      // ---- epilogue: out = O / l ----
      failed = __any_sync(0xffffffffu, !wait(&bar_o[t], (nk - 1) & 1));
      if (!failed) {
        tc::fence_after_sync();
        const bool store = qpos < L;
        const float inv = l > 0.f ? 1.f / l : 0.f;
        T* orow = static_cast<T*>(p.out) + (static_cast<int64_t>(a + qpos) * p.Hq + h) * D;
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 64) {
          uint32_t v[4][16];
#pragma unroll
          for (int i = 0; i < 4; ++i) tc::ld16(rbase + kColO + c0 + i * 16, v[i]);
          tc::wait_ld();
          if (store) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              float f[8];
#pragma unroll
              for (int k = 0; k < 8; ++k) f[k] = __uint_as_float(v[i][k]) * inv;
              *reinterpret_cast<uint4*>(orow + c0 + i * 16) = pack8<T>(f);
#pragma unroll
              for (int k = 0; k < 8; ++k) f[k] = __uint_as_float(v[i][8 + k]) * inv;
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
  // one head per box of 64 x B (only when the kernel reads or writes them)
  CUtensorMap tkc = tk, tvc = tv;
  const bool paged = a.cached_lens || a.slot_mapping;
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
  TcParams p;
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
  p.slot_mapping = a.slot_mapping;
  p.k_cache = a.k_cache;
  p.v_cache = a.v_cache;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(tiles, a.num_heads, a.num_seqs);
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = LY::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t err = cudaLaunchKernelEx(&cfg, prefill_tc_kernel<T, D>, p, tq, tk, tv, tkc, tvc);
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
  if ((a.cached_lens || a.slot_mapping) &&
      (!a.k_cache || !a.v_cache || !prefill_tc_paged_ok(a.block_size, a.num_blocks) ||
       (a.cached_lens && (!a.block_tables || a.max_blocks_per_seq < 1))))
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
