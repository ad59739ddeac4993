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
// 128 queries of one (prompt, head), 256 consecutive queries, and runs ten
// warps with separate jobs:
//   * warp 9 loads: Q of both tiles once, then each 64-key block of K and V
//     into a 3-stage ring, by tiled TMA with the 128-byte swizzle: the new
//     tokens from q, k, v (the [T][H][D] tensors seen as (D, H, T); boxes
//     64 x 1 x rows), the stored prefix from the cache pools (seen as
//     (D, B, H, N); one box of 64 x B rows per physical block, found in the
//     block table).  The CTA that holds a key block's own queries also
//     stores that block of the new keys and values in the cache: TMA stores
//     of the tiles already in shared memory, one box per physical block, when
//     the block's slots fill whole physical blocks in order (the usual case),
//     else row by row from the warp's lanes;
//   * warp 8 (one thread) issues the tensor-core products, tcgen05.mma
//     kind::f16, accumulating in tensor memory (TMEM): S_t = Q_t K^T (both
//     operands K-major in shared memory) and O_t += P_t V (P_t from TMEM, V
//     MN-major in shared memory), in the order S0, S1, then per block PV0,
//     S0', PV1, S1': while one tile's softmax runs, the tensor pipe works on
//     the other tile's products;
//   * warps 0-3 and 4-7: the softmax of tile 0 and tile 1, one thread per
//     query row (its warp's 32 TMEM lanes), so the row max and sum stay in
//     the thread.  Base 2; the running max is raised only when a score
//     passes it by more than 2^8, which then rescales that row of O in TMEM.
//     Two scores per packed fp32 instruction, maxima three at a time; in
//     blocks with no masked score half of the weights come from an FMA-pipe
//     polynomial (exp2poly.cuh) and half from the exponential unit, which
//     alone would take as long as the products.  P (and for bf16 the rest
//     P - P_hi, so P enters as about 16 significant bits) goes back to TMEM
//     as packed 16-bit pairs.
//   * After its last block each softmax thread divides its row of O by its
//     sum and stores it.
// Barriers: per stage full (TMA bytes) and empty (last product that reads
// it); per tile S ready, P ready (128 arrivals) and O done.  TMEM loads are
// issued in groups of four under one wait.  TMEM per tile:
// S 64 columns, P 32 + 32, O head_dim; 512 in all, one CTA per SM.
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
constexpr int kTcBN = 64;       // keys per block (MMA N of S, K of P V)
constexpr int kTcTiles = 2;     // query tiles per CTA
constexpr int kTcStages = 3;    // K/V ring depth
constexpr int kTcThreads = 320; // 8 softmax warps, the MMA warp, the load warp
constexpr int kMmaWarp = 8, kLoadWarp = 9;
constexpr uint32_t kColS = 0, kColPhi = 64, kColPlo = 96, kColO = 128;
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
#ifndef PA_TC_EARLY_S
#define PA_TC_EARLY_S 0
#endif
// 1: the softmax warps release S as soon as they hold the scores in
// registers, and the next block's S is issued then, ahead of this block's
// P V; each softmax waits for the previous P V only before it stores P and
// rescales O.  0: S(j+1) is issued after P(j) V.
constexpr bool kTcEarlyS = PA_TC_EARLY_S != 0;

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
  static constexpr int KV_BYTES = kTcBN * D * 2;  // one block of K (or V): 16 KB
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
  __shared__ uint64_t bar_q, bar_full[kTcStages], bar_empty[kTcStages];
  __shared__ uint64_t bar_s[kTcTiles], bar_p[kTcTiles], bar_o[kTcTiles], bar_sfree[kTcTiles];
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
    for (int i = 0; i < kTcStages; ++i) {
      mbar_init(&bar_full[i], 1);
      mbar_init(&bar_empty[i], 1);
    }
#pragma unroll
    for (int t = 0; t < kTcTiles; ++t) {
      mbar_init(&bar_s[t], 1);
      mbar_init(&bar_p[t], kTcBM);
      mbar_init(&bar_o[t], 1);
      mbar_init(&bar_sfree[t], kTcBM / 32);  // one arrival per softmax warp
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
    // jj - npre of the new keys.
    const int32_t* table = p.cached_lens ? p.block_tables + static_cast<int64_t>(s) * p.max_blocks
                                         : nullptr;
    auto load_block = [&](int jj, int st) {  // lane 0
      uint8_t* dst = sKV + st * LY::STAGE;
      mbar_arrive_expect_tx(&bar_full[st], LY::STAGE);
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
            } else {
              set_status(p.status, -7 /* PA_ERR_BAD_BLOCK */);
            }
          }
#pragma unroll
          for (int hf = 0; hf < LY::HALVES; ++hf) {
            tc::tma_load_4d(dst + hf * (kTcBN * 128) + r0 * 128, &tm_kc, hf * 64, 0, kvh, blk,
                            &bar_full[st]);
            tc::tma_load_4d(dst + LY::KV_BYTES + hf * (kTcBN * 128) + r0 * 128, &tm_vc, hf * 64,
                            0, kvh, blk, &bar_full[st]);
          }
        }
      } else {
        const int j = jj - npre;
#pragma unroll
        for (int hf = 0; hf < LY::HALVES; ++hf) {
          tc::tma_load_3d(dst + hf * (kTcBN * 128), &tm_k, hf * 64, kvh, a + j * kTcBN,
                          &bar_full[st]);
          tc::tma_load_3d(dst + LY::KV_BYTES + hf * (kTcBN * 128), &tm_v, hf * 64, kvh,
                          a + j * kTcBN, &bar_full[st]);
        }
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
    auto store_block = [&](int jj) -> bool {  // whole warp; block jj's data has landed
      const int st = jj % kTcStages;
      if (!wwait(&bar_full[st], (jj / kTcStages) & 1)) return false;
      const uint8_t* sK = sKV + st * LY::STAGE;
      const uint8_t* sV = sK + LY::KV_BYTES;
      const int j = jj - npre;
      bool plain = false;
      for (int r0 = 0; r0 < kTcBN; r0 += p.B) {
        // lane r < B takes row r0 + r of the block: new token j*64 + r0 + r
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
            for (int hf = 0; hf < LY::HALVES; ++hf) {
              tc::tma_store_4d(&tm_kc, sK + hf * (kTcBN * 128) + r0 * 128, hf * 64, 0, kvh, blk);
              tc::tma_store_4d(&tm_vc, sV + hf * (kTcBN * 128) + r0 * 128, hf * 64, 0, kvh, blk);
            }
            tc::bulk_commit();
          }
        } else if (lane < p.B && slot >= num_slots) {
          set_status(p.status, -9 /* PA_ERR_BAD_SLOT */);
        } else if (lane < p.B && slot >= 0) {
          // row by row: undo the swizzle (16-byte piece c of row r sits at
          // piece c ^ (r % 8)) and write the row at its slot
          const int r = r0 + lane;
          const int64_t row = ((slot / p.B) * p.Hkv + kvh) * p.B + slot % p.B;
          uint4* dk = reinterpret_cast<uint4*>(static_cast<T*>(p.k_cache) + row * D);
          uint4* dv = reinterpret_cast<uint4*>(static_cast<T*>(p.v_cache) + row * D);
#pragma unroll
          for (int hf = 0; hf < LY::HALVES; ++hf)
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const int off = hf * (kTcBN * 128) + r * 128 + ((c ^ (r & 7)) << 4);
              dk[hf * 8 + c] = *reinterpret_cast<const uint4*>(sK + off);
              dv[hf * 8 + c] = *reinterpret_cast<const uint4*>(sV + off);
            }
          plain = true;
        }
      }
      // generic reads of the stage before the next TMA load writes it
      if (plain) fence_proxy_async_smem();
      __syncwarp();
      return true;
    };
    int issued = 0, stored = own_lo;
    bool ok = true;
    for (int jj = 0; jj < nkb; ++jj) {
      const int st = jj % kTcStages;
      if (jj >= kTcStages) {
        if (!wwait(&bar_empty[st], ((jj / kTcStages) - 1) & 1)) break;
        // the stage still holds block jj - kTcStages: store it if it is ours,
        // and let the stores finish reading it before it is refilled
        if (stores && jj - kTcStages >= own_lo) {
          if (!(ok = store_block(jj - kTcStages))) break;
          stored = jj - kTcStages + 1;
          if (lane == 0) tc::bulk_wait_read_all();
          __syncwarp();
        }
      }
      if (lane == 0) load_block(jj, st);
      issued = jj + 1;
    }
    // our blocks still in the ring
    for (int jj = stored; stores && ok && jj < issued; ++jj) ok = store_block(jj);
    if (lane == 0) {
      // drain: the stores must have read their tiles, and the copies in
      // flight landed, before this CTA's shared memory goes (the stores'
      // global writes complete with the grid, like any other store)
      tc::bulk_wait_read_all();
      mbar_wait_bounded(&bar_q, 0, kTcDrainNs);
      for (int j = issued > kTcStages ? issued - kTcStages : 0; j < issued; ++j)
        mbar_wait_bounded(&bar_full[j % kTcStages], (j / kTcStages) & 1, kTcDrainNs);
    }
  } else if (warp == kMmaWarp) {
    // ---------------- tensor-core products ----------------
    if (lane == 0) {
      const uint32_t qa = smem_addr(sQ);
      int s_done[kTcTiles] = {0, 0}, o_done[kTcTiles] = {0, 0}, empties = 0;
      auto issue_s = [&](int t, int j) -> bool {  // S_t = Q_t K_j^T
        // (the previous block's scores were read: its P is written, P V issued)
        if (!wait(&bar_full[j % kTcStages], (j / kTcStages) & 1)) return false;
        tc::fence_after_sync();
        const uint32_t q = qa + t * LY::Q_BYTES;
        const uint32_t k = smem_addr(sKV + (j % kTcStages) * LY::STAGE);
        const uint32_t d = tmem + t * kTileCols + kColS;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          tc::mma_ss(d, tc::smem_desc(q + (ks >> 2) * (kTcBM * 128) + (ks & 3) * 32, 16, 1024),
                     tc::smem_desc(k + (ks >> 2) * (kTcBN * 128) + (ks & 3) * 32, 16, 1024),
                     IDESC_S, ks > 0);
        tc::commit(&bar_s[t]);
        ++s_done[t];
        return true;
      };
      auto issue_pv = [&](int t, int j) -> bool {  // O_t += P_t V_j
        if (!wait(&bar_p[t], j & 1)) return false;
        tc::fence_after_sync();
        const uint32_t v = smem_addr(sKV + (j % kTcStages) * LY::STAGE + LY::KV_BYTES);
        const uint32_t base = tmem + t * kTileCols;
#pragma unroll
        for (int ks = 0; ks < kTcBN / 16; ++ks) {
          const uint64_t dv = tc::smem_desc(v + ks * 2048, kTcBN * 128, 1024);
          tc::mma_ts(base + kColO, base + kColPhi + ks * 8, dv, IDESC_O, j > 0 || ks > 0);
          if constexpr (BF16) tc::mma_ts(base + kColO, base + kColPlo + ks * 8, dv, IDESC_O, true);
        }
        tc::commit(&bar_o[t]);
        ++o_done[t];
        return true;
      };
      bool ok = wait(&bar_q, 0);
      for (int t = 0; t < kTcTiles && ok; ++t)
        if (nkb_t[t] > 0) ok = issue_s(t, 0);
      for (int j = 0; j < nkb && ok; ++j) {
        if constexpr (kTcEarlyS) {
          // S(j+1) as soon as the softmax holds S(j) in registers, then P(j) V
          for (int t = 0; t < kTcTiles && ok; ++t) {
            if (j + 1 >= nkb_t[t]) continue;
            ok = wait(&bar_sfree[t], j & 1);
            if (ok) ok = issue_s(t, j + 1);
          }
          for (int t = 0; t < kTcTiles && ok; ++t)
            if (j < nkb_t[t]) ok = issue_pv(t, j);
        } else {
          for (int t = 0; t < kTcTiles && ok; ++t) {
            if (j >= nkb_t[t]) continue;
            ok = issue_pv(t, j);
            if (ok && j + 1 < nkb_t[t]) ok = issue_s(t, j + 1);
          }
        }
        if (ok) {
          tc::commit(&bar_empty[j % kTcStages]);  // block j's stage is read for good
          empties = j + 1;
        }
      }
      // drain: every product issued must finish, and every commit arrive,
      // before TMEM and this CTA's shared memory are given up
      for (int j = empties > kTcStages ? empties - kTcStages : 0; j < empties; ++j)
        mbar_wait_bounded(&bar_empty[j % kTcStages], (j / kTcStages) & 1, kTcDrainNs);
#pragma unroll
      for (int t = 0; t < kTcTiles; ++t) {
        if (s_done[t] > 0) mbar_wait_bounded(&bar_s[t], (s_done[t] - 1) & 1, kTcDrainNs);
        if (o_done[t] > 0) mbar_wait_bounded(&bar_o[t], (o_done[t] - 1) & 1, kTcDrainNs);
      }
    }
  } else {
    // ---------------- softmax of one query row ----------------
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
      float sv[kTcBN];
      {
        // four loads in flight, one wait
        uint32_t v[kTcBN / 16][16];
#pragma unroll
        for (int i = 0; i < kTcBN / 16; ++i) tc::ld16(rbase + kColS + i * 16, v[i]);
        tc::wait_ld();
#pragma unroll
        for (int i = 0; i < kTcBN / 16; ++i)
#pragma unroll
          for (int c = 0; c < 16; ++c) sv[i * 16 + c] = __uint_as_float(v[i][c]);
      }
      if constexpr (kTcEarlyS) {
        // the scores are in registers: the next block's S may overwrite them
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_sfree[t]);
      }
      // `below`: no score of this warp's rows is masked in this block, so part
      // of the weights may come from the polynomial
      bool below;
      if (jj < npre) {
        // stored prefix: its keys precede every new row; the last block may
        // run past the prefix (rows read as zeros), which is masked
        below = jj * kTcBN + kTcBN <= cl;
        if (!below) {
#pragma unroll
          for (int c = 0; c < kTcBN; ++c)
            if (jj * kTcBN + c >= cl) sv[c] = -INFINITY;
        }
      } else {
        // new keys: those past this row exist only in the diagonal blocks
        const int j = jj - npre;
        if (j * kTcBN + kTcBN - 1 > qpos) {
#pragma unroll
          for (int c = 0; c < kTcBN; ++c)
            if (j * kTcBN + c > qpos) sv[c] = -INFINITY;
        }
        below = j * kTcBN + kTcBN - 1 <= q0 + t * kTcBM + (warp & 3) * 32;
      }
      // four independent partial maxima (of three-input maxima)
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      if constexpr (kTcPacked) {
#pragma unroll
        for (int c = 0; c < kTcBN; c += 8) {
#pragma unroll
          for (int u = 0; u < 4; ++u) mx[u] = fmax3(mx[u], sv[c + 2 * u], sv[c + 2 * u + 1]);
        }
      } else {
#pragma unroll
        for (int c = 0; c < kTcBN; ++c) mx[c & 3] = fmaxf(mx[c & 3], sv[c]);
      }
      // base-2 logits: the scale (> 0) is applied in the exponent
      const float rmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * p.scale_log2;
      // P_t and O_t are in use by the previous block's product until it is
      // done (here, or after the weights when S runs a block ahead)
      auto wait_pv = [&]() -> bool {
        if (jj > 0) {
          if (__any_sync(0xffffffffu, !wait(&bar_o[t], (jj - 1) & 1))) return false;
          tc::fence_after_sync();
        }
        return true;
      };
      if constexpr (!kTcEarlyS) {
        failed = !wait_pv();
        if (failed) break;
      }
      const bool raise = rmax > m + 8.f;
      const float m_new = raise ? rmax : m;
      const float alpha = raise && m != -INFINITY ? fast_exp2(m - m_new) : 1.f;
      auto rescale_o = [&]() {
        if (!(jj > 0 && __any_sync(0xffffffffu, alpha != 1.f))) return;
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
      };
      if constexpr (!kTcEarlyS) rescale_o();
      l *= alpha;
      m = m_new;
      const float mm = m == -INFINITY ? 0.f : m;
      uint32_t ph[32], pl[32];
      float2 ls[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};  // partial sums
      const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
      const float2 nm2 = make_float2(-mm, -mm);
      // 2^(scale * s - m), two scores per packed fma (masked scores are -inf:
      // weight 0).  Below the diagonal, kTcPolyPairs of every four pairs of
      // weights come from the FMA-pipe polynomial and the rest from the
      // exponential unit, so the two units share the work.
      auto weights = [&](int c, bool poly) {
        float2 pw;
        if constexpr (kTcPacked) {
          const float2 x = __ffma2_rn(make_float2(sv[c], sv[c + 1]), sc2, nm2);
          pw = poly ? exp2_poly2(x) : make_float2(fast_exp2(x.x), fast_exp2(x.y));
          ls[(c >> 1) & 1] = __fadd2_rn(ls[(c >> 1) & 1], pw);
        } else {
          pw = make_float2(fast_exp2(fmaf(sv[c], p.scale_log2, -mm)),
                           fast_exp2(fmaf(sv[c + 1], p.scale_log2, -mm)));
          ls[(c >> 1) & 1].x += pw.x + pw.y;
        }
        ph[c / 2] = Elem<T>::from_float2(pw.x, pw.y);
        if constexpr (BF16) {
          const float2 back = Elem<T>::to_float2(ph[c / 2]);
          pl[c / 2] = Elem<T>::from_float2(pw.x - back.x, pw.y - back.y);
        }
      };
      if (below) {
#pragma unroll
        for (int c = 0; c < kTcBN; c += 2) weights(c, ((c >> 1) & 3) >= 4 - kTcPolyPairs);
      } else {
#pragma unroll
        for (int c = 0; c < kTcBN; c += 2) weights(c, false);
      }
      l += (ls[0].x + ls[0].y) + (ls[1].x + ls[1].y);
      if constexpr (kTcEarlyS) {
        failed = !wait_pv();
        if (failed) break;
        rescale_o();
      }
      tc::st16(rbase + kColPhi, *reinterpret_cast<uint32_t(*)[16]>(ph));
      tc::st16(rbase + kColPhi + 16, *reinterpret_cast<uint32_t(*)[16]>(ph + 16));
      if constexpr (BF16) {
        tc::st16(rbase + kColPlo, *reinterpret_cast<uint32_t(*)[16]>(pl));
        tc::st16(rbase + kColPlo + 16, *reinterpret_cast<uint32_t(*)[16]>(pl + 16));
      }
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
