// prefill_tc: the prompt phase on the 5th-generation tensor cores (tcgen05).
//
// What it computes is prefill.cu's function ("The KV Cache and
// PagedAttention", section "One Token at a Time"; "KV cache", section "How it
// works"): for prompt s, query head h and position t,
//     out[t][h] = sum_{u <= t} softmax_u(scale * q[t][h] . k[u]) v[u],
// query head h reading key/value head h / (Hq / Hkv).
//
// How (one CTA = 128 queries of one (prompt, head); 128 threads, one query
// row each; two CTAs per SM):
//   * Q (128 x D) and each 64-key block of K and V arrive by 3-D tiled TMA
//     (the [T][H][D] tensors seen as (D, H, T); boxes 64 x 1 x rows, 128-byte
//     swizzle) into shared memory; K and V are double-buffered in stages.
//   * S = Q K^T: thread 0 issues tcgen05.mma (M = 128, N = 64, K = 16 per
//     instruction, both operands K-major in shared memory) into tensor memory
//     (TMEM); a commit signals an mbarrier.
//   * Softmax: each thread reads its query's 64 scores from TMEM (its warp's
//     32 lanes), so the row max and sum need no shuffles.  Base 2; the
//     running max is raised only when a score passes it by more than 2^8,
//     which then rescales that row of O in TMEM.  P (and for bf16 the rest
//     P - P_hi, so P enters as about 16 significant bits) is written back to
//     TMEM as packed 16-bit pairs.
//   * O += P V: tcgen05.mma with A = P from TMEM and B = V (MN-major: head_dim
//     contiguous) from shared memory; O accumulates in TMEM.
//   * After the last block each thread reads its row of O, divides by its
//     sum and stores it.
// TMEM per CTA: S 64 columns, P 32 (+ 32 for bf16's low part), O head_dim.
// Every wait is bounded: a wait that gives up records PA_ERR_TIMEOUT, the CTA
// drains what it issued (bounded too), frees its TMEM and returns.
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

constexpr int kTcThreads = 128;  // one per query row
constexpr int kTcBM = 128;       // queries per CTA (MMA M)
constexpr int kTcBN = 64;        // keys per block (MMA N of S, K of P V)
constexpr uint32_t kColS = 0, kColPhi = 64, kColPlo = 96, kColO = 128, kTmemCols = 256;
constexpr int64_t kTcDrainNs = 1000000000;

template <int D>
struct TcLayout {
  static constexpr int HALVES = D / 64;             // 64-element (128-byte) column blocks
  static constexpr int Q_BYTES = kTcBM * D * 2;     // 32 KB at head_dim 128
  static constexpr int KV_BYTES = kTcBN * D * 2;    // 16 KB
  static constexpr int STAGE = 2 * KV_BYTES;        // K block, then V block
  // shared memory asked for: + 1 KB to align by hand; sized for head_dim 128
  // at every head_dim, which keeps two CTAs (2 x 256 TMEM columns) per SM
  static constexpr int SMEM = 1024 + 128 * 128 * 2 + 2 * 2 * 64 * 128 * 2;
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
};

template <typename T, int D>
__global__ void __launch_bounds__(kTcThreads, 2)
prefill_tc_kernel(const TcParams p, const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v) {
  using LY = TcLayout<D>;
  constexpr bool BF16 = std::is_same<T, __nv_bfloat16>::value;
  constexpr uint32_t IDESC_S = tc::idesc_f16(kTcBM, kTcBN, BF16, false);
  constexpr uint32_t IDESC_O = tc::idesc_f16(kTcBM, D, BF16, true);
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 128-byte swizzle patterns repeat every 1024 bytes of shared address: align by hand
  uint8_t* smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + LY::Q_BYTES;
  __shared__ uint64_t bar_q, bar_kv[2], bar_s, bar_o;
  __shared__ uint32_t tmem_base;

  griddep_wait();
  const int s = blockIdx.z, h = blockIdx.y;
  const int a = __ldg(p.cu_seqlens + s), b = __ldg(p.cu_seqlens + s + 1);
  if (a < 0 || b < a || b > p.num_tokens) {
    if (blockIdx.x == 0 && h == 0 && threadIdx.x == 0) set_status(p.status, -8 /* PA_ERR_BAD_LEN */);
    return;
  }
  const int L = b - a;
  if (L > p.max_seqlen && blockIdx.x == 0 && h == 0 && threadIdx.x == 0)
    set_status(p.status, -8 /* PA_ERR_BAD_LEN: a prompt longer than max_seqlen */);
  const int tile = gridDim.x - 1 - blockIdx.x;  // heaviest tiles first
  if (tile * kTcBM >= L) return;                 // the whole CTA leaves: nothing allocated yet
  const int kvh = h / (p.Hq / p.Hkv);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int q_end = min(L, (tile + 1) * kTcBM);  // this tile's queries end here
  const int nkb = (q_end + kTcBN - 1) / kTcBN;   // key blocks up to the diagonal

  if (tid == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_q)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_k)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_v)) : "memory");
    mbar_init(&bar_q, 1);
    mbar_init(&bar_kv[0], 1);
    mbar_init(&bar_kv[1], 1);
    mbar_init(&bar_s, 1);
    mbar_init(&bar_o, 1);
    fence_barrier_init();
  }
  if (warp == 0) tc::alloc(&tmem_base, kTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_base;
  const uint32_t row_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);

  // Producer bookkeeping (thread 0): what was issued, for the drain.
  int kv_issued = 0, s_commits = 0, o_commits = 0;
  auto load_kv = [&](int j) {  // key block j into stage j % 2
    uint8_t* st = sKV + (j & 1) * LY::STAGE;
    uint64_t* bar = &bar_kv[j & 1];
    mbar_arrive_expect_tx(bar, LY::STAGE);
#pragma unroll
    for (int hf = 0; hf < LY::HALVES; ++hf) {
      tc::tma_load_3d(st + hf * (kTcBN * 128), &tm_k, hf * 64, kvh, a + j * kTcBN, bar);
      tc::tma_load_3d(st + LY::KV_BYTES + hf * (kTcBN * 128), &tm_v, hf * 64, kvh, a + j * kTcBN,
                      bar);
    }
    ++kv_issued;
  };
  if (tid == 0) {
    mbar_arrive_expect_tx(&bar_q, LY::Q_BYTES);
#pragma unroll
    for (int hf = 0; hf < LY::HALVES; ++hf)
      tc::tma_load_3d(sQ + hf * (kTcBM * 128), &tm_q, hf * 64, h, a + tile * kTcBM, &bar_q);
    load_kv(0);
  }

  const int qpos = tile * kTcBM + tid;  // this thread's query, within the prompt
  float m = -INFINITY, l = 0.f;
  bool failed = false;
  int j = 0;
  for (; j < nkb; ++j) {
    // ---- S = Q K^T (thread 0 issues) ----
    if (tid == 0 && !failed) {
      bool ok = mbar_wait_bounded(&bar_kv[j & 1], (j >> 1) & 1, p.wait_limit_ns);
      if (ok && j == 0) ok = mbar_wait_bounded(&bar_q, 0, p.wait_limit_ns);
      if (!ok) {
        failed = true;
      } else {
        const uint32_t q0 = smem_addr(sQ), k0 = smem_addr(sKV + (j & 1) * LY::STAGE);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          tc::mma_ss(tmem + kColS,
                     tc::smem_desc(q0 + (ks >> 2) * (kTcBM * 128) + (ks & 3) * 32, 16, 1024),
                     tc::smem_desc(k0 + (ks >> 2) * (kTcBN * 128) + (ks & 3) * 32, 16, 1024),
                     IDESC_S, ks > 0);
        tc::commit(&bar_s);
        ++s_commits;
      }
    }
    // ---- softmax of this thread's row ----
    // tcgen05.ld/st are warp-collective: every guard around them is made
    // uniform across the warp by a vote
    float sv[kTcBN];
    if (!failed) failed = !mbar_wait_bounded(&bar_s, j & 1, p.wait_limit_ns);
    failed = __any_sync(0xffffffffu, failed);
    tc::fence_after_sync();
    if (!failed) {
#pragma unroll
      for (int c0 = 0; c0 < kTcBN; c0 += 16) {
        uint32_t v[16];
        tc::ld16(row_addr + kColS + c0, v);
        tc::wait_ld();
#pragma unroll
        for (int c = 0; c < 16; ++c) sv[c0 + c] = __uint_as_float(v[c]);
      }
    }
    float rmax = -INFINITY;
#pragma unroll
    for (int c = 0; c < kTcBN; ++c) {
      const int key = j * kTcBN + c;
      sv[c] = key <= qpos ? sv[c] * p.scale_log2 : -INFINITY;
      rmax = fmaxf(rmax, sv[c]);
    }
    // P and O are still in use by the previous block's P V until it completes
    if (j > 0 && !failed) failed = !mbar_wait_bounded(&bar_o, (j - 1) & 1, p.wait_limit_ns);
    failed = __any_sync(0xffffffffu, failed);
    tc::fence_after_sync();
    if (tid == 0 && !failed && j + 1 < nkb) load_kv(j + 1);  // its stage held block j - 1
    // Raise the running max of a row only past a slack of 2^8; a row whose
    // max rises after the first block rescales its O (the whole warp takes
    // part in the TMEM traffic, with factor 1 on rows that do not rise).
    const bool raise = rmax > m + 8.f;
    const float m_new = raise ? rmax : m;
    const float alpha = raise && m != -INFINITY ? fast_exp2(m - m_new) : 1.f;
    if (!failed && j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 16) {
        uint32_t v[16];
        tc::ld16(row_addr + kColO + c0, v);
        tc::wait_ld();
#pragma unroll
        for (int c = 0; c < 16; ++c) v[c] = __float_as_uint(__uint_as_float(v[c]) * alpha);
        tc::st16(row_addr + kColO + c0, v);
      }
      tc::wait_st();
    }
    l *= alpha;
    m = m_new;
    {
      const float mm = m == -INFINITY ? 0.f : m;
      uint32_t ph[32], pl[32];
#pragma unroll
      for (int c = 0; c < kTcBN; c += 2) {
        const float p0 = fast_exp2(sv[c] - mm), p1 = fast_exp2(sv[c + 1] - mm);
        l += p0 + p1;
        ph[c / 2] = Elem<T>::from_float2(p0, p1);
        if constexpr (BF16) {
          const float2 back = Elem<T>::to_float2(ph[c / 2]);
          pl[c / 2] = Elem<T>::from_float2(p0 - back.x, p1 - back.y);
        }
      }
      if (!failed) {
        tc::st16(row_addr + kColPhi, *reinterpret_cast<uint32_t(*)[16]>(ph));
        tc::st16(row_addr + kColPhi + 16, *reinterpret_cast<uint32_t(*)[16]>(ph + 16));
        if constexpr (BF16) {
          tc::st16(row_addr + kColPlo, *reinterpret_cast<uint32_t(*)[16]>(pl));
          tc::st16(row_addr + kColPlo + 16, *reinterpret_cast<uint32_t(*)[16]>(pl + 16));
        }
        tc::wait_st();
      }
    }
    tc::fence_before_sync();
    if (__syncthreads_or(failed ? 1 : 0)) {
      failed = true;
      break;
    }
    tc::fence_after_sync();
    // ---- O += P V (thread 0 issues) ----
    if (tid == 0) {
      const uint32_t v0 = smem_addr(sKV + (j & 1) * LY::STAGE + LY::KV_BYTES);
#pragma unroll
      for (int ks = 0; ks < kTcBN / 16; ++ks) {
        const uint64_t dv = tc::smem_desc(v0 + ks * 2048, kTcBN * 128, 1024);
        tc::mma_ts(tmem + kColO, tmem + kColPhi + ks * 8, dv, IDESC_O, j > 0 || ks > 0);
        if constexpr (BF16) tc::mma_ts(tmem + kColO, tmem + kColPlo + ks * 8, dv, IDESC_O, true);
      }
      tc::commit(&bar_o);
      ++o_commits;
    }
  }

  if (!failed) {
    // ---- epilogue: out = O / l ----
    failed = !mbar_wait_bounded(&bar_o, (nkb - 1) & 1, p.wait_limit_ns);
    failed = __any_sync(0xffffffffu, failed);
    tc::fence_after_sync();
    if (!failed) {
      const bool store = qpos < L;
      const float inv = l > 0.f ? 1.f / l : 0.f;
      T* orow = static_cast<T*>(p.out) + (static_cast<int64_t>(a + qpos) * p.Hq + h) * D;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 16) {
        uint32_t v[16];
        tc::ld16(row_addr + kColO + c0, v);
        tc::wait_ld();
        float f[8];
        if (store) {
#pragma unroll
          for (int k = 0; k < 8; ++k) f[k] = __uint_as_float(v[k]) * inv;
          *reinterpret_cast<uint4*>(orow + c0) = pack8<T>(f);
#pragma unroll
          for (int k = 0; k < 8; ++k) f[k] = __uint_as_float(v[8 + k]) * inv;
          *reinterpret_cast<uint4*>(orow + c0 + 8) = pack8<T>(f);
        }
      }
    }
  }
  if (failed) {
    if (tid == 0) {
      set_status(p.status, -10 /* PA_ERR_TIMEOUT */);
      // drain what this CTA issued before its memory goes away (bounded):
      // the last load into each stage, the last commit of each barrier
      for (int i = kv_issued > 2 ? kv_issued - 2 : 0; i < kv_issued; ++i)
        mbar_wait_bounded(&bar_kv[i & 1], (i >> 1) & 1, kTcDrainNs);
      mbar_wait_bounded(&bar_q, 0, kTcDrainNs);
      if (s_commits > 0) mbar_wait_bounded(&bar_s, (s_commits - 1) & 1, kTcDrainNs);
      if (o_commits > 0) mbar_wait_bounded(&bar_o, (o_commits - 1) & 1, kTcDrainNs);
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
  const int tiles = (a.max_seqlen + kTcBM - 1) / kTcBM;
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
  const uint32_t bq[3] = {64u, 1u, static_cast<uint32_t>(kTcBM)};
  const uint32_t bk[3] = {64u, 1u, static_cast<uint32_t>(kTcBN)};
  const bool bf16 = std::is_same<T, __nv_bfloat16>::value;
  if (!encode_swizzled_map(&tq, a.q, bf16, 3, dq, sq, bq) ||
      !encode_swizzled_map(&tk, a.k, bf16, 3, dk, sk, bk) ||
      !encode_swizzled_map(&tv, a.v, bf16, 3, dk, sk, bk))
    return cudaErrorInvalidValue;
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
  cudaError_t err = cudaLaunchKernelEx(&cfg, prefill_tc_kernel<T, D>, p, tq, tk, tv);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_tc(const PrefillArgs& a, cudaStream_t stream) {
  if (a.head_dim == 128)
    return a.is_bf16 ? launch_prefill_tc_typed<__nv_bfloat16, 128>(a, stream)
                     : launch_prefill_tc_typed<__half, 128>(a, stream);
  if (a.head_dim == 64)
    return a.is_bf16 ? launch_prefill_tc_typed<__nv_bfloat16, 64>(a, stream)
                     : launch_prefill_tc_typed<__half, 64>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace pa
