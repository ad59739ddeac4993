// prefill: the prompt phase.  Every prompt's tokens attend causally over the
// prompt's own keys and values ("The KV Cache and PagedAttention", section
// "One Token at a Time": the prompt is processed all at once and its keys and
// values are what later steps reuse; "KV cache", section "How it works":
// position t attends over positions 0..t), and those keys and values are
// stored in their blocks (the cache write kernel, launched first).
//
// Prompts are packed: prompt s is rows cu_seqlens[s] .. cu_seqlens[s+1]-1 of
// q [T][Hq][D] and of k, v [T][Hkv][D]; query head h reads key/value head
// h / (Hq / Hkv).  For prompt s, head h, position t:
//     out[t][h] = sum_{u <= t} softmax_u(scale * q[t][h] . k[u]) v[u].
//
// Dense and compute-bound (4 * D flops per (query, key) pair, half the pairs
// of a prompt), so it runs on the tensor cores: warp-level mma.sync m16n8k16
// (fp16 or bf16 in, fp32 accumulate).  A CTA of 4 warps takes 64 queries of
// one (prompt, head), 16 per warp, and walks the prompt's keys in blocks of
// 64 up to the diagonal:
//   * K and V blocks are double-buffered in shared memory by 16-byte
//     cp.async copies; rows are 16-byte pieces XOR-swizzled by the row index
//     so that the 8 rows an ldmatrix reads lie in distinct banks;
//   * S = Q K^T (queries on the rows, keys on the columns), Q in registers;
//   * online softmax per query row in base 2, the running max and sum
//     reduced over the 4 lanes that hold a row;
//   * O += P V with P taken straight from the S accumulators as the A
//     operand, V through the transposing ldmatrix; for bf16 P goes in as two
//     bf16 values P_hi + P_lo (one bf16 value alone carries 8 bits).
// Tiles run heaviest (most key blocks) first.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>
#include <set>
#include <type_traits>

#include "dtype.cuh"
#include "kernels.h"
#include "mma_ptx.cuh"
#include "ptx.cuh"

namespace pa {

namespace {

constexpr int kPfWarps = 4;
constexpr int kBM = 16 * kPfWarps;  // queries per CTA
constexpr int kBN = 64;             // keys per block

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool fill) {
  // fill == false: 16 zero bytes, nothing read
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(fill ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Shared tile of 64 rows x D: 16-byte piece c of row r at piece c ^ (r % 8).
template <int D>
__device__ __forceinline__ uint32_t tile_addr(uint32_t base, int r, int c) {
  return base + r * (D * 2) + ((c ^ (r & 7)) << 4);
}

// Load rows [row0, row0 + 64) of head `head` of a [T][heads][D] tensor into
// a swizzled tile; rows at or past `row_end` become zeros.
template <int D>
__device__ __forceinline__ void load_tile(uint32_t tile, const uint8_t* base, int64_t row0,
                                          int64_t row_end, int heads, int head, int tid) {
  constexpr int PIECES = D / 8;  // 16-byte pieces per row
  for (int i = tid; i < 64 * PIECES; i += kPfWarps * 32) {
    const int r = i / PIECES, c = i - (i / PIECES) * PIECES;
    const int64_t row = row0 + r;
    const bool ok = row < row_end;
    const uint8_t* src = base + ((ok ? row : row0) * heads + head) * (D * 2) + c * 16;
    cp_async16(tile_addr<D>(tile, r, c), src, ok);
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kPfWarps * 32, 2)
prefill_kernel(T* __restrict__ out, const T* __restrict__ q, const T* __restrict__ k,
               const T* __restrict__ v, const int32_t* __restrict__ cu_seqlens, int num_tokens,
               int max_seqlen, int Hq, int Hkv, float scale_log2, int32_t* status) {
  constexpr int KD = D / 16;   // head_dim steps of the product
  constexpr int NT = kBN / 8;  // key tiles of 8 per block
  constexpr int DT = D / 8;    // head_dim tiles of 8 in O
  constexpr int TILE = 64 * D * 2;
  constexpr bool SPLIT = sizeof(T) == 2 && !std::is_same<T, __half>::value;  // bf16
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sQ = smem_addr(smem);
  const uint32_t sK0 = sQ + TILE, sV0 = sQ + 3 * TILE;  // two buffers each

  griddep_wait();
  const int s = blockIdx.z, h = blockIdx.y;
  const int a = __ldg(cu_seqlens + s), b = __ldg(cu_seqlens + s + 1);
  if (a < 0 || b < a || b > num_tokens) {
    if (blockIdx.x == 0 && h == 0 && threadIdx.x == 0) set_status(status, -8 /* PA_ERR_BAD_LEN */);
    return;
  }
  const int L = b - a;
  // A prompt longer than max_seqlen breaks the call's contract: report it
  // (positions past the grid's tiles are not computed).
  if (L > max_seqlen && blockIdx.x == 0 && h == 0 && threadIdx.x == 0)
    set_status(status, -8 /* PA_ERR_BAD_LEN */);
  const int tile = gridDim.x - 1 - blockIdx.x;  // heaviest tiles first
  if (tile * kBM >= L) return;
  const int kvh = h / (Hq / Hkv);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nkb = tile + 1;  // key blocks up to the diagonal (kBM == kBN)

  const uint8_t* qb = reinterpret_cast<const uint8_t*>(q);
  const uint8_t* kb8 = reinterpret_cast<const uint8_t*>(k);
  const uint8_t* vb8 = reinterpret_cast<const uint8_t*>(v);
  load_tile<D>(sQ, qb, a + tile * kBM, b, Hq, h, tid);
  load_tile<D>(sK0, kb8, a, b, Hkv, kvh, tid);
  load_tile<D>(sV0, vb8, a, b, Hkv, kvh, tid);
  cp_async_commit();

  uint32_t qa[KD][4];
  float o[DT][4];
#pragma unroll
  for (int i = 0; i < DT; ++i)
#pragma unroll
    for (int c = 0; c < 4; ++c) o[i][c] = 0.f;
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
  const int q_row0 = tile * kBM + warp * 16 + (lane >> 2);  // query of c0, c1 (c2, c3: +8)

  for (int kb = 0; kb < nkb; ++kb) {
    const int buf = kb & 1;
    if (kb + 1 < nkb) {
      const int nb = (kb + 1) & 1;
      load_tile<D>(sK0 + nb * TILE, kb8, a + (kb + 1) * kBN, b, Hkv, kvh, tid);
      load_tile<D>(sV0 + nb * TILE, vb8, a + (kb + 1) * kBN, b, Hkv, kvh, tid);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (kb == 0) {
      // Q fragments of this warp's 16 rows
#pragma unroll
      for (int ks = 0; ks < KD; ++ks)
        ldsm_x4(tile_addr<D>(sQ, warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8, ks * 2 + (lane >> 4)),
                qa[ks]);
    }
    const uint32_t sK = sK0 + buf * TILE, sV = sV0 + buf * TILE;

    // ---- S = Q K^T: 16 queries x 64 keys per warp ----
    float sc[NT][4];
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int c = 0; c < 4; ++c) sc[j][c] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KD; ++ks)
#pragma unroll
      for (int j = 0; j < NT; j += 2) {
        uint32_t r[4];
        ldsm_x4(tile_addr<D>(sK, (j + (lane >> 4)) * 8 + (lane & 7), ks * 2 + ((lane >> 3) & 1)), r);
        mma_16816<T>(sc[j], qa[ks], r[0], r[1]);
        mma_16816<T>(sc[j + 1], qa[ks], r[2], r[3]);
      }

    // ---- online softmax per row (base 2) ----
    const bool diag = kb == tile;
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int key = kb * kBN + j * 8 + (lane & 3) * 2 + (c & 1);
        const int qry = q_row0 + (c >> 1) * 8;
        float x = sc[j][c] * scale_log2;
        if (diag && key > qry) x = -INFINITY;
        sc[j][c] = x;
        mx[c >> 1] = fmaxf(mx[c >> 1], x);
      }
    float alpha[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
      const float m_new = fmaxf(m[r], mx[r]);  // finite: every row sees its own key
      alpha[r] = fast_exp2(m[r] - m_new);
      m[r] = m_new;
      l[r] *= alpha[r];
    }
#pragma unroll
    for (int i = 0; i < DT; ++i) {
      o[i][0] *= alpha[0];
      o[i][1] *= alpha[0];
      o[i][2] *= alpha[1];
      o[i][3] *= alpha[1];
    }
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        sc[j][c] = fast_exp2(sc[j][c] - m[c >> 1]);
        l[c >> 1] += sc[j][c];
      }

    // ---- O += P V ----
#pragma unroll
    for (int kk = 0; kk < kBN / 16; ++kk) {
      uint32_t pa[4], pl[4];
      const float* p0 = sc[2 * kk];
      const float* p1 = sc[2 * kk + 1];
      const float pv[8] = {p0[0], p0[1], p0[2], p0[3], p1[0], p1[1], p1[2], p1[3]};
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        pa[r] = Elem<T>::from_float2(pv[2 * r], pv[2 * r + 1]);
        if constexpr (SPLIT) {
          const float2 back = Elem<T>::to_float2(pa[r]);
          pl[r] = Elem<T>::from_float2(pv[2 * r] - back.x, pv[2 * r + 1] - back.y);
        }
      }
#pragma unroll
      for (int dn = 0; dn < DT; dn += 2) {
        uint32_t r[4];
        ldsm_x4_trans(tile_addr<D>(sV, kk * 16 + ((lane >> 3) & 1) * 8 + (lane & 7), dn + (lane >> 4)), r);
        mma_16816<T>(o[dn], pa, r[0], r[1]);
        mma_16816<T>(o[dn + 1], pa, r[2], r[3]);
        if constexpr (SPLIT) {
          mma_16816<T>(o[dn], pl, r[0], r[1]);
          mma_16816<T>(o[dn + 1], pl, r[2], r[3]);
        }
      }
    }
    __syncthreads();  // every warp is done with this buffer before it is refilled
  }

  // ---- epilogue: out = O / l ----
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    l[r] += __shfl_xor_sync(0xffffffffu, l[r], 1);
    l[r] += __shfl_xor_sync(0xffffffffu, l[r], 2);
  }
  const float inv0 = 1.f / l[0], inv1 = 1.f / l[1];
  const int q0 = q_row0, q1 = q_row0 + 8;
#pragma unroll
  for (int dn = 0; dn < DT; ++dn) {
    const int d = dn * 8 + (lane & 3) * 2;
    if (q0 < L)
      *reinterpret_cast<uint32_t*>(out + (static_cast<int64_t>(a + q0) * Hq + h) * D + d) =
          Elem<T>::from_float2(o[dn][0] * inv0, o[dn][1] * inv0);
    if (q1 < L)
      *reinterpret_cast<uint32_t*>(out + (static_cast<int64_t>(a + q1) * Hq + h) * D + d) =
          Elem<T>::from_float2(o[dn][2] * inv1, o[dn][3] * inv1);
  }
}

template <typename T, int D>
cudaError_t launch_prefill_typed(const PrefillArgs& a, cudaStream_t stream) {
  constexpr size_t smem = 5 * 64 * D * 2;  // Q + two K + two V tiles
  {
    // the shared-memory limit is a per-device attribute: raise it once per device
    static std::mutex mu;
    static std::set<int> raised;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaGetLastError();
    std::lock_guard<std::mutex> lock(mu);
    if (!raised.count(dev)) {
      if (cudaFuncSetAttribute(prefill_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem)) != cudaSuccess)
        return cudaGetLastError();
      raised.insert(dev);
    }
  }
  const int tiles = (a.max_seqlen + kBM - 1) / kBM;
  if (tiles <= 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(tiles, a.num_heads, a.num_seqs);
  cfg.blockDim = dim3(kPfWarps * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t err = cudaLaunchKernelEx(
      &cfg, prefill_kernel<T, D>, static_cast<T*>(a.out), static_cast<const T*>(a.q),
      static_cast<const T*>(a.k), static_cast<const T*>(a.v), a.cu_seqlens, a.num_tokens,
      a.max_seqlen, a.num_heads, a.num_kv_heads, a.scale * 1.4426950408889634f, a.status);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const PrefillArgs& a, cudaStream_t stream) {
  if (a.head_dim == 128)
    return a.is_bf16 ? launch_prefill_typed<__nv_bfloat16, 128>(a, stream)
                     : launch_prefill_typed<__half, 128>(a, stream);
  if (a.head_dim == 64)
    return a.is_bf16 ? launch_prefill_typed<__nv_bfloat16, 64>(a, stream)
                     : launch_prefill_typed<__half, 64>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace pa
