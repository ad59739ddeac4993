// Tiled TMA tensor maps with the 128-byte swizzle (16-bit tensors, and the
// 8-bit cache's one-byte codes), encoded
// through the driver's cuTensorMapEncodeTiled, which is looked up once
// through the runtime (the library does not link the driver library).
#include <cuda.h>
#include <cuda_runtime.h>

#include "kernels.h"

namespace pa {

namespace {

#ifndef PA_TMA_L2_PROMOTION
#define PA_TMA_L2_PROMOTION 256
#endif
// L2 promotion of the tiled loads' requests (0, 64, 128 or 256 bytes).
CUtensorMapL2promotion l2_promotion() {
  switch (PA_TMA_L2_PROMOTION) {
    case 0: return CU_TENSOR_MAP_L2_PROMOTION_NONE;
    case 64: return CU_TENSOR_MAP_L2_PROMOTION_L2_64B;
    case 128: return CU_TENSOR_MAP_L2_PROMOTION_L2_128B;
    default: return CU_TENSOR_MAP_L2_PROMOTION_L2_256B;
  }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault,
                                         &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      cudaGetLastError();
      return static_cast<EncodeTiledFn>(nullptr);
    }
    return reinterpret_cast<EncodeTiledFn>(f);
  }();
  return fn;
}

}  // namespace

bool encode_swizzled_map(CUtensorMap* map, const void* base, bool bf16, int rank,
                         const uint64_t* dims, const uint64_t* strides_bytes,
                         const uint32_t* box) {
  return encode_tiled_map(map, base,
                          bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                          rank, dims, strides_bytes, box);
}

namespace {
bool encode_with(CUtensorMap* map, const void* base, CUtensorMapDataType type, int rank,
                 const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                 CUtensorMapSwizzle swizzle) {
  const EncodeTiledFn fn = encode_tiled();
  if (!fn || rank < 1 || rank > 5) return false;
  cuuint64_t d[5], st[4];
  cuuint32_t b[5], e[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    e[i] = 1u;
    if (i + 1 < rank) st[i] = strides_bytes[i];
  }
  return fn(map, type, static_cast<cuuint32_t>(rank), const_cast<void*>(base), d, st, b, e,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, l2_promotion(),
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
}  // namespace

bool encode_tiled_map(CUtensorMap* map, const void* base, CUtensorMapDataType type, int rank,
                      const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box) {
  return encode_with(map, base, type, rank, dims, strides_bytes, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

bool encode_plain_map(CUtensorMap* map, const void* base, CUtensorMapDataType type, int rank,
                      const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box) {
  return encode_with(map, base, type, rank, dims, strides_bytes, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}

}  // namespace pa
