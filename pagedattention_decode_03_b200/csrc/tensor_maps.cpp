// TMA tensor maps of the KV cache, shared by the pool (api.cpp) and the
// no-allocation entry point (noalloc.cu).
//
// The cache [L][NB][H][B][128] is viewed as rows of 128 elements, one row per
// (layer, block, head, slot).  A staged tile is 16 rows (16 token slots of one
// KV head), read into shared memory with the 128-byte swizzle so the ldmatrix
// and UMMA reads of its rows are free of bank conflicts.
//   2-D map [rows][128]: boxes of 16 rows x 128 bytes (64 16-bit or 128 FP8
//     elements): two boxes per 16-bit tile (the two d-halves), one per FP8 tile.
//   3-D map of a 16-bit cache, [2 d-halves][rows][64] (strides 128 B and
//     256 B): one box {64, 16, 2} brings a whole 16-row tile, d-half 0 then
//     d-half 1, the same shared-memory layout as the two 2-D boxes with half the
//     copy instructions.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "pa_internal.h"

namespace pa {
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encoder() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

}  // namespace

const char* encode_cache_maps(void* k_cache, void* v_cache, int kv_dtype, int64_t rows, CacheMaps* m) {
  EncodeTiledFn encode = encoder();
  if (!encode) return "cuTensorMapEncodeTiled not available from the driver";
  const bool fp8 = kv_dtype == kFP8;
  const CUtensorMapDataType dt = fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kHeadDim) * (fp8 ? 1 : 2)};
  const cuuint32_t box[2] = {fp8 ? 128u : 64u, 16u};
  const cuuint32_t estr[3] = {1, 1, 1};
  void* base[2] = {k_cache, v_cache};
  CUtensorMap* m2[2] = {&m->k, &m->v};
  for (int i = 0; i < 2; ++i)
    if (encode(m2[i], dt, 2, base[i], dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return "cuTensorMapEncodeTiled (2-D cache view) failed";
  m->k3 = m->k;
  m->v3 = m->v;
  if (fp8) return nullptr;
  const cuuint64_t dims3[3] = {64, static_cast<cuuint64_t>(rows), 2};
  const cuuint64_t strides3[2] = {256, 128};
  const cuuint32_t box3[3] = {64u, 16u, 2u};
  CUtensorMap* m3[2] = {&m->k3, &m->v3};
  for (int i = 0; i < 2; ++i)
    if (encode(m3[i], dt, 3, base[i], dims3, strides3, box3, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return "cuTensorMapEncodeTiled (3-D cache view) failed";
  return nullptr;
}

}  // namespace pa
