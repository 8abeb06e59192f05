// Host-side helpers for TMA tensor maps: the driver's cuTensorMapEncodeTiled,
// looked up once through the runtime's driver entry-point query (no link
// dependency on libcuda), and a checked fp32 map builder.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace lla {

typedef CUresult (*TmapEncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline TmapEncodeFn tmap_encoder() {
  static TmapEncodeFn fn = []() -> TmapEncodeFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<TmapEncodeFn>(p);
  }();
  return fn;
}

// fp32 tiled map of `rank` dimensions (innermost first).  strides[i] is the
// byte stride of dimension i + 1.  Out-of-range elements of a box read as 0.
// Returns false when the driver rejects the map (alignment, sizes).
inline bool tmap_f32(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
                     const cuuint32_t* box, CUtensorMapSwizzle swizzle) {
  TmapEncodeFn enc = tmap_encoder();
  if (!enc || !base || (reinterpret_cast<uintptr_t>(base) & 15)) return false;
  for (int i = 0; i < rank - 1; ++i)
    if (strides[i] % 16 || strides[i] >= (1ull << 40)) return false;
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, (cuuint32_t)rank, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace lla
