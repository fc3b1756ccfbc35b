// tmap.h -- host-side encoding of TMA tensor maps.
//
// The driver's encoder is looked up through the runtime so the library does
// not link against libcuda: it still loads where no driver is installed, and
// the entry point is resolved on first use on a GPU machine.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

namespace strata {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Tiled map of a rank-`rank` tensor: dims[0] innermost (contiguous), byte
// strides of dims 1..rank-1, box extents per dim.  Returns false when the
// encoder is unavailable or rejects the description (alignment, extents).
inline bool make_tmap(CUtensorMap* map, CUtensorMapDataType dtype, int rank, const void* base,
                      const cuuint64_t* dims, const cuuint64_t* byte_strides,
                      const cuuint32_t* box, CUtensorMapSwizzle swizzle) {
  EncodeTiledFn enc = encode_tiled();
  if (!enc) return false;
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const CUresult r =
      enc(map, dtype, (cuuint32_t)rank, const_cast<void*>(base), dims, byte_strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace strata
