// Host-side TMA tensor maps for the tcgen05 kernels: cuTensorMapEncodeTiled, reached through
// the runtime's driver entry point so that the library needs no -lcuda. Every map this
// library builds is the same kind: dense row-major bytes (or 16 x U4 rows), 128-byte
// swizzle, 256-byte L2 promotion, zero fill outside the tensor (a box that runs past the
// last row reads zeros and still counts its full size toward the mbarrier transaction).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mxmoe {

using TmapEncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline TmapEncodeFn tmap_encoder() {
  static TmapEncodeFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<TmapEncodeFn>(ptr);
  }
  return fn;
}

inline bool tmap_available() { return tmap_encoder() != nullptr; }

// rank <= 3; dims[0] is the innermost (contiguous) extent in elements, strides_bytes the
// byte strides of dims 1.. (multiples of 16), box the tile copied per load.
inline bool tmap_encode(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base, const uint64_t* dims,
                        const uint64_t* strides_bytes, const uint32_t* box) {
  TmapEncodeFn fn = tmap_encoder();
  if (!fn || rank < 1 || rank > 3) return false;
  cuuint64_t d[3], s[2];
  cuuint32_t b[3], es[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) { d[i] = dims[i]; b[i] = box[i]; }
  for (int i = 0; i + 1 < rank; ++i) s[i] = strides_bytes[i];
  return fn(m, dt, static_cast<cuuint32_t>(rank), const_cast<void*>(base), d, s, b, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace mxmoe
