// The pieces of the small-batch tensor-core paths that turn a real value into MXFP4 "parts"
// and feed them to tcgen05.mma kind::mxf4 (shared by csrc/gemm_decode_sm100.cu and
// csrc/decode_layer_sm100.cu): a value is written as the sum of four e2m1 codes, each
// with the e8m0 scale of its 32-value block chosen from the largest residual, so that
// the FP4 x FP4 tensor core contracts it against the checkpoint's MXFP4 weights. The
// MXFP4 element and scale encodings are those of "quantization_mxfp4" (KerasFormers),
// Primitives.
#pragma once

#include <cuda_fp4.h>

#include "common.cuh"

namespace mxmoe {

// Instruction descriptor, kind::mxf4 block-scaled (scale_vec::2X): A = B = E2M1 (1), e8m0
// scales; sf_id (0 or 2) selects the scale-byte pair of a K = 64 step.
__host__ __device__ constexpr uint32_t idesc_mxf4(int M, int N) {
  return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) | (1u << 23) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ float pow2f(int s) {   // exact 2^s for s in [-126, 127]
  return __uint_as_float(static_cast<uint32_t>(s + 127) << 23);
}

// Scale exponent of an e2m1 part: the smallest s with amax / 2^s <= 6 (the e2m1 maximum),
// clamped to [-126, 125]; amax == 0 gives 0. Branch-free: a subnormal amax reads as
// floor(log2) = -127, which the clamp maps to -126 exactly as its true exponent would.
__device__ __forceinline__ int e2m1_part_exponent(float amax) {
  const int fl = static_cast<int>(__float_as_uint(amax) >> 23) - 127;   // amax >= 0
  int s = max(-126, min(125, fl - 2));                                   // amax / 2^s in [4, 8)
  s = (amax > 6.0f * pow2f(s)) ? min(125, s + 1) : s;
  return amax > 0.0f ? s : 0;
}

// The e2m1 code of v (already divided by its part scale, |v| <= 6), round to nearest
// even, in the low nibble; and the value that code stands for.
__device__ __forceinline__ uint32_t e2m1_code(float v) {
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp4x2(make_float2(v, 0.0f), __NV_E2M1, cudaRoundNearest)) & 0xFu;
}
__device__ __forceinline__ float e2m1_value(uint32_t code) {
  const __half2_raw h = __nv_cvt_fp4x2_to_halfraw2(static_cast<__nv_fp4x2_storage_t>(code), __NV_E2M1);
  return __half2float(__half(__half_raw{h.x}));
}

}  // namespace mxmoe
