// Shared device helpers for libmxfp4moe (sm_100a only).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "mxfp4_moe.h"

#if !defined(__CUDA_ARCH__) || (__CUDA_ARCH__ >= 1000)
#else
#error "libmxfp4moe is built for sm_100a only"
#endif

namespace mxmoe {

// ----------------------------------------------------------------- device error word
// Kernels never trap: a bad input or an expired wait writes the first error code into
// the per-device error word (a library-owned int in device memory, passed to the
// kernels that can fail) and the kernel skips the offending access. mxmoe_check()
// reads and clears it.
__device__ __forceinline__ void set_device_error(int* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

// ------------------------------------------------------------------ small utilities
__host__ __device__ __forceinline__ int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t h) {
  return __uint_as_float(static_cast<uint32_t>(h) << 16);
}

__device__ __forceinline__ uint16_t f32_to_bf16_bits_rn(float f) {
  __nv_bfloat16 b = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&b);
}

// FP8 E4M3 ("fn") of q with round-to-nearest-even and saturation to +-448 (hardware cvt).
__device__ __forceinline__ uint8_t f32_to_e4m3_satfinite(float q) {
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(q, __NV_SATFINITE, __NV_E4M3));
}

// Exact E4M3 -> fp32 (via the hardware e4m3 -> f16 conversion; every e4m3 value is an f16).
__device__ __forceinline__ float e4m3_to_f32(uint8_t c) {
  __half_raw hr = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(c), __NV_E4M3);
  return __half2float(__half(hr));
}

// The A-FP8 activation cast: one IEEE fp32 division, then RNE/satfinite to E4M3.
__device__ __forceinline__ uint8_t act_quant_e4m3(float x, float s) {
  return f32_to_e4m3_satfinite(__fdiv_rn(x, s));
}

// fp32 bit pattern of 2^(s - 127) for an e8m0 byte s in [0, 254] (s = 0 is the fp32
// subnormal 2^-127). s = 255 is handled by callers that need it.
__device__ __forceinline__ float e8m0_to_f32(uint32_t s) {
  return s == 0u ? __uint_as_float(0x00400000u) : __uint_as_float(s << 23);
}

__device__ __forceinline__ float silu_mul(float gate, float up) {
  return __fdiv_rn(gate, 1.0f + expf(-gate)) * up;
}

// One 32-byte store of eight fp32 values (sm_100's 256-bit global store); dst 32-byte
// aligned. Measured on the down GEMM's fp32 outputs: a full sector per thread and half the
// store instructions of two 16-byte stores, 0.700 against 0.815 ms at 65,536 routed rows.
__device__ __forceinline__ void st_global_v8(float* dst, const float (&v)[8]) {
  asm volatile("st.global.v8.f32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};\n" ::"l"(dst), "f"(v[0]), "f"(v[1]),
               "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7])
               : "memory");
}

// Programmatic dependent launch: a kernel launched with programmatic stream serialization
// may start once every CTA of the previous kernel in the stream has called
// griddep_launch_dependents() (or exited); griddep_wait() returns once that kernel has
// completed and its memory operations are visible. Both are no-ops without the attribute.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

// ------------------------------------------------------------------ warp utilities
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }


// -------------------------------------------------------------- legacy MMA (mma.sync)
// m16n8k16, bf16 x bf16 -> fp32. a: 4 regs, b: 2 regs, c/d: 4 fp32.
__device__ __forceinline__ void mma_bf16_16816(float d[4], const uint32_t a[4], const uint32_t b[2],
                                               const float c[4]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%11,%12,%13};\n"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]), "f"(c[0]), "f"(c[1]),
        "f"(c[2]), "f"(c[3]));
}

__device__ __forceinline__ uint32_t ld_nc_u32(const void* p) {
  uint32_t v;
  asm volatile("ld.global.nc.u32 %0, [%1];\n" : "=r"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

}  // namespace mxmoe
