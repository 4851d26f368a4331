// Standalone MXFP4 codec kernels: quantize (fp32 -> blocks + e8m0 scales) and
// dequantize (-> fp32 or bf16), bit-exact.
//
// Format ("quantization_mxfp4" (KerasFormers), intro and Primitives): e2m1 values, two
// per byte (element 2j in the low nibble), one e8m0 scale byte 2^(s-127) per 32 values
// along the contracting dim. Quantize: block exponent floor(log2(amax)) - 2, then each
// value to the nearest grid point. Both kernels treat the (rows, K) tensor as a flat
// run of 32-value blocks (K % 32 == 0), so block b owns bytes [16b, 16b+16) and scale b.
//
// Memory layout per thread: quantize reads one float4 (4 values) per lane, 8 lanes per
// block, so every warp-wide load is 512 contiguous bytes; dequantize reads one 32-bit
// word (8 values) per lane, 4 lanes per block. Both kernels are HBM-bound streams with
// several loads in flight per thread (quantize 4 float4, dequantize 8 words).
#include <algorithm>

#include "common.cuh"

namespace mxmoe {

namespace {

// floor(log2(m)) for a finite m > 0, exact (normal and subnormal fp32).
__device__ __forceinline__ int floor_log2_pos(float m) {
  uint32_t u = __float_as_uint(m);
  int ex = static_cast<int>(u >> 23);
  if (ex > 0) return ex - 127;
  return (31 - __clz(u)) - 149;  // subnormal: u = mantissa, value = u * 2^-149
}

// Nearest E2M1 magnitude code for r = |x| / 2^e in [0, 8): each comparison is one
// midpoint of the grid {0, .5, 1, 1.5, 2, 3, 4, 6}; '>' at a midpoint whose lower
// neighbour has the even code, '>=' where the upper one has it (ties to even). Everything
// above 5 becomes 6 (code 7), i.e. magnitudes past 6 saturate.
__device__ __forceinline__ uint32_t e2m1_code(float r) {
  return static_cast<uint32_t>(r > 0.25f) + static_cast<uint32_t>(r >= 0.75f) +
         static_cast<uint32_t>(r > 1.25f) + static_cast<uint32_t>(r >= 1.75f) +
         static_cast<uint32_t>(r > 2.5f) + static_cast<uint32_t>(r >= 3.5f) +
         static_cast<uint32_t>(r > 5.0f);
}

constexpr int kQuantUnroll = 4;

__global__ void __launch_bounds__(256) quantize_kernel(const float4* __restrict__ w,
                                                        int64_t nquads,
                                                        uint16_t* __restrict__ blocks16,
                                                        uint8_t* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int64_t warp_global = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  // each warp iteration covers kQuantUnroll * 32 consecutive quads (= 4 * 4 blocks)
  for (int64_t base = warp_global * (32 * kQuantUnroll); base < nquads;
       base += nwarps * (32 * kQuantUnroll)) {
    float4 v[kQuantUnroll];
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
      const int64_t q = base + u * 32 + lane;
      v[u] = q < nquads ? __ldcs(&w[q]) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
      const int64_t q = base + u * 32 + lane;
      float m = fmaxf(fmaxf(fabsf(v[u].x), fabsf(v[u].y)), fmaxf(fabsf(v[u].z), fabsf(v[u].w)));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
      int e = (m > 0.0f) ? floor_log2_pos(m) - 2 : -127;
      e = max(-127, min(127, e));
      // 2^-e: exponent field 127 - e lies in [2, 254] because floor(log2 amax) <= 127
      const float inv = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
      const float xs[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
      uint32_t packed = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t sign = (__float_as_uint(xs[i]) >> 31) << 3;
        packed |= (e2m1_code(fabsf(xs[i]) * inv) | sign) << (4 * i);
      }
      if (q < nquads) {
        __stcs(&blocks16[q], static_cast<uint16_t>(packed));
        if ((lane & 7) == 0) scales[q >> 3] = static_cast<uint8_t>(e + 127);
      }
    }
  }
}

// fp32 bits of the unscaled E2M1 magnitude for code c in [0, 8).
__device__ __forceinline__ uint32_t e2m1_mag_bits(uint32_t c) {
  return c < 2u ? c * 0x3F000000u : (((126u + (c >> 1)) << 23) | ((c & 1u) << 22));
}

constexpr int kDeqUnroll = 8;

template <bool kBf16>
__global__ void __launch_bounds__(256) dequantize_kernel(const uint32_t* __restrict__ blocks32,
                                                          const uint8_t* __restrict__ scales,
                                                          int64_t nwords, void* __restrict__ out) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  // kDeqUnroll words per thread and iteration, stride apart (each warp-wide access stays
  // contiguous), all loaded before the first is decoded
  for (int64_t base = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; base < nwords;
       base += kDeqUnroll * stride) {
    uint32_t wds[kDeqUnroll], scs[kDeqUnroll];
#pragma unroll
    for (int j = 0; j < kDeqUnroll; ++j) {
      const int64_t u = base + j * stride;
      wds[j] = u < nwords ? __ldcs(&blocks32[u]) : 0u;
      scs[j] = u < nwords ? scales[u >> 2] : 127u;
    }
#pragma unroll
    for (int j = 0; j < kDeqUnroll; ++j) {
      const int64_t u = base + j * stride;
      if (u >= nwords) break;
      const uint32_t wd = wds[j], s = scs[j];
      // value = c * 2^(s-127) = (c * s1) * s2 with every factor exact in fp32
      const float s1 = s == 255u ? __uint_as_float(254u << 23) : e8m0_to_f32(s);
      float v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t nib = (wd >> (4 * i)) & 15u;
        const float c = __uint_as_float(e2m1_mag_bits(nib & 7u) | ((nib & 8u) << 28));
        v[i] = c * s1;
      }
      if (s == 255u) {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] *= 2.0f;
      }
      if constexpr (kBf16) {
        // every value has at most two significant bits: its bf16 is the top half of fp32
        uint4 o;
        o.x = (__float_as_uint(v[0]) >> 16) | (__float_as_uint(v[1]) & 0xFFFF0000u);
        o.y = (__float_as_uint(v[2]) >> 16) | (__float_as_uint(v[3]) & 0xFFFF0000u);
        o.z = (__float_as_uint(v[4]) >> 16) | (__float_as_uint(v[5]) & 0xFFFF0000u);
        o.w = (__float_as_uint(v[6]) >> 16) | (__float_as_uint(v[7]) & 0xFFFF0000u);
        __stcs(reinterpret_cast<uint4*>(out) + u, o);
      } else {
        float4* o = reinterpret_cast<float4*>(out) + 2 * u;
        __stcs(o, make_float4(v[0], v[1], v[2], v[3]));
        __stcs(o + 1, make_float4(v[4], v[5], v[6], v[7]));
      }
    }
  }
}

// ------------------------------------------------ along an arbitrary contracting axis --
// The tensor as (outer, K, inner) with the contracting axis in the middle; the packed
// result has that axis last: blocks (outer, inner, K/2), scales (outer, inner, K/32)
// ("quantization_mxfp4" (KerasFormers), Primitives: MXFP4Quantizer quantizes along one
// axis, moved to the end). One thread per (outer, block, inner) with inner fastest, so a
// warp reads each of its 32 values as one contiguous run across inner; it writes its 16
// block bytes as one 16-byte store. The same exponent and rounding as quantize_kernel.
__global__ void __launch_bounds__(256) quantize_axis_kernel(const float* __restrict__ w, int64_t outer, int64_t K,
                                                             int64_t inner, uint8_t* __restrict__ blocks,
                                                             uint8_t* __restrict__ scales) {
  const int64_t nb = K / 32;
  const int64_t n = outer * nb * inner;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < n; idx += stride) {
    const int64_t i = idx % inner, ob = idx / inner;
    const int64_t b = ob % nb, o = ob / nb;
    const float* src = w + (o * K + 32 * b) * inner + i;
    float v[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = __ldcs(src + j * inner);
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < 32; ++j) m = fmaxf(m, fabsf(v[j]));
    int e = (m > 0.0f) ? floor_log2_pos(m) - 2 : -127;
    e = max(-127, min(127, e));
    const float inv = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
    uint32_t wd[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const uint32_t sign = (__float_as_uint(v[j]) >> 31) << 3;
      wd[j >> 3] |= (e2m1_code(fabsf(v[j]) * inv) | sign) << (4 * (j & 7));
    }
    const int64_t r = o * inner + i;
    *reinterpret_cast<uint4*>(blocks + r * (K / 2) + 16 * b) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
    scales[r * nb + b] = static_cast<uint8_t>(e + 127);
  }
}

// The inverse: (outer, inner, K/2) + (outer, inner, K/32) -> (outer, K, inner) fp32 or
// bf16, the values of dequantize_kernel; a warp's stores of each value index are one
// contiguous run across inner.
template <bool kBf16>
__global__ void __launch_bounds__(256) dequantize_axis_kernel(const uint8_t* __restrict__ blocks,
                                                               const uint8_t* __restrict__ scales, int64_t outer,
                                                               int64_t K, int64_t inner, void* __restrict__ out) {
  const int64_t nb = K / 32;
  const int64_t n = outer * nb * inner;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < n; idx += stride) {
    const int64_t i = idx % inner, ob = idx / inner;
    const int64_t b = ob % nb, o = ob / nb;
    const int64_t r = o * inner + i;
    const uint4 q = *reinterpret_cast<const uint4*>(blocks + r * (K / 2) + 16 * b);
    const uint32_t s = scales[r * nb + b];
    const float s1 = s == 255u ? __uint_as_float(254u << 23) : e8m0_to_f32(s);
    const uint32_t wd[4] = {q.x, q.y, q.z, q.w};
    const int64_t dst = (o * K + 32 * b) * inner + i;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const uint32_t nib = (wd[j >> 3] >> (4 * (j & 7))) & 15u;
      float v = __uint_as_float(e2m1_mag_bits(nib & 7u) | ((nib & 8u) << 28)) * s1;
      if (s == 255u) v *= 2.0f;
      if constexpr (kBf16)
        reinterpret_cast<uint16_t*>(out)[dst + j * inner] = static_cast<uint16_t>(__float_as_uint(v) >> 16);
      else
        reinterpret_cast<float*>(out)[dst + j * inner] = v;
    }
  }
}

// Grid of a grid-stride stream kernel: at most the CTAs that fit on the GPU at once, so
// every CTA of the grid is resident from the start (a second, partial wave would run the
// last share of the stream at lower occupancy).
template <typename Kernel>
int grid_for(Kernel kernel, int64_t work_items, int threads, int sms) {
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, 0) != cudaSuccess || per_sm < 1)
    per_sm = 1;
  const int64_t g = cdiv(work_items, threads);
  const int64_t cap = static_cast<int64_t>(sms) * per_sm;
  return static_cast<int>(g < 1 ? 1 : (g > cap ? cap : g));
}

}  // namespace

cudaError_t launch_quantize(const float* w, int64_t rows, int64_t K, uint8_t* blocks,
                            uint8_t* scales, cudaStream_t st, int sms) {
  const int64_t nquads = rows * K / 4;
  if (nquads == 0) return cudaSuccess;
  // 8 CTAs per SM although fewer are resident at once (48 registers a thread): measured
  // on one B200 over the 12.7 GB fp32 expert set, 3.60 ms against 3.74 ms on the grid of
  // resident CTAs, and a variant that loads the next iteration's values before encoding
  // this one's was slower still (3.90 ms)
  const int64_t want = std::max<int64_t>(cdiv(cdiv(nquads, kQuantUnroll), 256), 1);
  const int grid = static_cast<int>(std::min<int64_t>(want, static_cast<int64_t>(sms) * 8));
  quantize_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const float4*>(w), nquads,
                                        reinterpret_cast<uint16_t*>(blocks), scales);
  return cudaGetLastError();
}

cudaError_t launch_dequantize(const uint8_t* blocks, const uint8_t* scales, int64_t rows,
                              int64_t K, void* out, int out_dtype, cudaStream_t st, int sms) {
  const int64_t nwords = rows * K / 8;
  if (nwords == 0) return cudaSuccess;
  const int grid = out_dtype == MXMOE_OUT_BF16 ? grid_for(dequantize_kernel<true>, cdiv(nwords, kDeqUnroll), 256, sms)
                                               : grid_for(dequantize_kernel<false>, cdiv(nwords, kDeqUnroll), 256, sms);
  if (out_dtype == MXMOE_OUT_BF16)
    dequantize_kernel<true><<<grid, 256, 0, st>>>(reinterpret_cast<const uint32_t*>(blocks),
                                                  scales, nwords, out);
  else
    dequantize_kernel<false><<<grid, 256, 0, st>>>(reinterpret_cast<const uint32_t*>(blocks),
                                                   scales, nwords, out);
  return cudaGetLastError();
}

cudaError_t launch_quantize_axis(const float* w, int64_t outer, int64_t K, int64_t inner, uint8_t* blocks,
                                 uint8_t* scales, cudaStream_t st, int sms) {
  if (inner == 1) return launch_quantize(w, outer, K, blocks, scales, st, sms);
  const int64_t n = outer * (K / 32) * inner;
  if (n == 0) return cudaSuccess;
  quantize_axis_kernel<<<grid_for(quantize_axis_kernel, n, 256, sms), 256, 0, st>>>(w, outer, K, inner, blocks,
                                                                                   scales);
  return cudaGetLastError();
}

cudaError_t launch_dequantize_axis(const uint8_t* blocks, const uint8_t* scales, int64_t outer, int64_t K,
                                   int64_t inner, void* out, int out_dtype, cudaStream_t st, int sms) {
  if (inner == 1) return launch_dequantize(blocks, scales, outer, K, out, out_dtype, st, sms);
  const int64_t n = outer * (K / 32) * inner;
  if (n == 0) return cudaSuccess;
  if (out_dtype == MXMOE_OUT_BF16)
    dequantize_axis_kernel<true><<<grid_for(dequantize_axis_kernel<true>, n, 256, sms), 256, 0, st>>>(
        blocks, scales, outer, K, inner, out);
  else
    dequantize_axis_kernel<false><<<grid_for(dequantize_axis_kernel<false>, n, 256, sms), 256, 0, st>>>(
        blocks, scales, outer, K, inner, out);
  return cudaGetLastError();
}

}  // namespace mxmoe
