// The dense all-experts path ("quantization_mxfp4" (KerasFormers), As GPT-OSS's native
// format: long prefills can run every expert on every token instead of dispatching the
// routed ones, with the same output). Every token goes through all E experts; the router's
// gates weight the k selected experts and are zero for the others, so the weighted sum
// over all experts equals the routed one.
//
// dense_setup_kernel: the (T, E) gate matrix (the token's softmax weight at its selected
// experts, 0 elsewhere) and the expert offsets e * T of the expert-major (E * T) row
// layout the grouped GEMMs then work on (every expert owns all T tokens, in token order).
// dense_combine_kernel: out[t] = bf16(sum over e = 0 .. E-1 of G[t, e] * y[e * T + t]),
// fp32, one rounding per multiply and per add, experts in ascending order.
// Also here: the set-up and the fp32 -> bf16 rounding of a plain MXFP4 linear layer, which
// runs as the same grouped GEMMs with one expert that every token reaches.
#include "common.cuh"

namespace mxmoe {

namespace {

__global__ void __launch_bounds__(256) dense_setup_kernel(const int32_t* __restrict__ topk_idx,
                                                          const float* __restrict__ topk_w, int T, int E, int k,
                                                          float* __restrict__ gates, int32_t* __restrict__ offsets) {
  const int64_t n = static_cast<int64_t>(T) * E;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
    const int64_t t = i / E;
    const int e = static_cast<int>(i % E);
    float g = 0.0f;
    for (int j = 0; j < k; ++j)
      if (topk_idx[t * k + j] == e) g = topk_w[t * k + j];
    gates[i] = g;
  }
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e <= E; e += stride)
    offsets[e] = static_cast<int32_t>(e * T);
}

__global__ void __launch_bounds__(256) dense_combine_kernel(const float* __restrict__ y,
                                                            const float* __restrict__ gates, int T, int H, int E,
                                                            uint16_t* __restrict__ out) {
  const int h8 = H / 8;
  const int64_t n = static_cast<int64_t>(T) * h8;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t expert_stride = static_cast<int64_t>(T) * H;   // floats between experts' rows
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
    const int64_t t = i / h8;
    const int c = static_cast<int>(i % h8);
    const float* src = y + t * H + 8 * c;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int e = 0; e < E; ++e) {
      const float g = gates[t * E + e];
      const float4 a = __ldcs(reinterpret_cast<const float4*>(src + e * expert_stride));
      const float4 b = __ldcs(reinterpret_cast<const float4*>(src + e * expert_stride) + 1);
      const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
      for (int r = 0; r < 8; ++r) acc[r] = __fadd_rn(acc[r], __fmul_rn(g, v[r]));
    }
    uint4 o;
    o.x = f32_to_bf16_bits_rn(acc[0]) | (static_cast<uint32_t>(f32_to_bf16_bits_rn(acc[1])) << 16);
    o.y = f32_to_bf16_bits_rn(acc[2]) | (static_cast<uint32_t>(f32_to_bf16_bits_rn(acc[3])) << 16);
    o.z = f32_to_bf16_bits_rn(acc[4]) | (static_cast<uint32_t>(f32_to_bf16_bits_rn(acc[5])) << 16);
    o.w = f32_to_bf16_bits_rn(acc[6]) | (static_cast<uint32_t>(f32_to_bf16_bits_rn(acc[7])) << 16);
    reinterpret_cast<uint4*>(out)[i] = o;
  }
}

// The one-expert routing of a plain linear layer (offsets {0, T}, active {0}, one active
// expert) and, where the caller passes no bias, a zero bias of N values.
__global__ void linear_setup_kernel(int T, int N, int32_t* __restrict__ offsets, int32_t* __restrict__ active,
                                    int32_t* __restrict__ n_active, float* __restrict__ zero_bias) {
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    offsets[0] = 0;
    offsets[1] = T;
    active[0] = 0;
    *n_active = 1;
  }
  if (zero_bias)
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < N;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
      zero_bias[i] = 0.0f;
}

__global__ void __launch_bounds__(256) f32_to_bf16_kernel(const float4* __restrict__ y, int64_t n4,
                                                          uint2* __restrict__ out) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride) {
    const float4 v = __ldcs(y + i);
    out[i] = make_uint2(f32_to_bf16_bits_rn(v.x) | (static_cast<uint32_t>(f32_to_bf16_bits_rn(v.y)) << 16),
                        f32_to_bf16_bits_rn(v.z) | (static_cast<uint32_t>(f32_to_bf16_bits_rn(v.w)) << 16));
  }
}

unsigned grid_for(int64_t n, int sms) {
  const int64_t g = cdiv(n, 256);
  const int64_t cap = static_cast<int64_t>(sms) * 8;
  return static_cast<unsigned>(g < 1 ? 1 : (g > cap ? cap : g));
}

}  // namespace

cudaError_t launch_dense_setup(const int32_t* topk_idx, const float* topk_w, int T, int E, int k, float* gates,
                               int32_t* offsets, cudaStream_t st, int sms) {
  dense_setup_kernel<<<grid_for(static_cast<int64_t>(T) * E, sms), 256, 0, st>>>(topk_idx, topk_w, T, E, k, gates,
                                                                                offsets);
  return cudaGetLastError();
}

cudaError_t launch_dense_combine(const float* y, const float* gates, int T, int H, int E, uint16_t* out,
                                 cudaStream_t st, int sms) {
  dense_combine_kernel<<<grid_for(static_cast<int64_t>(T) * (H / 8), sms), 256, 0, st>>>(y, gates, T, H, E, out);
  return cudaGetLastError();
}

cudaError_t launch_linear_setup(int T, int N, int32_t* offsets, int32_t* active, int32_t* n_active, float* zero_bias,
                                cudaStream_t st, int sms) {
  linear_setup_kernel<<<grid_for(zero_bias ? N : 1, sms), 256, 0, st>>>(T, N, offsets, active, n_active, zero_bias);
  return cudaGetLastError();
}

cudaError_t launch_f32_to_bf16(const float* y, int64_t n, uint16_t* out, cudaStream_t st, int sms) {
  if (n == 0) return cudaSuccess;
  f32_to_bf16_kernel<<<grid_for(n / 4, sms), 256, 0, st>>>(reinterpret_cast<const float4*>(y), n / 4,
                                                           reinterpret_cast<uint2*>(out));
  return cudaGetLastError();
}

}  // namespace mxmoe
