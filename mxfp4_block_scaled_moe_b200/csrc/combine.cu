// Weighted un-permute / combine: out[t, :] = bf16( sum_j w[t, j] * y[pos(t, j), :] ),
// the sum taken in fp32 over the token's k experts in ascending expert id (one rounding
// per multiply and per add), then one round-to-nearest-even to bf16.
// ("quantization_mxfp4" (KerasFormers), As GPT-OSS's native format: the expert outputs
// are summed with their router gates.)
#include "common.cuh"

namespace mxmoe {

namespace {

__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ y,
                                                       const int32_t* __restrict__ topk_idx,
                                                       const float* __restrict__ topk_w,
                                                       const int32_t* __restrict__ inv, int T,
                                                       int H, int k, uint16_t* __restrict__ out) {
  const int h8 = H / 8;
  const int64_t n = static_cast<int64_t>(T) * h8;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
    const int t = static_cast<int>(i / h8), c = static_cast<int>(i % h8);
    // order the k slots by expert id (k <= 8, insertion sort)
    int ord[8], eid[8];
    for (int j = 0; j < k; ++j) {
      const int e = topk_idx[static_cast<int64_t>(t) * k + j];
      int q = j;
      while (q > 0 && eid[q - 1] > e) { eid[q] = eid[q - 1]; ord[q] = ord[q - 1]; --q; }
      eid[q] = e;
      ord[q] = j;
    }
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int q = 0; q < k; ++q) {
      const int j = ord[q];
      const float w = topk_w[static_cast<int64_t>(t) * k + j];
      const int64_t pos = inv[static_cast<int64_t>(t) * k + j];
      const float4* src = reinterpret_cast<const float4*>(y + pos * H) + 2 * c;
      const float4 a = src[0], b = src[1];
      const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
      for (int r = 0; r < 8; ++r) acc[r] = __fadd_rn(acc[r], __fmul_rn(w, v[r]));
    }
    uint4 o;
    o.x = f32_to_bf16_bits_rn(acc[0]) | (static_cast<uint32_t>(f32_to_bf16_bits_rn(acc[1])) << 16);
    o.y = f32_to_bf16_bits_rn(acc[2]) | (static_cast<uint32_t>(f32_to_bf16_bits_rn(acc[3])) << 16);
    o.z = f32_to_bf16_bits_rn(acc[4]) | (static_cast<uint32_t>(f32_to_bf16_bits_rn(acc[5])) << 16);
    o.w = f32_to_bf16_bits_rn(acc[6]) | (static_cast<uint32_t>(f32_to_bf16_bits_rn(acc[7])) << 16);
    reinterpret_cast<uint4*>(out)[i] = o;
  }
}

}  // namespace

cudaError_t launch_combine(const float* y, const int32_t* topk_idx, const float* topk_w,
                           const int32_t* inv, int T, int H, int k, uint16_t* out, cudaStream_t st,
                           int sms) {
  const int64_t n = static_cast<int64_t>(T) * (H / 8);
  const int64_t g = cdiv(n, 256);
  const int64_t cap = static_cast<int64_t>(sms) * 8;
  combine_kernel<<<static_cast<unsigned>(g < 1 ? 1 : (g > cap ? cap : g)), 256, 0, st>>>(
      y, topk_idx, topk_w, inv, T, H, k, out);
  return cudaGetLastError();
}

}  // namespace mxmoe
