// The warp-level top-k softmax of one token's router logits, shared by the routing kernels
// (csrc/route.cu) and the fused small-batch routing of the decode path
// (csrc/gemm_decode_sm100.cu). Ranking: larger logit first, NaN after every number, equal
// values -> lower expert id first ("gpt-oss-120b-mxfp4-fp8attn-v2", Model Details: top-4
// routing; ties to the lower id); softmax over the k selected logits.
#pragma once

#include "common.cuh"

namespace mxmoe {

// Ranking: larger logit first, NaN after every number, equal values -> lower id first.
__device__ __forceinline__ bool ranks_before(float a, int ia, float b, int ib) {
  const bool na = isnan(a), nb = isnan(b);
  if (na != nb) return nb;
  if (!na && a != b) return a > b;
  return ia < ib;
}

// One warp selects the k largest of a token's E logits (E <= 256, each lane holds up to 8)
// and writes the indices and the softmax over them.
__device__ __forceinline__ void topk_warp(const float* __restrict__ l, int E, int k,
                                          int32_t* __restrict__ idx_out, float* __restrict__ w_out) {
  const int lane = threadIdx.x & 31;
  float v[8];
  int taken = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane + 32 * i;
    v[i] = e < E ? l[e] : 0.0f;
  }
  float sel[8];
  int sidx[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j >= k) break;
    float bv = 0.0f;
    int bi = -1;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !((taken >> i) & 1) && (bi < 0 || ranks_before(v[i], e, bv, bi))) {
        bv = v[i];
        bi = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (oi >= 0 && (bi < 0 || ranks_before(ov, oi, bv, bi))) { bv = ov; bi = oi; }
    }
    sel[j] = bv;
    sidx[j] = bi;
    if ((bi & 31) == lane) taken |= 1 << (bi >> 5);
  }
  // softmax over the k selected logits: lane j < k takes term j; every lane adds the terms
  // in order j = 0 .. k-1 (the same sum as a sequential loop)
  float my_sel = sel[0];
  int my_idx = sidx[0];
#pragma unroll
  for (int j = 1; j < 8; ++j)
    if (j < k && lane == j) { my_sel = sel[j]; my_idx = sidx[j]; }
  const float pj = lane < k ? expf(my_sel - sel[0]) : 0.0f;
  float z = 0.0f;
  for (int j = 0; j < k; ++j) z += __shfl_sync(0xffffffffu, pj, j);
  if (lane < k) {
    idx_out[lane] = my_idx;
    w_out[lane] = __fdiv_rn(pj, z);
  }
}


}  // namespace mxmoe
