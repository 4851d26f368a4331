// Warp-level routing pieces shared by the routing kernels (csrc/route.cu) and the one-launch
// decode layer (csrc/decode_layer_sm100.cu), so that both compute bit-identical logits and
// selections: one router logit as a warp's dot product, and the top-k softmax of one
// token's router logits. Ranking: larger logit first, NaN after every number, equal
// values -> lower expert id first ("gpt-oss-120b-mxfp4-fp8attn-v2", Model Details: top-4
// routing; ties to the lower id); softmax over the k selected logits.
#pragma once

#include "common.cuh"

namespace mxmoe {

// One router logit <x, w> over H bf16 values (H % 8 == 0, rows 16-byte aligned) by one
// warp, fp32: each lane takes 16-byte chunks lane, lane + 32, ..., twelve in flight (one
// memory round trip per 3072 values), and adds their products in chunk order (low then
// high half of each 32-bit word); the lanes' sums are then added by a butterfly. Every
// lane returns the same sum.
__device__ __forceinline__ float router_logit_warp(const uint16_t* __restrict__ x, const uint16_t* __restrict__ w,
                                                   int H) {
  const int lane = threadIdx.x & 31;
  const uint4* xr = reinterpret_cast<const uint4*>(x);
  const uint4* wr = reinterpret_cast<const uint4*>(w);
  float acc = 0.0f;
  constexpr int kChunks = 12;
  for (int c0 = lane; c0 < H / 8; c0 += kChunks * 32) {
    uint4 a[kChunks], b[kChunks];
#pragma unroll
    for (int u = 0; u < kChunks; ++u) {
      const int c = c0 + 32 * u;
      if (c < H / 8) { a[u] = ld_nc_v4(xr + c); b[u] = ld_nc_v4(wr + c); }
    }
#pragma unroll
    for (int u = 0; u < kChunks; ++u) {
      if (c0 + 32 * u >= H / 8) break;
      const uint32_t av[4] = {a[u].x, a[u].y, a[u].z, a[u].w}, bv[4] = {b[u].x, b[u].y, b[u].z, b[u].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc = fmaf(__uint_as_float(av[i] << 16), __uint_as_float(bv[i] << 16), acc);
        acc = fmaf(__uint_as_float(av[i] & 0xFFFF0000u), __uint_as_float(bv[i] & 0xFFFF0000u), acc);
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  return acc;
}

// An unsigned key whose order is the ranking's order of logits: larger logit, larger key;
// -0 and +0 equal; NaN the smallest key (0), below every number.
__device__ __forceinline__ unsigned rank_key(float v) {
  if (isnan(v)) return 0u;
  const unsigned u = __float_as_uint(v == 0.0f ? 0.0f : v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// One warp selects the k largest of a token's E logits (E <= 256, each lane holds up to 8)
// and writes the indices and the softmax over them. Each of the k rounds takes the lane's
// best untaken logit and two warp reductions (redux.sync): the largest key, then the
// lowest expert id among the lanes that hold it; lane j keeps round j's value and index.
__device__ __forceinline__ void topk_warp(const float* __restrict__ l, int E, int k,
                                          int32_t* __restrict__ idx_out, float* __restrict__ w_out) {
  const int lane = threadIdx.x & 31;
  float v[8];
  unsigned key[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane + 32 * i;
    v[i] = e < E ? l[e] : 0.0f;
    key[i] = rank_key(v[i]);
  }
  unsigned avail = 0u;   // bit i: value i exists and is not taken yet
#pragma unroll
  for (int i = 0; i < 8; ++i) avail |= (lane + 32 * i < E ? 1u : 0u) << i;
  float my_sel = 0.0f, sel0 = 0.0f;
  int my_idx = -1;
#pragma unroll 1
  for (int j = 0; j < k; ++j) {
    // the lane's best: the largest key, the lowest id on equal keys (ids rise with i)
    unsigned bk = 0u, bi = 0xFFFFu;
    float bv = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (((avail >> i) & 1u) && (bi == 0xFFFFu || key[i] > bk)) {
        bk = key[i];
        bi = static_cast<unsigned>(lane + 32 * i);
        bv = v[i];
      }
    }
    const unsigned gk = __reduce_max_sync(0xffffffffu, bi == 0xFFFFu ? 0u : bk);
    const unsigned gi = __reduce_min_sync(0xffffffffu, (bi != 0xFFFFu && bk == gk) ? bi : 0xFFFFu);
    const float gv = __shfl_sync(0xffffffffu, bv, static_cast<int>(gi & 31u));
    if (j == 0) sel0 = gv;
    if (lane == j) { my_sel = gv; my_idx = static_cast<int>(gi); }
    if ((gi & 31u) == static_cast<unsigned>(lane)) avail &= ~(1u << (gi >> 5));
  }
  // softmax over the k selected logits: lane j < k takes term j; every lane adds the terms
  // in order j = 0 .. k-1 (the same sum as a sequential loop)
  const float pj = lane < k ? expf(my_sel - sel0) : 0.0f;
  float z = 0.0f;
  for (int j = 0; j < k; ++j) z += __shfl_sync(0xffffffffu, pj, j);
  if (lane < k) {
    idx_out[lane] = my_idx;
    w_out[lane] = __fdiv_rn(pj, z);
  }
}

}  // namespace mxmoe
