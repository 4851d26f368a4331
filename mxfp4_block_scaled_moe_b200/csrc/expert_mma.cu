// Routed expert GEMMs with the MXFP4 weights dequantized in registers (the decode path:
// few tokens per expert, bound by streaming the packed weight bytes from HBM).
//
// Page: "quantization_mxfp4" (KerasFormers), As GPT-OSS's native format -- on decode only
// the top-k routed experts' blocks are dequantized; Primitives -- w = codebook[nibble] *
// 2^(scale - 127).
//
// Shape of the work: for every active expert e and its n_e routed rows (positions
// [off_e, off_e + n_e) of the expert-grouped order), y = s * (X_e . W_e^T) + bias.
// Weights are the M side of mma.sync m16n8k16 (16 weight rows per warp), the routed
// tokens the N side (8 per n-tile), so the bytes of each weight are read once whatever
// n_e is. Per 32-value block (one e8m0 scale) a warp issues two k16 MMAs into a scratch
// accumulator and folds it into the running sum with the block's fp32 scale, so the
// nibbles are decoded without their scale.
//
// Nibble decoding: a 32-bit word holds 8 consecutive e2m1 values v0..v7 (v_i in bits
// 4i..4i+3). The pair (v_i, v_{i+4}) sits 16 bits apart, so one shift per field places
// the 3 magnitude bits at bf16 bits 6..8 (exponent LSBs + mantissa MSB) and the sign at
// bit 15 of both halves at once. That bf16 equals the e2m1 value times 2^-126 (code 1
// becomes the bf16 subnormal 2^-127); one bf16x2 multiply by 2^126 makes it exact.
// The K order inside every group of 8 is therefore (0,4,1,5,2,6,3,7) on both operands;
// activations get the same order with two byte permutes per register pair.
//
// Lane (g = lane/4, t = lane%4) owns weight rows g and g+8 and, within each 32-value
// block, values 8t..8t+7 (bytes 4t..4t+3 of the 16-byte block). A CTA owns one 16-row
// group; its warps split the K blocks so that many loads are in flight per SM even when
// few experts are active, and their partial sums are added in a fixed order.
#include "common.cuh"
#include "launchers.h"

namespace mxmoe {

namespace {

constexpr int kWarps = 4;       // warps per CTA, splitting K
constexpr int kUnroll = 8;      // 32-value blocks per load chunk (two chunks in flight)

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;\n" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// bf16x2 (v_i, v_{i+4}) of an e2m1 word, exact (see the file comment).
template <int i>
__device__ __forceinline__ uint32_t e2m1_pair_bf16x2(uint32_t w) {
  constexpr uint32_t kMag = 0x01C001C0u, kSign = 0x80008000u, k2p126 = 0x7E807E80u;
  uint32_t mag, sgn;
  if constexpr (i == 0) { mag = (w << 6) & kMag; sgn = (w << 12) & kSign; }
  if constexpr (i == 1) { mag = (w << 2) & kMag; sgn = (w << 8) & kSign; }
  if constexpr (i == 2) { mag = (w >> 2) & kMag; sgn = (w << 4) & kSign; }
  if constexpr (i == 3) { mag = (w >> 6) & kMag; sgn = w & kSign; }
  return bf16x2_mul(mag | sgn, k2p126);
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;\n" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 1-D bulk copy global -> shared, completion counted on an mbarrier (16-byte aligned,
// size a multiple of 16).
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// Wait for phase 0 of a single-use mbarrier, giving up after ~1 s.
__device__ __forceinline__ bool wait_phase0(uint64_t* bar) {
  const long long t0 = clock64();
  while (true) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_addr(bar))
        : "memory");
    if (ok) return true;
    if (clock64() - t0 > 2000000000LL) return false;
  }
}

struct ExpertGemmArgs {
  const uint8_t* blocks;   // (E, rows_total, K/2)
  const uint8_t* scales;   // (E, rows_total, K/32)
  const float* bias;       // (E, rows_total)
  int rows_total;          // 2I for gate_up, H for down
  int K;                   // H for gate_up, I for down
  const uint16_t* act;     // activation rows (bf16 bits), K wide
  const int32_t* act_row;  // nullptr: row = position; else row = act_row[position]
  const int32_t* offsets;  // (E+1)
  const int32_t* active;   // active expert ids
  const int32_t* n_active;
  float s_in;              // scale applied to the dot product before the bias
  // outputs
  int mode;                // 0: gate_up + SwiGLU -> act_out; 1: down -> y_out
  int I;                   // gate_up: intermediate size (gate rows [0,I), up rows [I,2I))
  float s_mid;             // fp8 path: a is quantized with this scale; 0: bf16 rounding
  uint16_t* act_out;       // (P, I) bf16 bits (mode 0)
  float* y_out;            // (P, rows_total) fp32 (mode 1)
  unsigned* amax_bits;     // optional: running max |a| (fp32 bits), mode 0
  int* err;                // device error word (bounded-wait timeout)
  // mode 1 with the combine folded in (combine_out != nullptr): the last CTA of each
  // 16-row group writes out[t, rows] = bf16(sum_j w[t,j] * y[inv[t,j], rows])
  uint16_t* combine_out;   // (T, rows_total) bf16
  const int32_t* topk_idx; // (T, k)
  const float* topk_w;     // (T, k)
  const int32_t* inv;      // (T*k) pair -> position
  unsigned* tickets;       // one per 16-row group, zero between calls
  int T, k;
};

// One CTA = one 16-row weight group of one active expert (gate_up: 8 gate + the 8
// matching up rows; down: 16 rows); its kWarps warps split the K blocks, then warp 0 adds
// the partial sums of warps 1.. in a fixed order and runs the epilogue.
template <int NT>
__global__ void __launch_bounds__(kWarps * 32) expert_mma_kernel(ExpertGemmArgs p) {
  // shared: the group's 16 weight rows [16][K/2] bytes, their scales [16][nb] fp32, the
  // partial sums [kWarps-1][NT][4][32] fp32, one mbarrier
  extern __shared__ __align__(16) uint8_t s_dyn[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int slot = blockIdx.y;
  if (slot >= *p.n_active) return;
  const int e = p.active[slot];
  const int pos0 = p.offsets[e], n_e = p.offsets[e + 1] - pos0;
  const int nb = p.K / 32;

  int lo0, hi0;   // first lo row and first hi row of the group
  if (p.mode == 0) {
    lo0 = blockIdx.x * 8;
    hi0 = p.I + lo0;
  } else {
    lo0 = blockIdx.x * 16;
    hi0 = lo0 + 8;
  }
  const int row_lo = lo0 + g, row_hi = hi0 + g;
  const int64_t erow = static_cast<int64_t>(e) * p.rows_total;
  const int rb = p.K / 2;   // packed bytes per row
  uint8_t* wbuf = s_dyn;
  float* sc = reinterpret_cast<float*>(s_dyn + 16 * rb);
  float* red = sc + 16 * nb;
  uint64_t* bar = reinterpret_cast<uint64_t*>(red + (kWarps - 1) * NT * 4 * 32);

  // the 8 lo rows and the 8 hi rows are each 8 * K/2 contiguous bytes: two bulk copies
  // bring the whole group into shared memory while the scales are staged below
  if (threadIdx.x == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(smem_addr(bar)));
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_addr(bar)), "r"(16 * rb)
                 : "memory");
    bulk_copy_g2s(wbuf, p.blocks + (erow + lo0) * rb, 8 * rb, bar);
    bulk_copy_g2s(wbuf + 8 * rb, p.blocks + (erow + hi0) * rb, 8 * rb, bar);
  }

  // scales of the 16 rows as fp32 (slots 0..7 lo rows, 8..15 hi rows); the 8 lo rows (and
  // the 8 hi rows) are 8 * nb contiguous bytes, loaded 16 bytes at a time when aligned
  {
    const uint8_t* half_src[2] = {p.scales + (erow + lo0) * nb, p.scales + (erow + hi0) * nb};
    const int half_bytes = 8 * nb;
    const bool vec = ((reinterpret_cast<uintptr_t>(half_src[0]) | reinterpret_cast<uintptr_t>(half_src[1]) |
                       static_cast<uintptr_t>(half_bytes)) & 15u) == 0;
    if (vec) {
      const int n16 = half_bytes / 16;
      for (int c = threadIdx.x; c < 2 * n16; c += blockDim.x) {
        const int h = c >= n16 ? 1 : 0, o = (c - h * n16) * 16;
        const uint4 v = ld_nc_v4(half_src[h] + o);
        const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
        float* dst = sc + h * half_bytes + o;
#pragma unroll
        for (int j = 0; j < 16; ++j) dst[j] = e8m0_to_f32((wv[j >> 2] >> (8 * (j & 3))) & 0xFFu);
      }
    } else {
      for (int i = threadIdx.x; i < 2 * half_bytes; i += blockDim.x) {
        const int h = i >= half_bytes ? 1 : 0;
        sc[i] = e8m0_to_f32(half_src[h][i - h * half_bytes]);
      }
    }
  }
  __syncthreads();
  if (!wait_phase0(bar)) {
    set_device_error(p.err, MXMOE_ETIMEOUT);
    const long long t0 = clock64();   // let the copies in flight land before leaving
    while (clock64() - t0 < 200000) {
    }
    return;
  }
  const float* sc_lo = sc + g * nb;
  const float* sc_hi = sc + (8 + g) * nb;
  const uint8_t* wlo = wbuf + g * rb + 4 * t;
  const uint8_t* whi = wbuf + (8 + g) * rb + 4 * t;
  const int b_begin = (warp * nb) / kWarps, b_end = ((warp + 1) * nb) / kWarps;

  for (int tp = 0; tp < n_e; tp += 8 * NT) {
    const uint16_t* arow[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int j = tp + nt * 8 + g;
      if (j < n_e) {
        const int pos = pos0 + j;
        const int64_t r = p.act_row ? p.act_row[pos] : pos;
        arow[nt] = p.act + r * p.K + 8 * t;
      } else {
        arow[nt] = nullptr;
      }
    }
    const int nt_live = min(NT, (n_e - tp + 7) / 8);

    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int r = 0; r < 4; ++r) acc[nt][r] = 0.0f;

    // weight words double-buffered: the loads of chunk c+1 are in flight while chunk c
    // is decoded and multiplied (two named buffers, so every index stays static)
    uint32_t wlA[kUnroll], whA[kUnroll], wlB[kUnroll], whB[kUnroll];
    auto load_chunk = [&](uint32_t (&wl)[kUnroll], uint32_t (&wh)[kUnroll], int b0) {
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int b = b0 + u;
        wl[u] = b < b_end ? *reinterpret_cast<const uint32_t*>(wlo + 16 * b) : 0u;
        wh[u] = b < b_end ? *reinterpret_cast<const uint32_t*>(whi + 16 * b) : 0u;
      }
    };
    auto compute_chunk = [&](const uint32_t (&wl)[kUnroll], const uint32_t (&wh)[kUnroll], int b0) {
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int b = b0 + u;
        if (b >= b_end) break;
        uint32_t a0[4], a1[4];
        a0[0] = e2m1_pair_bf16x2<0>(wl[u]);
        a0[1] = e2m1_pair_bf16x2<0>(wh[u]);
        a0[2] = e2m1_pair_bf16x2<1>(wl[u]);
        a0[3] = e2m1_pair_bf16x2<1>(wh[u]);
        a1[0] = e2m1_pair_bf16x2<2>(wl[u]);
        a1[1] = e2m1_pair_bf16x2<2>(wh[u]);
        a1[2] = e2m1_pair_bf16x2<3>(wl[u]);
        a1[3] = e2m1_pair_bf16x2<3>(wh[u]);
        const float sl = sc_lo[b], sh = sc_hi[b];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          if (nt >= nt_live) break;
          uint4 v = make_uint4(0u, 0u, 0u, 0u);
          if (arow[nt]) v = ld_nc_v4(arow[nt] + 32 * b);
          // natural (x0..x7) -> k-step 0: (x0,x4),(x1,x5); k-step 1: (x2,x6),(x3,x7)
          const uint32_t b0r[2] = {prmt(v.x, v.z, 0x5410u), prmt(v.x, v.z, 0x7632u)};
          const uint32_t b1r[2] = {prmt(v.y, v.w, 0x5410u), prmt(v.y, v.w, 0x7632u)};
          float tmp[4] = {0.f, 0.f, 0.f, 0.f};
          mma_bf16_16816(tmp, a0, b0r, tmp);
          mma_bf16_16816(tmp, a1, b1r, tmp);
          acc[nt][0] = fmaf(tmp[0], sl, acc[nt][0]);
          acc[nt][1] = fmaf(tmp[1], sl, acc[nt][1]);
          acc[nt][2] = fmaf(tmp[2], sh, acc[nt][2]);
          acc[nt][3] = fmaf(tmp[3], sh, acc[nt][3]);
        }
      }
    };
    load_chunk(wlA, whA, b_begin);
    for (int b0 = b_begin; b0 < b_end; b0 += 2 * kUnroll) {
      if (b0 + kUnroll < b_end) load_chunk(wlB, whB, b0 + kUnroll);
      compute_chunk(wlA, whA, b0);
      if (b0 + kUnroll >= b_end) break;
      if (b0 + 2 * kUnroll < b_end) load_chunk(wlA, whA, b0 + 2 * kUnroll);
      compute_chunk(wlB, whB, b0 + kUnroll);
    }

    // partial sums of warps 1.. to shared memory; warp 0 adds them in warp order
    if (warp > 0) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        if (nt >= nt_live) break;
#pragma unroll
        for (int r = 0; r < 4; ++r) red[(((warp - 1) * NT + nt) * 4 + r) * 32 + lane] = acc[nt][r];
      }
    }
    __syncthreads();
    if (warp == 0) {
      for (int w = 1; w < kWarps; ++w)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          if (nt >= nt_live) break;
#pragma unroll
          for (int r = 0; r < 4; ++r) acc[nt][r] += red[(((w - 1) * NT + nt) * 4 + r) * 32 + lane];
        }
      // epilogue: acc[nt][0..1] = row_lo, tokens 2t, 2t+1; acc[nt][2..3] = row_hi
      const float b_lo = p.bias[erow + row_lo], b_hi = p.bias[erow + row_hi];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        if (nt >= nt_live) break;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int j = tp + nt * 8 + 2 * t + c;
          if (j >= n_e) continue;
          const int64_t pos = pos0 + j;
          const float lo = __fadd_rn(__fmul_rn(p.s_in, acc[nt][c]), b_lo);
          const float hi = __fadd_rn(__fmul_rn(p.s_in, acc[nt][2 + c]), b_hi);
          if (p.mode == 0) {
            const float a = silu_mul(lo, hi);
            if (p.amax_bits) atomicMax(p.amax_bits, __float_as_uint(fabsf(a)));
            uint16_t bits;
            if (p.s_mid > 0.0f)
              bits = static_cast<uint16_t>(__float_as_uint(e4m3_to_f32(act_quant_e4m3(a, p.s_mid))) >> 16);
            else
              bits = f32_to_bf16_bits_rn(a);
            p.act_out[pos * p.I + row_lo] = bits;
          } else {
            p.y_out[pos * p.rows_total + row_lo] = lo;
            p.y_out[pos * p.rows_total + row_hi] = hi;
          }
        }
      }
    }
    __syncthreads();
  }

  if (p.mode == 1 && p.combine_out != nullptr) {
    // every CTA of this row group (one per active expert) stores its y rows and takes a
    // ticket; the last one adds the group's rows for all tokens in ascending expert id
    __shared__ unsigned s_last;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(&p.tickets[blockIdx.x], 1u) == static_cast<unsigned>(*p.n_active) - 1u;
    __syncthreads();
    if (s_last) {
      __threadfence();
      for (int i = threadIdx.x; i < p.T * 16; i += blockDim.x) {
        const int t = i >> 4, r = lo0 + (i & 15);
        int ord[8], eid[8];
        for (int j = 0; j < p.k; ++j) {
          const int ex = p.topk_idx[static_cast<int64_t>(t) * p.k + j];
          int q = j;
          while (q > 0 && eid[q - 1] > ex) { eid[q] = eid[q - 1]; ord[q] = ord[q - 1]; --q; }
          eid[q] = ex;
          ord[q] = j;
        }
        float acc = 0.0f;
        for (int q = 0; q < p.k; ++q) {
          const int j = ord[q];
          const int64_t pos = p.inv[static_cast<int64_t>(t) * p.k + j];
          acc = __fadd_rn(acc, __fmul_rn(p.topk_w[static_cast<int64_t>(t) * p.k + j],
                                         __ldcg(p.y_out + pos * p.rows_total + r)));
        }
        p.combine_out[static_cast<int64_t>(t) * p.rows_total + r] = f32_to_bf16_bits_rn(acc);
      }
      if (threadIdx.x == 0) p.tickets[blockIdx.x] = 0u;
    }
  }
}

size_t smem_bytes(int K, int nt) {
  return static_cast<size_t>(16) * (K / 2) + static_cast<size_t>(16) * (K / 32) * sizeof(float) +
         static_cast<size_t>(kWarps - 1) * nt * 4 * 32 * sizeof(float) + 16;
}

}  // namespace

cudaError_t launch_expert_mma(const uint8_t* blocks, const uint8_t* scales, const float* bias,
                              int rows_total, int K, const uint16_t* act, const int32_t* act_row,
                              const int32_t* offsets, const int32_t* active,
                              const int32_t* n_active, int max_active, float s_in, int mode, int I,
                              float s_mid, uint16_t* act_out, float* y_out, unsigned* amax_bits,
                              int max_tokens_per_expert, int* err, const CombineArgs* combine,
                              cudaStream_t st) {
  ExpertGemmArgs a{blocks, scales, bias, rows_total, K, act, act_row, offsets, active, n_active,
                   s_in, mode, I, s_mid, act_out, y_out, amax_bits, err,
                   combine ? combine->out : nullptr, combine ? combine->topk_idx : nullptr,
                   combine ? combine->topk_w : nullptr, combine ? combine->inv : nullptr,
                   combine ? combine->tickets : nullptr, combine ? combine->T : 0, combine ? combine->k : 0};
  const int groups = mode == 0 ? I / 8 : rows_total / 16;
  dim3 grid(static_cast<unsigned>(groups), static_cast<unsigned>(max_active));
  // one n-tile (8 tokens) per pass for up to 8 routed tokens, else two per pass; a group's
  // weights stay in shared memory across passes
  const int ntc = max_tokens_per_expert <= 8 ? 1 : 2;
  const size_t smem = smem_bytes(K, ntc);
  if (ntc == 1)
    expert_mma_kernel<1><<<grid, kWarps * 32, smem, st>>>(a);
  else
    expert_mma_kernel<2><<<grid, kWarps * 32, smem, st>>>(a);
  return cudaGetLastError();
}

cudaError_t expert_mma_set_smem_limits(int max_K) {
  const int smem = static_cast<int>(smem_bytes(max_K, 2));
  cudaError_t e = cudaSuccess;
  if (smem > 48 * 1024) {
    if ((e = cudaFuncSetAttribute(expert_mma_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem))) return e;
    if ((e = cudaFuncSetAttribute(expert_mma_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem))) return e;
  }
  return e;
}

}  // namespace mxmoe
