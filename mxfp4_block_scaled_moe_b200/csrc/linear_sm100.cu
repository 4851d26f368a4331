// FP8 E4M3 static per-tensor linear on the 5th-generation tensor cores:
//   out[t, n] = bf16( fp32(s * acc[t, n]) + b[n] ),  acc = sum_k xq[t, k] * wq[n, k],
//   s = fp32(s_x * s_w), xq = e4m3(fp32(x / s_x)) (cast by the library's FP8 cast kernel).
// Page "gpt-oss-120b-mxfp4-fp8attn-v2", Model Details and Quantization Recipe: the
// attention projections (Q, K, V, O) hold FP8 E4M3 weights with a static per-tensor
// weight scale, and their inputs are cast to FP8 E4M3 with a static per-tensor input
// scale.
//
// MMA: tcgen05.mma.cta_group::1.kind::f8f6f4 (no block scales: both per-tensor scales
// are applied once in the epilogue), A = xq (M = 128 token rows), B = wq (N = 256 weight
// rows), K = 32 per instruction, fp32 accumulators in tensor memory, two 256-column slots
// so one unit's epilogue overlaps the next unit's MMAs. Operands arrive by TMA with
// 128-byte swizzle, 128 values of K per stage, four stages (192 KB).
//
// Persistent schedule: one CTA per SM walks the units (m-tile, n-tile, K split). When the
// tiles alone would leave SMs idle (few tokens: decode), K is split; each split writes its
// fp32 partial and a second kernel adds the partials in split order, then applies the
// scale, the bias and the bf16 rounding (deterministic whichever CTA finishes first).
//
// Roles (320 threads): warp 0 TMA producer, warp 1 tensor-memory owner and MMA issuer (one
// thread), warps 2..9 epilogue (warp w reads tensor-memory lane quarter w % 4 and one of
// the two 128-column halves). Every mbarrier wait gives up after ~1 s: the kernel then
// records MXMOE_ETIMEOUT, lets in-flight copies land, frees its tensor memory and returns.
#include <algorithm>

#include <cuda.h>

#include "common.cuh"
#include "launchers.h"
#include "tc_common.cuh"
#include "tmap.h"

namespace mxmoe {
namespace lin {

using namespace tc;

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;
constexpr int kStages = 4;
constexpr int kAStage = BM * BK;   // 16 KB
constexpr int kBStage = BN * BK;   // 32 KB
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kTmemCols = 512;
constexpr int kSmemBytes = 1024 + kStages * (kAStage + kBStage) + 256;

// kind::f8f6f4 instruction descriptor: D = F32 (bit 4), A = B = E4M3 (format 0 at bits
// 7-9 and 10-12), both K-major, N/8 at bits 17..22, M/16 at bits 24..28.
__host__ __device__ constexpr uint32_t idesc_f8_e4m3(int M, int N) {
  return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void tc_mma_f8(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n}\n" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

struct Params {
  int T, K, N;
  int m_tiles, n_tiles, nk, ksplit, units;
  float s;              // fp32(s_x * s_w)
  const float* bias;    // (N) or null
  uint16_t* out;        // (T, N) bf16 bits
  float* part;          // ksplit > 1: (ksplit, T, N) fp32 partial accumulators
  int* err;
};

struct Unit {
  int mt, nt, ks, k0, k1;
};

__device__ __forceinline__ Unit unit_at(const Params& p, int u) {
  Unit w;
  w.ks = u % p.ksplit;
  const int t = u / p.ksplit;
  w.nt = t % p.n_tiles;
  w.mt = t / p.n_tiles;
  w.k0 = w.ks * p.nk / p.ksplit;
  w.k1 = (w.ks + 1) * p.nk / p.ksplit;
  return w;
}

__global__ void __launch_bounds__(kThreads, 1)
fp8_linear_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b, Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + kStages * kAStage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + kStages * kBStage);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* acc_full = bars + 2 * kStages;
  uint64_t* acc_empty = acc_full + 2;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(acc_empty + 2);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acc_empty + 2) + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&tmap_a)) : "memory");
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&tmap_b)) : "memory");
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);    // the producer's expect_tx
      mbar_init(&empty[s], 1);   // the MMA commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kEpiWarps);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(tmem_holder)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer -----
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
        const Unit w = unit_at(p, u);
        for (int kt = w.k0; kt < w.k1; ++kt) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[stage], kAStage + kBStage);
          tma_load_2d(sA + stage * kAStage, &tmap_a, &full[stage], kt * BK, w.mt * BM);
          tma_load_2d(sB + stage * kBStage, &tmap_b, &full[stage], kt * BK, w.nt * BN);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer -----
    int stage = 0;
    uint32_t phase = 0;
    int it = 0;
    const uint32_t idesc = idesc_f8_e4m3(BM, BN);
    bool ok = true;
    for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x, ++it) {
      const Unit w = unit_at(p, u);
      const int ab = it & 1;
      if (!mbar_wait(&acc_empty[ab], ((it >> 1) & 1) ^ 1, abort_flag, p.err)) break;
      tc_fence_after();
      const uint32_t dacc = tmem + ab * BN;
      for (int kt = w.k0; kt < w.k1; ++kt) {
        if (!mbar_wait(&full[stage], phase, abort_flag, p.err)) { ok = false; break; }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t a0 = smem_u32(sA + stage * kAStage), b0 = smem_u32(sB + stage * kBStage);
          const int nks = min(4, (p.K - kt * BK) / 32);   // K % 32 == 0: the last stage may hold fewer steps
          for (int kk = 0; kk < nks; ++kk)
            tc_mma_f8(dacc, smem_desc(a0 + 32 * kk, 16, 1024, 2), smem_desc(b0 + 32 * kk, 16, 1024, 2), idesc,
                      (kt > w.k0 || kk > 0) ? 1u : 0u);
          tc_commit(&empty[stage]);
        }
        __syncwarp();
        if (++stage == kStages) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
      if (lane == 0) tc_commit(&acc_full[ab]);
      __syncwarp();
    }
  } else {
    // --------------------------------------------------------------- epilogue -----
    const int q = warp & 3;              // tensor-memory lane quarter of this warp
    const int half = (warp - 2) >> 2;    // columns [128 half, 128 half + 128)
    const int row = 32 * q + lane;
    int it = 0;
    for (int u = blockIdx.x; u < p.units; u += gridDim.x, ++it) {
      const Unit w = unit_at(p, u);
      const int ab = it & 1;
      if (!mbar_wait(&acc_full[ab], (it >> 1) & 1, abort_flag, p.err)) break;
      tc_fence_after();
      const uint32_t tbase = tmem + ab * BN + (static_cast<uint32_t>(32 * q) << 16);
      const int64_t t = static_cast<int64_t>(w.mt) * BM + row;
      const bool valid = t < p.T;
      for (int c0 = 128 * half; c0 < 128 * half + 128; c0 += 8) {
        uint32_t v[8];
        tc_ld_32x32b_x8(tbase + c0, v);
        const int n = w.nt * BN + c0;
        const bool live = n < p.N;       // N % 8 == 0: a group of 8 columns is wholly in or out
        float bb[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (live && p.bias && p.ksplit == 1) {
          const float4 b0 = __ldg(reinterpret_cast<const float4*>(p.bias + n));
          const float4 b1 = __ldg(reinterpret_cast<const float4*>(p.bias + n) + 1);
          bb[0] = b0.x; bb[1] = b0.y; bb[2] = b0.z; bb[3] = b0.w; bb[4] = b1.x; bb[5] = b1.y; bb[6] = b1.z; bb[7] = b1.w;
        }
        tc_wait_ld(v);
        if (valid && live && p.ksplit == 1) {
          uint32_t o[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float y0 = __fadd_rn(__fmul_rn(p.s, __uint_as_float(v[2 * i])), bb[2 * i]);
            const float y1 = __fadd_rn(__fmul_rn(p.s, __uint_as_float(v[2 * i + 1])), bb[2 * i + 1]);
            o[i] = f32_to_bf16_bits_rn(y0) | (static_cast<uint32_t>(f32_to_bf16_bits_rn(y1)) << 16);
          }
          *reinterpret_cast<uint4*>(p.out + t * p.N + n) = make_uint4(o[0], o[1], o[2], o[3]);
        } else if (valid && live) {
          float4* dst = reinterpret_cast<float4*>(p.part + (static_cast<int64_t>(w.ks) * p.T + t) * p.N + n);
          dst[0] = make_float4(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2]), __uint_as_float(v[3]));
          dst[1] = make_float4(__uint_as_float(v[4]), __uint_as_float(v[5]), __uint_as_float(v[6]), __uint_as_float(v[7]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[ab]);
    }
  }

  // --------------------------------------------------------------------- teardown ---
  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {   // let copies already issued land before the CTA's shared memory goes
    const long long t0 = clock64();
    while (clock64() - t0 < 200000) {
    }
  }
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTmemCols));
  }
}

// The split-K finish: out = bf16( fp32(s * sum of the partials in split order) + b ).
__global__ void __launch_bounds__(256) fp8_linear_reduce_kernel(const float* __restrict__ part, int ksplit,
                                                                 int64_t TN, int N, float s,
                                                                 const float* __restrict__ bias,
                                                                 uint16_t* __restrict__ out) {
  const int64_t n4 = TN / 4;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 a = __ldcs(reinterpret_cast<const float4*>(part) + i);
    for (int k = 1; k < ksplit; ++k) {
      const float4 b = __ldcs(reinterpret_cast<const float4*>(part + k * TN) + i);
      a.x = __fadd_rn(a.x, b.x); a.y = __fadd_rn(a.y, b.y); a.z = __fadd_rn(a.z, b.z); a.w = __fadd_rn(a.w, b.w);
    }
    const int n = static_cast<int>((4 * i) % N);
    float4 bb = make_float4(0.f, 0.f, 0.f, 0.f);
    if (bias) bb = __ldg(reinterpret_cast<const float4*>(bias + n));
    const float y0 = __fadd_rn(__fmul_rn(s, a.x), bb.x), y1 = __fadd_rn(__fmul_rn(s, a.y), bb.y);
    const float y2 = __fadd_rn(__fmul_rn(s, a.z), bb.z), y3 = __fadd_rn(__fmul_rn(s, a.w), bb.w);
    reinterpret_cast<uint2*>(out)[i] =
        make_uint2(f32_to_bf16_bits_rn(y0) | (static_cast<uint32_t>(f32_to_bf16_bits_rn(y1)) << 16),
                   f32_to_bf16_bits_rn(y2) | (static_cast<uint32_t>(f32_to_bf16_bits_rn(y3)) << 16));
  }
}

}  // namespace lin

namespace {

// (rows, K) bytes, K-major, box (BK, box_rows), 128-byte swizzle, zero fill outside
bool encode_rows(CUtensorMap* m, const void* base, int64_t rows, int64_t K, uint32_t box_rows) {
  const uint64_t dims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(rows > 0 ? rows : 1)};
  const uint64_t strides[1] = {static_cast<uint64_t>(K)};
  const uint32_t box[2] = {static_cast<uint32_t>(lin::BK), box_rows};
  return tmap_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base, dims, strides, box);
}

constexpr size_t kLinPartBudget = 64u << 20;   // bytes of split-K partials at most

}  // namespace

int fp8_linear_ksplit(int T, int K, int N, int sms) {
  const int64_t tiles = static_cast<int64_t>((T + lin::BM - 1) / lin::BM) * ((N + lin::BN - 1) / lin::BN);
  const int nk = (K + lin::BK - 1) / lin::BK;
  if (tiles >= sms) return 1;
  int64_t s = sms / tiles;
  s = std::min<int64_t>(s, nk);
  const int64_t per = static_cast<int64_t>(T) * N * 4;
  if (per > 0) s = std::min<int64_t>(s, static_cast<int64_t>(kLinPartBudget / per));
  return static_cast<int>(std::max<int64_t>(1, s));
}

cudaError_t launch_fp8_linear(const uint8_t* xq, int T, int K, const uint8_t* wq, int N, float s, const float* bias,
                              uint16_t* out, float* part, int ksplit, int* err, int sms, cudaStream_t st) {
  static bool ready = false;
  if (!ready) {
    cudaError_t e = cudaFuncSetAttribute(lin::fp8_linear_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         lin::kSmemBytes);
    if (e != cudaSuccess) return e;
    ready = true;
  }
  CUtensorMap ma, mb;
  if (!encode_rows(&ma, xq, T, K, lin::BM) || !encode_rows(&mb, wq, N, K, lin::BN)) return cudaErrorInvalidValue;
  lin::Params p{};
  p.T = T;
  p.K = K;
  p.N = N;
  p.m_tiles = (T + lin::BM - 1) / lin::BM;
  p.n_tiles = (N + lin::BN - 1) / lin::BN;
  p.nk = (K + lin::BK - 1) / lin::BK;
  p.ksplit = ksplit;
  p.units = p.m_tiles * p.n_tiles * ksplit;
  p.s = s;
  p.bias = bias;
  p.out = out;
  p.part = part;
  p.err = err;
  const int grid = std::max(1, std::min(sms, p.units));
  lin::fp8_linear_kernel<<<grid, lin::kThreads, lin::kSmemBytes, st>>>(ma, mb, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || ksplit == 1) return e;
  const int64_t TN = static_cast<int64_t>(T) * N;
  const int64_t g = std::min<int64_t>(cdiv(TN / 4, 256), static_cast<int64_t>(sms) * 8);
  lin::fp8_linear_reduce_kernel<<<static_cast<unsigned>(std::max<int64_t>(g, 1)), 256, 0, st>>>(part, ksplit, TN, N,
                                                                                                s, bias, out);
  return cudaGetLastError();
}

bool fp8_linear_supported() { return tmap_available(); }

}  // namespace mxmoe
