// Tensor-pipe rate probe (mxmoe_tc_rate_probe): the block-scaled MMA the prefill GEMMs
// issue -- tcgen05.mma kind::mxf8f6f4 with E4M3 A (M = 128) against E2M1 B, K = 32 per
// instruction, e8m0 block scales -- issued back to back by one thread per SM from operands
// that stay in shared memory, so nothing but the tensor pipe limits it. Its FLOP rate is
// the denominator the benchmark divides the prefill GEMMs' rate by: a measured ceiling
// for this instruction on this GPU at the clock it runs, instead of a nominal figure or a
// ratio applied to another instruction's measured rate.
//
// One CTA per SM (the shared-memory request keeps a second one off the SM). Per loop
// iteration: four MMAs covering 128 of K (the prefill GEMM's stage), optionally preceded
// by one tcgen05.cp.128x256b of B scale factors (the prefill's per-stage scale copy), all
// accumulating into one 128 x N fp32 accumulator. The operands are pseudo-random bytes
// (E4M3 A without NaN encodings; any byte is an E2M1 container) with unit scales, or zeros;
// zero operands switch fewer bits, draw less power and run ~12 % faster under the power
// cap, so the random ones give the rate GEMMs on real data can reach. The result is
// discarded. Every wait is bounded (MXMOE_ETIMEOUT on expiry).
#include "launchers.h"
#include "tc_common.cuh"

namespace mxmoe {

namespace {

using namespace tc;

constexpr int kProbeThreads = 128;
constexpr int kProbeA = 128 * 128;      // A: 128 rows x 128 bytes (e4m3, K = 128)
constexpr int kProbeB = 256 * 128;      // B: up to 256 rows x 128 bytes (e2m1 in byte containers)
constexpr int kProbeSf = 4096;          // one 128x256b copy source (128 lanes x 32 bytes)
constexpr int kProbeSmem = 120 * 1024;  // more than half the SM's shared memory: one CTA per SM
constexpr int kProbeTmemCols = 512;
constexpr int kProbeSfaCol = 256;       // A scales (8 columns)
constexpr int kProbeSfbCol = 264;       // B scales (8 columns: rows 0..127, then 128..255)

__global__ void __launch_bounds__(kProbeThreads, 1) tc_rate_kernel(int n, int with_copy, int random, int iters,
                                                                     int* err) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + kProbeA;
  uint8_t* sSF = sB + kProbeB;
  uint64_t* done = reinterpret_cast<uint64_t*>(sSF + kProbeSf);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  const int warp = threadIdx.x >> 5;

  for (int i = threadIdx.x; i < (kProbeA + kProbeB) / 4; i += blockDim.x) {
    uint32_t h = static_cast<uint32_t>(i) * 2654435761u;   // a multiplicative hash of the index
    h ^= h >> 15;
    h *= 2246822519u;
    h ^= h >> 13;
    // clearing bit 3 of every byte keeps the E4M3 exponent below 15: no NaN encodings
    reinterpret_cast<uint32_t*>(sA)[i] = random ? (h & 0xF7F7F7F7u) : 0u;
  }
  for (int i = threadIdx.x; i < kProbeSf / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(sSF)[i] = make_uint4(0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);   // 2^0
  fence_async_smem();
  if (threadIdx.x == 0) {
    mbar_init(done, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(tmem_holder)),
                 "r"(kProbeTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  if (threadIdx.x == 0) {
    const uint64_t sfd = smem_desc(smem_u32(sSF), 2048, 128, 0);
    tc_cp_128x256b(tmem + kProbeSfaCol, sfd);
    tc_cp_128x256b(tmem + kProbeSfbCol, sfd);
    const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
    const uint32_t id0 = idesc_mxf8f6f4(128, n);
    for (int it = 0; it < iters; ++it) {
      if (with_copy) tc_cp_128x256b(tmem + kProbeSfbCol, sfd);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t ad = smem_desc(a0 + 32 * kk, 16, 1024, 2);
        const uint64_t bd = smem_desc(b0 + 32 * kk, 16, 1024, 2);
        const uint32_t id = id0 | (static_cast<uint32_t>(kk) << 4) | (static_cast<uint32_t>(kk) << 29);
        const uint32_t sel = static_cast<uint32_t>(kk) << 30;
        tc_mma_mxf8f6f4(tmem, ad, bd, id, (tmem + kProbeSfaCol) | sel, (tmem + kProbeSfbCol) | sel,
                        (it > 0 || kk > 0) ? 1u : 0u);
      }
    }
    tc_commit(done);
    mbar_wait(done, 0, abort_flag, err);
  }
  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {   // the pipe may still be working on this CTA's tensor memory
    const long long t0 = clock64();
    while (clock64() - t0 < 200000) {
    }
  }
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kProbeTmemCols));
  }
}

}  // namespace

cudaError_t launch_tc_rate(int n, int with_copy, int random, int iters, int ctas, int* err, cudaStream_t st) {
  static bool ready = false;
  if (!ready) {
    cudaError_t e = cudaFuncSetAttribute(tc_rate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kProbeSmem);
    if (e != cudaSuccess) return e;
    ready = true;
  }
  tc_rate_kernel<<<ctas, kProbeThreads, kProbeSmem, st>>>(n, with_copy, random, iters, err);
  return cudaGetLastError();
}

}  // namespace mxmoe
