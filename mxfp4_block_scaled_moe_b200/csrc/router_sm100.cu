// Router GEMM on the 5th-generation tensor cores: logits = x · Wrᵀ + br (bf16 operands,
// fp32 accumulation; the bias is added to the first K range's partial).
//
// Pages: "openai/gpt-oss-120b" config.json (the router stays in bf16: modules_to_not_convert)
// and Model Details (128 experts, top-4); "amd/gpt-oss-20b-MoE-Quant-W-MXFP4-A-FP8-KV-FP8"
// Quantization recipe (router kept in full precision).
//
// One CTA per (128 tokens, one of S contiguous K ranges), all experts at once; S (1..4)
// brings the grid near one CTA per SM without reading any byte twice, and the top-k kernel
// adds the S partial logits in range order. tcgen05.mma.cta_group::1.kind::f16 with
// M = 128 tokens, N = E rounded up to 16 (<= 256), K = 16 per instruction, operands staged by
// TMA with 128-byte swizzle (64 bf16 = 128 bytes of K per stage), accumulators in tensor
// memory. Roles (192 threads): warp 0 TMA producer, warp 1 tensor-memory owner and MMA
// issuer, warps 2-5 epilogue (warp w reads tensor-memory lanes 32*(w%4) .. +31, one token
// per lane, 32 columns per wait). The top-k softmax stays a separate warp-per-token kernel:
// selecting in this epilogue (one thread per token) measured slower than that kernel.
// Every mbarrier wait is bounded: on expiry the kernel flags MXMOE_ETIMEOUT, lets in-flight
// copies land, frees its tensor memory and returns.
#include <cuda.h>

#include <atomic>

#include "common.cuh"
#include "launchers.h"
#include "tc_common.cuh"

namespace mxmoe {
namespace rt {

using namespace tc;

constexpr int BM = 128;              // tokens per CTA (MMA M)
constexpr int BK = 64;               // bf16 values of K per stage (128 bytes per row)
constexpr int kThreads = 192;        // warp 0 TMA, 1 MMA, 2-5 epilogue
constexpr int kMaxStages = 8;
constexpr int kTmemCols = 256;
constexpr int kAStage = BM * BK * 2;  // 16 KB
constexpr int kSmemBudget = 200 * 1024;

// Instruction descriptor, kind::f16: D = F32 (bit 4), A = B = BF16 (bits 7-9, 10-12 = 1),
// both K-major, N/8 at bits 17..22, M/16 at bits 24..28.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void tc_mma_bf16(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tc_wait_ld32(uint32_t (&a)[8], uint32_t (&b)[8], uint32_t (&c)[8], uint32_t (&d)[8]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;\n"
               : "+r"(a[0]), "+r"(a[1]), "+r"(a[2]), "+r"(a[3]), "+r"(a[4]), "+r"(a[5]), "+r"(a[6]), "+r"(a[7]),
                 "+r"(b[0]), "+r"(b[1]), "+r"(b[2]), "+r"(b[3]), "+r"(b[4]), "+r"(b[5]), "+r"(b[6]), "+r"(b[7]),
                 "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3]), "+r"(c[4]), "+r"(c[5]), "+r"(c[6]), "+r"(c[7]),
                 "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3]), "+r"(d[4]), "+r"(d[5]), "+r"(d[6]), "+r"(d[7])
               :
               : "memory");
}

__global__ void __launch_bounds__(kThreads, 1)
router_tc_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
                 const uint16_t* __restrict__ br, int T, int H, int E, int NP, int stages, int stage_bytes,
                 float* __restrict__ logits0, float* __restrict__ logits_rest, int* __restrict__ err) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + stages * stage_bytes);
  uint64_t* empty = full + kMaxStages;
  uint64_t* acc_full = empty + kMaxStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(acc_full + 1);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acc_full + 1) + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * BM;
  // this CTA's K range (stages k_lo .. k_lo + nk - 1) and its partial of the logits
  const int nk_all = H / BK, S = static_cast<int>(gridDim.y), ks = static_cast<int>(blockIdx.y);
  const int k_lo = ks * nk_all / S;
  const int nk = (ks + 1) * nk_all / S - k_lo;
  float* __restrict__ logits =
      ks == 0 ? logits0 : logits_rest + static_cast<int64_t>(ks - 1) * static_cast<int64_t>(T) * E;
  if (ks != 0) br = nullptr;

  if (threadIdx.x == 0) {
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&map_x)) : "memory");
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&map_w)) : "memory");
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
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
  auto sA = [&](int s) { return smem + s * stage_bytes; };
  auto sB = [&](int s) { return smem + s * stage_bytes + kAStage; };

  if (warp == 0) {
    // ------------------------------------------------------------------ producer ---
    if (lane == 0) {
      const uint32_t tx = static_cast<uint32_t>(kAStage + NP * BK * 2);
      for (int kt = 0; kt < nk; ++kt) {
        const int s = kt % stages;
        const uint32_t ph = (kt / stages) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, err)) break;
        mbar_arrive_expect_tx(&full[s], tx);
        tma_load_2d(sA(s), &map_x, &full[s], (k_lo + kt) * BK, m0);
        tma_load_2d(sB(s), &map_w, &full[s], (k_lo + kt) * BK, 0);
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------------- MMA ---
    const uint32_t id = idesc_bf16(BM, NP);
    bool ok = true;
    for (int kt = 0; kt < nk; ++kt) {
      const int s = kt % stages;
      if (!mbar_wait(&full[s], (kt / stages) & 1, abort_flag, err)) { ok = false; break; }
      tc_fence_after();
      if (lane == 0) {
        const uint32_t a0 = smem_u32(sA(s)), b0 = smem_u32(sB(s));
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          tc_mma_bf16(tmem, smem_desc(a0 + 32 * kk, 16, 1024, 2), smem_desc(b0 + 32 * kk, 16, 1024, 2), id,
                      (kt > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&empty[s]);
      }
      __syncwarp();
    }
    if (ok && lane == 0) tc_commit(acc_full);
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue ---
    const int q = warp & 3;
    const int row = m0 + 32 * q + lane;
    const bool valid = row < T;
    if (mbar_wait(acc_full, 0, abort_flag, err)) {
      tc_fence_after();
      const uint32_t tbase = tmem + (static_cast<uint32_t>(32 * q) << 16);
      for (int c0 = 0; c0 < E; c0 += 32) {   // E % 8 == 0; NP >= E columns hold results
        uint32_t r[4][8];
        tc_ld_32x32b_x8(tbase + c0, r[0]);
        tc_ld_32x32b_x8(tbase + c0 + 8, r[1]);
        tc_ld_32x32b_x8(tbase + c0 + 16, r[2]);
        tc_ld_32x32b_x8(tbase + c0 + 24, r[3]);
        tc_wait_ld32(r[0], r[1], r[2], r[3]);
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int c = c0 + 8 * g;
          if (c >= E || !valid) continue;
          float v[8];
#pragma unroll
          for (int i = 0; i < 8; ++i)
            v[i] = br ? __uint_as_float(r[g][i]) + bf16_bits_to_f32(br[c + i]) : __uint_as_float(r[g][i]);
          float4* dst = reinterpret_cast<float4*>(logits + static_cast<int64_t>(row) * E + c);
          dst[0] = make_float4(v[0], v[1], v[2], v[3]);
          dst[1] = make_float4(v[4], v[5], v[6], v[7]);
        }
      }
    }
  }

  // ---------------------------------------------------------------------- teardown ---
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

}  // namespace rt

namespace {

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled rt_encoder() {
  static EncodeTiled fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiled>(p);
  }
  return fn;
}

// 2-D bf16 map over rows x H, box of 64 values x box_rows rows, 128-byte swizzle; rows
// past the tensor read as zeros.
bool rt_encode(CUtensorMap* m, const void* base, int64_t rows, int H, int box_rows) {
  EncodeTiled fn = rt_encoder();
  if (!fn) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(H) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(rt::BK), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int rt_np(int E) { return (E + 15) & ~15; }
int rt_stage_bytes(int E) { return rt::kAStage + rt_np(E) * rt::BK * 2; }
int rt_stages(int E) { return std::min(rt::kMaxStages, rt::kSmemBudget / rt_stage_bytes(E)); }
size_t rt_smem(int E) { return 1024 + static_cast<size_t>(rt_stages(E)) * rt_stage_bytes(E) + (2 * rt::kMaxStages + 2) * 8 + 16; }
constexpr size_t kRtSmemMax = 1024 + rt::kSmemBudget + (2 * rt::kMaxStages + 2) * 8 + 16;   // any E

}  // namespace

int router_tc_ksplit(int T, int H, int sms) {
  const int tiles = static_cast<int>(cdiv(T, rt::BM));
  const int s = std::max(1, std::min(4, sms / std::max(tiles, 1)));
  return std::min(s, H / rt::BK);
}

bool router_tc_supported(int T, int H, int E, const void* x, const void* wr, const void* logits) {
  if (T <= 0 || H % rt::BK || H < rt::BK || E % 8 || E < 8 || E > 256) return false;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(wr) | reinterpret_cast<uintptr_t>(logits)) & 15u)
    return false;
  return rt_encoder() != nullptr;
}

cudaError_t launch_router_tc(const uint16_t* x, const uint16_t* wr, const uint16_t* br, int T, int H, int E,
                             int ksplit, float* logits, float* logits_rest, int* err, cudaStream_t st) {
  static std::atomic<uint64_t> smem_set{0};   // one bit per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  if (!(smem_set.load() & bit)) {
    e = cudaFuncSetAttribute(rt::router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kRtSmemMax));
    if (e != cudaSuccess) return e;
    smem_set.fetch_or(bit);
  }
  CUtensorMap mx, mw;
  if (!rt_encode(&mx, x, T, H, rt::BM) || !rt_encode(&mw, wr, E, H, rt_np(E))) return cudaErrorInvalidValue;
  if (ksplit < 1 || ksplit > H / rt::BK || (ksplit > 1 && !logits_rest)) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(cdiv(T, rt::BM)), static_cast<unsigned>(ksplit));
  rt::router_tc_kernel<<<grid, rt::kThreads, rt_smem(E), st>>>(mx, mw, br, T, H, E, rt_np(E), rt_stages(E),
                                                                rt_stage_bytes(E), logits, logits_rest, err);
  return cudaGetLastError();
}

}  // namespace mxmoe
