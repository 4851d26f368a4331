// Routing kernels: router logits (GEMV for few tokens, mma.sync GEMM for many), top-k
// softmax, the deterministic token -> expert permutation, and the activation casts.
//
// Router: GPT-OSS top-k routing with the router kept in bf16 ("gpt-oss-120b-mxfp4-
// fp8attn-v2", config.json modules_to_not_convert; "xpuenabler/gpt-oss-15.5b-23E-nf4-
// GPU", Quantization recipe: router kept unquantized). Top-k ties go to the lower expert
// id; the softmax runs over the k selected logits.
// Permutation: the routed dispatch of "quantization_mxfp4", As GPT-OSS's native format:
// pairs (token, slot) grouped by expert, ascending token inside an expert.
#include <atomic>

#include "common.cuh"
#include "topk.cuh"

namespace mxmoe {

// ------------------------------------------------------------------ router GEMV -----
// One warp per (token, expert): 16-byte loads along H, fp32 FMA, fixed-order warp sum.
__global__ void __launch_bounds__(256) router_gemv_kernel(const uint16_t* __restrict__ x,
                                                           const uint16_t* __restrict__ wr,
                                                           const uint16_t* __restrict__ br,
                                                           int T, int H, int E,
                                                           float* __restrict__ logits) {
  const int lane = threadIdx.x & 31;
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (wid >= static_cast<int64_t>(T) * E) return;
  const int t = static_cast<int>(wid / E), e = static_cast<int>(wid % E);
  const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(t) * H);
  const uint4* wrow = reinterpret_cast<const uint4*>(wr + static_cast<int64_t>(e) * H);
  float acc = 0.0f;
  for (int c0 = lane; c0 < H / 8; c0 += 4 * 32) {
    uint4 a[4], b[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = c0 + 32 * u;
      if (c < H / 8) { a[u] = ld_nc_v4(xr + c); b[u] = ld_nc_v4(wrow + c); }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
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
  if (lane == 0) logits[wid] = br ? acc + bf16_bits_to_f32(br[e]) : acc;
}

// ------------------------------------------------------------------ router GEMM -----
// logits (T, E) = x (T, H) . Wr (E, H)^T with mma.sync m16n8k16 (bf16 in, fp32 acc).
// CTA tile 64 tokens x 64 experts, 4 warps as 2 x 2 (each 32 x 32), K in steps of 128
// staged by cp.async into padded shared rows (272-byte pitch: ldmatrix conflict-free).
// The work is small (2*T*H*E FLOP) and each K step ends in a CTA barrier, so the steps are
// wide: 23 of them at H = 2880 rather than 90.
namespace rg {
constexpr int BM = 64, BN = 64, BK = 128, PITCH = 136, STAGES = 3;  // pitch in bf16 elements
constexpr int kSmemBytes = STAGES * (BM + BN) * PITCH * 2;
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool pred) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  const int n = pred ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(n));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

__device__ __forceinline__ void ldmatrix_x4(uint32_t r[4], const void* smem) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(s));
}

__global__ void __launch_bounds__(128) router_gemm_kernel(const uint16_t* __restrict__ x,
                                                           const uint16_t* __restrict__ wr,
                                                           const uint16_t* __restrict__ br,
                                                           int T, int H, int E,
                                                           float* __restrict__ logits) {
  using namespace rg;
  extern __shared__ __align__(16) uint16_t rg_smem[];
  uint16_t (*sa)[BM * PITCH] = reinterpret_cast<uint16_t (*)[BM * PITCH]>(rg_smem);
  uint16_t (*sb)[BN * PITCH] = reinterpret_cast<uint16_t (*)[BN * PITCH]>(rg_smem + STAGES * BM * PITCH);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m0 = blockIdx.x * BM, n0 = blockIdx.y * BN;
  const int wm = (warp >> 1) * 32, wn = (warp & 1) * 32;
  const int nk = (H + BK - 1) / BK;   // the last K step may be partial (H % 32 == 0)

  auto load_stage = [&](int stage, int kt) {
    // 64 rows x 256 bytes per operand = 1024 chunks of 16 B each; 128 threads x 8
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int c = tid + i * 128, row = c >> 4, col = (c & 15) * 8;
      const int gm = m0 + row, gn = n0 + row;
      const int gmc = gm < T ? gm : T - 1, gnc = gn < E ? gn : E - 1;
      const int kc = kt * BK + col;
      const bool kin = kc < H;   // columns past H read as zeros
      cp_async16(&sa[stage][row * PITCH + col], x + static_cast<int64_t>(gmc) * H + (kin ? kc : 0), gm < T && kin);
      cp_async16(&sb[stage][row * PITCH + col], wr + static_cast<int64_t>(gnc) * H + (kin ? kc : 0), gn < E && kin);
    }
  };

  float acc[2][4][4];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int r = 0; r < 4; ++r) acc[i][j][r] = 0.0f;

#pragma unroll
  for (int s = 0; s < STAGES - 1; ++s) {
    if (s < nk) load_stage(s, s);
    cp_async_commit();
  }
  for (int kt = 0; kt < nk; ++kt) {
    cp_async_wait<STAGES - 2>();
    __syncthreads();
    const int nxt = kt + STAGES - 1;
    if (nxt < nk) load_stage(nxt % STAGES, nxt);
    cp_async_commit();
    const int st = kt % STAGES;
#pragma unroll
    for (int ks = 0; ks < BK; ks += 16) {
      uint32_t af[2][4], bfr[4][2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        // x4: matrices (rows 0-7, k 0-7), (rows 8-15, k 0-7), (rows 0-7, k 8-15), (rows 8-15, k 8-15)
        const int r = wm + i * 16 + (lane & 15), c = ks + (lane >> 4) * 8;
        ldmatrix_x4(af[i], &sa[st][r * PITCH + c]);
      }
#pragma unroll
      for (int j = 0; j < 4; j += 2) {
        // x4 over two n8 tiles: (n 0-7, k 0-7), (n 0-7, k 8-15), (n 8-15, k 0-7), (n 8-15, k 8-15)
        const int r = wn + j * 8 + (lane & 7) + ((lane >> 4) << 3), c = ks + ((lane >> 3) & 1) * 8;
        uint32_t t4[4];
        ldmatrix_x4(t4, &sb[st][r * PITCH + c]);
        bfr[j][0] = t4[0]; bfr[j][1] = t4[1]; bfr[j + 1][0] = t4[2]; bfr[j + 1][1] = t4[3];
      }
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) mma_bf16_16816(acc[i][j], af[i], bfr[j], acc[i][j]);
    }
  }
  cp_async_wait<0>();
  // epilogue: c0,c1 -> (row g, cols 2t, 2t+1); c2,c3 -> (row g+8, ...)
  const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int row = m0 + wm + i * 16 + g + (r >> 1) * 8;
        const int col = n0 + wn + j * 8 + 2 * t4 + (r & 1);
        if (row < T && col < E)
          logits[static_cast<int64_t>(row) * E + col] =
              br ? acc[i][j][r] + bf16_bits_to_f32(br[col]) : acc[i][j][r];
      }
}

// ----------------------------------------------------------------------- top-k -----
// topk_warp (csrc/topk.cuh): one warp per token.

// n_rest > 0: the router wrote its logits as 1 + n_rest partials over K ranges (rest:
// n_rest arrays of T*E after logits); a token's logits are their sum in range order,
// written back to logits before the selection.
__global__ void __launch_bounds__(256) topk_kernel(float* __restrict__ logits, const float* __restrict__ rest,
                                                    int n_rest, int T, int E, int k, int32_t* __restrict__ idx,
                                                    float* __restrict__ wts) {
  __shared__ float s_row[8][256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (t >= T) return;
  const float* row = logits + static_cast<int64_t>(t) * E;
  if (n_rest > 0) {
    float* rw = logits + static_cast<int64_t>(t) * E;
    if ((E & 3) == 0) {   // four consecutive logits per lane, 16-byte loads (rows are 16-byte aligned)
      for (int e = 4 * lane; e < E; e += 128) {
        float4 v = *reinterpret_cast<const float4*>(rw + e);
        for (int s = 0; s < n_rest; ++s) {
          const float4 u = *reinterpret_cast<const float4*>(rest + (static_cast<int64_t>(s) * T + t) * E + e);
          v.x += u.x; v.y += u.y; v.z += u.z; v.w += u.w;
        }
        *reinterpret_cast<float4*>(rw + e) = v;
        s_row[warp][e] = v.x; s_row[warp][e + 1] = v.y; s_row[warp][e + 2] = v.z; s_row[warp][e + 3] = v.w;
      }
    } else {
      for (int e = lane; e < E; e += 32) {
        float v = rw[e];
        for (int s = 0; s < n_rest; ++s) v += rest[(static_cast<int64_t>(s) * T + t) * E + e];
        rw[e] = v;
        s_row[warp][e] = v;
      }
    }
    __syncwarp();
    row = s_row[warp];
  }
  topk_warp(row, E, k, idx + static_cast<int64_t>(t) * k, wts + static_cast<int64_t>(t) * k);
}

// --------------------------------------------------------------------- permute -----
// Stable counting sort of the P = T*k pairs by expert, in two passes over chunks of
// `chunk` pairs (a multiple of kPermThreads, at most kPermMaxChunks chunks): (1) per-chunk
// histograms, (2) every CTA rebuilds the global offsets and its own start per expert from
// the histograms, then places its pairs in order. Within a sub-chunk of kPermThreads pairs
// the rank of a pair among equal experts is its rank in its warp (match_any) plus the
// counts of the same expert in lower warps. Small chunks keep many CTAs busy: at 16K
// pairs there are 32 CTAs and each places its pairs in one round.
constexpr int kPermThreads = 512;
constexpr int kPermMaxChunks = 128;

__host__ __device__ __forceinline__ int64_t permute_chunk_size(int64_t P) {
  const int64_t subs = cdiv(P, kPermThreads);
  return kPermThreads * (subs < kPermMaxChunks ? 1 : cdiv(subs, kPermMaxChunks));
}

__global__ void __launch_bounds__(kPermThreads) permute_count_kernel(
    const int32_t* __restrict__ idx, int64_t P, int E, int32_t* __restrict__ counts, int* __restrict__ err) {
  __shared__ int hist[256];
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int64_t chunk = permute_chunk_size(P);
  const int64_t lo = static_cast<int64_t>(blockIdx.x) * chunk;
  const int64_t hi = min(P, lo + chunk);
  for (int64_t p = lo + threadIdx.x; p < hi; p += blockDim.x) {
    const int e = idx[p];
    if (e >= 0 && e < E) atomicAdd(&hist[e], 1);
    else set_device_error(err, MXMOE_EDEVICE);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) counts[static_cast<int64_t>(blockIdx.x) * E + e] = hist[e];
}

struct PermuteSmem {
  int base[256];
  int total[256];
  int wc[kPermThreads / 32][256];
  int scan_tmp[256];
};

// The scatter pass, run by one CTA of kPermThreads threads for chunk `cta` (counts ==
// nullptr: single-CTA mode, the CTA builds its own histogram of all P pairs first).
__device__ void permute_scatter_body(
    PermuteSmem& sm, int cta, const int32_t* __restrict__ idx, int64_t P, int E, int k,
    const int32_t* __restrict__ counts, int32_t* __restrict__ offsets, int32_t* __restrict__ perm_token,
    int32_t* __restrict__ perm_slot, int32_t* __restrict__ inv, int32_t* __restrict__ active,
    int32_t* __restrict__ n_active, int* __restrict__ err) {
  int* base = sm.base;
  int* total = sm.total;
  int (*wc)[256] = sm.wc;
  int* scan_tmp = sm.scan_tmp;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t chunk = permute_chunk_size(P);
  const int nchunks = static_cast<int>(cdiv(P, chunk));
  const int64_t lo = static_cast<int64_t>(cta) * chunk;
  const int64_t hi = min(P, lo + chunk);

  if (counts == nullptr) {
    for (int e = tid; e < E; e += blockDim.x) total[e] = 0;
    __syncthreads();
    for (int64_t p = tid; p < P; p += blockDim.x) {
      const int e = __ldcg(idx + p);   // may have been written by other CTAs of this launch
      if (e >= 0 && e < E) atomicAdd(&total[e], 1);
      else set_device_error(err, MXMOE_EDEVICE);
    }
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x) base[e] = 0;
  } else {
    for (int e = tid; e < E; e += blockDim.x) {
      int before = 0, all = 0;
      for (int c = 0; c < nchunks; ++c) {
        const int v = counts[static_cast<int64_t>(c) * E + e];
        if (c < cta) before += v;
        all += v;
      }
      total[e] = all;
      base[e] = before;
    }
  }
  __syncthreads();
  // exclusive scan of total[] over experts (E <= 256) by one warp, in expert order
  if (warp == 0) {
    int carry = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int e = e0 + lane;
      const int v = e < E ? total[e] : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
      }
      if (e < E) scan_tmp[e] = carry + incl - v;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (cta == 0 && lane == 0) offsets[E] = carry;
  }
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) {
    base[e] += scan_tmp[e];
    if (cta == 0) offsets[e] = scan_tmp[e];
  }
  if (cta == 0 && tid == 0) {
    int n = 0;
    for (int e = 0; e < E; ++e)
      if (total[e] > 0) active[n++] = e;
    *n_active = n;
  }
  __syncthreads();

  const int64_t my_lo = counts == nullptr ? 0 : lo;
  const int64_t my_hi = counts == nullptr ? P : hi;
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int64_t sub = my_lo; sub < my_hi; sub += blockDim.x) {
    const int64_t p = sub + tid;
    int e = p < my_hi ? __ldcg(idx + p) : -1;
    if (e >= E) e = -1;
    for (int i = tid; i < (kPermThreads / 32) * 256; i += blockDim.x) (&wc[0][0])[i] = 0;  // all slots
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & lt_mask);
    __syncthreads();
    if (e >= 0 && rank == 0) wc[warp][e] = __popc(peers);
    __syncthreads();
    // exclusive prefix over warps, per expert; total of this sub-chunk into scan_tmp
    for (int ee = tid; ee < E; ee += blockDim.x) {
      int run = 0;
      for (int w = 0; w < kPermThreads / 32; ++w) {
        const int c = wc[w][ee];
        wc[w][ee] = run;
        run += c;
      }
      scan_tmp[ee] = run;
    }
    __syncthreads();
    if (e >= 0) {
      const int pos = base[e] + wc[warp][e] + rank;
      perm_token[pos] = static_cast<int32_t>(p / k);
      perm_slot[pos] = static_cast<int32_t>(p % k);
      if (inv) inv[p] = pos;
    }
    __syncthreads();
    for (int ee = tid; ee < E; ee += blockDim.x) base[ee] += scan_tmp[ee];
    __syncthreads();
  }
}

__global__ void __launch_bounds__(kPermThreads) permute_scatter_kernel(
    const int32_t* __restrict__ idx, int64_t P, int E, int k, const int32_t* __restrict__ counts,
    int32_t* __restrict__ offsets, int32_t* __restrict__ perm_token,
    int32_t* __restrict__ perm_slot, int32_t* __restrict__ inv, int32_t* __restrict__ active,
    int32_t* __restrict__ n_active, int* __restrict__ err) {
  __shared__ PermuteSmem sm;
  permute_scatter_body(sm, blockIdx.x, idx, P, E, k, counts, offsets, perm_token, perm_slot, inv, active,
                       n_active, err);
}

// ----------------------------------------------------------- fused small-batch routing -
// One launch for the routing of a small batch: every warp computes one (token, expert)
// logit (the router GEMV's arithmetic). The CTA that completes a token's logits last (a
// per-token arrival counter) runs that token's top-k softmax, so the tokens' top-k run in
// parallel across CTAs; the CTA that finishes last overall (a second counter) runs the
// single-CTA permutation. Every counter is reset by the CTA that consumed it. Saves two
// launches on the latency-bound decode path.
constexpr int kSmallT = 64, kSmallE = 256;
constexpr int kSmallPairs = 64;   // routed pairs placed by the direct count in route_small_kernel

__global__ void __launch_bounds__(kPermThreads) route_small_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ wr, const uint16_t* __restrict__ br,
    int T, int H, int E, int k, float* __restrict__ logits, unsigned* __restrict__ ticket,
    unsigned* __restrict__ tok_tickets, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
    int32_t* __restrict__ offsets, int32_t* __restrict__ perm_token, int32_t* __restrict__ perm_slot,
    int32_t* __restrict__ inv, int32_t* __restrict__ active, int32_t* __restrict__ n_active,
    int* __restrict__ err) {
  __shared__ PermuteSmem sm;
  __shared__ unsigned s_last;
  __shared__ int s_tok[kPermThreads / 32], s_ntok;
  // the decode token split may launch now and load its rows; it waits for this kernel
  // before reading any routing output
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int64_t wid = static_cast<int64_t>(blockIdx.x) * nwarps + warp;
  if (wid < static_cast<int64_t>(T) * E) {
    const int t = static_cast<int>(wid / E), e = static_cast<int>(wid % E);
    const float acc = router_logit_warp(x + static_cast<int64_t>(t) * H, wr + static_cast<int64_t>(e) * H, H);
    if (lane == 0) logits[wid] = br ? acc + bf16_bits_to_f32(br[e]) : acc;
  }
  // tokens whose logits this CTA helped compute: the last of a token's CTAs runs its top-k
  __threadfence();
  if (threadIdx.x == 0) s_ntok = 0;
  __syncthreads();
  {
    const int64_t w_lo = static_cast<int64_t>(blockIdx.x) * nwarps;
    const int64_t w_hi = min(static_cast<int64_t>(T) * E, w_lo + nwarps);   // > w_lo: the grid covers T*E warps
    const int t_lo = static_cast<int>(w_lo / E), t_hi = static_cast<int>((w_hi - 1) / E);
    if (static_cast<int>(threadIdx.x) <= t_hi - t_lo) {
      const int t = t_lo + static_cast<int>(threadIdx.x);
      const int64_t c_first = static_cast<int64_t>(t) * E / nwarps;
      const int64_t c_last = (static_cast<int64_t>(t) * E + E - 1) / nwarps;
      const unsigned need = static_cast<unsigned>(c_last - c_first + 1);
      if (atomicAdd(&tok_tickets[t], 1u) == need - 1u) {
        tok_tickets[t] = 0u;   // every CTA of the token has arrived
        s_tok[atomicAdd(&s_ntok, 1)] = t;
      }
    }
  }
  __syncthreads();
  __threadfence();
  for (int i = warp; i < s_ntok; i += nwarps) {
    const int t = s_tok[i];
    // the other CTAs' logits: read through L2
    float lv[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane + 32 * j;
      lv[j] = e < E ? __ldcg(logits + static_cast<int64_t>(t) * E + e) : 0.0f;
    }
    __shared__ float s_row[kPermThreads / 32][256];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane + 32 * j;
      if (e < E) s_row[warp][e] = lv[j];
    }
    __syncwarp();
    topk_warp(s_row[warp], E, k, topk_idx + static_cast<int64_t>(t) * k, topk_w + static_cast<int64_t>(t) * k);
    __syncwarp();
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(ticket, 1u) == gridDim.x - 1u;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  __syncthreads();   // the CTA's global writes of topk_idx are visible to all its threads
  const int P = T * k;
  if (P <= kSmallPairs) {
    // A handful of pairs (a decode step): each pair's position is the number of valid pairs
    // with a smaller expert id plus the earlier valid pairs with the same one -- the order of
    // the general scatter, without its passes and barriers.
    int* s_e = sm.scan_tmp;   // P <= 256 expert ids
    int* s_off = &sm.wc[0][0];   // E + 1 <= 257 offsets
    for (int q = threadIdx.x; q < P; q += blockDim.x) {
      int e = __ldcg(topk_idx + q);
      if (e < 0 || e >= E) {
        set_device_error(err, MXMOE_EDEVICE);
        e = -1;
      }
      s_e[q] = e;
    }
    __syncthreads();
    for (int q = threadIdx.x; q < P; q += blockDim.x) {
      const int e = s_e[q];
      if (e < 0) continue;
      int pos = 0;
      for (int r = 0; r < P; ++r) {
        const int f = s_e[r];
        pos += (f >= 0 && (f < e || (f == e && r < q))) ? 1 : 0;
      }
      perm_token[pos] = q / k;
      perm_slot[pos] = q % k;
      inv[q] = pos;
    }
    for (int e = threadIdx.x; e <= E; e += blockDim.x) {
      int c = 0;
      for (int r = 0; r < P; ++r) c += (s_e[r] >= 0 && s_e[r] < e) ? 1 : 0;
      s_off[e] = c;
      offsets[e] = c;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int n = 0;
      for (int e = 0; e < E; ++e)
        if (s_off[e + 1] > s_off[e]) active[n++] = e;
      *n_active = n;
      *ticket = 0u;
    }
    return;
  }
  permute_scatter_body(sm, 0, topk_idx, static_cast<int64_t>(T) * k, E, k, nullptr, offsets, perm_token,
                       perm_slot, inv, active, n_active, err);
  if (threadIdx.x == 0) *ticket = 0u;
}

bool route_small_supported(int T, int E, int k) {
  return T <= kSmallT && E <= kSmallE && static_cast<int64_t>(T) * k <= 4096;   // one CTA places at most 4096 pairs
}

cudaError_t launch_route_small(const uint16_t* x, const uint16_t* wr, const uint16_t* br, int T, int H, int E,
                               int k, float* logits, unsigned* ticket, unsigned* tok_tickets, int32_t* topk_idx,
                               float* topk_w, int32_t* offsets, int32_t* perm_token, int32_t* perm_slot, int32_t* inv,
                               int32_t* active, int32_t* n_active, int* err, cudaStream_t st) {
  const int64_t warps = static_cast<int64_t>(T) * E;
  const unsigned grid = static_cast<unsigned>(cdiv(warps, kPermThreads / 32));
  route_small_kernel<<<grid, kPermThreads, 0, st>>>(x, wr, br, T, H, E, k, logits, ticket, tok_tickets, topk_idx, topk_w,
                                                    offsets, perm_token, perm_slot, inv, active, n_active, err);
  return cudaGetLastError();
}

// ------------------------------------------------------------ activation casts -----
// q = e4m3(fp32(x / s)); x bf16 (n), n % 8 == 0 not required.
__global__ void __launch_bounds__(256) fp8_quant_kernel(const uint16_t* __restrict__ x, int64_t n,
                                                         float s, uint8_t* __restrict__ q) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride)
    q[i] = act_quant_e4m3(bf16_bits_to_f32(x[i]), s);
}

// The A-FP8 input of the register-dequant path: xq[i] = bf16 bits of e4m3(x[i] / s),
// exact (every e4m3 value is a bf16 value). Vectorized by 8 (H % 32 == 0).
__global__ void __launch_bounds__(256) fp8_quant_as_bf16_kernel(const uint4* __restrict__ x,
                                                                 int64_t n8, float s,
                                                                 uint4* __restrict__ xq) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8; i += stride) {
    const uint4 v = x[i];
    const uint32_t in[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float lo = e4m3_to_f32(act_quant_e4m3(__uint_as_float(in[j] << 16), s));
      const float hi = e4m3_to_f32(act_quant_e4m3(__uint_as_float(in[j] & 0xFFFF0000u), s));
      o[j] = (__float_as_uint(lo) >> 16) | (__float_as_uint(hi) & 0xFFFF0000u);
    }
    xq[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// The A-FP8 cast fused with the scatter into expert-grouped order (one pass over x, one cast
// per token): a1[inv[t*k + j], :] = e4m3(fp32(x[t, :] / s)) for each of token t's k routed
// slots. One warp per token, eight values per lane and chunk, four chunks in flight; a slot
// whose expert id or position is out of range is skipped (the permute has flagged it).
__global__ void __launch_bounds__(256) quant_scatter_fp8_kernel(const uint16_t* __restrict__ x,
                                                                 const int32_t* __restrict__ topk_idx,
                                                                 const int32_t* __restrict__ inv, int T,
                                                                 int k, int E, int64_t P, int H, float s,
                                                                 uint8_t* __restrict__ a1) {
  griddep_launch_dependents();   // the gate_up GEMM may start its setup and weight stream
  const int lane = threadIdx.x & 31;
  const int nw = static_cast<int>((static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5);
  const int n8 = H / 8;
  for (int t = static_cast<int>((static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5); t < T;
       t += nw) {
    int my_pos = -1;
    if (lane < k) {
      const int64_t p = static_cast<int64_t>(t) * k + lane;
      const int e = topk_idx[p];
      const int pos = inv[p];
      if (e >= 0 && e < E && pos >= 0 && pos < P) my_pos = pos;
    }
    const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(t) * H);
    for (int c0 = lane; c0 < n8; c0 += 4 * 32) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (c0 + 32 * u < n8) v[u] = ld_nc_v4(src + c0 + 32 * u);   // four chunks in flight
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (c0 + 32 * u >= n8) break;
        const uint32_t in[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
        uint32_t q[2] = {0u, 0u};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t lo = act_quant_e4m3(__uint_as_float(in[j] << 16), s);
          const uint32_t hi = act_quant_e4m3(__uint_as_float(in[j] & 0xFFFF0000u), s);
          q[j >> 1] |= (lo | (hi << 8)) << (16 * (j & 1));
        }
        const uint2 qv = make_uint2(q[0], q[1]);
        for (int j = 0; j < k; ++j) {
          const int pos = __shfl_sync(0xffffffffu, my_pos, j);
          if (pos >= 0) reinterpret_cast<uint2*>(a1 + static_cast<int64_t>(pos) * H)[c0 + 32 * u] = qv;
        }
      }
    }
  }
}

// amax |x| over a bf16 tensor, folded into *amax_bits (float bits; |x| >= 0 orders as int)
__global__ void __launch_bounds__(256) amax_bf16_kernel(const uint16_t* __restrict__ x, int64_t n,
                                                         unsigned* __restrict__ amax_bits) {
  float m = 0.0f;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride)
    m = fmaxf(m, fabsf(bf16_bits_to_f32(x[i])));
  m = warp_max(m);
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, __float_as_uint(m));
}

__global__ void finalize_scales_kernel(const unsigned* __restrict__ amax_bits, float* __restrict__ out) {
  if (threadIdx.x < 2) out[threadIdx.x] = __fdiv_rn(__uint_as_float(amax_bits[threadIdx.x]), 448.0f);
}

// ------------------------------------------------------------------- launchers -----
cudaError_t launch_router(const uint16_t* x, const uint16_t* wr, const uint16_t* br, int T, int H,
                          int E, float* logits, cudaStream_t st) {
  if (T <= 32) {
    const int64_t warps = static_cast<int64_t>(T) * E;
    router_gemv_kernel<<<static_cast<unsigned>(cdiv(warps * 32, 256)), 256, 0, st>>>(x, wr, br, T, H, E, logits);
  } else {
    static std::atomic<uint64_t> smem_set{0};   // one bit per device
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = 1ull << (dev & 63);
    if (!(smem_set.load() & bit)) {
      e = cudaFuncSetAttribute(router_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, rg::kSmemBytes);
      if (e != cudaSuccess) return e;
      smem_set.fetch_or(bit);
    }
    dim3 grid(static_cast<unsigned>(cdiv(T, rg::BM)), static_cast<unsigned>(cdiv(E, rg::BN)));
    router_gemm_kernel<<<grid, 128, rg::kSmemBytes, st>>>(x, wr, br, T, H, E, logits);
  }
  return cudaGetLastError();
}

cudaError_t launch_topk(float* logits, const float* rest, int n_rest, int T, int E, int k, int32_t* idx, float* w,
                        cudaStream_t st) {
  if (n_rest > 0 && E > 256) return cudaErrorInvalidValue;
  topk_kernel<<<static_cast<unsigned>(cdiv(static_cast<int64_t>(T) * 32, 256)), 256, 0, st>>>(logits, rest, n_rest, T,
                                                                                             E, k, idx, w);
  return cudaGetLastError();
}

int permute_chunks(int64_t P) { return static_cast<int>(cdiv(P, permute_chunk_size(P))); }

// counts_ws: int32 scratch of permute_chunks(P) * E entries (unused for one chunk).
cudaError_t launch_permute(const int32_t* idx, int T, int E, int k, int32_t* counts_ws,
                           int32_t* offsets, int32_t* perm_token, int32_t* perm_slot,
                           int32_t* inv, int32_t* active, int32_t* n_active, int* err,
                           cudaStream_t st, int* launches) {
  const int64_t P = static_cast<int64_t>(T) * k;
  const int nc = permute_chunks(P);
  if (nc <= 1) {
    permute_scatter_kernel<<<1, kPermThreads, 0, st>>>(idx, P, E, k, nullptr, offsets, perm_token,
                                                       perm_slot, inv, active, n_active, err);
    *launches += 1;
  } else {
    permute_count_kernel<<<nc, kPermThreads, 0, st>>>(idx, P, E, counts_ws, err);
    permute_scatter_kernel<<<nc, kPermThreads, 0, st>>>(idx, P, E, k, counts_ws, offsets,
                                                        perm_token, perm_slot, inv, active, n_active,
                                                        err);
    *launches += 2;
  }
  return cudaGetLastError();
}

cudaError_t launch_fp8_quant(const uint16_t* x, int64_t n, float s, uint8_t* q, cudaStream_t st,
                             int sms) {
  const int64_t g = cdiv(n, 256);
  fp8_quant_kernel<<<static_cast<unsigned>(g < sms * 8 ? (g < 1 ? 1 : g) : sms * 8), 256, 0, st>>>(x, n, s, q);
  return cudaGetLastError();
}

cudaError_t launch_fp8_quant_as_bf16(const uint16_t* x, int64_t n, float s, uint16_t* xq,
                                     cudaStream_t st, int sms) {
  const int64_t n8 = n / 8;
  const int64_t g = cdiv(n8, 256);
  fp8_quant_as_bf16_kernel<<<static_cast<unsigned>(g < sms * 8 ? (g < 1 ? 1 : g) : sms * 8), 256, 0, st>>>(
      reinterpret_cast<const uint4*>(x), n8, s, reinterpret_cast<uint4*>(xq));
  return cudaGetLastError();
}

cudaError_t launch_quant_scatter_fp8(const uint16_t* x, const int32_t* topk_idx, const int32_t* inv, int T,
                                    int k, int E, int64_t P, int H, float s, uint8_t* a1, cudaStream_t st,
                                    int sms) {
  if (k > 32) return cudaErrorInvalidValue;
  const int64_t g = cdiv(static_cast<int64_t>(T) * 32, 256);
  quant_scatter_fp8_kernel<<<static_cast<unsigned>(g < sms * 16 ? (g < 1 ? 1 : g) : sms * 16), 256, 0, st>>>(
      x, topk_idx, inv, T, k, E, P, H, s, a1);
  return cudaGetLastError();
}

cudaError_t launch_amax_bf16(const uint16_t* x, int64_t n, unsigned* amax_bits, cudaStream_t st,
                             int sms) {
  const int64_t g = cdiv(n, 256);
  amax_bf16_kernel<<<static_cast<unsigned>(g < sms * 4 ? (g < 1 ? 1 : g) : sms * 4), 256, 0, st>>>(x, n, amax_bits);
  return cudaGetLastError();
}

cudaError_t launch_finalize_scales(const unsigned* amax_bits, float* out, cudaStream_t st) {
  finalize_scales_kernel<<<1, 32, 0, st>>>(amax_bits, out);
  return cudaGetLastError();
}

}  // namespace mxmoe
