// Grouped expert GEMMs for bf16 activations on the 5th-generation tensor cores (tcgen05):
// the prefill path of the weight-only W-MXFP4 layer (no activation quantization).
//
// Pages: "quantization_mxfp4" (KerasFormers), As GPT-OSS's native format (gate_up_proj
// (E, 2I, H) and down_proj (E, H, I) as e2m1 blocks + one e8m0 scale per 32 values along
// the contracting dim, biases in full precision, the routed dispatch) and Primitives
// (e8m0 block scales, codebook[nibble] * 2^(scale - 127)).
//
// Activations as two e4m3 parts. A bf16 value x has 8 significant bits. Per 32-value block
// of a row, part 1 is e4m3(x / 2^s1) (round to nearest even) with s1 = floor(log2(amax)) - 7,
// so |x| / 2^s1 < 256 and nothing saturates; the residual r = x - part1 * 2^s1 is a multiple
// of x's ulp no larger than half of part 1's ulp, i.e. at most 4 significant bits, and
// part 2 = e4m3(r / 2^s2) with s2 = floor(log2(max |r|)) - 7 holds it exactly wherever it
// lies in e4m3's range under s2. So the two parts reproduce every element down to about
// 2^-14 of its block's maximum exactly, and smaller ones to within max(2^(s2 - 10),
// 2^(s1 - 14)), about 2^-21 of the block's maximum. Both parts
// are A operands of kind::mxf8f6f4 block-scaled MMAs with their e8m0 bytes as the A scale
// factors, accumulating into one fp32 accumulator: the MMA sees x * w exactly (up to the
// tiny elements above), at twice the FP8 path's MMA count (the bf16 MMA rate).
//
//   split:   x rows in expert-grouped order -> parts (2, P, H) e4m3 + scales (2, P, H/32)
//   gate_up: acc = sum_p A1_p . Wgu_e^T on [gate rows n0.., up rows I+n0..];
//            a = bf16(silu(acc_g + b_g) * (acc_u + b_u))                    (bf16, (P, I))
//   split:   a rows -> parts (2, P, I) + scales
//   down:    acc = sum_p A2_p . Wd_e^T;  y = acc + b_d                      (fp32, (P, H))
//
// The GEMM has the structure of the FP8 prefill GEMM (persistent, one CTA per SM, tiles of
// 128 grouped rows x 240 weight rows, TMA for A and the 4-bit weights, scale converters,
// a tensor-memory accumulator pair, 16 epilogue warps), with three stages of 128 K values
// (each stage now holds two A tiles) and, per stage, one tcgen05.cp 128x256b of the two
// parts' A scales beside the one of the weights' scales.
//
// Roles (640 threads):
//   warp 0: TMA producer (both A parts, the weight tile)   warp 1: TMEM owner + MMA issuer
//   warp 2: weight scales of tile rows 0..127 + part 1's A scales
//   warp 3: weight scales of tile rows 128..255 + part 2's A scales; first builds the schedule
//   warps 4..19: epilogue (TMEM lane quarter w % 4, every (w-4)/4-th group of 8 columns)
// Every mbarrier wait gives up after ~1 s (clock64): the kernel then records MXMOE_ETIMEOUT
// in the error word, lets in-flight copies land, frees its tensor memory and returns.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "tc_common.cuh"
#include "tmap.h"

namespace mxmoe {
namespace g100b {

using namespace tc;

constexpr int BM = 128;             // rows of A per tile (MMA M)
constexpr int BN = 240;             // MMA N (gate_up: 120 gate + 120 up rows)
constexpr int BK = 128;             // K values per pipeline stage
constexpr int kParts = 2;           // e4m3 parts per activation
constexpr int kStages = 3;
constexpr int kEpiWarps = 16;
constexpr int kThreads = 128 + 32 * kEpiWarps;
constexpr int kAStage = BM * BK;            // 16 KB per part
constexpr int kBStage = BN * BK;            // 30 KB (e2m1 spread to one byte per value)
constexpr int kSfStage = 4096;              // weight scales: 128 lanes x 32 bytes
constexpr int kSfaStage = 4096;             // A scales: part 1 at 0, part 2 at 2048
constexpr int kAccCols = 256;
constexpr int kTmemCols = 512;
constexpr int kSfaCol = 240;                // two 8-column slots of A scales (240, 248)
constexpr int kSfbCol = 496;                // two 8-column slots of weight scales (496, 504)

struct Params {
  const uint8_t* b_scales;   // weight e8m0 scales, (groups, rows_per_group, nb)
  const uint8_t* a_scales;   // part scales, (2, P, nb): part p of grouped row m at (p * P + m) * nb
  const float* bias;         // (E, rows_total)
  const int32_t* offsets;    // (E+1)
  int64_t P;                 // rows of each part of A (grouped rows; a_shared: T)
  int a_shared;              // 1: every expert reads the same A rows (the dense all-experts
                             // path: A row = row within the expert), 0: A row = grouped row
  int E;
  int K;
  int nb;                    // K / 32
  int rows_per_group;        // gate_up: I; down: H
  int rows_total;            // gate_up: 2I; down: H
  int n_out;                 // gate_up: I; down: H
  int n_tiles;
  int nk_full;               // K / 128
  int tail_steps;            // 32-value K-steps of the final partial tile (0 or 2)
  uint16_t* a_out;           // gate_up output (P, I) bf16 bits
  float* y_out;              // down output (P, H) fp32
  int* err;
};

struct Tile {
  int e, mt, nt, m0, rows;
};

__device__ __forceinline__ Tile tile_of(int t, const int* prefix, const int32_t* offsets, int E, int n_tiles) {
  int lo = 0, hi = E;  // largest e with prefix[e] <= t
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] <= t) lo = mid; else hi = mid;
  }
  int e = lo;
  while (e + 1 < E && prefix[e + 1] <= t) ++e;
  const int rem = t - prefix[e];
  Tile tl;
  tl.e = e;
  tl.mt = rem / n_tiles;
  tl.nt = rem % n_tiles;
  const int off = offsets[e];
  tl.m0 = off + tl.mt * BM;
  tl.rows = min(BM, offsets[e + 1] - tl.m0);
  return tl;
}

// 2^e as fp32 for e in [-127, 127] (2^-127 is the subnormal 0x00400000).
__device__ __forceinline__ float pow2i(int e) {
  return e >= -126 ? __uint_as_float(static_cast<uint32_t>(e + 127) << 23) : __uint_as_float(0x00400000u);
}

// Block scale exponent of a part: floor(log2(amax)) - 7, clamped to the e8m0 range (an
// all-zero block gets 0; a subnormal amax counts as 2^-127).
__device__ __forceinline__ int part_exponent(float amax) {
  const int ex = static_cast<int>(__float_as_uint(amax) >> 23);
  const int fl = ex == 0 ? -127 : ex - 127;
  return amax > 0.0f ? max(-127, min(127, fl - 7)) : 0;
}

// ----------------------------------------------------------------- split kernel ---
// One warp per grouped row m (grid-stride); lane l takes the row's 32-value blocks l,
// l + 32, ... The row is src[perm[m]] (the token's x row) when perm is given, else src[m].
// A row whose token index is outside [0, T) gets zero parts with unit scales.
__global__ void __launch_bounds__(256) split_parts_kernel(const uint16_t* __restrict__ src,
                                                           const int32_t* __restrict__ perm, int T,
                                                           int64_t P, int K, uint8_t* __restrict__ parts,
                                                           uint8_t* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int nb = K / 32;
  const int64_t warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t m = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; m < P; m += warps) {
    int64_t row = m;
    bool ok = true;
    if (perm) {
      const int t = perm[m];
      ok = t >= 0 && t < T;
      row = ok ? t : 0;
    }
    const uint4* s = reinterpret_cast<const uint4*>(src + row * K);
    uint8_t* p1 = parts + m * K;
    uint8_t* p2 = parts + (P + m) * K;
    for (int b = lane; b < nb; b += 32) {
      float v[32];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 w = ok ? s[4 * b + q] : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          v[8 * q + 2 * j] = __uint_as_float(wv[j] << 16);
          v[8 * q + 2 * j + 1] = __uint_as_float(wv[j] & 0xFFFF0000u);
        }
      }
      float amax = 0.0f;
#pragma unroll
      for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
      const int s1 = part_exponent(amax);
      const float d1 = pow2i(-s1), u1 = pow2i(s1);
      uint32_t c1[8];
      float rmax = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) c1[i] = 0u;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const uint8_t c = f32_to_e4m3_satfinite(v[i] * d1);
        c1[i >> 2] |= static_cast<uint32_t>(c) << (8 * (i & 3));
        v[i] = v[i] - e4m3_to_f32(c) * u1;   // the residual (exact)
        rmax = fmaxf(rmax, fabsf(v[i]));
      }
      const int s2 = part_exponent(rmax);
      const float d2 = pow2i(-s2);
      uint32_t c2[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) c2[i] = 0u;
#pragma unroll
      for (int i = 0; i < 32; ++i)
        c2[i >> 2] |= static_cast<uint32_t>(f32_to_e4m3_satfinite(v[i] * d2)) << (8 * (i & 3));
      uint4* o1 = reinterpret_cast<uint4*>(p1 + 32 * b);
      uint4* o2 = reinterpret_cast<uint4*>(p2 + 32 * b);
      o1[0] = make_uint4(c1[0], c1[1], c1[2], c1[3]);
      o1[1] = make_uint4(c1[4], c1[5], c1[6], c1[7]);
      o2[0] = make_uint4(c2[0], c2[1], c2[2], c2[3]);
      o2[1] = make_uint4(c2[4], c2[5], c2[6], c2[7]);
      scales[m * nb + b] = static_cast<uint8_t>(s1 + 127);
      scales[(P + m) * nb + b] = static_cast<uint8_t>(s2 + 127);
    }
  }
}

// ------------------------------------------------------------------------ kernel ---
template <bool kGateUp>
__global__ void __launch_bounds__(kThreads, 1)
moe_gemm_parts_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                      const __grid_constant__ CUtensorMap tmap_bt, Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;                                   // kStages x (part 1, part 2)
  uint8_t* sB = sA + kStages * kParts * kAStage;
  uint8_t* sSF = sB + kStages * kBStage;                // weight scales
  uint8_t* sSFA = sSF + kStages * kSfStage;             // A (part) scales
  uint64_t* bars = reinterpret_cast<uint64_t*>(sSFA + kStages * kSfaStage);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* acc_full = bars + 2 * kStages;
  uint64_t* acc_empty = acc_full + 2;
  int* prefix = reinterpret_cast<int*>(acc_empty + 2);           // E + 1
  volatile int* abort_flag = prefix + (p.E + 1);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(prefix + p.E + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bn_rows = kGateUp ? BN / 2 : BN;
  griddep_launch_dependents();

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 3);     // TMA producer (expect_tx) + the two scale-converter warps
      mbar_init(&empty[s], 1);    // MMA commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kEpiWarps);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == 3) {
    int carry = 0;
    for (int e0 = 0; e0 < p.E; e0 += 32) {
      const int e = e0 + lane;
      const int m = e < p.E ? p.offsets[e + 1] - p.offsets[e] : 0;
      const int tiles = ((m + BM - 1) / BM) * p.n_tiles;
      int incl = tiles;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
      }
      if (e < p.E) prefix[e] = carry + incl - tiles;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) prefix[p.E] = carry;
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
  const int total_tiles = prefix[p.E];
  const int nkt = p.nk_full + (p.tail_steps > 0 ? 1 : 0);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer -----
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool dep_ready = false;
      const uint32_t tx = kParts * kAStage + (kGateUp ? 2 : 1) * bn_rows * (BK / 2);
      for (int t = blockIdx.x; t < total_tiles && !*abort_flag; t += gridDim.x) {
        const Tile tl = tile_of(t, prefix, p.offsets, p.E, p.n_tiles);
        const int n0 = tl.nt * bn_rows;
        for (int kt = 0; kt < nkt; ++kt) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err)) break;
          mbar_arrive_expect_tx(&full[stage], tx);
          const bool tail = kt >= p.nk_full;
          const CUtensorMap* mb = tail ? &tmap_bt : &tmap_b;
          const int kx = tail ? p.K - BK : kt * BK;
          const int bx = tail ? 0 : kt * BK;
          if (kGateUp) {
            tma_load_3d(sB + stage * kBStage, mb, &full[stage], bx, n0, 2 * tl.e);
            tma_load_3d(sB + stage * kBStage + bn_rows * BK, mb, &full[stage], bx, n0, 2 * tl.e + 1);
          } else {
            tma_load_3d(sB + stage * kBStage, mb, &full[stage], bx, n0, tl.e);
          }
          if (!dep_ready) {
            griddep_wait();     // the parts are the previous kernel's output
            dep_ready = true;
          }
          uint8_t* a_dst = sA + stage * kParts * kAStage;
          const int arow = p.a_shared ? tl.m0 - p.offsets[tl.e] : tl.m0;
          tma_load_2d(a_dst, &tmap_a, &full[stage], kx, arow);
          tma_load_2d(a_dst + kAStage, &tmap_a, &full[stage], kx, static_cast<int>(p.P) + arow);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer -----
    int stage = 0;
    uint32_t phase = 0;
    int it = 0;
    uint32_t kc = 0;   // k-steps issued so far: its parity picks the scale slots
    const uint32_t idesc0 = idesc_mxf8f6f4(BM, BN);
    for (int t = blockIdx.x; t < total_tiles && !*abort_flag; t += gridDim.x, ++it) {
      const int ab = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      if (!mbar_wait(&acc_empty[ab], acc_phase ^ 1, abort_flag, p.err)) break;
      tc_fence_after();
      const uint32_t dacc = tmem + ab * kAccCols;
      bool ok = true;
      for (int kt = 0; kt < nkt; ++kt, ++kc) {
        if (!mbar_wait(&full[stage], phase, abort_flag, p.err)) { ok = false; break; }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t slot = 8u * (kc & 1u);
          const uint32_t sfb = tmem + kSfbCol + slot, sfa = tmem + kSfaCol + slot;
          tc_cp_128x256b(sfb, smem_desc(smem_u32(sSF + stage * kSfStage), 2048, 128, 0));
          tc_cp_128x256b(sfa, smem_desc(smem_u32(sSFA + stage * kSfaStage), 2048, 128, 0));
          const uint32_t a0 = smem_u32(sA + stage * kParts * kAStage), b0 = smem_u32(sB + stage * kBStage);
          const int first = kt < p.nk_full ? 0 : 4 - p.tail_steps;
          for (int kk = first; kk < 4; ++kk) {
            const uint64_t bd = smem_desc(b0 + 32 * kk, 16, 1024, 2);
            const uint32_t id = idesc0 | (static_cast<uint32_t>(kk) << 4) | (static_cast<uint32_t>(kk) << 29);
            const uint32_t sel = static_cast<uint32_t>(kk) << 30;
#pragma unroll
            for (int pp = 0; pp < kParts; ++pp) {
              const uint64_t ad = smem_desc(a0 + pp * kAStage + 32 * kk, 16, 1024, 2);
              tc_mma_mxf8f6f4(dacc, ad, bd, id, (sfa + 4 * pp) | sel, sfb | sel,
                              (kt > 0 || kk > first || pp > 0) ? 1u : 0u);
            }
          }
          tc_commit(&empty[stage]);
        }
        __syncwarp();
        if (++stage == kStages) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
      if (lane == 0) tc_commit(&acc_full[ab]);
      __syncwarp();
    }
  } else if (warp == 2 || warp == 3) {
    // -------------------------------------------------------- scale converters -----
    // Weight scales: warp 2 fills columns 0-3 (tile rows 0..127), warp 3 columns 4-7 (rows
    // 128..255); lane l owns rows l, l+32, l+64, l+96 of its half, whose four words sit side
    // by side (byte 16*L + 4*i for tensor-memory lane L = 32*q + l), stored once per
    // quarter q. A scales: warp 2 + pp holds part pp's bytes of grouped rows m0 + l + 32 i in
    // the same layout (columns 0-3 of the A slot for part 1, 4-7 for part 2). A stage's 4
    // bytes of a row are two aligned 16-bit words (nb is even, k-blocks start at multiples
    // of 4), loaded kStages stages ahead and combined only at the store; a row outside the
    // tile (or past the grouped rows) reads the array's first row and stores unit scales.
    const int w2 = warp - 2;
    const int halves = kGateUp ? 2 : 1;
    uint32_t phase = 0;
    auto rows_of = [&](int t, const uint16_t* (&rp)[8], uint32_t& ok) {
      const Tile tl = tile_of(t, prefix, p.offsets, p.E, p.n_tiles);
      const int n0 = tl.nt * bn_rows;
      const int valid = min(bn_rows, p.rows_per_group - n0);
      ok = 0u;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = 128 * w2 + lane + 32 * i;
        const int h = r >= bn_rows ? 1 : 0;
        const int rr = r - h * bn_rows;
        const int group = kGateUp ? 2 * tl.e + h : tl.e;
        const bool in = r < BN && rr < valid && h < halves;
        rp[i] = reinterpret_cast<const uint16_t*>(
            p.b_scales + (in ? (static_cast<int64_t>(group) * p.rows_per_group + n0 + rr) * p.nb : 0));
        ok |= (in ? 1u : 0u) << i;
        const int64_t m = static_cast<int64_t>(p.a_shared ? tl.m0 - p.offsets[tl.e] : tl.m0) + lane + 32 * i;
        const bool ain = m < p.P;
        rp[4 + i] = reinterpret_cast<const uint16_t*>(
            p.a_scales + (ain ? (static_cast<int64_t>(w2) * p.P + m) * p.nb : 0));
        ok |= (ain ? 1u : 0u) << (4 + i);
      }
    };
    auto load = [&](const uint16_t* const (&rp)[8], int kt, uint32_t (&wv)[16]) {
      const int kw = (kt < p.nk_full ? 4 * kt : p.nb - 4) >> 1;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        wv[2 * i] = __ldg(rp[i] + kw);
        wv[2 * i + 1] = __ldg(rp[i] + kw + 1);
      }
    };
    int lt = blockIdx.x, lkt = 0;
    int st = blockIdx.x, skt = 0;
    const uint16_t* rp[8] = {nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr};
    uint32_t rows_ok = 0u;
    uint32_t buf[kStages][16] = {};
    uint32_t buf_ok[kStages] = {};
    auto load_next = [&](uint32_t (&wv)[16]) -> uint32_t {
      if (lt >= total_tiles) return 0u;
      if (lkt == 0) rows_of(lt, rp, rows_ok);
      load(rp, lkt, wv);
      if (++lkt == nkt) { lkt = 0; lt += gridDim.x; }
      return rows_ok;
    };
#pragma unroll
    for (int j = 0; j < kStages; ++j) buf_ok[j] = load_next(buf[j]);
    bool run = true;
    while (run) {
#pragma unroll
      for (int j = 0; j < kStages; ++j) {
        if (st >= total_tiles || *abort_flag || !mbar_wait(&empty[j], phase ^ 1, abort_flag, p.err)) {
          run = false;
          break;
        }
        uint32_t wq[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
          wq[i] = ((buf_ok[j] >> i) & 1u) ? ((buf[j][2 * i] & 0xFFFFu) | (buf[j][2 * i + 1] << 16)) : 0x7F7F7F7Fu;
        const uint4 wb = make_uint4(wq[0], wq[1], wq[2], wq[3]);
        const uint4 wa = make_uint4(wq[4], wq[5], wq[6], wq[7]);
        uint8_t* db = sSF + j * kSfStage + 2048 * w2 + 16 * lane;
        uint8_t* da = sSFA + j * kSfaStage + 2048 * w2 + 16 * lane;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          *reinterpret_cast<uint4*>(db + 512 * q) = wb;
          *reinterpret_cast<uint4*>(da + 512 * q) = wa;
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[j]);
        if (++skt == nkt) { skt = 0; st += gridDim.x; }
        buf_ok[j] = load_next(buf[j]);
      }
      phase ^= 1;
    }
  } else if (warp >= 4) {
    // --------------------------------------------------------------- epilogue -----
    const int q = warp & 3;
    const int slice = (warp - 4) >> 2;
    constexpr int kSlices = kEpiWarps / 4;
    const int row = 32 * q + lane;
    int it = 0;
    for (int t = blockIdx.x; t < total_tiles && !*abort_flag; t += gridDim.x, ++it) {
      const Tile tl = tile_of(t, prefix, p.offsets, p.E, p.n_tiles);
      const int n0 = tl.nt * bn_rows;
      const int ab = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      if (!mbar_wait(&acc_full[ab], acc_phase, abort_flag, p.err)) break;
      tc_fence_after();
      const uint32_t tbase = tmem + ab * kAccCols + (static_cast<uint32_t>(32 * q) << 16);
      const bool valid = row < tl.rows;
      const int64_t pos = tl.m0 + row;
      if (kGateUp) {
        for (int c0 = 8 * slice; c0 < bn_rows; c0 += 8 * kSlices) {
          uint32_t g[8], u[8];
          tc_ld_32x32b_x8(tbase + c0, g);
          tc_ld_32x32b_x8(tbase + bn_rows + c0, u);
          const bool live = n0 + c0 < p.n_out;
          float bg[8], bu[8];
          if (live) {
            const float4* bp = reinterpret_cast<const float4*>(p.bias + static_cast<int64_t>(tl.e) * p.rows_total + n0 + c0);
            const float4* bq = reinterpret_cast<const float4*>(p.bias + static_cast<int64_t>(tl.e) * p.rows_total + p.n_out + n0 + c0);
            const float4 b0 = bp[0], b1 = bp[1], b2 = bq[0], b3 = bq[1];
            bg[0] = b0.x; bg[1] = b0.y; bg[2] = b0.z; bg[3] = b0.w; bg[4] = b1.x; bg[5] = b1.y; bg[6] = b1.z; bg[7] = b1.w;
            bu[0] = b2.x; bu[1] = b2.y; bu[2] = b2.z; bu[3] = b2.w; bu[4] = b3.x; bu[5] = b3.y; bu[6] = b3.z; bu[7] = b3.w;
          } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) bg[i] = bu[i] = 0.0f;
          }
          tc_wait_ld(g, u);
          uint32_t o[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float a0 = silu_mul(__fadd_rn(__uint_as_float(g[2 * i]), bg[2 * i]),
                                      __fadd_rn(__uint_as_float(u[2 * i]), bu[2 * i]));
            const float a1 = silu_mul(__fadd_rn(__uint_as_float(g[2 * i + 1]), bg[2 * i + 1]),
                                      __fadd_rn(__uint_as_float(u[2 * i + 1]), bu[2 * i + 1]));
            o[i] = static_cast<uint32_t>(f32_to_bf16_bits_rn(a0)) | (static_cast<uint32_t>(f32_to_bf16_bits_rn(a1)) << 16);
          }
          if (valid && live)
            *reinterpret_cast<uint4*>(p.a_out + pos * p.n_out + n0 + c0) = make_uint4(o[0], o[1], o[2], o[3]);
        }
      } else {
        for (int c0 = 8 * slice; c0 < BN; c0 += 8 * kSlices) {
          uint32_t v[8];
          tc_ld_32x32b_x8(tbase + c0, v);
          const bool live = n0 + c0 < p.n_out;
          float bb[8];
          if (live) {
            const float4* bp = reinterpret_cast<const float4*>(p.bias + static_cast<int64_t>(tl.e) * p.rows_total + n0 + c0);
            const float4 b0 = bp[0], b1 = bp[1];
            bb[0] = b0.x; bb[1] = b0.y; bb[2] = b0.z; bb[3] = b0.w; bb[4] = b1.x; bb[5] = b1.y; bb[6] = b1.z; bb[7] = b1.w;
          } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) bb[i] = 0.0f;
          }
          tc_wait_ld(v);
          float o[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) o[i] = __fadd_rn(__uint_as_float(v[i]), bb[i]);
          if (valid && live) {
            st_global_v8(p.y_out + pos * p.n_out + n0 + c0, o);
          }
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
  if (*abort_flag) {
    const long long t0 = clock64();
    while (clock64() - t0 < 200000) {
    }
  }
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTmemCols));
  }
}

size_t smem_bytes(int E) {
  return 1024 + kStages * (kParts * kAStage + kBStage + kSfStage + kSfaStage) + (2 * kStages + 4) * sizeof(uint64_t) +
         (E + 3) * sizeof(int) + 16;
}

}  // namespace g100b

// ---------------------------------------------------------------- host side -------

// src rows (bf16, K values) -> two e4m3 parts (2, P, K) + e8m0 scales (2, P, K/32); row m
// is src[perm[m]] when perm is given (tokens in expert-grouped order), else src[m].
cudaError_t launch_split_parts(const uint16_t* src, const int32_t* perm, int T, int64_t P, int K, uint8_t* parts,
                               uint8_t* scales, int sms, cudaStream_t st) {
  if (P == 0) return cudaSuccess;
  const int64_t blocks = cdiv(P, 8);
  const int grid = static_cast<int>(std::min<int64_t>(blocks, static_cast<int64_t>(sms) * 16));
  g100b::split_parts_kernel<<<grid, 256, 0, st>>>(src, perm, T, P, K, parts, scales);
  return cudaGetLastError();
}

cudaError_t tc_parts_gemm_prepare(int E) {
  const size_t smem = g100b::smem_bytes(E);
  cudaError_t e = cudaFuncSetAttribute(g100b::moe_gemm_parts_kernel<true>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e) return e;
  return cudaFuncSetAttribute(g100b::moe_gemm_parts_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(smem));
}

// parts/a_scales: the split of the grouped activation rows, (2, P_rows, K) and
// (2, P_rows, K/32); blocks/scales: (E, rows_total, K/2) and (E, rows_total, K/32);
// gate_up: rows_total = 2I, n_out = I, writes a_out (P_rows, I) bf16; down: rows_total =
// n_out = H, writes y_out (P_rows, H) fp32.
cudaError_t launch_tc_parts_gemm(bool gate_up, const uint8_t* parts, const uint8_t* a_scales, int64_t P_rows, int K,
                                 const uint8_t* blocks, const uint8_t* scales, const float* bias, int E, int n_out,
                                 const int32_t* offsets, uint16_t* a_out, float* y_out, int* err, int sms,
                                 cudaStream_t st, bool a_shared) {
  using namespace g100b;
  const int rows_per_group = n_out;
  const int groups = gate_up ? 2 * E : E;
  const int bn_rows = gate_up ? BN / 2 : BN;
  CUtensorMap ma, mb, mbt;
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(P_rows > 0 ? 2 * P_rows : 1)};
    const uint64_t strides[1] = {static_cast<uint64_t>(K)};
    const uint32_t box[2] = {BK, BM};
    if (!tmap_encode(&ma, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, parts, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t row_bytes = static_cast<uint64_t>(K) / 2;
    const uint64_t dims[3] = {static_cast<uint64_t>((K / BK) * BK), static_cast<uint64_t>(rows_per_group),
                              static_cast<uint64_t>(groups)};
    const uint64_t strides[2] = {row_bytes, row_bytes * rows_per_group};
    const uint32_t box[3] = {BK, static_cast<uint32_t>(bn_rows), 1};
    if (!tmap_encode(&mb, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 3, blocks, dims, strides, box))
      return cudaErrorInvalidValue;
    const uint64_t tdims[3] = {BK, static_cast<uint64_t>(rows_per_group), static_cast<uint64_t>(groups)};
    if (!tmap_encode(&mbt, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 3, blocks + (K - BK) / 2, tdims, strides, box))
      return cudaErrorInvalidValue;
  }
  Params prm;
  prm.b_scales = scales;
  prm.a_scales = a_scales;
  prm.bias = bias;
  prm.offsets = offsets;
  prm.P = P_rows;
  prm.a_shared = a_shared ? 1 : 0;
  prm.E = E;
  prm.K = K;
  prm.nb = K / 32;
  prm.rows_per_group = rows_per_group;
  prm.rows_total = gate_up ? 2 * n_out : n_out;
  prm.n_out = n_out;
  prm.n_tiles = (n_out + bn_rows - 1) / bn_rows;
  prm.nk_full = K / BK;
  prm.tail_steps = (K % BK) / 32;
  prm.a_out = a_out;
  prm.y_out = y_out;
  prm.err = err;
  // programmatic dependent launch: the kernel starts during its predecessor (the split of
  // its input rows) and waits for it only before loading those rows
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(sms));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem_bytes(E);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (gate_up) return cudaLaunchKernelEx(&cfg, moe_gemm_parts_kernel<true>, ma, mb, mbt, prm);
  return cudaLaunchKernelEx(&cfg, moe_gemm_parts_kernel<false>, ma, mb, mbt, prm);
}

}  // namespace mxmoe
