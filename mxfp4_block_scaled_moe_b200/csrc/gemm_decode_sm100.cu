// Routed expert GEMMs for small batches on the tensor cores, with the MXFP4 weights as
// the MMA's A operand: the tensor core decodes the e2m1 nibbles and applies their e8m0
// block scales (tcgen05.mma kind::mxf8f6f4 block_scale), TMA streams the packed weight
// bytes, and no instruction of the SM touches a nibble. This is the decode path of
// "quantization_mxfp4" (KerasFormers), As GPT-OSS's native format: only the routed
// experts' blocks are read, once per layer.
//
// Operands of one expert e with n_e routed rows:
//   A = 128 weight rows (gate_up: 128 gate rows and, in a second MMA, the 128 matching up
//       rows; down: 128 rows of down_proj), e2m1 with the checkpoint's e8m0 scales;
//   B = the expert's token rows as FP8 E4M3 "parts" with their own e8m0 block scales
//       (MX-FP8). With FP8 activations a token is one part (its static-scale e4m3 code,
//       unit block scales; the per-tensor scale multiplies in the epilogue). With bf16
//       activations a token is np = 3 parts: p1 = e4m3(x / 2^s1), p2 = e4m3((x - p1)/2^s2),
//       p3 the same on the next residual, each s from its block's amax, so that
//       p1 + p2 + p3 reproduces x to about 2^-12 of the block's largest value.
//   D = 128 x N fp32 in tensor memory, N = np * n_e rounded up to 16; the epilogue adds a
//       token's np columns.
// The gate_up epilogue applies bias + SwiGLU and writes a directly as the down GEMM's B
// operand (its 32-row warp is exactly one 32-value block of the down contraction, so the
// block amax is a warp reduction); the down epilogue writes y and, in the last CTA of
// each 128-row tile (an atomic ticket reset for the next call), the weighted combine.
//
// Scale-factor records of the B operand ("SFB"): for expert e and k-tile kt, 1024 bytes
// = two 512-byte tcgen05.cp atoms (rows 0..127, 128..255), row r of an atom at byte
// 16*(r%32) + 4*((r/32)%4) + j for the tile's k-block j. The final (tail) k-tile of a
// K = 22.5 x 128 contraction holds k-blocks nb-4 .. nb-1, consumed by k-steps 2 and 3.
#include <cuda.h>

#include "common.cuh"
#include "launchers.h"
#include "tc_common.cuh"

namespace mxmoe {
namespace dec {

using namespace tc;

constexpr int BM = 128;
constexpr int BK = 128;
constexpr int kBoxRows = 32;       // token-part rows per TMA box of B
constexpr int kMaxN = 192;         // largest B width (np * n_e rounded up) this path takes
constexpr int kThreads = 256;      // warp 0 TMA, 1 MMA, 2-3 A-scale converters, 4-7 epilogue
constexpr int kMaxStages = 8;
constexpr int kTmemCols = 512;
constexpr int kAccUpCol = 256;     // second accumulator (up rows)
constexpr int kSfaCol0 = 192;      // A scales: gate (or down) at 192..195, up at 196..199
constexpr int kSfbCol = 200;       // B scales: 200..207 (two atoms)
constexpr int kSfRecord = 1024;

// instruction descriptor, kind::mxf8f6f4 block-scaled: A = E2M1 (5), B = E4M3 (0)
__host__ __device__ constexpr uint32_t idesc_w_by_x(int M, int N) {
  return (5u << 7) | (0u << 10) | (static_cast<uint32_t>(N >> 3) << 17) | (1u << 23) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// Where the scale of k-block kb lives: k-tile and byte within the tile's 4 blocks. The
// tail tile (K % 128 == 64) holds blocks nb-4 .. nb-1.
__device__ __forceinline__ void sf_slot(int kb, int nb, int nk_full, int& kt, int& j) {
  if (kb < 4 * nk_full) {
    kt = kb >> 2;
    j = kb & 3;
  } else {
    kt = nk_full;
    j = kb - (nb - 4);
  }
}

__device__ __forceinline__ int sf_atom_byte(int r, int j) {
  return (r >> 7) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + j;
}

// e8m0 exponent s for a block whose largest magnitude is amax: amax / 2^s in [128, 256),
// inside e4m3's range. amax == 0 gives 0.
__device__ __forceinline__ int part_exponent(float amax) {
  if (!(amax > 0.0f)) return 0;
  const uint32_t u = __float_as_uint(amax);
  int ex = static_cast<int>(u >> 23);
  int fl = ex > 0 ? ex - 127 : (31 - __clz(u)) - 149;
  return max(-127, min(127, fl - 7));
}

__device__ __forceinline__ float pow2f(int s) {   // exact 2^s for s in [-126, 127]
  return __uint_as_float(static_cast<uint32_t>(s + 127) << 23);
}

// Split v (this lane's element of a 32-value block held by the warp) into np e4m3 parts.
// Writes part bytes and scale exponents (same in every lane). Lanes outside the data pass
// v = 0.
template <int NP>
__device__ __forceinline__ void split_parts(float v, uint8_t (&q)[NP], int (&s)[NP]) {
  float r = v;
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const float amax = warp_max(fabsf(r));
    s[p] = part_exponent(amax);
    const int sc = max(s[p], -126);
    q[p] = f32_to_e4m3_satfinite(r * pow2f(-sc));   // power-of-two scaling: exact
    r = r - e4m3_to_f32(q[p]) * pow2f(sc);         // exact residual
  }
}

// Bytes of one pipeline stage: A tiles, B tile, A scale atoms, B scale record, rounded up
// to 1024 so that every stage's tiles keep the 1024-byte alignment of 128-byte swizzle.
__host__ __device__ constexpr int stage_size(int kA, int b_stage_bytes) {
  return ((kA * BM * BK + b_stage_bytes + kA * 512 + kSfRecord) + 1023) & ~1023;
}

struct Params {
  // A: weights
  const uint8_t* w_scales;   // (groups, rows_per_group, nb) e8m0
  const float* bias;         // (E, rows_total)
  int rows_per_group;        // gate_up: I (a half); down: H
  int rows_total;            // 2I or H
  int n_out;                 // I or H
  // shapes
  int E, K, nb, nk_full, tail_steps, np;
  const int32_t* offsets;
  const int32_t* active;
  const int32_t* n_active;
  const uint8_t* sfb;        // B scale records [E][nkt][1024]
  float s_in;                // per-tensor scale of the B operand (FP8) or 1
  // gate_up outputs (the down GEMM's B operand)
  uint8_t* xs_out;           // (P * np_out, I) e4m3
  uint8_t* sfb_out;          // [E][nkt_out][1024]
  int np_out, nb_out, nk_full_out, nkt_out;
  float s_out;               // FP8: static scale of a; 0: bf16 split
  unsigned* amax_bits;       // calibration: running max |a|
  // down outputs
  float* y_out;              // (P, H) fp32
  uint16_t* out;             // (T, H) bf16, combine
  const int32_t* topk_idx;
  const float* topk_w;
  const int32_t* inv;
  unsigned* tickets;         // per 128-row tile
  int T, k;
  int* err;
  int stages, b_stage_bytes;
};

template <bool kGateUp, int NP>
__global__ void __launch_bounds__(kThreads, 1)
decode_gemm_kernel(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_wt,
                   const __grid_constant__ CUtensorMap map_x, Params p) {
  const int slot = blockIdx.y;
  if (slot >= *p.n_active) return;   // the whole CTA, before any barrier or allocation
  const int e = p.active[slot];
  const int off = p.offsets[e], n_e = p.offsets[e + 1] - off;
  const int ncols = ((p.np * n_e + 15) / 16) * 16;
  const int nboxes = (p.np * n_e + kBoxRows - 1) / kBoxRows;
  const int row0 = blockIdx.x * BM;
  const int nkt = p.nk_full + (p.tail_steps > 0 ? 1 : 0);
  const int S = p.stages;
  constexpr int kA = kGateUp ? 2 : 1;   // A tiles per stage

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int a_bytes = kA * BM * BK;                       // unpacked e2m1, one byte per value
  const int stage_bytes = stage_size(kA, p.b_stage_bytes);  // a multiple of 1024
  uint8_t* sRaw = smem + S * stage_bytes;                 // kA * 128 rows * nb raw scale bytes
  const int raw_bytes = ((kA * BM * p.nb) + 15) & ~15;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sRaw + raw_bytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + kMaxStages;
  uint64_t* acc_full = bars + 2 * kMaxStages;
  uint64_t* raw_full = acc_full + 1;                      // [2]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(raw_full + 2);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(raw_full + 2) + 1;
  unsigned* last_flag = tmem_holder + 1;

  auto sA = [&](int s, int h) { return smem + s * stage_bytes + h * BM * BK; };
  auto sB = [&](int s) { return smem + s * stage_bytes + a_bytes; };
  auto sSFA = [&](int s, int h) { return smem + s * stage_bytes + a_bytes + p.b_stage_bytes + h * 512; };
  auto sSFB = [&](int s) { return smem + s * stage_bytes + a_bytes + p.b_stage_bytes + kA * 512; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1 + kA);   // TMA producer (expect_tx) + one scale converter per A tile
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(&raw_full[0], 1);
    mbar_init(&raw_full[1], 1);
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
    // ---------------------------------------------------------------- producer -----
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      const uint32_t tx = kA * BM * (BK / 2) + nboxes * kBoxRows * BK + kSfRecord;
      for (int kt = 0; kt < nkt; ++kt) {
        if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err)) break;
        mbar_arrive_expect_tx(&full[stage], tx);
        const bool tail = kt >= p.nk_full;
        const CUtensorMap* mw = tail ? &map_wt : &map_w;
        const int wx = tail ? 0 : kt * BK;
        const int kx = tail ? p.K - BK : kt * BK;
        if (kGateUp) {
          tma_load_3d(sA(stage, 0), mw, &full[stage], wx, row0, 2 * e);
          tma_load_3d(sA(stage, 1), mw, &full[stage], wx, row0, 2 * e + 1);
        } else {
          tma_load_3d(sA(stage, 0), mw, &full[stage], wx, row0, e);
        }
        for (int b = 0; b < nboxes; ++b)
          tma_load_2d(sB(stage) + b * kBoxRows * BK, &map_x, &full[stage], kx, p.np * off + b * kBoxRows);
        bulk_g2s(sSFB(stage), p.sfb + (static_cast<int64_t>(e) * nkt + kt) * kSfRecord, kSfRecord, &full[stage]);
        if (++stage == S) { stage = 0; phase ^= 1; }
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------------------- MMA -----
    int stage = 0;
    uint32_t phase = 0;
    const uint32_t id0 = idesc_w_by_x(BM, ncols);
    bool ok = true;
    for (int kt = 0; kt < nkt; ++kt) {
      if (!mbar_wait(&full[stage], phase, abort_flag, p.err)) { ok = false; break; }
      tc_fence_after();
      if (lane == 0) {
        for (int h = 0; h < kA; ++h)
          tc_cp_32x128b_x4(tmem + kSfaCol0 + 4 * h, smem_desc(smem_u32(sSFA(stage, h)), 0, 128, 0));
        const uint32_t sfb = smem_u32(sSFB(stage));
        tc_cp_32x128b_x4(tmem + kSfbCol, smem_desc(sfb, 0, 128, 0));
        tc_cp_32x128b_x4(tmem + kSfbCol + 4, smem_desc(sfb + 512, 0, 128, 0));
        const uint32_t b0 = smem_u32(sB(stage));
        const int first = kt < p.nk_full ? 0 : 4 - p.tail_steps;
        for (int kk = first; kk < 4; ++kk) {
          const uint64_t bd = smem_desc(b0 + 32 * kk, 16, 1024, 2);
          const uint32_t id = id0 | (static_cast<uint32_t>(kk) << 4) | (static_cast<uint32_t>(kk) << 29);
          const uint32_t sel = static_cast<uint32_t>(kk) << 30;
          const uint32_t acc = (kt > 0 || kk > first) ? 1u : 0u;
          for (int h = 0; h < kA; ++h) {
            const uint64_t ad = smem_desc(smem_u32(sA(stage, h)) + 32 * kk, 16, 1024, 2);
            tc_mma_mxf8f6f4(tmem + h * kAccUpCol, ad, bd, id, (tmem + kSfaCol0 + 4 * h) | sel,
                            (tmem + kSfbCol) | sel, acc);
          }
        }
        tc_commit(&empty[stage]);
      }
      __syncwarp();
      if (++stage == S) { stage = 0; phase ^= 1; }
    }
    if (ok && lane == 0) tc_commit(acc_full);
    __syncwarp();
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------ A (weight) scale converters -----
    const int h = warp - 2;   // 0: gate / down rows, 1: up rows
    if (h < kA) {
      const int group = kGateUp ? 2 * e + h : e;
      const int valid = min(BM, p.rows_per_group - row0);
      const int bytes = valid * p.nb;
      const uint8_t* src = p.w_scales + (static_cast<int64_t>(group) * p.rows_per_group + row0) * p.nb;
      uint8_t* dst = sRaw + h * BM * p.nb;
      const bool bulk = ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst) |
                          static_cast<uintptr_t>(bytes)) & 15u) == 0;
      bool ok = true;
      if (bulk) {
        if (lane == 0) {
          mbar_arrive_expect_tx(&raw_full[h], static_cast<uint32_t>(bytes));
          bulk_g2s(dst, src, static_cast<uint32_t>(bytes), &raw_full[h]);
        }
        ok = mbar_wait(&raw_full[h], 0, abort_flag, p.err);
      } else {
        for (int c0 = 0; c0 < bytes; c0 += 32 * 8) {
          uint8_t v[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int c = c0 + u * 32 + lane;
            v[u] = c < bytes ? src[c] : 0;
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int c = c0 + u * 32 + lane;
            if (c < bytes) dst[c] = v[u];
          }
        }
      }
      __syncwarp();
      if (ok) {
        // lane l owns atom rows l, l+32, l+64, l+96: bytes 16*l .. 16*l+15 of the atom
        int src_off[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = lane + 32 * i;
          src_off[i] = r < valid ? (h * BM + r) * p.nb : -1;
        }
        int stage = 0;
        uint32_t phase = 0;
        for (int kt = 0; kt < nkt; ++kt) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err)) break;
          const int kb0 = kt < p.nk_full ? 4 * kt : p.nb - 4;
          uint32_t wv[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if (src_off[i] < 0) {
              wv[i] = 0x7F7F7F7Fu;
            } else {
              const uint8_t* s8 = sRaw + src_off[i] + kb0;
              wv[i] = static_cast<uint32_t>(s8[0]) | (static_cast<uint32_t>(s8[1]) << 8) |
                      (static_cast<uint32_t>(s8[2]) << 16) | (static_cast<uint32_t>(s8[3]) << 24);
            }
          }
          *reinterpret_cast<uint4*>(sSFA(stage, h) + 16 * lane) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
          fence_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&full[stage]);
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
      }
    }
  } else {
    // ----------------------------------------------------------------- epilogue -----
    const int q = warp & 3;
    const int m = 32 * q + lane;           // accumulator row = TMEM lane
    const int row = row0 + m;              // weight row within the half / down_proj
    const bool live = row < p.n_out;
    if (mbar_wait(acc_full, 0, abort_flag, p.err)) {
      tc_fence_after();
      const uint32_t tb = tmem + (static_cast<uint32_t>(32 * q) << 16);
      // NP (parts per token) is a template parameter and every loop over accumulator
      // columns is unrolled, so the tcgen05.ld destinations stay in registers until the
      // wait that makes them valid
      const float* bias_e = p.bias + static_cast<int64_t>(e) * p.rows_total;
      if (kGateUp) {
        const float bg = live ? bias_e[row] : 0.0f;
        const float bu = live ? bias_e[p.n_out + row] : 0.0f;
        const int kb = row >> 5;           // k-block of the down contraction (warp-uniform)
        int okt, oj;
        sf_slot(kb, p.nb_out, p.nk_full_out, okt, oj);
        uint8_t* rec = p.sfb_out + (static_cast<int64_t>(e) * p.nkt_out + okt) * kSfRecord;
        const bool warp_live = (row0 + 32 * q) < p.n_out;
        for (int j0 = 0; j0 < n_e; j0 += 8) {
          uint32_t g[NP][8], u[NP][8];
#pragma unroll
          for (int c = 0; c < NP; ++c) {
            tc_ld_32x32b_x8(tb + NP * j0 + 8 * c, g[c]);
            tc_ld_32x32b_x8(tb + kAccUpCol + NP * j0 + 8 * c, u[c]);
            tc_wait_ld(g[c], u[c]);
          }
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            if (j0 + jj < n_e) {
              float gs = 0.0f, us = 0.0f;
#pragma unroll
              for (int pp = 0; pp < NP; ++pp) {
                gs += __uint_as_float(g[(NP * jj + pp) >> 3][(NP * jj + pp) & 7]);
                us += __uint_as_float(u[(NP * jj + pp) >> 3][(NP * jj + pp) & 7]);
              }
              const float gv = __fadd_rn(__fmul_rn(p.s_in, gs), bg);
              const float uv = __fadd_rn(__fmul_rn(p.s_in, us), bu);
              const float a = live ? silu_mul(gv, uv) : 0.0f;
              if (p.amax_bits && live) atomicMax(p.amax_bits, __float_as_uint(fabsf(a)));
              const int64_t pos = off + j0 + jj;
              if (p.s_out > 0.0f) {
                // FP8 intermediate: one part, unit block scale
                if (live) p.xs_out[pos * p.n_out + row] = act_quant_e4m3(a, p.s_out);
                if (warp_live && lane == 0) rec[sf_atom_byte(j0 + jj, oj)] = 127;
              } else {
                // bf16 intermediate, split into 3 MX-FP8 parts over this warp's 32 rows
                const float ar = bf16_bits_to_f32(f32_to_bf16_bits_rn(a));
                uint8_t qv[3];
                int sv[3];
                split_parts<3>(live ? ar : 0.0f, qv, sv);
                if (warp_live) {
#pragma unroll
                  for (int pp = 0; pp < 3; ++pp) {
                    if (live) p.xs_out[(pos * 3 + pp) * p.n_out + row] = qv[pp];
                    if (lane == 0) rec[sf_atom_byte(3 * (j0 + jj) + pp, oj)] = static_cast<uint8_t>(sv[pp] + 127);
                  }
                }
              }
            }
          }
        }
      } else {
        const float bd = live ? bias_e[row] : 0.0f;
        for (int j0 = 0; j0 < n_e; j0 += 8) {
          uint32_t v[NP][8];
#pragma unroll
          for (int c = 0; c < NP; ++c) {
            tc_ld_32x32b_x8(tb + NP * j0 + 8 * c, v[c]);
            tc_wait_ld(v[c]);
          }
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            if (j0 + jj < n_e) {
              float ys = 0.0f;
#pragma unroll
              for (int pp = 0; pp < NP; ++pp) ys += __uint_as_float(v[(NP * jj + pp) >> 3][(NP * jj + pp) & 7]);
              if (live)
                p.y_out[static_cast<int64_t>(off + j0 + jj) * p.n_out + row] = __fadd_rn(__fmul_rn(p.s_in, ys), bd);
            }
          }
        }
      }
    }
  }

  // ---------------------------------------------------------------------- teardown ---
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
  if (!kGateUp && p.out != nullptr && !*abort_flag) {
    // weighted combine of this 128-row tile, by the last of the tile's CTAs
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0)
      *last_flag = atomicAdd(&p.tickets[blockIdx.x], 1u) == static_cast<unsigned>(*p.n_active) - 1u;
    __syncthreads();
    if (*last_flag) {
      __threadfence();
      for (int i = threadIdx.x; i < p.T * BM; i += blockDim.x) {
        const int t = i / BM, r = row0 + (i % BM);
        if (r >= p.n_out) continue;
        int ord[8], eid[8];
        for (int j = 0; j < p.k; ++j) {
          const int ex = p.topk_idx[static_cast<int64_t>(t) * p.k + j];
          int qq = j;
          while (qq > 0 && eid[qq - 1] > ex) { eid[qq] = eid[qq - 1]; ord[qq] = ord[qq - 1]; --qq; }
          eid[qq] = ex;
          ord[qq] = j;
        }
        float acc = 0.0f;
        for (int qq = 0; qq < p.k; ++qq) {
          const int j = ord[qq];
          const int64_t pos = p.inv[static_cast<int64_t>(t) * p.k + j];
          acc = __fadd_rn(acc, __fmul_rn(p.topk_w[static_cast<int64_t>(t) * p.k + j],
                                         __ldcg(p.y_out + pos * p.n_out + r)));
        }
        p.out[static_cast<int64_t>(t) * p.n_out + r] = f32_to_bf16_bits_rn(acc);
      }
      if (threadIdx.x == 0) p.tickets[blockIdx.x] = 0u;
    }
  }
}

// ------------------------------------------------ token operand of the gate_up GEMM --
// One warp per (routed pair, 32-value block): x's block as np MX-FP8 parts (bf16 path) or
// its static-scale e4m3 code with a unit block scale (FP8 path), written in expert-grouped
// row order with the block scales into the expert's scale records.
template <int NP>
__global__ void __launch_bounds__(256) split_tokens_kernel(
    const uint16_t* __restrict__ x, const int32_t* __restrict__ perm_token, const int32_t* __restrict__ perm_slot,
    const int32_t* __restrict__ topk_idx, const int32_t* __restrict__ offsets, int64_t P, int H, int k,
    float s0, uint8_t* __restrict__ xs, uint8_t* __restrict__ sfb, int nb, int nk_full, int nkt) {
  const int lane = threadIdx.x & 31;
  const int64_t w = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (w >= P * nb) return;
  const int64_t pos = w / nb;
  const int kb = static_cast<int>(w % nb);
  const int t = perm_token[pos];
  const int e = topk_idx[static_cast<int64_t>(t) * k + perm_slot[pos]];
  const int j = static_cast<int>(pos - offsets[e]);
  const float v = bf16_bits_to_f32(x[static_cast<int64_t>(t) * H + 32 * kb + lane]);
  int kt, jb;
  sf_slot(kb, nb, nk_full, kt, jb);
  uint8_t* rec = sfb + (static_cast<int64_t>(e) * nkt + kt) * kSfRecord;
  if (NP == 1) {
    xs[pos * H + 32 * kb + lane] = act_quant_e4m3(v, s0);
    if (lane == 0) rec[sf_atom_byte(j, jb)] = 127;
  } else {
    uint8_t qv[NP];
    int sv[NP];
    split_parts<NP>(v, qv, sv);
#pragma unroll
    for (int pp = 0; pp < NP; ++pp) {
      xs[(pos * NP + pp) * H + 32 * kb + lane] = qv[pp];
      if (lane == 0) rec[sf_atom_byte(NP * j + pp, jb)] = static_cast<uint8_t>(sv[pp] + 127);
    }
  }
}

size_t smem_bytes(bool gate_up, int stages, int b_stage_bytes, int nb) {
  const int kA = gate_up ? 2 : 1;
  const size_t stage = static_cast<size_t>(stage_size(kA, b_stage_bytes));
  return 1024 + stages * stage + ((kA * BM * nb + 15) & ~15) + (2 * kMaxStages + 3) * sizeof(uint64_t) + 32;
}

}  // namespace dec

namespace {

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encoder() {
  static EncodeTiled fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiled>(ptr);
  }
  return fn;
}

bool encode(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base, const uint64_t* dims,
            const uint64_t* strides_bytes, const uint32_t* box) {
  EncodeTiled fn = encoder();
  if (!fn) return false;
  cuuint64_t d[3], s[2];
  cuuint32_t b[3], es[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) { d[i] = dims[i]; b[i] = box[i]; }
  for (int i = 0; i + 1 < rank; ++i) s[i] = strides_bytes[i];
  return fn(m, dt, rank, const_cast<void*>(base), d, s, b, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int stages_for(bool gate_up, int b_stage_bytes, int nb) {
  for (int s = dec::kMaxStages; s >= 2; --s)
    if (dec::smem_bytes(gate_up, s, b_stage_bytes, nb) <= 227 * 1024) return s;
  return 0;
}

}  // namespace

bool decode_tc_supported(int H, int I, int np, int max_tokens_per_expert, const void* gu_blocks,
                         const void* d_blocks) {
  if (H % 64 || I % 64 || H < dec::BK || I < dec::BK) return false;
  if (np * max_tokens_per_expert > dec::kMaxN) return false;
  if ((reinterpret_cast<uintptr_t>(gu_blocks) | reinterpret_cast<uintptr_t>(d_blocks)) & 31u) return false;
  const int bst = ((np * max_tokens_per_expert + dec::kBoxRows - 1) / dec::kBoxRows) * dec::kBoxRows * dec::BK;
  if (stages_for(true, bst, std::max(H, I) / 32) < 2) return false;
  return encoder() != nullptr;
}

cudaError_t decode_tc_prepare() {
  const int smem = 227 * 1024;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(dec::decode_gemm_kernel<true, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem))) return e;
  if ((e = cudaFuncSetAttribute(dec::decode_gemm_kernel<true, 3>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem))) return e;
  if ((e = cudaFuncSetAttribute(dec::decode_gemm_kernel<false, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem))) return e;
  return cudaFuncSetAttribute(dec::decode_gemm_kernel<false, 3>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
}

size_t decode_tc_sfb_bytes(int E, int K) {
  const int nkt = K / dec::BK + (K % dec::BK ? 1 : 0);
  return static_cast<size_t>(E) * nkt * dec::kSfRecord;
}

cudaError_t launch_split_tokens(int np, const uint16_t* x, const int32_t* perm_token, const int32_t* perm_slot,
                                const int32_t* topk_idx, const int32_t* offsets, int64_t P, int H, int k, float s0,
                                uint8_t* xs, uint8_t* sfb, cudaStream_t st) {
  const int nb = H / 32, nk_full = H / dec::BK, nkt = nk_full + (H % dec::BK ? 1 : 0);
  const int64_t warps = P * nb;
  const unsigned grid = static_cast<unsigned>(cdiv(warps * 32, 256));
  if (np == 1)
    dec::split_tokens_kernel<1><<<grid, 256, 0, st>>>(x, perm_token, perm_slot, topk_idx, offsets, P, H, k, s0,
                                                      xs, sfb, nb, nk_full, nkt);
  else
    dec::split_tokens_kernel<3><<<grid, 256, 0, st>>>(x, perm_token, perm_slot, topk_idx, offsets, P, H, k, s0,
                                                      xs, sfb, nb, nk_full, nkt);
  return cudaGetLastError();
}

// gate_up (gate_up = true): A = gu weights, B = xs (np parts per row), writes xs_out /
// sfb_out for the down GEMM. down: A = d weights, B = xs_out, writes y and the combine.
cudaError_t launch_decode_gemm(bool gate_up, const DecodeGemmArgs& a, cudaStream_t st) {
  using namespace dec;
  const int K = gate_up ? a.H : a.I;
  const int n_out = gate_up ? a.I : a.H;
  const int groups = gate_up ? 2 * a.E : a.E;
  const int np = gate_up ? a.np : a.np_mid;
  const int64_t b_rows = a.P * np;
  const int nb = K / 32, nk_full = K / BK, tail = (K % BK) / 32;
  const int nkt = nk_full + (tail ? 1 : 0);
  const int n_max = np * a.max_tokens_per_expert;
  const int bst = ((n_max + kBoxRows - 1) / kBoxRows) * kBoxRows * BK;
  const int S = stages_for(gate_up, bst, std::max(a.H, a.I) / 32);
  if (S < 2) return cudaErrorInvalidValue;
  CUtensorMap mw, mwt, mx;
  {
    const uint64_t row_bytes = static_cast<uint64_t>(K) / 2;
    const uint64_t dims[3] = {static_cast<uint64_t>(nk_full * BK), static_cast<uint64_t>(n_out),
                              static_cast<uint64_t>(groups)};
    const uint64_t strides[2] = {row_bytes, row_bytes * n_out};
    const uint32_t box[3] = {BK, BM, 1};
    const uint8_t* blocks = gate_up ? a.gu_blocks : a.d_blocks;
    if (!encode(&mw, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 3, blocks, dims, strides, box)) return cudaErrorInvalidValue;
    const uint64_t tdims[3] = {BK, static_cast<uint64_t>(n_out), static_cast<uint64_t>(groups)};
    if (!encode(&mwt, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 3, blocks + (K - BK) / 2, tdims, strides, box))
      return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(b_rows > 0 ? b_rows : 1)};
    const uint64_t strides[1] = {static_cast<uint64_t>(K)};
    const uint32_t box[2] = {BK, kBoxRows};
    if (!encode(&mx, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, gate_up ? a.xs : a.xs_mid, dims, strides, box))
      return cudaErrorInvalidValue;
  }
  Params prm{};
  prm.w_scales = gate_up ? a.gu_scales : a.d_scales;
  prm.bias = gate_up ? a.gu_bias : a.d_bias;
  prm.rows_per_group = n_out;
  prm.rows_total = gate_up ? 2 * a.I : a.H;
  prm.n_out = n_out;
  prm.E = a.E;
  prm.K = K;
  prm.nb = nb;
  prm.nk_full = nk_full;
  prm.tail_steps = tail;
  prm.np = np;
  prm.offsets = a.offsets;
  prm.active = a.active;
  prm.n_active = a.n_active;
  prm.sfb = gate_up ? a.sfb : a.sfb_mid;
  prm.s_in = gate_up ? a.s0 : a.s1_in;
  prm.xs_out = a.xs_mid;
  prm.sfb_out = a.sfb_mid;
  prm.np_out = a.np_mid;
  prm.nb_out = a.I / 32;
  prm.nk_full_out = a.I / BK;
  prm.nkt_out = a.I / BK + (a.I % BK ? 1 : 0);
  prm.s_out = a.s1_quant;
  prm.amax_bits = a.amax_bits;
  prm.y_out = a.y;
  prm.out = a.out;
  prm.topk_idx = a.topk_idx;
  prm.topk_w = a.topk_w;
  prm.inv = a.inv;
  prm.tickets = a.tickets;
  prm.T = a.T;
  prm.k = a.k;
  prm.err = a.err;
  prm.stages = S;
  prm.b_stage_bytes = bst;
  dim3 grid(static_cast<unsigned>((n_out + BM - 1) / BM), static_cast<unsigned>(a.max_active));
  const size_t smem = smem_bytes(gate_up, S, bst, std::max(a.H, a.I) / 32);
  if (np != 1 && np != 3) return cudaErrorInvalidValue;
  if (gate_up && np == 1)
    decode_gemm_kernel<true, 1><<<grid, kThreads, smem, st>>>(mw, mwt, mx, prm);
  else if (gate_up)
    decode_gemm_kernel<true, 3><<<grid, kThreads, smem, st>>>(mw, mwt, mx, prm);
  else if (np == 1)
    decode_gemm_kernel<false, 1><<<grid, kThreads, smem, st>>>(mw, mwt, mx, prm);
  else
    decode_gemm_kernel<false, 3><<<grid, kThreads, smem, st>>>(mw, mwt, mx, prm);
  return cudaGetLastError();
}

}  // namespace mxmoe
