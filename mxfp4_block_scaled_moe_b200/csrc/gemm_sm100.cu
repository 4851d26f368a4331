// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05) with block-scaled
// MXFP4 weights and FP8 E4M3 activations: the prefill path of the W-MXFP4 / A-FP8 layer.
//
// Pages: "quantization_mxfp4" (KerasFormers), As GPT-OSS's native format (gate_up_proj
// (E, 2I, H) and down_proj (E, H, I) as e2m1 blocks + one e8m0 scale per 32 values along
// the contracting dim, biases in full precision); "amd/gpt-oss-20b-MoE-Quant-W-MXFP4-A-
// FP8-KV-FP8", Quantization schemes (FP8 per-tensor activations).
//
// One kernel, two epilogues:
//   gate_up: acc = A1_e . Wgu_e^T on [gate rows n0.., up rows I+n0..]; a = silu(s0*acc_g
//            + b_g) * (s0*acc_u + b_u); A2 = e4m3(a / s1)            (bytes, (P, I))
//   down:    acc = A2_e . Wd_e^T;  y = s1 * acc + b_d                 (fp32, (P, H))
// where A1 / A2 hold the routed rows grouped by expert (offsets[e] .. offsets[e+1]).
//
// MMA: tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale, M = 128, N = 240, K = 32 per
// instruction, fp32 accumulators in tensor memory. A (e4m3) carries unit scales (e8m0
// 127) and its per-tensor scale is applied in the epilogue; B (e2m1) carries the
// checkpoint's e8m0 block scales. Operands arrive by TMA with 128-byte swizzle; the e2m1
// weights use the 4-bit "16 x U4 in 16 bytes" tensor-map type, which spreads each 8 packed
// bytes over 16 bytes of shared memory as the kind::mxf8f6f4 operand layout requires.
// K = 2880 is 22.5 tiles of 128: the last tile reads the final 128 values through a
// second tensor map and issues only its last two K-steps.
//
// Scale factors: two converter warps read the checkpoint's e8m0 bytes of the stage's 4
// k-blocks for the tile's rows (L1-cached loads issued kStages stages ahead) and write them
// in the layout the MMA reads from tensor memory: weight row n at column n/32, lane n%32 of
// every 32-lane quarter, byte j for k-block j. The stage's 8 columns go in with ONE tcgen05.cp
// 128x256b from a 4 KB source that repeats the 32 lanes for each quarter: in the tensor
// pipe a scale copy costs about as much as an MMA whatever its size (measured: 4 MMAs of
// N = 240 take ~550 cycles; adding two 32x128b.warpx4 copies ~880, one 128x256b ~730).
//
// Roles (640 threads, one CTA per SM, persistent over the tile list):
//   warp 0: TMA producer          warp 1: TMEM owner + MMA issuer (one thread)
//   warps 2-3: scale converters (rows 0..127 / 128..255); warp 3 first builds the schedule
//   warps 4..19: epilogue; warp w reads TMEM lane quarter w % 4 and every (w-4)/4-th group
//   of 8 accumulator columns, so each sub-partition runs 4 epilogue warps
// Every mbarrier wait gives up after ~1 s (clock64): the kernel then records MXMOE_ETIMEOUT
// in the error word, lets in-flight copies land, frees its tensor memory and returns.
#include <cuda.h>

#include "common.cuh"
#include "tc_common.cuh"
#include "tmap.h"

namespace mxmoe {
namespace g100 {

using namespace tc;

constexpr int BM = 128;             // rows of A per tile (MMA M)
constexpr int BN = 240;             // MMA N (gate_up: 120 gate + 120 up rows)
constexpr int BK = 128;             // K values per pipeline stage
constexpr int kStages = 4;
constexpr int kEpiWarps = 16;                // 4 per SM sub-partition: hides the epilogue's latency
constexpr int kThreads = 128 + 32 * kEpiWarps;  // warps 0-3 producer/MMA/scales/schedule
constexpr int kAStage = BM * BK;            // 16 KB (e4m3, one byte per value)
constexpr int kBStage = BN * BK;            // 30 KB (e2m1 spread to one byte per value)
constexpr int kSfStage = 4096;              // 128 lanes x 32 bytes: columns 0-3 at 0, 4-7 at 2048
constexpr int kAccCols = 256;               // column stride between the two accumulators
constexpr int kTmemCols = 512;
constexpr int kSfaCol = 240;                // 4 columns of unit A scales (gap after accumulator 0)
constexpr int kSfbCol = 496;                // two 8-column slots of B scales (rows 0..255),
                                            // alternated per stage so the copy of stage s+1
                                            // never overwrites scales stage s still reads

struct Params {
  const uint8_t* b_scales;   // raw e8m0 scales, (groups, rows_per_group, nb)
  const float* bias;         // (E, rows_total)
  const int32_t* offsets;    // (E+1)
  int E;
  int K;                     // contracting length (multiple of 64)
  int nb;                    // K / 32
  int rows_per_group;        // gate_up: I (one half); down: H
  int rows_total;            // bias row length: gate_up 2I, down H
  int n_out;                 // gate_up: I; down: H
  int n_tiles;               // output tiles along N per m-tile
  int nk_full;               // K / 128
  int tail_steps;            // K-steps of 32 in the final partial tile (0 or 2)
  float s_in;                // scale of the A operand (s0 gate_up / s1 down)
  float s_out;               // gate_up: quantization scale s1 of a
  int a_shared;              // 1: every expert reads the same A rows (the dense all-experts
                             // path: A row = row within the expert), 0: A row = grouped row
  uint8_t* a_out;            // gate_up output (P, I) e4m3
  float* y_out;              // down output (P, H) fp32
  int* err;
};

// ---------------------------------------------------------------- tile schedule ---
struct Tile {
  int e, mt, nt, m0, rows;  // expert, m-tile, n-tile, first grouped row, valid rows
};

__device__ __forceinline__ Tile tile_of(int t, const int* prefix, const int32_t* offsets, int E, int n_tiles) {
  int lo = 0, hi = E;  // largest e with prefix[e] <= t
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] <= t) lo = mid; else hi = mid;
  }
  // skip experts with no tiles (equal prefixes)
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

// ------------------------------------------------------------------------ kernel ---
template <bool kGateUp>
__global__ void __launch_bounds__(kThreads, 1)
moe_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                const __grid_constant__ CUtensorMap tmap_bt, Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + kStages * kAStage;
  uint8_t* sSF = sB + kStages * kBStage;
  uint8_t* sSFA = sSF + kStages * kSfStage;       // 512 B of unit scales
  uint64_t* bars = reinterpret_cast<uint64_t*>(sSFA + 512);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* acc_full = bars + 2 * kStages;
  uint64_t* acc_empty = acc_full + 2;
  int* prefix = reinterpret_cast<int*>(acc_empty + 2);           // E + 1
  volatile int* abort_flag = prefix + (p.E + 1);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(prefix + p.E + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bn_rows = kGateUp ? BN / 2 : BN;      // rows per B load (one half for gate_up)
  // The next kernel (down after gate_up) may launch now: its CTAs take the SMs this grid
  // frees and wait for this grid's results only where they read them.
  griddep_launch_dependents();

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 3);     // TMA producer (expect_tx) + the two scale-converter warps
      mbar_init(&empty[s], 1);    // MMA commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kEpiWarps);  // one arrive per epilogue warp
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == 3) {
    // tile schedule: prefix[e] = number of tiles of experts < e
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
    // tensor memory: 512 columns (two 240-column accumulators + scale factors)
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(tmem_holder)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
    // unit A scales (e8m0 127) in the atom layout, then into tensor memory below
    for (int i = lane; i < 128; i += 32) reinterpret_cast<uint32_t*>(sSFA)[i] = 0x7F7F7F7Fu;
    fence_async_smem();
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
      const uint32_t tx = kAStage + (kGateUp ? 2 : 1) * bn_rows * (BK / 2);
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
            // the activation rows are the previous kernel's output: setup and the first
            // weight stage overlap that kernel's tail
            griddep_wait();
            dep_ready = true;
          }
          tma_load_2d(sA + stage * kAStage, &tmap_a, &full[stage], kx, p.a_shared ? tl.m0 - p.offsets[tl.e] : tl.m0);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer -----
    if (lane == 0) {
      tc_fence_after();
      tc_cp_32x128b_x4(tmem + kSfaCol, smem_desc(smem_u32(sSFA), 0, 128, 0));
    }
    __syncwarp();
    int stage = 0;
    uint32_t phase = 0;
    int it = 0;
    const uint32_t idesc0 = idesc_mxf8f6f4(BM, BN);
    for (int t = blockIdx.x; t < total_tiles && !*abort_flag; t += gridDim.x, ++it) {
      const int ab = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      if (!mbar_wait(&acc_empty[ab], acc_phase ^ 1, abort_flag, p.err)) break;
      tc_fence_after();
      const uint32_t dacc = tmem + ab * kAccCols;
      bool ok = true;
      for (int kt = 0; kt < nkt; ++kt) {
        if (!mbar_wait(&full[stage], phase, abort_flag, p.err)) { ok = false; break; }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t sf = smem_u32(sSF + stage * kSfStage);
          const uint32_t sfb = tmem + kSfbCol + 8 * (stage & 1);
          tc_cp_128x256b(sfb, smem_desc(sf, 2048, 128, 0));
          const uint32_t a0 = smem_u32(sA + stage * kAStage), b0 = smem_u32(sB + stage * kBStage);
          const int first = kt < p.nk_full ? 0 : 4 - p.tail_steps;
          for (int kk = first; kk < 4; ++kk) {
            const uint64_t ad = smem_desc(a0 + 32 * kk, 16, 1024, 2);
            const uint64_t bd = smem_desc(b0 + 32 * kk, 16, 1024, 2);
            const uint32_t id = idesc0 | (static_cast<uint32_t>(kk) << 4) | (static_cast<uint32_t>(kk) << 29);
            const uint32_t sel = static_cast<uint32_t>(kk) << 30;
            tc_mma_mxf8f6f4(dacc, ad, bd, id, (tmem + kSfaCol) | sel, sfb | sel,
                            (kt > 0 || kk > first) ? 1u : 0u);
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
    // warp 2 fills columns 0-3 (tile rows 0..127), warp 3 columns 4-7 (rows 128..255);
    // lane l owns rows l, l+32, l+64, l+96 of its half, whose four words sit side by side
    // (byte 16*L + 4*i for tensor-memory lane L = 32*q + l), stored once per quarter q.
    // The scale bytes come straight from the checkpoint's (groups, rows, nb) array through
    // the L1 cache, loaded kStages stages ahead (also across tile boundaries): a stage's 4 bytes
    // of a row are two aligned 16-bit words (nb is even, k-blocks start at multiples of 4).
    const int w2 = warp - 2;
    const int halves = kGateUp ? 2 : 1;
    uint32_t phase = 0;
    // rows of tile t this lane converts; a row outside the tile reads the array's first
    // row and its bit in ok is clear (its words become unit scales at the store)
    auto rows_of = [&](int t, const uint16_t* (&rp)[4], uint32_t& ok) {
      const Tile tl = tile_of(t, prefix, p.offsets, p.E, p.n_tiles);
      const int n0 = tl.nt * bn_rows;
      const int valid = min(bn_rows, p.rows_per_group - n0);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = 128 * w2 + lane + 32 * i;
        const int h = r >= bn_rows ? 1 : 0;
        const int rr = r - h * bn_rows;
        const int group = kGateUp ? 2 * tl.e + h : tl.e;
        const bool in = r < BN && rr < valid && h < halves;
        rp[i] = reinterpret_cast<const uint16_t*>(
            p.b_scales + (in ? (static_cast<int64_t>(group) * p.rows_per_group + n0 + rr) * p.nb : 0));
        ok = (ok & ~(1u << i)) | ((in ? 1u : 0u) << i);
      }
    };
    // the stage's two 16-bit words of each row, kept apart until the store (combining
    // them here would wait for the loads)
    auto load = [&](const uint16_t* const (&rp)[4], int kt, uint32_t (&wv)[8]) {
      const int kw = (kt < p.nk_full ? 4 * kt : p.nb - 4) >> 1;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        wv[2 * i] = __ldg(rp[i] + kw);
        wv[2 * i + 1] = __ldg(rp[i] + kw + 1);
      }
    };
    // A ring of kStages register sets, unrolled so that no set is ever moved: the loads of
    // a stage are issued kStages stages before its store (a register move would wait for
    // them at once).
    int lt = blockIdx.x, lkt = 0;   // next stage to load
    int st = blockIdx.x, skt = 0;   // next stage to store
    const uint16_t* rp[4] = {nullptr, nullptr, nullptr, nullptr};
    uint32_t rows_ok = 0u;
    uint32_t buf[kStages][8] = {};
    uint32_t buf_ok[kStages] = {};   // the rows_ok of each set's tile
    auto load_next = [&](uint32_t (&wv)[8]) -> uint32_t {
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
        uint32_t wq4[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          wq4[i] = ((buf_ok[j] >> i) & 1u) ? ((buf[j][2 * i] & 0xFFFFu) | (buf[j][2 * i + 1] << 16)) : 0x7F7F7F7Fu;
        const uint4 wq = make_uint4(wq4[0], wq4[1], wq4[2], wq4[3]);
        uint8_t* dst = sSF + j * kSfStage + 2048 * w2 + 16 * lane;
#pragma unroll
        for (int q = 0; q < 4; ++q) *reinterpret_cast<uint4*>(dst + 512 * q) = wq;
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
    const int q = warp & 3;                 // tensor-memory lane quarter of this warp
    const int slice = (warp - 4) >> 2;      // which groups of 8 columns it takes
    constexpr int kSlices = kEpiWarps / 4;
    const int row = 32 * q + lane;          // tile row = TMEM lane
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
        // 15 groups of 8 gate columns (and the 8 matching up columns), round-robin over slices
        for (int c0 = 8 * slice; c0 < bn_rows; c0 += 8 * kSlices) {
          uint32_t g[8], u[8];
          tc_ld_32x32b_x8(tbase + c0, g);
          tc_ld_32x32b_x8(tbase + bn_rows + c0, u);
          // n_out % 8 == 0: a group of 8 columns is wholly inside or wholly past the tile
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
          uint32_t lo = 0, hi = 0;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float gv = __fadd_rn(__fmul_rn(p.s_in, __uint_as_float(g[i])), bg[i]);
            const float uv = __fadd_rn(__fmul_rn(p.s_in, __uint_as_float(u[i])), bu[i]);
            const uint32_t qb = act_quant_e4m3(silu_mul(gv, uv), p.s_out);
            if (i < 4) lo |= qb << (8 * i); else hi |= qb << (8 * (i - 4));
          }
          if (valid && live)
            *reinterpret_cast<uint2*>(p.a_out + pos * p.n_out + n0 + c0) = make_uint2(lo, hi);
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
          for (int i = 0; i < 8; ++i) o[i] = __fadd_rn(__fmul_rn(p.s_in, __uint_as_float(v[i])), bb[i]);
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
    // let copies already issued land before the CTA's shared memory goes away
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
  return 1024 + kStages * (kAStage + kBStage + kSfStage) + 512 + (2 * kStages + 4) * sizeof(uint64_t) +
         (E + 3) * sizeof(int) + 16;
}

}  // namespace g100

// ---------------------------------------------------------------- host side -------

// Whether the tcgen05 path can run these shapes/pointers (else the register-dequant path).
bool tc_gemm_supported(int H, int I, const void* gu_blocks, const void* d_blocks, const void* gu_scales,
                       const void* d_scales) {
  if (H % 64 || I % 64) return false;          // 16 x U4 rows: K/2 bytes a multiple of 32
  if (H < g100::BK || I < g100::BK) return false;
  if ((reinterpret_cast<uintptr_t>(gu_blocks) | reinterpret_cast<uintptr_t>(d_blocks)) & 31u) return false;
  // the scale converters read the e8m0 bytes as 16-bit words
  if ((reinterpret_cast<uintptr_t>(gu_scales) | reinterpret_cast<uintptr_t>(d_scales)) & 1u) return false;
  return tmap_available();
}

cudaError_t tc_gemm_prepare(int E) {
  const size_t smem = g100::smem_bytes(E);
  cudaError_t e = cudaFuncSetAttribute(g100::moe_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e) return e;
  return cudaFuncSetAttribute(g100::moe_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(smem));
}


// a: grouped activation rows (P_rows, K) e4m3 (a_shared: the T rows every expert reads);
// blocks/scales: (E, rows_total, K/2) and
// (E, rows_total, K/32); gate_up: rows_total = 2I, n_out = I; down: rows_total = n_out = H.
cudaError_t launch_tc_gemm(bool gate_up, const uint8_t* a, int64_t P_rows, int K, const uint8_t* blocks,
                           const uint8_t* scales, const float* bias, int E, int n_out, const int32_t* offsets,
                           float s_in, float s_out, uint8_t* a_out, float* y_out, int* err, int sms,
                           cudaStream_t st, bool a_shared) {
  using namespace g100;
  const int rows_per_group = n_out;          // one half of gate_up, or all of down
  const int groups = gate_up ? 2 * E : E;
  const int bn_rows = gate_up ? BN / 2 : BN;
  CUtensorMap ma, mb, mbt;
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(P_rows > 0 ? P_rows : 1)};
    const uint64_t strides[1] = {static_cast<uint64_t>(K)};
    const uint32_t box[2] = {BK, BM};
    if (!tmap_encode(&ma, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, a, dims, strides, box)) return cudaErrorInvalidValue;
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
  prm.bias = bias;
  prm.offsets = offsets;
  prm.E = E;
  prm.K = K;
  prm.nb = K / 32;
  prm.rows_per_group = rows_per_group;
  prm.rows_total = gate_up ? 2 * n_out : n_out;
  prm.n_out = n_out;
  prm.n_tiles = (n_out + bn_rows - 1) / bn_rows;
  prm.nk_full = K / BK;
  prm.tail_steps = (K % BK) / 32;
  prm.s_in = s_in;
  prm.s_out = s_out;
  prm.a_shared = a_shared ? 1 : 0;
  prm.a_out = a_out;
  prm.y_out = y_out;
  prm.err = err;
  // programmatic dependent launch: the kernel starts during its predecessor (the FP8 cast
  // and scatter, or gate_up for down) and waits for it only before reading its output
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
  if (gate_up) return cudaLaunchKernelEx(&cfg, moe_gemm_kernel<true>, ma, mb, mbt, prm);
  return cudaLaunchKernelEx(&cfg, moe_gemm_kernel<false>, ma, mb, mbt, prm);
}

}  // namespace mxmoe
