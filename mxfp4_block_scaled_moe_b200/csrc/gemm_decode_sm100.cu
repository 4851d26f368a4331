// Routed expert GEMMs for small batches on the tensor cores (tcgen05.mma kind::mxf4
// block_scale): both operands are packed e2m1 with e8m0 block scales, so TMA copies the
// checkpoint's MXFP4 bytes into shared memory as they are and the tensor core decodes the
// nibbles and applies the scales. This is the decode path of "quantization_mxfp4"
// (KerasFormers), As GPT-OSS's native format: only the routed experts' blocks are read,
// once per layer.
//
// Operands of one expert e (or one group of at most 56 of its routed rows):
//   A = two 128-row weight tiles per stage, each its own MMA and accumulator (gate_up: 128
//       gate rows and the 128 matching up rows; down: 256 consecutive rows of down_proj),
//       with the checkpoint's e8m0 scales; both share the stage's B tile, so a stage moves
//       32 KB of weights for one B load and one set of B-scale copies;
//   B = the routed token rows as four MXFP4 "parts" each: p1 = e2m1(x / 2^s1), p2 the same
//       on the residual x - p1, and so on, each s chosen from the largest residual of its
//       32-value block so that nothing saturates. Every part removes about three bits of
//       the residual, and four parts change a 2880-long dot product by about 1.5e-4 of
//       the largest output; a block scale keeps that bound when one channel is 1000x the
//       others (a row-wide scale would not: the other values would keep only the bits
//       below the outlier's). The per-tensor FP8 path splits the e4m3 value of x / s0 the
//       same way.
//   D = 128 x N fp32 in tensor memory, N = 4 * rows rounded up to 16; the epilogue adds a
//       token's four columns.
// Why not FP8 tokens against FP4 weights (kind::mxf8f6f4): a block-scaled MMA costs the
// tensor pipe about 100 cycles whatever N is, and kind::mxf4 covers K = 64 per
// instruction instead of 32, so it moves twice the weight bytes per instruction; with
// K = 32 the pipe, not HBM, bounded decode. The packed operands also halve the shared
// memory per weight byte (no 8-bit containers), which doubles the bytes in flight.
//
// Persistent schedule. One CTA per SM walks the work units u = blockIdx.x, +gridDim.x, ...
// of the list (row group, unit rows, K split; a unit is 128 rows of gate with the matching
// 128 of up, or 256 rows of down_proj), so the TMA ring stays full across unit boundaries
// and two TMEM accumulator slots let the epilogue of one unit overlap the MMAs of the
// next. Few units are split along K so that every SM streams: each
// split writes its fp32 partial accumulator, and the last split of a 32-row slice (an
// atomic ticket) adds the partials in split order, so results do not depend on which CTA
// finishes last.
//
// The gate_up epilogue applies bias + SwiGLU and writes a directly as the down GEMM's B
// operand (its 32-row warp is exactly one 32-value block of the down contraction, so a
// part's block amax stays inside the warp: after a four-row transpose through shared
// memory it is three xor-shuffles); the down epilogue writes y (fp32), which the combine
// kernel reduces per token.
//
// Scale-factor records of the B operand ("SFB"), one of 5 KB per (row group, 256-deep
// stage). Tensor memory holds a 128-wide k-tile's scales of B rows 0..127 in four columns
// (column i, lane 32q + l: the four k-block scales of row 32i + l, the same for the four
// 32-lane quarters q). The first 4 KB are the tcgen05.cp.128x256b source of the stage's
// two k-tiles for rows 0..127 (k-tile kt's 16 bytes of lane L at 2048 kt + 16 L): one
// copy per stage for B tiles of at most 128 rows. Wider tiles (up to 224 rows) take the
// four 32x128b.warpx4 atoms instead: rows 0..127 of k-tile kt from the first 512 bytes of
// its 2 KB, rows 128..255 from the 512 bytes at 4096 + 512 kt. Row r < 128, k-block j of
// k-tile kt: bytes 2048 kt + 512 q + 16 (r % 32) + 4 (r / 32) + j for q = 0..3; row
// r >= 128: byte 4096 + 512 kt + 16 (r % 32) + 4 ((r - 128) / 32) + j.
#include <climits>

#include <cuda.h>
#include <cuda_fp4.h>

#include "common.cuh"
#include "launchers.h"
#include "mx_parts.cuh"
#include "tc_common.cuh"
#include "tmap.h"

namespace mxmoe {
namespace dec {

using namespace tc;

constexpr int BM = 128;
constexpr int BKS = 256;           // K per pipeline stage (128 packed bytes per row)
constexpr int kRowBytes = 128;     // packed bytes of a row per stage
constexpr int kParts = 4;          // e2m1 parts per token row
constexpr int kGroupRows = 56;     // routed rows per row group: N = 4 * 56 = 224 at most
constexpr int kMaxN = kParts * kGroupRows;
constexpr int kThreads = 256;      // warp 0 TMA, 1 MMA, 2-3 A-scale converters, 4-7 epilogue
constexpr int kEpiWarps = 4;
constexpr int kMaxStages = 10;
constexpr int kTmemCols = 512;
constexpr int kSlot1 = 240;        // accumulator slot 1 starts here (slot 0 at column 0)
constexpr int kBigCols = 112;      // gate_up units wider than this take both slots
constexpr int kSfaCol = 480;       // A scales: tile h, atom a at 480 + 8h + 4a
constexpr int kSfbCol = 496;       // B scales: tiles <= 128 rows: k-tile t at 496 + 4t;
                                   // wider: k-tile t, atom b at 496 + 8t + 4b
constexpr int kSfRecord = 5120;    // B scale record per (row group, 256-deep stage)
constexpr int kSfNarrow = 4096;    // its part that B tiles of at most 128 rows use
// Per stage: the A (weight) scales of each tile as one 128x256b tcgen05.cp source (4 KB:
// the two 128-wide k-tiles' atoms, repeated for the four 32-lane quarters), then the
// stage's B scale record.
__host__ __device__ constexpr int sf_stage_bytes(int kA) { return kA * 4096 + kSfRecord; }
constexpr int kSfStageMax = sf_stage_bytes(2);
constexpr int kMaxE = 256;
constexpr int kMaxGrp = kDecodeMaxGroups;
constexpr int kMaxSplit = 8;
constexpr int kMaxTopK = 8;
constexpr int kSmemBytes = 227 * 1024;

// Store the e8m0 byte v of B row r (< 256), k-block j of k-tile ktl (0 or 1) of a stage
// into the stage's record (every copy of it: four for rows below 128).
__device__ __forceinline__ void sfb_store(uint8_t* rec, int r, int ktl, int j, uint8_t v) {
  if (r < 128) {
    uint8_t* b = rec + 2048 * ktl + 16 * (r & 31) + 4 * (r >> 5) + j;
#pragma unroll
    for (int q = 0; q < 4; ++q) b[512 * q] = v;
  } else {
    rec[4096 + 512 * ktl + 16 * (r & 31) + 4 * ((r - 128) >> 5) + j] = v;
  }
}

struct Params {
  // A: weights
  const uint8_t* w_scales;   // (groups, rows_per_group, nb) e8m0
  const float* bias;         // (E, rows_total)
  int rows_per_group;        // gate_up: I (a half); down: H
  int rows_total;            // 2I or H
  int n_out;                 // I or H
  // shapes
  int E, K, nb, nst, n_m, box_rows, split_cap, max_chunks;
  int smem_bytes;            // dynamic shared memory of the launch
  int64_t P;
  const int32_t* offsets;
  const int32_t* active;
  const int32_t* n_active;
  const uint8_t* sfb;        // B scale records [E][max_chunks][nst][kSfRecord]
  float s_in;                // per-tensor scale of the B operand (FP8) or 1
  // gate_up outputs (the down GEMM's B operand)
  uint8_t* xs_out;           // (P * 4, I / 2) packed e2m1 parts
  uint8_t* sfb_out;          // [E][max_chunks][2*nst_out][1024]
  int nst_out;
  float s_out;               // FP8: static scale of a; 0: bf16 intermediate
  // down output
  float* y_out;              // (P, H) fp32
  // split-K
  float* part;               // [split][planes][P * 4][n_out] fp32 partial accumulators
                             // (gate_up: planes gate and up; down: one, rows as they are)
  unsigned* split_tickets;   // [kMaxGrp][n_m][4], zero between calls
  int* err;
};

// Per-CTA schedule, in shared memory, identical in every CTA: the row groups (an expert's
// routed rows in chunks of at most kGroupRows) and the derived unit count.
struct Sched {
  int n_active, n_grp, nsplit, units, stages, stage_bytes;
  int act[kMaxE];
  int off[kMaxE + 1];
  int g_e[kMaxGrp];          // expert of the group
  int g_c[kMaxGrp];          // chunk index within the expert
  int g_off[kMaxGrp];        // first routed row (expert-grouped order)
  int g_n[kMaxGrp];          // rows in the group
};

struct Unit {
  int g, e, c, m, s, k0, k1, off, j0, n, cols, ncols, nbox;
};

__device__ __forceinline__ Unit unit_at(const Sched& sc, const Params& p, int u) {
  Unit w;
  w.s = u % sc.nsplit;
  const int t = u / sc.nsplit;
  w.m = t % p.n_m;
  w.g = t / p.n_m;
  w.e = sc.g_e[w.g];
  w.c = sc.g_c[w.g];
  w.off = sc.g_off[w.g];
  w.j0 = w.c * kGroupRows;   // first row of the group within its expert
  w.n = sc.g_n[w.g];
  w.k0 = w.s * p.nst / sc.nsplit;
  w.k1 = (w.s + 1) * p.nst / sc.nsplit;
  w.cols = kParts * w.n;
  w.ncols = max(16, (w.cols + 15) & ~15);
  w.nbox = (w.cols + p.box_rows - 1) / p.box_rows;
  return w;
}

// Byte offsets of the fixed part of the shared-memory layout (host and device agree).
__host__ __device__ constexpr int sched_bytes() { return (static_cast<int>(sizeof(Sched)) + 127) & ~127; }
__host__ __device__ constexpr int bar_bytes() { return 256; }
constexpr int kEpiStageBytes = 512;   // per epilogue warp: 4 rows x 32 fp32 values
__host__ __device__ constexpr int epi_stage_offset() { return sched_bytes() + bar_bytes(); }
__host__ __device__ constexpr int ring_offset() {
  return (epi_stage_offset() + kEpiWarps * kEpiStageBytes + 1023) & ~1023;
}
__host__ __device__ inline int stage_bytes_for(int kA, int b_rows) {
  return ((kA * BM * kRowBytes + b_rows * kRowBytes) + 1023) & ~1023;
}

// ------------------------------------------------------------------- epilogue pieces --
// Accumulator columns of 8 rows (kParts per row, row-major) for this warp's 32 lanes.
// Every index is static, so the tcgen05.ld destinations stay in registers until the wait
// that makes them valid.
template <bool kGateUp>
__device__ __forceinline__ void read_tmem8(uint32_t tg, uint32_t tu, int j0, float (&vg)[8 * kParts],
                                           float (&vu)[8 * kParts]) {
  uint32_t g[kParts][8], u[kParts][8];
#pragma unroll
  for (int c = 0; c < kParts; ++c) {
    tc_ld_32x32b_x8(tg + kParts * j0 + 8 * c, g[c]);
    if (kGateUp) tc_ld_32x32b_x8(tu + kParts * j0 + 8 * c, u[c]);
  }
#pragma unroll
  for (int c = 0; c < kParts; ++c) {
    tc_wait_ld(g[c]);
    if (kGateUp) tc_wait_ld(u[c]);
  }
#pragma unroll
  for (int f = 0; f < 8 * kParts; ++f) {
    vg[f] = __uint_as_float(g[f >> 3][f & 7]);
    vu[f] = kGateUp ? __uint_as_float(u[f >> 3][f & 7]) : 0.0f;
  }
}

// Address of the fp32 partial of (split s, accumulator h, global column c, row).
__device__ __forceinline__ float* part_at(const Params& p, int planes, int s, int h, int64_t c, int row) {
  return p.part + ((static_cast<int64_t>(s) * planes + h) * (p.P * kParts) + c) * p.n_out + row;
}

// Sum a row's kParts part columns (in part order) for the 8 rows of a group.
__device__ __forceinline__ void sum_parts(const float (&v)[8 * kParts], float (&s)[8]) {
#pragma unroll
  for (int jj = 0; jj < 8; ++jj) {
    float a = 0.0f;
#pragma unroll
    for (int pp = 0; pp < kParts; ++pp) a += v[kParts * jj + pp];
    s[jj] = a;
  }
}

// gate_up: bias, SwiGLU and the down GEMM's B operand for rows j0 .. j0+7 of the unit's
// group (gs / us: the accumulators summed over a row's parts, before the per-tensor
// scale; lane = intermediate index within the warp's 32-value block of the down
// contraction). The intermediate a = silu(g) * u is rounded as the layer defines it
// (e4m3(a / s1) with FP8 activations, else bf16); silu uses the fast exponential and
// division (a few ulp, far inside the layer tolerance; branch-free, so the eight rows'
// chains overlap). It is then written as kParts e2m1 parts, part p the residual of the
// parts before it rounded to nearest-even at the scale 2^s (s: the smallest with
// max|residual| / 2^s <= 6 over the 32-value block). The warp first transposes four
// rows at a time through its 512-byte shared staging area so that each lane holds four
// consecutive values of one row: a block maximum is then three shuffles, and a lane's
// four codes leave as one 16-bit store (even value in the low nibble).
// dry: the same instructions with every global store masked off (warms the instruction
// cache). Not inlined, so that the warm-up call and the real ones run the same code.
__device__ __noinline__ void finish_gate_up(uint8_t* xs_out, uint8_t* sfb_out, float* stage, int n_out, int nst_out,
                                            int max_chunks, float s_in, float s_out, int e, int c, int off, int n,
                                            int j0, const float (&gs)[8], const float (&us)[8], float bg, float bu,
                                            int row, int lane, bool dry) {
  const int kb = row >> 5;   // the warp's 32 rows: one 32-value block of the down contraction
  const int nv = min(8, n - j0);
  uint8_t* rec = sfb_out + ((static_cast<int64_t>(e) * max_chunks + c) * nst_out + (kb >> 3)) * kSfRecord;
  const int64_t row_bytes = n_out / 2;
  float a[8];
#pragma unroll
  for (int jj = 0; jj < 8; ++jj) {
    const float gv = __fadd_rn(__fmul_rn(s_in, gs[jj]), bg);
    const float uv = __fadd_rn(__fmul_rn(s_in, us[jj]), bu);
    const float v = __fmul_rn(__fdividef(gv, 1.0f + __expf(-gv)), uv);
    a[jj] = s_out > 0.0f ? e4m3_to_f32(act_quant_e4m3(v, s_out)) : bf16_bits_to_f32(f32_to_bf16_bits_rn(v));
  }
  const int j = lane >> 3, sub = lane & 7;   // after the transpose: row p0 + j, values 4 sub .. 4 sub + 3
#pragma unroll
  for (int p0 = 0; p0 < 8; p0 += 4) {
    if (p0 >= nv) break;
    __syncwarp();   // the previous pass has read the staging area
#pragma unroll
    for (int t = 0; t < 4; ++t) stage[32 * t + lane] = a[p0 + t];
    __syncwarp();
    const float4 v4 = *reinterpret_cast<const float4*>(stage + 32 * j + 4 * sub);
    float v[4] = {v4.x, v4.y, v4.z, v4.w};
    const bool mine = p0 + j < nv && !dry;
    uint8_t* dst = xs_out + (static_cast<int64_t>(off + j0 + p0 + j) * kParts) * row_bytes + 16 * kb + 2 * sub;
#pragma unroll 1
    for (int pp = 0; pp < kParts; ++pp) {
      float m = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
      const int sc = e2m1_part_exponent(m);
      const float down = pow2f(-sc), up = pow2f(sc);
      const uint32_t b0 = __nv_cvt_float2_to_fp4x2(make_float2(v[0] * down, v[1] * down), __NV_E2M1, cudaRoundNearest);
      const uint32_t b1 = __nv_cvt_float2_to_fp4x2(make_float2(v[2] * down, v[3] * down), __NV_E2M1, cudaRoundNearest);
      const __half2_raw h0 = __nv_cvt_fp4x2_to_halfraw2(static_cast<__nv_fp4x2_storage_t>(b0), __NV_E2M1);
      const __half2_raw h1 = __nv_cvt_fp4x2_to_halfraw2(static_cast<__nv_fp4x2_storage_t>(b1), __NV_E2M1);
      // the residual update is exact: a part value has two significant bits, its scale is a power of two
      v[0] -= __half2float(__half(__half_raw{h0.x})) * up;
      v[1] -= __half2float(__half(__half_raw{h0.y})) * up;
      v[2] -= __half2float(__half(__half_raw{h1.x})) * up;
      v[3] -= __half2float(__half(__half_raw{h1.y})) * up;
      if (mine) {
        *reinterpret_cast<uint16_t*>(dst + pp * row_bytes) = static_cast<uint16_t>(b0 | (b1 << 8));
        if (sub == 0) sfb_store(rec, kParts * (j0 + p0 + j) + pp, (kb >> 2) & 1, kb & 3, static_cast<uint8_t>(sc + 127));
      }
    }
  }
  __syncwarp();   // the staging area is reused by the next call
}

// down: y = s_in * acc + bias for rows j0 .. j0+7 of the unit's group.
__device__ __forceinline__ void finish_down(const Params& p, const Unit& w, int j0, const float (&ys)[8], float bd,
                                            int row) {
#pragma unroll
  for (int jj = 0; jj < 8; ++jj)
    if (j0 + jj < w.n)
      p.y_out[static_cast<int64_t>(w.off + j0 + jj) * p.n_out + row] = __fadd_rn(__fmul_rn(p.s_in, ys[jj]), bd);
}

// ---------------------------------------------------------------------- the kernel --
template <bool kGateUp>
__global__ void __launch_bounds__(kThreads, 1)
decode_gemm_kernel(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_x, Params p) {
  constexpr int kA = 2;                       // A tiles (accumulators) per unit
  constexpr int kPlanes = kGateUp ? 2 : 1;    // planes of the split-K partials
  constexpr int kUnitRows = kGateUp ? BM : 2 * BM;   // output rows a unit covers
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Sched& sc = *reinterpret_cast<Sched*>(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + sched_bytes());
  uint64_t* full = bars;                       // [kMaxStages]
  uint64_t* empty = bars + kMaxStages;         // [kMaxStages]
  uint64_t* acc_full = bars + 2 * kMaxStages;  // [2]
  uint64_t* acc_empty = acc_full + 2;          // [2]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(acc_empty + 2);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acc_empty + 2) + 1;
  uint8_t* ring = smem + ring_offset();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // The next kernel (down after gate_up) may launch now: its CTAs take the SMs this grid
  // leaves free or frees, and wait for this grid's results only where they read them.
  griddep_launch_dependents();
  if (threadIdx.x == 0) {
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&map_w)) : "memory");
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&map_x)) : "memory");
    for (int s = 0; s < kMaxStages; ++s) {
      mbar_init(&full[s], 1 + kA);   // TMA producer (expect_tx) + one scale converter per A tile
      mbar_init(&empty[s], 1);
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
  for (int i = threadIdx.x; i <= p.E; i += blockDim.x) sc.off[i] = p.offsets[i];
  for (int i = threadIdx.x; i < p.E; i += blockDim.x) sc.act[i] = p.active[i];
  if (threadIdx.x == 0) sc.n_active = *p.n_active;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) {
    // row groups: an exclusive scan of the active experts' chunk counts, 32 at a time
    const int na = min(max(sc.n_active, 0), p.E);
    int base = 0, maxcols = 0;
    bool fits = true;
    for (int i0 = 0; i0 < na; i0 += 32) {
      const int i = i0 + lane;
      int e = 0, off = 0, n_e = 0, nch = 0;
      if (i < na) {
        e = sc.act[i];
        off = sc.off[e];
        n_e = sc.off[e + 1] - off;
        nch = (n_e + kGroupRows - 1) / kGroupRows;
      }
      int incl = nch;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (nch > p.max_chunks) fits = false;
      for (int c = 0, g = base + incl - nch; c < nch; ++c, ++g) {
        const int n = min(kGroupRows, n_e - c * kGroupRows);
        if (g < kMaxGrp) {
          sc.g_e[g] = e;
          sc.g_c[g] = c;
          sc.g_off[g] = off + c * kGroupRows;
          sc.g_n[g] = n;
        }
        maxcols = max(maxcols, kParts * n);
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) maxcols = max(maxcols, __shfl_xor_sync(0xffffffffu, maxcols, o));
    fits = __all_sync(0xffffffffu, fits) && base <= kMaxGrp;
    if (lane == 0) {
      const int ng = base;
      sc.n_grp = ng;
      const int ncols_max = max(16, (maxcols + 15) & ~15);
      const int nbox_max = (maxcols + p.box_rows - 1) / p.box_rows;
      const int b_rows = max(ncols_max, nbox_max * p.box_rows);
      sc.stage_bytes = stage_bytes_for(kA, b_rows);
      const int avail = static_cast<int>((smem_raw + p.smem_bytes) - ring);
      sc.stages = min(kMaxStages, avail / (sc.stage_bytes + sf_stage_bytes(kA)));
      // K split: fewest stages on the busiest CTA, counting about four stages for each
      // split unit's partial write, ticket and the finisher's reduction (measured: at one
      // token, three splits of four stages instead of one unit of twelve made gate_up
      // slower, 39.7 against 26.7 us)
      const int tiles = ng * p.n_m, G = gridDim.x;
      int best = 1, best_cost = INT_MAX;
      for (int s = 1; s <= min(p.split_cap, p.nst); ++s) {
        const int per = (tiles * s + G - 1) / G;
        const int cost = per * ((p.nst + s - 1) / s) + (s > 1 ? 4 * per : 0);
        if (cost < best_cost) { best_cost = cost; best = s; }
      }
      sc.nsplit = best;
      sc.units = tiles * best;
      if (!fits || sc.stages < 2) {   // the host's checks exclude both; never expected
        set_device_error(p.err, MXMOE_EUNSUPPORTED);
        sc.units = 0;
      }
    }
  }
  __syncthreads();
  const uint32_t tmem = *tmem_holder;
  const int S = sc.stages;
  auto sA = [&](int s, int h) { return ring + s * sc.stage_bytes + h * BM * kRowBytes; };
  auto sB = [&](int s) { return ring + s * sc.stage_bytes + kA * BM * kRowBytes; };
  uint8_t* sf_base = ring + S * sc.stage_bytes;
  constexpr int kSfStage = sf_stage_bytes(kA);
  auto sSFA = [&](int s, int h) { return sf_base + s * kSfStage + h * 4096; };
  auto sSFB = [&](int s) { return sf_base + s * kSfStage + kA * 4096; };
  auto n_ksteps = [&](int kst) { return min(4, (p.K - BKS * kst + 63) / 64); };

  if (warp == 0) {
    // ---------------------------------------------------------------- producer -----
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      bool dep_ready = false;
      for (int u = blockIdx.x; u < sc.units && ok; u += gridDim.x) {
        const Unit w = unit_at(sc, p, u);
        // B scales: the stage's record (its first 4 KB for B tiles of at most 128 rows)
        const uint32_t sfb_bytes = w.ncols > 128 ? kSfRecord : kSfNarrow;
        const uint32_t tx = kA * BM * kRowBytes + w.nbox * p.box_rows * kRowBytes + sfb_bytes;
        const uint8_t* rec = p.sfb + (static_cast<int64_t>(w.e) * p.max_chunks + w.c) * p.nst * kSfRecord;
        for (int kst = w.k0; kst < w.k1; ++kst) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[stage], tx);
          // gate_up: rows m*128.. of gate (matrix 2e) and up (2e+1); down: rows m*256 .. +255
          tma_load_3d(sA(stage, 0), &map_w, &full[stage], kRowBytes * kst, w.m * kUnitRows, kGateUp ? 2 * w.e : w.e);
          if (!dep_ready) {
            // the token operand and its scales are the previous kernel's output: everything
            // before this point (setup, the first weight stage, the scale converters' start)
            // overlaps that kernel's tail
            griddep_wait();
            dep_ready = true;
          }
          for (int b = 0; b < w.nbox; ++b)
            tma_load_2d(sB(stage) + b * p.box_rows * kRowBytes, &map_x, &full[stage], kRowBytes * kst,
                        kParts * w.off + b * p.box_rows);
          bulk_g2s(sSFB(stage), rec + static_cast<int64_t>(kst) * kSfRecord, sfb_bytes, &full[stage]);
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------------------- MMA -----
    int stage = 0;
    uint32_t phase = 0;
    uint32_t use0 = 0u, use1 = 0u;   // completed uses of each accumulator slot
    int nxt = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < sc.units && ok; u += gridDim.x) {
      const Unit w = unit_at(sc, p, u);
      const bool big = w.ncols > kBigCols;
      const int slot = big ? 0 : nxt;
      if (big) {
        ok = mbar_wait(&acc_empty[0], (use0 & 1u) ^ 1u, abort_flag, p.err) &&
             mbar_wait(&acc_empty[1], (use1 & 1u) ^ 1u, abort_flag, p.err);
      } else {
        ok = mbar_wait(&acc_empty[slot], ((slot ? use1 : use0) & 1u) ^ 1u, abort_flag, p.err);
      }
      if (!ok) break;
      tc_fence_after();
      const uint32_t dg = big ? 0u : static_cast<uint32_t>(slot * kSlot1);
      const uint32_t du = big ? static_cast<uint32_t>(kSlot1) : dg + static_cast<uint32_t>(w.ncols);
      const uint32_t id0 = idesc_mxf4(BM, w.ncols);
      const bool wide = w.ncols > 128;   // B rows past 128: per-k-tile atoms, 8 columns a k-tile
      const int sfb_step = wide ? 8 : 4;  // tensor-memory columns of B scales per k-tile
      for (int kst = w.k0; kst < w.k1; ++kst) {
        if (!mbar_wait(&full[stage], phase, abort_flag, p.err)) { ok = false; break; }
        tc_fence_after();
        if (lane == 0) {
          const int nks = n_ksteps(kst);
          const int nkt = (nks + 1) >> 1;   // 128-wide k-tiles this stage uses
          // each tile's weight scales for both k-tiles: 8 columns in one copy (a scale copy
          // costs the tensor pipe about as much as an MMA whatever its size)
#pragma unroll
          for (int h = 0; h < kA; ++h)
            tc_cp_128x256b(tmem + kSfaCol + 8 * h, smem_desc(smem_u32(sSFA(stage, h)), 2048, 128, 0));
          if (!wide) {
            tc_cp_128x256b(tmem + kSfbCol, smem_desc(smem_u32(sSFB(stage)), 2048, 128, 0));
          } else {
            for (int t = 0; t < nkt; ++t) {
              tc_cp_32x128b_x4(tmem + kSfbCol + 8 * t, smem_desc(smem_u32(sSFB(stage) + 2048 * t), 0, 128, 0));
              tc_cp_32x128b_x4(tmem + kSfbCol + 8 * t + 4,
                               smem_desc(smem_u32(sSFB(stage) + 4096 + 512 * t), 0, 128, 0));
            }
          }
          const uint32_t b0 = smem_u32(sB(stage));
          for (int sk = 0; sk < nks; ++sk) {
            const int t = sk >> 1;
            const uint32_t sfid = static_cast<uint32_t>(sk & 1) * 2u;
            const uint32_t id = id0 | (sfid << 4) | (sfid << 29);
            const uint32_t sel = sfid << 30;
            const uint64_t bd = smem_desc(b0 + 32 * sk, 16, 1024, 2);
            const uint32_t acc = (kst > w.k0 || sk > 0) ? 1u : 0u;
#pragma unroll
            for (int h = 0; h < kA; ++h) {
              const uint64_t ad = smem_desc(smem_u32(sA(stage, h)) + 32 * sk, 16, 1024, 2);
              tc_mma_mxf4(tmem + (h ? du : dg), ad, bd, id, (tmem + kSfaCol + 8 * h + 4 * t) | sel,
                          (tmem + kSfbCol + sfb_step * t) | sel, acc);
            }
          }
          tc_commit(&empty[stage]);
        }
        __syncwarp();
        if (++stage == S) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
      if (lane == 0) {
        tc_commit(&acc_full[slot]);
        if (big) tc_commit(&acc_full[1]);
      }
      __syncwarp();
      if (big) {
        ++use0;
        ++use1;
        nxt = 0;
      } else {
        if (slot) ++use1; else ++use0;
        nxt ^= 1;
      }
    }
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------ A (weight) scale converters -----
    const int h = warp - 2;   // gate_up: 0 gate rows, 1 up rows; down: the unit's first / second 128 rows
    if (h < kA) {
      // lane l owns rows l, l+32, l+64, l+96 of the tile; a stage's 8 scale bytes of a row
      // are four aligned 16-bit words (nb is even). They are loaded kRing stages ahead
      // into an unrolled ring of register sets (never moved, always from a valid address,
      // with a mask of the words that exist beside them, and combined only at the store,
      // so no instruction waits for them before that) and stored as the 128x256b copy
      // source: k-tile 0's word of row 32i + l at 16*L + 4*i, k-tile 1's at 2048 + 16*L + 4*i,
      // for each tensor-memory lane L = 32*q + l.
      // one set: each unrolled copy of the loop body is more code fetched cold at every
      // launch, and after a unit's first stages the rows' scale bytes hit L1 (measured on one
      // B200, layer forward at T = 1 / 8 / 64: one set 98 / 151 / 190 us, two 107 / 157 /
      // 196, three 110 / 161 / 201, five 18 us slower than three)
      constexpr int kRing = 1;
      int stage = 0;
      uint32_t phase = 0;
      const uint16_t* rp[4] = {nullptr, nullptr, nullptr, nullptr};
      uint32_t rows_ok = 0u;                  // bit i: row lane + 32 i is in the tile
      int lu = blockIdx.x, lk = 0, lk1 = 0;   // load cursor: unit, stage, end stage
      auto start_unit = [&](int u) {
        const Unit w = unit_at(sc, p, u);
        const int row0 = w.m * kUnitRows + (kGateUp ? 0 : h * BM);
        const int valid = max(0, min(BM, p.rows_per_group - row0));
        const int group = kGateUp ? 2 * w.e + h : w.e;
        // a tile wholly past the last row (down's last pair) reads the group's first row, masked
        const uint8_t* blk = p.w_scales + (static_cast<int64_t>(group) * p.rows_per_group + (valid > 0 ? row0 : 0)) * p.nb;
        rows_ok = 0u;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = lane + 32 * i;
          rp[i] = reinterpret_cast<const uint16_t*>(blk + static_cast<int64_t>(r < valid ? r : 0) * p.nb);
          rows_ok |= (r < valid ? 1u : 0u) << i;
        }
        lk = w.k0;
        lk1 = w.k1;
      };
      // wd: the raw words; returns the mask of those that exist (bit 4 i + q)
      auto load_next = [&](uint32_t (&wd)[16]) -> uint32_t {
        if (lu >= sc.units) return 0u;
        const int b0 = 8 * lk;
        uint32_t ok = 0u;
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            wd[4 * i + q] = __ldg(rp[i] + min(b0 / 2 + q, p.nb / 2 - 1));
            ok |= (((rows_ok >> i) & 1u) && b0 + 2 * q < p.nb ? 1u : 0u) << (4 * i + q);
          }
        if (++lk == lk1) {
          lu += gridDim.x;
          if (lu < sc.units) start_unit(lu);
        }
        return ok;
      };
      if (lu < sc.units) start_unit(lu);
      int su = blockIdx.x, sk = 0, sk1 = 0;    // store cursor
      if (su < sc.units) {
        const Unit w = unit_at(sc, p, su);
        sk = w.k0;
        sk1 = w.k1;
      }
      uint32_t ring[kRing][16] = {};
      uint32_t ring_ok[kRing] = {};
#pragma unroll
      for (int j = 0; j < kRing; ++j) ring_ok[j] = load_next(ring[j]);
      bool run = su < sc.units;
      while (run) {
#pragma unroll
        for (int j = 0; j < kRing; ++j) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err)) { run = false; break; }
          uint32_t wv[16];
#pragma unroll
          for (int f = 0; f < 16; ++f) wv[f] = ((ring_ok[j] >> f) & 1u) ? (ring[j][f] & 0xFFFFu) : 0x7F7Fu;
          const uint4 c0 = make_uint4(wv[0] | (wv[1] << 16), wv[4] | (wv[5] << 16), wv[8] | (wv[9] << 16),
                                      wv[12] | (wv[13] << 16));
          const uint4 c1 = make_uint4(wv[2] | (wv[3] << 16), wv[6] | (wv[7] << 16), wv[10] | (wv[11] << 16),
                                      wv[14] | (wv[15] << 16));
          uint8_t* dst = sSFA(stage, h) + 16 * lane;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            *reinterpret_cast<uint4*>(dst + 512 * q) = c0;
            *reinterpret_cast<uint4*>(dst + 2048 + 512 * q) = c1;
          }
          fence_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&full[stage]);
          if (++stage == S) { stage = 0; phase ^= 1; }
          if (++sk == sk1) {
            su += gridDim.x;
            if (su >= sc.units) { run = false; break; }
            const Unit w = unit_at(sc, p, su);
            sk = w.k0;
            sk1 = w.k1;
          }
          ring_ok[j] = load_next(ring[j]);
        }
      }
    }
  } else {
    // ----------------------------------------------------------------- epilogue -----
    const int q = warp & 3;
    float* epi_stage = reinterpret_cast<float*>(smem + epi_stage_offset() + (warp - 4) * kEpiStageBytes);
    if (kGateUp && blockIdx.x < sc.units) {
      // The part-splitting epilogue runs once per unit, long after the kernel starts, and
      // its instructions would come cold from memory that the weight stream saturates:
      // run it once now, stores masked off, while the first stages load.
      float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      finish_gate_up(p.xs_out, p.sfb_out, epi_stage, p.n_out, p.nst_out, p.max_chunks, p.s_in, p.s_out, 0, 0, 0, 8, 0, z, z,
                     0.0f, 0.0f, lane, lane, true);
    }
    uint32_t use0 = 0u, use1 = 0u;
    int nxt = 0;
    for (int u = blockIdx.x; u < sc.units; u += gridDim.x) {
      const Unit w = unit_at(sc, p, u);
      const bool big = w.ncols > kBigCols;
      const int slot = big ? 0 : nxt;
      // this warp's rows: gate_up one row of both accumulators (gate, up); down row0 of the
      // first accumulator and row1 = row0 + 128 of the second
      const int row0 = w.m * kUnitRows + 32 * q + lane;
      const int row1 = kGateUp ? row0 : row0 + BM;
      const bool live0 = (w.m * kUnitRows + 32 * q) < p.n_out;   // n_out % 64 == 0: whole warps
      const bool live1 = kGateUp ? live0 : (w.m * kUnitRows + BM + 32 * q) < p.n_out;
      // this warp's biases, loaded before the wait so that their latency overlaps the MMAs
      const float* bias_e = p.bias + static_cast<int64_t>(w.e) * p.rows_total;
      const float bias0 = __ldg(bias_e + min(row0, p.n_out - 1));
      const float bias1 = __ldg(bias_e + (kGateUp ? p.n_out : 0) + min(row1, p.n_out - 1));
      bool ok = mbar_wait(&acc_full[slot], (slot ? use1 : use0) & 1u, abort_flag, p.err);
      if (ok && big) ok = mbar_wait(&acc_full[1], use1 & 1u, abort_flag, p.err);
      if (!ok) break;
      tc_fence_after();
      const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * q) << 16);
      const uint32_t tg = lane_base + (big ? 0u : static_cast<uint32_t>(slot * kSlot1));
      const uint32_t tu = lane_base + (big ? static_cast<uint32_t>(kSlot1)
                                           : static_cast<uint32_t>(slot * kSlot1 + w.ncols));
      const bool live = live0 || live1;
      const bool split = sc.nsplit > 1;
      const int64_t col0 = static_cast<int64_t>(w.off) * kParts;
      // the partial of accumulator h: gate_up plane h at the shared row, down plane 0 at its own row
      const int ph1 = kGateUp ? 1 : 0;
      if (live && split) {
        // this split's partials
        for (int j0 = 0; j0 < w.n; j0 += 8) {
          float vg[8 * kParts], vu[8 * kParts];
          read_tmem8<true>(tg, tu, j0, vg, vu);
#pragma unroll
          for (int f = 0; f < 8 * kParts; ++f) {
            if (j0 + f / kParts < w.n) {
              if (live0) *part_at(p, kPlanes, w.s, 0, col0 + kParts * j0 + f, row0) = vg[f];
              if (live1) *part_at(p, kPlanes, w.s, ph1, col0 + kParts * j0 + f, row1) = vu[f];
            }
          }
        }
      }
      bool finished = live && !split;
      unsigned* stk = p.split_tickets + (static_cast<int64_t>(w.g) * p.n_m + w.m) * 4 + q;
      if (live && split) {
        // the last split of this 32-row slice adds the partials in split order
        __threadfence();
        __syncwarp();
        unsigned t = 0;
        if (lane == 0) t = atomicAdd(stk, 1u);
        t = __shfl_sync(0xffffffffu, t, 0);
        finished = t == static_cast<unsigned>(sc.nsplit - 1);
        if (finished) __threadfence();
      }
      if (finished) {
        for (int j0 = 0; j0 < w.n; j0 += 8) {
          float vg[8 * kParts], vu[8 * kParts];
          if (!split) {
            read_tmem8<true>(tg, tu, j0, vg, vu);
          } else {
#pragma unroll
            for (int f = 0; f < 8 * kParts; ++f) { vg[f] = 0.0f; vu[f] = 0.0f; }
            for (int s = 0; s < sc.nsplit; ++s) {
#pragma unroll
              for (int f = 0; f < 8 * kParts; ++f) {
                if (j0 + f / kParts < w.n) {
                  if (live0) vg[f] += __ldcg(part_at(p, kPlanes, s, 0, col0 + kParts * j0 + f, row0));
                  if (live1) vu[f] += __ldcg(part_at(p, kPlanes, s, ph1, col0 + kParts * j0 + f, row1));
                }
              }
            }
          }
          float gs[8], us[8];
          sum_parts(vg, gs);
          sum_parts(vu, us);
          if (kGateUp) {
            finish_gate_up(p.xs_out, p.sfb_out, epi_stage, p.n_out, p.nst_out, p.max_chunks, p.s_in, p.s_out, w.e, w.c, w.off,
                           w.n, j0, gs, us, bias0, bias1, row0, lane, false);
          } else {
            if (live0) finish_down(p, w, j0, gs, bias0, row0);
            if (live1) finish_down(p, w, j0, us, bias1, row1);
          }
        }
        if (split && lane == 0) *stk = 0u;   // ready for the next call
      }
      // the accumulator slot is free for the unit after next
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&acc_empty[slot]);
        if (big) mbar_arrive(&acc_empty[1]);
      }
      if (big) {
        ++use0;
        ++use1;
        nxt = 0;
      } else {
        if (slot) ++use1; else ++use0;
        nxt ^= 1;
      }
    }
  }

  // ---------------------------------------------------------------------- teardown ---
  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {   // let copies still in flight land before the CTA's memory goes
    const long long t0 = clock64();
    while (clock64() - t0 < 200000) {
    }
  }
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTmemCols));
  }
}

// ------------------------------------------------ token operand of the gate_up GEMM --
// One CTA per token: the token's x (or, with FP8 activations, the e4m3 value of x / s0)
// as four e2m1 parts, each 32-value block with its own e8m0 scale per part (the smallest
// s with the block's largest residual / 2^s <= 6), written to each of the token's k
// routed rows in expert-grouped order (its position inv[t*k + j]). Scale records: per
// (expert, row group, 256-deep stage) one record as the down GEMM's B operand has them
// (sfb_store). The row's loads are issued
// first (they depend on nothing), the routing lookups beside them; each thread holds 16
// consecutive values (half a block: a block's maximum is one shuffle with the
// neighbouring lane), so a part leaves as one 8-byte store per routed row.
constexpr int kSplitThreads = 256;
constexpr int kSplitVals = 16;   // values per thread: H <= 4096
__global__ void __launch_bounds__(kSplitThreads) split_tokens_kernel(
    const uint16_t* __restrict__ x, const int32_t* __restrict__ topk_idx, const int32_t* __restrict__ inv,
    const int32_t* __restrict__ offsets, int E, int64_t P, int H, int k, float s0, int fp8,
    uint8_t* __restrict__ xs, uint8_t* __restrict__ sfb, int max_chunks, int nst) {
  __shared__ int s_pos[kMaxTopK];
  __shared__ long long s_rec[kMaxTopK];   // byte offset of the routed row's first record, or -1
  __shared__ int s_jr[kMaxTopK];          // the routed row within its row group
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x;
  const int i0 = kSplitVals * static_cast<int>(threadIdx.x);
  const bool act = i0 < H;   // H % 64 == 0: a thread's 16 values are all in or all out
  uint4 raw[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
  if (act) {
    const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(t) * H + i0);
    raw[0] = ld_nc_v4(src);
    raw[1] = ld_nc_v4(src + 1);
  }
  // This kernel starts during the routing kernel (programmatic dependent launch): the row
  // above is the layer input, the routing lookups below are that kernel's output. Only
  // once routing is complete may the gate_up GEMM launch, since its setup reads the
  // routing's expert offsets before it waits for this kernel. (Letting it launch at this
  // kernel's start instead, with the set-up waiting, measured 7 us slower per decode step.)
  griddep_wait();
  griddep_launch_dependents();
  if (static_cast<int>(threadIdx.x) < k) {   // thread j < k: the token's routed row j
    const int64_t pr = static_cast<int64_t>(t) * k + threadIdx.x;
    const int e = topk_idx[pr];
    const int pos = inv[pr];
    int ps = -1, jr = 0;
    long long rec = -1;
    if (e >= 0 && e < E && pos >= 0 && pos < P) {   // else the permutation has flagged it
      const int je = pos - offsets[e];   // row within the expert
      rec = (static_cast<long long>(e) * max_chunks + je / kGroupRows) * nst * kSfRecord;
      jr = je % kGroupRows;
      ps = pos;
    }
    s_pos[threadIdx.x] = ps;
    s_rec[threadIdx.x] = rec;
    s_jr[threadIdx.x] = jr;
  }
  float r[kSplitVals];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t w4[4] = {raw[h].x, raw[h].y, raw[h].z, raw[h].w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float lo = __uint_as_float(w4[q] << 16), hi = __uint_as_float(w4[q] & 0xFFFF0000u);
      r[8 * h + 2 * q] = fp8 ? e4m3_to_f32(act_quant_e4m3(lo, s0)) : lo;
      r[8 * h + 2 * q + 1] = fp8 ? e4m3_to_f32(act_quant_e4m3(hi, s0)) : hi;
    }
  }
  const int64_t row_bytes = H / 2;
  const int kb = static_cast<int>(threadIdx.x) >> 1;   // this thread's 32-value block
  const int64_t rec_st = static_cast<int64_t>(kb >> 3) * kSfRecord;   // this block's stage record
  const bool writes_scale = act && (lane & 1) == 0;
  __syncthreads();   // s_pos, s_rec, s_jr
#pragma unroll 1
  for (int pp = 0; pp < kParts; ++pp) {
    float m = 0.0f;
#pragma unroll
    for (int v = 0; v < kSplitVals; ++v) m = fmaxf(m, fabsf(r[v]));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));   // the other half of the block
    const int sc = e2m1_part_exponent(m);
    const float down = pow2f(-sc), up = pow2f(sc);
    uint32_t packed[2] = {0u, 0u};
#pragma unroll
    for (int j = 0; j < kSplitVals / 2; ++j) {
      const uint32_t byte =
          __nv_cvt_float2_to_fp4x2(make_float2(r[2 * j] * down, r[2 * j + 1] * down), __NV_E2M1, cudaRoundNearest);
      const __half2_raw hv = __nv_cvt_fp4x2_to_halfraw2(static_cast<__nv_fp4x2_storage_t>(byte), __NV_E2M1);
      r[2 * j] -= __half2float(__half(__half_raw{hv.x})) * up;       // exact
      r[2 * j + 1] -= __half2float(__half(__half_raw{hv.y})) * up;
      packed[j >> 2] |= byte << (8 * (j & 3));
    }
    if (act)
      for (int j = 0; j < k; ++j) {
        const int pos = s_pos[j];
        if (pos < 0) continue;
        *reinterpret_cast<uint2*>(xs + (static_cast<int64_t>(pos) * kParts + pp) * row_bytes + i0 / 2) =
            make_uint2(packed[0], packed[1]);
        if (writes_scale)
          sfb_store(sfb + s_rec[j] + rec_st, kParts * s_jr[j] + pp, (kb >> 2) & 1, kb & 3, static_cast<uint8_t>(sc + 127));
      }
  }
}

}  // namespace dec

namespace {

constexpr size_t kPartBudget = 16u << 20;   // split-K partials, bytes

int split_cap(int kA, int64_t P, int n_out) {
  const double per = static_cast<double>(kA) * P * dec::kParts * n_out * 4.0;
  const int64_t c = per > 0 ? static_cast<int64_t>(kPartBudget / per) : dec::kMaxSplit;
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(dec::kMaxSplit, c)));
}

int box_rows_for(int T) {
  const int n = dec::kParts * T;
  return n <= 8 ? 8 : (n <= 64 ? 16 : 32);
}

int max_chunks_for(int T) { return std::max(1, (T + dec::kGroupRows - 1) / dec::kGroupRows); }
int nst_for(int K) { return (K + dec::BKS - 1) / dec::BKS; }

}  // namespace

bool decode_tc_supported(int H, int I, int T, const void* gu_blocks, const void* d_blocks, const void* gu_scales,
                         const void* d_scales) {
  if (H % 64 || I % 64 || H < 64 || I < 64 || T < 1 || T > kDecodeMaxT) return false;
  if (H > dec::kSplitThreads * dec::kSplitVals) return false;   // the token split holds a row
  if ((reinterpret_cast<uintptr_t>(gu_blocks) | reinterpret_cast<uintptr_t>(d_blocks)) & 15u) return false;
  // the weight-scale converters read the e8m0 bytes as 16-bit words
  if ((reinterpret_cast<uintptr_t>(gu_scales) | reinterpret_cast<uintptr_t>(d_scales)) & 1u) return false;
  // the widest B tile must still leave two pipeline stages
  const int worst = dec::ring_offset() + 2 * (dec::stage_bytes_for(2, dec::kMaxN) + dec::kSfStageMax);
  if (worst + 1024 > dec::kSmemBytes) return false;
  return tmap_available();
}

cudaError_t decode_tc_prepare() {
  const int smem = dec::kSmemBytes;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(dec::decode_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem))) return e;
  return cudaFuncSetAttribute(dec::decode_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
}

size_t decode_tc_xs_bytes(int64_t P, int K) { return static_cast<size_t>(P) * dec::kParts * (K / 2); }

size_t decode_tc_sfb_bytes(int E, int K, int T) {
  return static_cast<size_t>(E) * max_chunks_for(T) * nst_for(K) * dec::kSfRecord;
}

size_t decode_tc_part_bytes(int64_t P, int H, int I) {
  const size_t gu = static_cast<size_t>(split_cap(2, P, I)) * 2 * P * dec::kParts * I * 4;
  const size_t d = static_cast<size_t>(split_cap(1, P, H)) * 1 * P * dec::kParts * H * 4;
  return std::max(gu, d);
}

size_t decode_tc_ticket_count(int H, int I) {
  // split-K tickets per (row group, unit rows, epilogue warp): gate_up units of 128 rows of
  // I, down units of 256 rows of H (sized here for 128, a bound)
  const size_t m_gu = (I + dec::BM - 1) / dec::BM, m_d = (H + dec::BM - 1) / dec::BM;
  return static_cast<size_t>(dec::kMaxGrp) * (m_gu + m_d) * 4;
}

cudaError_t launch_split_tokens(bool fp8, const uint16_t* x, const int32_t* topk_idx, const int32_t* inv,
                                const int32_t* offsets, int T, int E, int H, int k, float s0, uint8_t* xs, uint8_t* sfb,
                                cudaStream_t st) {
  if (T <= 0) return cudaSuccess;
  if (k > dec::kMaxTopK || H > dec::kSplitThreads * dec::kSplitVals || H % 64) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(T));
  cfg.blockDim = dim3(dec::kSplitThreads);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, dec::split_tokens_kernel, x, topk_idx, inv, offsets, E, static_cast<int64_t>(T) * k, H,
                            k, s0, fp8 ? 1 : 0, xs, sfb, max_chunks_for(T), nst_for(H));
}

// gate_up (gate_up = true): A = gu weights, B = xs (4 parts per routed row), writes xs_mid
// / sfb_mid for the down GEMM. down: A = d weights, B = xs_mid, writes y.
cudaError_t launch_decode_gemm(bool gate_up, const DecodeGemmArgs& a, cudaStream_t st) {
  using namespace dec;
  const int K = gate_up ? a.H : a.I;
  const int n_out = gate_up ? a.I : a.H;
  const int groups = gate_up ? 2 * a.E : a.E;
  const int64_t b_rows = a.P * kParts;
  const int unit_rows = gate_up ? BM : 2 * BM;   // output rows per unit (down: two 128-row tiles)
  const int n_m = (n_out + unit_rows - 1) / unit_rows;
  const int box_rows = box_rows_for(a.T);
  if (a.E > kMaxE || a.k > kMaxTopK || a.T > kDecodeMaxT)
    return cudaErrorInvalidValue;
  CUtensorMap mw, mx;
  {
    const uint64_t row_bytes = static_cast<uint64_t>(K) / 2;
    const uint64_t dims[3] = {row_bytes, static_cast<uint64_t>(n_out), static_cast<uint64_t>(groups)};
    const uint64_t strides[2] = {row_bytes, row_bytes * n_out};
    // gate_up: 128 rows of gate (matrix 2e) and of up (2e+1); down: 256 rows of matrix e
    const uint32_t box[3] = {static_cast<uint32_t>(kRowBytes), static_cast<uint32_t>(gate_up ? BM : 2 * BM),
                             gate_up ? 2u : 1u};
    if (!tmap_encode(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, gate_up ? a.gu_blocks : a.d_blocks, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(K) / 2, static_cast<uint64_t>(b_rows > 0 ? b_rows : 1)};
    const uint64_t strides[1] = {static_cast<uint64_t>(K) / 2};
    const uint32_t box[2] = {static_cast<uint32_t>(kRowBytes), static_cast<uint32_t>(box_rows)};
    if (!tmap_encode(&mx, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, gate_up ? a.xs : a.xs_mid, dims, strides, box)) return cudaErrorInvalidValue;
  }
  Params prm{};
  prm.w_scales = gate_up ? a.gu_scales : a.d_scales;
  prm.bias = gate_up ? a.gu_bias : a.d_bias;
  prm.rows_per_group = n_out;
  prm.rows_total = gate_up ? 2 * a.I : a.H;
  prm.n_out = n_out;
  prm.E = a.E;
  prm.K = K;
  prm.nb = K / 32;
  prm.nst = nst_for(K);
  prm.n_m = n_m;
  prm.box_rows = box_rows;
  prm.split_cap = split_cap(gate_up ? 2 : 1, a.P, n_out);
  prm.max_chunks = max_chunks_for(a.T);
  prm.smem_bytes = kSmemBytes;
  prm.P = a.P;
  prm.offsets = a.offsets;
  prm.active = a.active;
  prm.n_active = a.n_active;
  prm.sfb = gate_up ? a.sfb : a.sfb_mid;
  prm.s_in = gate_up ? a.s0 : a.s1_in;
  prm.xs_out = a.xs_mid;
  prm.sfb_out = a.sfb_mid;
  prm.nst_out = nst_for(a.I);
  prm.s_out = a.s1_quant;
  prm.y_out = a.y;
  prm.part = a.part;
  prm.split_tickets = gate_up ? a.split_tickets_gu : a.split_tickets_d;
  prm.err = a.err;
  const int64_t max_grp = std::min<int64_t>(kMaxGrp, static_cast<int64_t>(a.max_active) + a.P / kGroupRows + 1);
  const int64_t max_units = max_grp * n_m * prm.split_cap;
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(a.sms, max_units)));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = st;
  // programmatic dependent launch: the kernel starts during its predecessor (the token
  // split, or gate_up for down) and waits for it only before reading its output
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (gate_up) return cudaLaunchKernelEx(&cfg, decode_gemm_kernel<true>, mw, mx, prm);
  return cudaLaunchKernelEx(&cfg, decode_gemm_kernel<false>, mw, mx, prm);
}

}  // namespace mxmoe
