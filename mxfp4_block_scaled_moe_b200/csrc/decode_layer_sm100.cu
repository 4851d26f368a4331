// The whole routed MoE layer of a handful of tokens (T <= 8) in one persistent launch on
// the tensor cores: router logits, top-k softmax, the token operand, gate_up + SwiGLU,
// down and the weighted combine. This is the decode path of "quantization_mxfp4"
// (KerasFormers), As GPT-OSS's native format: only the routed experts' MXFP4 blocks are
// read, once per layer, and each expert's output is weighted by its softmax gate.
//
// Why one launch. At one token the layer moves 53 MB of weights (E32, H = I = 2880): about
// 8 us of HBM time. Split into routing, token split, gate_up and down launches, every
// programmatic-dependent hop between them measured 5-6 us from the trigger to the next
// grid's first CTA, and the routing launch alone 11 us, so the weight stream was a fifth
// of the step. Here every CTA (one per SM, all resident) takes part in each step and the
// steps meet at counters in global memory:
//   1. every warp of the grid computes router logits and 32-value blocks of the token
//      operand (each token as four e2m1 parts with e8m0 block scales, as below) and the
//      grid meets at one counter;
//   2. every CTA reads all logits and runs the same top-k, so every CTA knows the routed
//      experts without another exchange;
//   3. gate_up, then down, as work lists of (expert, tile, 256-deep K stage) units (a
//      gate_up tile: 128 rows of gate and the matching 128 of up; a down tile: two
//      consecutive 128-row tiles): whole tiles per CTA, stream-K (one contiguous range of
//      stages per CTA, so
//      every SM streams the same weight bytes) or a hybrid of the two, chosen on the
//      device from the tile count (down is always stream-K). A gate_up tile cut between
//      CTAs is finished by the last of them (a ticket), which adds the fp32 partials in
//      CTA order;
//   4. down's token operand for one 256-deep stage of expert a waits (a counter per
//      expert and stage) for the gate_up warps that write those 256 intermediate rows; its
//      weights are in flight before that, so the ring fills across the boundary;
//   5. every down piece parks its fp32 partial; after a second meeting of the grid, every
//      warp of the grid takes (32-row slice, token) items of the output: each token's
//      experts in ascending id, each expert's pieces in CTA order, scaled, biased and
//      weighted by the token's softmax gate.
//
// Operands of every MMA (tcgen05.mma kind::mxf4 block_scale, M = 128, K = 64):
//   A = weight rows, the checkpoint's packed e2m1 bytes by TMA, with their e8m0 scales;
//       two A tiles per stage: gate_up the gate and the matching up rows, down two
//       consecutive 128-row tiles;
//   B = all T tokens as 4 T rows: token t's four parts in rows 4t .. 4t+3 (p1 = e2m1(x /
//       2^s1), p2 the same on the residual x - p1, ...; each s the smallest with the
//       block's largest residual / 2^s <= 6), padded with zero rows to N = 16 or 32. Every
//       expert multiplies all tokens (a small-N MMA costs the tensor pipe the same whatever
//       N is) and the epilogue keeps the columns of the tokens routed to it;
//   D = 128 x N fp32 in tensor memory per A tile; a token's value is the sum of its four
//       part columns.
// The down GEMM's B is the intermediate a = silu(g) * u, rounded as the layer defines it
// (bf16, or e4m3(a / s1) with FP8 activations), written by the gate_up epilogue as the
// same four parts (its 32-row warp is one 32-value block of the down contraction).
//
// Scale sources in shared memory: one tcgen05.cp.128x256b per 256-deep stage and operand
// (8 tensor-memory columns: two 128-wide k-tiles of four columns). Lane L = 32q + l,
// column 4kt + i holds the four block scales (k-blocks 4kt .. 4kt+3 of the stage) of row
// 32i + l, the same for the four 32-lane quarters q; the source keeps k-tile kt's 16 bytes
// of lane L at 2048 kt + 16 L.
//
// Every wait is bounded (about a second; then the error word reads MXMOE_ETIMEOUT and the
// kernel winds down) and every counter is returned to zero by the CTA that consumes it
// last, so the next call starts from zeros.
#include <climits>

#include <cuda.h>

#include "common.cuh"
#include "launchers.h"
#include "mx_parts.cuh"
#include "tc_common.cuh"
#include "tmap.h"
#include "topk.cuh"

namespace mxmoe {
namespace dl {

using namespace tc;

constexpr int kThreads = 288;   // warp 0 weight TMA, 1 MMA, 2-3 weight-scale converters, 4-7 epilogue, 8 token TMA
constexpr int kWarps = kThreads / 32;
constexpr int kEpiWarps = 4;
constexpr int kMaxT = kDecodeLayerMaxT;
constexpr int kMaxK = 8;
constexpr int kMaxE = 256;
constexpr int kMaxActive = kMaxT * kMaxK;
constexpr int kParts = 4;
constexpr int BM = 128;
constexpr int kRowBytes = 128;                  // packed bytes of a row per stage (K = 256)
constexpr int kStages = 4;
constexpr int kABytes = 2 * BM * kRowBytes;     // two 128-row A tiles
constexpr int kBBytesMax = 32 * kRowBytes;      // B: at most 32 rows
constexpr int kSfSrc = 4096;                    // one 128x256b tcgen05.cp source
constexpr int kOffB = kABytes;
constexpr int kOffSfa = kOffB + kBBytesMax;     // two sources, one per A tile
constexpr int kOffSfb = kOffSfa + 2 * kSfSrc;
constexpr int kStageBytes = kOffSfb + kSfSrc;   // 48 KB
constexpr int kTmemCols = 256;
constexpr int kSlotCols = 64;                   // accumulator slot s at 64 s: A tile h at + 32 h
constexpr int kSfaCol = 128;                    // A tile h's scales at 128 + 8 h
constexpr int kSfbCol = 144;
constexpr int kSmemBytes = 227 * 1024;
constexpr int kMaxHI = 8192;                    // H, I at most (the work lists' 32-bit arithmetic)
constexpr int kMaxNmD = kMaxHI / 256;           // down tiles (row-tile pairs) per expert
constexpr int kMaxGrid = 256;
constexpr int kMaxPieces = 48;                  // a CTA's pieces of one GEMM at most

// One GEMM's work list. A tile is one (active expert, 128-row tile) of the weights (down:
// a pair of consecutive row tiles), tile = active expert * nm + m, and takes nst 256-deep
// stages. Three ways to share the tiles among the G CTAs, chosen per call from the tile
// count (every CTA makes the same choice):
//   whole:     tile t to CTA t mod G, every tile on one CTA (no partial sums);
//   stream-K:  the tiles' nst * tiles stages cut into G contiguous ranges, so every CTA
//              streams the same bytes; a tile cut between CTAs costs a partial-sum
//              exchange through global memory (a store, a ticket, the last piece's loads:
//              about kExchangeStages stages of latency on the path);
//   hybrid:    tiles / G whole tiles per CTA after a stream-K share of the tiles % G
//              remaining ones, which each CTA takes first so that their exchange overlaps
//              its whole tiles.
// The choice takes the least of the busiest CTA's stage count (plus the exchange where it
// is on the path).
constexpr int kExchangeStages = 6;
enum : int { kWhole = 0, kStreamK = 1, kHybrid = 2 };

struct Phase {
  int nm, nst, K;   // tiles per expert, 256-deep stages per tile, contraction length
  int tiles;        // na * nm
  int mode;
  int Nr;           // tiles 0 .. Nr-1 go by stream-K
  int w;            // hybrid: whole tiles per CTA
  unsigned W;       // stream-K units: Nr * nst (< 2^17 for H, I <= 8192: the products
                    // below stay in 32 bits)
  int Gp;           // CTAs with stream-K work: min(grid, W), so every range is non-empty
};

struct PieceRec {    // one piece of a CTA's work list, as the CTA stores it
  uint16_t tile;
  uint8_t a, m, k0, k1, whole, slot;
};

struct Sched {
  int na;                      // routed (active) experts
  int act[kMaxActive];         // their ids, ascending
  unsigned tmask[kMaxActive];  // tokens routed to each (bit t)
  int tk_idx[kMaxT][kMaxK];    // top-k of each token: expert ids
  float tk_w[kMaxT][kMaxK];    // and softmax weights
  int a_of[kMaxE];             // active index of an expert id, or -1
  int cb_a[kMaxT][kMaxK];      // token t's experts as active indices, ascending
  float cb_w[kMaxT][kMaxK];    // and their weights
  Phase phs[2];                        // the work lists of gate_up and down
  int npc[2];                          // this CTA's pieces per GEMM
  PieceRec pcs[2][kMaxPieces];
  // the down work list's pieces, for the combine: per down tile its first CTA, its piece
  // count and the number of pieces of the tiles before it (the tile's pieces are stored
  // there, in CTA order)
  uint8_t dcf[kMaxActive * kMaxNmD];
  uint8_t dcn[kMaxActive * kMaxNmD];
  uint16_t poff[kMaxActive * kMaxNmD];
};
constexpr int kSchedBytes = (static_cast<int>(sizeof(Sched)) + 127) & ~127;
constexpr int kBarBytes = 256;
constexpr int kRingOffset = (kSchedBytes + kBarBytes + 1023) & ~1023;
static_assert(kRingOffset + kStages * kStageBytes + 1024 <= kSmemBytes, "shared memory");

struct Params {
  const uint16_t* x;          // (T, H) bf16
  const uint16_t* wr;         // (E, H) bf16 router weight
  const uint16_t* br;         // (E) bf16 router bias or null
  const uint8_t* gu_scales;   // (E, 2I, H/32) e8m0
  const float* gu_bias;       // (E, 2I)
  const uint8_t* d_scales;    // (E, H, I/32)
  const float* d_bias;        // (E, H)
  int T, H, I, E, k;
  int npad;                   // B rows per MMA: 4T rounded up to 16
  int fp8;                    // activations as e4m3(x / s0), intermediate as e4m3(a / s1)
  float s0, s1;
  float* logits;              // (T, E)
  uint8_t* xs;                // (4T, H/2) token parts
  uint8_t* sfx;               // [ceil(H/256)][4096] their scale sources
  uint8_t* xs_mid;            // (kMaxActive * npad, I/2) intermediate parts
  uint8_t* sf_mid;            // [kMaxActive][ceil(I/256)][4096]
  float* part;                // [grid][2 pieces][2 tiles][T][128] gate_up stream-K partials
  float* dpart;               // [down pieces][2 tiles][T][128] down pieces' values, tile-major
  unsigned* bar;              // [0] grid meeting after routing, [1] CTAs done, [2] grid meeting before the output
  unsigned* done_gu;          // [kMaxActive][ceil(I/256)] gate_up warps finished per expert and down stage
  unsigned* tk_gu;            // [kMaxActive * ceil(I/128)][4] gate_up partial-tile tickets
  int32_t* topk_idx;          // (T, k) routing outputs (nullable)
  float* topk_w;
  uint16_t* out;              // (T, H) bf16
  int* err;
};

// ------------------------------------------------------------------- small helpers --
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;\n" ::: "memory");
}

__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];\n" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Bounded wait until *p >= target (another CTA's release). False on timeout or abort.
__device__ __forceinline__ bool wait_count(const unsigned* p, unsigned target, volatile int* abort_flag, int* err) {
  if (ld_acquire(p) >= target) return true;
  const long long t0 = clock64();
  while (ld_acquire(p) < target) {
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitCycles) {
      *abort_flag = 1;
      set_device_error(err, MXMOE_ETIMEOUT);
      return false;
    }
    __nanosleep(64);
  }
  return true;
}

__device__ __forceinline__ Phase phase_of(const Params& p, int na, int ph) {
  Phase d;
  if (ph == 0) {
    d.nm = (p.I + BM - 1) / BM;
    d.nst = (p.H + 255) / 256;
    d.K = p.H;
  } else {
    d.nm = (p.H + 2 * BM - 1) / (2 * BM);
    d.nst = (p.I + 255) / 256;
    d.K = p.I;
  }
  const int G = gridDim.x;
  d.tiles = na * d.nm;
  const int w = d.tiles / G, rem = d.tiles % G;
  const int c_whole = (d.tiles + G - 1) / G * d.nst;
  const int c_sk = (d.tiles * d.nst + G - 1) / G + kExchangeStages;
  const int c_hyb = w * d.nst + (rem ? (rem * d.nst + G - 1) / G + (w == 0 ? kExchangeStages : 0) : 0);
  if (ph == 1) {
    // down: always stream-K; its partial sums are added by the combine of each output
    // slice, so a cut tile costs no extra exchange
    d.mode = kStreamK;
    d.Nr = d.tiles;
  } else if (c_whole <= c_sk && c_whole <= c_hyb) {
    d.mode = kWhole;
    d.Nr = 0;
  } else if (c_hyb < c_sk && w > 0) {
    d.mode = kHybrid;
    d.Nr = rem;
  } else {
    d.mode = kStreamK;
    d.Nr = d.tiles;
  }
  d.w = w;
  d.W = static_cast<unsigned>(d.Nr * d.nst);
  d.Gp = static_cast<int>(min(static_cast<unsigned>(G), d.W));
  return d;
}

__device__ __forceinline__ unsigned range_begin(const Phase& d, int c) {
  return static_cast<unsigned>(c) * d.W / static_cast<unsigned>(d.Gp);
}
// the CTA whose stream-K range holds unit s
__device__ __forceinline__ int cta_of(const Phase& d, unsigned s) {
  return static_cast<int>(((s + 1) * static_cast<unsigned>(d.Gp) - 1) / d.W);
}

struct Piece {
  int a, m, k0, k1;
  int slot;        // stream-K pieces: 0 the CTA's first, 1 a later one (its last)
  int tile;
  bool whole;      // no other CTA works on the tile
};

// This CTA's pieces of GEMM ph in order, into sc.pcs[ph] (one warp; the integer divisions
// of the work list run once, lanes in parallel, instead of in every role's loop).
__device__ __forceinline__ void build_pieces(Sched& sc, const Phase& d, int ph, int* err) {
  const int lane = threadIdx.x & 31, c = blockIdx.x, G = gridDim.x;
  int n_sk = 0;
  unsigned b0 = 0, b1 = 0, t0 = 0;
  if (c < d.Gp) {
    b0 = range_begin(d, c);
    b1 = range_begin(d, c + 1);
    t0 = b0 / static_cast<unsigned>(d.nst);
    n_sk = static_cast<int>((b1 - 1) / static_cast<unsigned>(d.nst) - t0) + 1;
  }
  int wt = 0, ws = 1, wn = 0;
  if (d.mode == kWhole) {
    wt = c;
    ws = G;
    wn = c < d.tiles ? (d.tiles - c + G - 1) / G : 0;
  } else if (d.mode == kHybrid) {
    wt = d.Nr + c * d.w;
    wn = d.w;
  }
  const int n = n_sk + wn;
  if (n > kMaxPieces) {   // the host's size checks exclude this; never expected
    if (lane == 0) {
      set_device_error(err, MXMOE_EUNSUPPORTED);
      sc.npc[ph] = 0;
    }
    return;
  }
  for (int i = lane; i < n; i += 32) {
    PieceRec r;
    int tile;
    if (i < n_sk) {
      tile = static_cast<int>(t0) + i;
      const unsigned ts = static_cast<unsigned>(tile * d.nst);
      r.k0 = static_cast<uint8_t>(max(b0, ts) - ts);
      r.k1 = static_cast<uint8_t>(min(b1, ts + d.nst) - ts);
      r.whole = r.k0 == 0 && r.k1 == d.nst;
      r.slot = i == 0 ? 0 : 1;
    } else {
      tile = wt + (i - n_sk) * ws;
      r.k0 = 0;
      r.k1 = static_cast<uint8_t>(d.nst);
      r.whole = 1;
      r.slot = 0;
    }
    r.tile = static_cast<uint16_t>(tile);
    r.a = static_cast<uint8_t>(tile / d.nm);
    r.m = static_cast<uint8_t>(tile - r.a * d.nm);
    sc.pcs[ph][i] = r;
  }
  if (lane == 0) sc.npc[ph] = n;
}

__device__ __forceinline__ Piece piece_at(const Sched& sc, int ph, int i) {
  const PieceRec r = sc.pcs[ph][i];
  Piece pc;
  pc.tile = r.tile;
  pc.a = r.a;
  pc.m = r.m;
  pc.k0 = r.k0;
  pc.k1 = r.k1;
  pc.whole = r.whole != 0;
  pc.slot = r.slot;
  return pc;
}

__device__ __forceinline__ int n_ksteps(int K, int kst) { return min(4, (K - 256 * kst + 63) / 64); }

// ------------------------------------------------------------------ token operand --
// Writes the four e2m1 parts of one 32-value block of x (or of e4m3(x / s0)) for token t,
// k-block kb: lane l holds value 32 kb + l. The part bytes go to rows 4t .. 4t+3 of xs, the
// scale bytes into the stage's scale source (once per 32-lane quarter).
__device__ __forceinline__ void split_block(float v, uint8_t* row0, int64_t row_stride, uint8_t* sf, int r0,
                                            int lane) {
#pragma unroll 1
  for (int pp = 0; pp < kParts; ++pp) {
    // the block's largest |residual| (non-negative floats order as their bit patterns; a
    // NaN counts as 0, as a maximum by fmaxf leaves it out)
    const unsigned u = __float_as_uint(fabsf(v));
    const float m = __uint_as_float(__reduce_max_sync(0xffffffffu, u > 0x7F800000u ? 0u : u));
    const int s = e2m1_part_exponent(m);
    const uint32_t code = e2m1_code(v * pow2f(-s));
    v -= e2m1_value(code) * pow2f(s);   // exact: two significant bits at a power-of-two scale
    const uint32_t byte = code | (__shfl_down_sync(0xffffffffu, code, 1) << 4);
    const uint32_t word = byte | (__shfl_down_sync(0xffffffffu, byte, 2) << 8) |
                          (__shfl_down_sync(0xffffffffu, byte, 4) << 16) | (__shfl_down_sync(0xffffffffu, byte, 6) << 24);
    if ((lane & 7) == 0) *reinterpret_cast<uint32_t*>(row0 + pp * row_stride + 4 * (lane >> 3)) = word;
    if (lane < 4) sf[16 * (32 * lane + r0 + pp)] = static_cast<uint8_t>(s + 127);
  }
}

// ------------------------------------------------------------- routing, per CTA ----
// One warp: the routed experts in ascending id and each one's token mask, from
// sc.tk_idx (the masks gather by shared-memory atomics in sc.a_of, which then takes the
// experts' active indices). g_idx / g_w (nullable): the top-k written out as (T, k).
__device__ __forceinline__ void build_sched(Sched& sc, int T, int E, int k, int* err, int32_t* g_idx, float* g_w) {
  const int lane = threadIdx.x & 31;
  unsigned* mask_of = reinterpret_cast<unsigned*>(sc.a_of);
  for (int e = lane; e < E; e += 32) mask_of[e] = 0u;
  __syncwarp();
  for (int q = lane; q < T * k; q += 32) {
    const int t = q / k, j = q - t * k;
    const int e = sc.tk_idx[t][j];
    if (e >= 0 && e < E) {
      atomicOr(&mask_of[e], 1u << t);
    } else {
      set_device_error(err, MXMOE_EDEVICE);
    }
    if (g_idx) {
      g_idx[q] = e;
      g_w[q] = sc.tk_w[t][j];
    }
  }
  __syncwarp();
  int base = 0;
#pragma unroll
  for (int i = 0; i < kMaxE / 32; ++i) {
    if (32 * i >= E) break;
    const int e = lane + 32 * i;
    const unsigned tm = e < E ? mask_of[e] : 0u;
    const unsigned bal = __ballot_sync(0xffffffffu, tm != 0u);
    if (tm) {
      const int a = base + __popc(bal & ((1u << lane) - 1u));
      sc.a_of[e] = a;
      sc.act[a] = e;
      sc.tmask[a] = tm;
    }
    base += __popc(bal);
  }
  if (lane == 0) sc.na = base;
  __syncwarp();
}

// Lanes t < T: token t's experts in ascending id with their weights (the output's order);
// an id out of range (flagged by build_sched) stays in the list as expert slot 0 with
// weight 0.
__device__ __forceinline__ void build_token_lists(Sched& sc, int T, int E, int k) {
  const int t = threadIdx.x & 31;
  if (t >= T) return;
  for (int j = 0; j < k; ++j) {
    const int e = sc.tk_idx[t][j];
    const bool valid = e >= 0 && e < E;
    const int a = valid ? sc.a_of[e] : 0;
    const float w = valid ? sc.tk_w[t][j] : 0.0f;
    int i = j;
    while (i > 0 && sc.cb_a[t][i - 1] > a) {
      sc.cb_a[t][i] = sc.cb_a[t][i - 1];
      sc.cb_w[t][i] = sc.cb_w[t][i - 1];
      --i;
    }
    sc.cb_a[t][i] = a;
    sc.cb_w[t][i] = w;
  }
}

// ------------------------------------------------------------------ epilogue piece --
// The epilogue warp's work on one gate_up piece once its accumulators are in registers
// (g0 / g1: the per-token gate and up values on this warp's 32 rows): a tile cut between
// CTAs parks its partials and the last of its pieces adds them; the tile's last piece
// then applies bias + SwiGLU and writes the intermediate as four parts.
template <int kTp>
__device__ __forceinline__ void epi_gate_up(const Params& p, const Sched& sc, const Phase& d, const Piece& pc,
                                            float (&g0)[kTp], float (&g1)[kTp], int q, int lane) {
  const int T = p.T;
  if (!pc.whole) {
    // park this piece's per-token values; the last piece adds the CTAs' values in CTA order
    const int64_t per = 2 * static_cast<int64_t>(T) * BM;
    float* mine = p.part + (static_cast<int64_t>(blockIdx.x) * 2 + pc.slot) * per + 32 * q + lane;
#pragma unroll
    for (int t = 0; t < kTp; ++t) {
      if (t < T) {
        mine[static_cast<int64_t>(t) * BM] = g0[t];
        mine[static_cast<int64_t>(T + t) * BM] = g1[t];
      }
    }
    __threadfence();
    __syncwarp();
    unsigned* tk = p.tk_gu + pc.tile * 4 + q;
    const unsigned s_first = static_cast<unsigned>(pc.tile * d.nst);
    const int c_first = cta_of(d, s_first), c_last = cta_of(d, s_first + d.nst - 1);
    unsigned old = 0;
    if (lane == 0) old = atomicAdd(tk, 1u);
    old = __shfl_sync(0xffffffffu, old, 0);
    if (old != static_cast<unsigned>(c_last - c_first)) return;
    __threadfence();
#pragma unroll
    for (int t = 0; t < kTp; ++t) { g0[t] = 0.0f; g1[t] = 0.0f; }
    // up to four CTAs' partials in flight at once, added in CTA order
    for (int c0 = c_first; c0 <= c_last; c0 += 4) {
      float v0[4][kTp], v1[4][kTp];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = min(c0 + u, c_last);
        const int sl = range_begin(d, c) < s_first ? 1 : 0;
        const float* src = p.part + (static_cast<int64_t>(c) * 2 + sl) * per + 32 * q + lane;
#pragma unroll
        for (int t = 0; t < kTp; ++t) {
          v0[u][t] = t < T ? __ldcg(src + static_cast<int64_t>(t) * BM) : 0.0f;
          v1[u][t] = t < T ? __ldcg(src + static_cast<int64_t>(T + t) * BM) : 0.0f;
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (c0 + u <= c_last) {
#pragma unroll
          for (int t = 0; t < kTp; ++t) {
            g0[t] += v0[u][t];
            g1[t] += v1[u][t];
          }
        }
      }
    }
    if (lane == 0) *tk = 0u;   // ready for the next call
  }
  const int rr0 = pc.m * BM + 32 * q;   // the warp's first intermediate row
  const int nst_d = (p.I + 255) / 256;
  if (rr0 < p.I) {
    const int e = sc.act[pc.a];
    const float bias0 = __ldg(p.gu_bias + static_cast<int64_t>(e) * 2 * p.I + rr0 + lane);
    const float bias1 = __ldg(p.gu_bias + static_cast<int64_t>(e) * 2 * p.I + p.I + rr0 + lane);
    const unsigned mask = sc.tmask[pc.a];
    const int kb = rr0 / 32;   // the warp's block of the down contraction
    const int64_t row_stride = p.I / 2;
    uint8_t* rows = p.xs_mid + static_cast<int64_t>(pc.a) * p.npad * row_stride + 16 * kb;
    uint8_t* sf = p.sf_mid + (static_cast<int64_t>(pc.a) * nst_d + (kb >> 3)) * kSfSrc + ((kb >> 2) & 1) * 2048 +
                  (kb & 3);
#pragma unroll
    for (int t = 0; t < kTp; ++t) {
      if (t >= T) break;
      if (!((mask >> t) & 1u)) continue;
      const float gv = __fadd_rn(__fmul_rn(p.s0, g0[t]), bias0);
      const float uv = __fadd_rn(__fmul_rn(p.s0, g1[t]), bias1);
      const float v = __fmul_rn(__fdividef(gv, 1.0f + __expf(-gv)), uv);
      const float a = p.fp8 ? e4m3_to_f32(act_quant_e4m3(v, p.s1)) : bf16_bits_to_f32(f32_to_bf16_bits_rn(v));
      split_block(a, rows + static_cast<int64_t>(kParts * t) * row_stride, row_stride, sf, kParts * t, lane);
    }
  }
  // every gate_up warp counts once, live or not, toward the down stage its rows feed:
  // down stage s of this expert waits for the 4 warps of each of gate_up tiles 2s, 2s + 1
  fence_proxy_async_global();
  __threadfence();
  __syncwarp();
  if (lane == 0) atomicAdd(&p.done_gu[pc.a * nst_d + (pc.m >> 1)], 1u);
}

// The down side: every piece parks its per-token values of both row tiles (no bias),
// [piece][row tile][token][128 rows]; the output is formed after the whole grid has
// parked its pieces (combine_items below).
template <int kTp>
__device__ __forceinline__ void epi_down(const Params& p, const Sched& sc, const Piece& pc, const float (&g0)[kTp],
                                         const float (&g1)[kTp], int q, int lane) {
  const int T = p.T;
  const int slot = sc.poff[pc.tile] + static_cast<int>(blockIdx.x) - sc.dcf[pc.tile];   // the tile's pieces in CTA order
  float* mine = p.dpart + static_cast<int64_t>(slot) * 2 * T * BM + 32 * q + lane;
#pragma unroll
  for (int t = 0; t < kTp; ++t) {
    if (t < T) {
      mine[t * BM] = g0[t];
      mine[(T + t) * BM] = g1[t];
    }
  }
}

// One (32-row slice, token) item of the output, by one warp (lane = row): the token's
// experts in ascending id, each y = s * (the expert tile's pieces added in CTA order) +
// bias, weighted and added. All of a token's expert pieces (kCombinePc each) and biases
// are in flight at once, and every warp of the grid takes items.
// Not inlined, and with plain arguments, so that its one copy of code serves the real
// items and a dry run (dry: the same loads, no store) that every CTA makes early on: the
// output runs once per call, right after the weights have streamed through the caches,
// and its instructions would otherwise come from memory there, a few microseconds.
struct ItemArgs {
  const float* dpart;
  const float* d_bias;
  uint16_t* out;
  int H, T, k, nm;
  float s_in;
};
constexpr int kCombinePc = 6;
__device__ __noinline__ void combine_item(const ItemArgs x, const Sched* __restrict__ sc, int s, int t, bool dry) {
  const int lane = threadIdx.x & 31;
  const int r = 32 * s + lane;
  const int m = s / 8, h = (s / 4) & 1;                 // tile pair, row tile within it
  const int off = (h * x.T + t) * BM + 32 * (s & 3) + lane;
  const int per = 2 * x.T * BM;
  float v[kMaxK][kCombinePc], bd[kMaxK];
  int np[kMaxK];
  const float* src[kMaxK];
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) {
    const bool on = j < x.k;
    const int a = sc->cb_a[t][on ? j : 0];
    const int tile = a * x.nm + m;
    np[j] = on ? sc->dcn[tile] : 0;
    src[j] = x.dpart + static_cast<int64_t>(sc->poff[tile]) * per + off;
    bd[j] = on ? __ldg(x.d_bias + static_cast<int64_t>(sc->act[a]) * x.H + r) : 0.0f;
#pragma unroll
    for (int i = 0; i < kCombinePc; ++i) v[j][i] = i < np[j] ? __ldcg(src[j] + i * per) : 0.0f;
  }
  float acc = 0.0f;
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) {
    if (j >= x.k) break;
    float y = 0.0f;
#pragma unroll
    for (int i = 0; i < kCombinePc; ++i)
      if (i < np[j]) y += v[j][i];
    for (int i = kCombinePc; i < np[j]; ++i) y += __ldcg(src[j] + i * per);   // a tile in more pieces
    acc = __fadd_rn(acc, __fmul_rn(sc->cb_w[t][j], __fadd_rn(__fmul_rn(x.s_in, y), bd[j])));
  }
  if (!dry) x.out[static_cast<int64_t>(t) * x.H + r] = f32_to_bf16_bits_rn(acc);
}

__device__ __forceinline__ ItemArgs item_args(const Params& p, int nm) {
  ItemArgs x;
  x.dpart = p.dpart;
  x.d_bias = p.d_bias;
  x.out = p.out;
  x.H = p.H;
  x.T = p.T;
  x.k = p.k;
  x.nm = nm;
  x.s_in = p.fp8 ? p.s1 : 1.0f;
  return x;
}

// ---------------------------------------------------------------------- the kernel --
template <int kTp>   // token values a thread holds: 1 (T = 1), 4 (T <= 4) or 8
__global__ void __launch_bounds__(kThreads, 1)
decode_layer_kernel(const __grid_constant__ CUtensorMap map_gu, const __grid_constant__ CUtensorMap map_d,
                    const __grid_constant__ CUtensorMap map_xs, const __grid_constant__ CUtensorMap map_mid,
                    const __grid_constant__ Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Sched& sc = *reinterpret_cast<Sched*>(smem);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kSchedBytes);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* down_ready = acc_empty + 2;         // down's work list and the output's tables are built
  volatile int* abort_flag = reinterpret_cast<volatile int*>(down_ready + 1);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(down_ready + 1) + 1;
  volatile unsigned* last_out = reinterpret_cast<volatile unsigned*>(down_ready + 1) + 2;
  uint8_t* ring = smem + kRingOffset;
  auto sA = [&](int s, int h) { return ring + s * kStageBytes + h * (BM * kRowBytes); };
  auto sB = [&](int s) { return ring + s * kStageBytes + kOffB; };
  auto sSfa = [&](int s, int h) { return ring + s * kStageBytes + kOffSfa + h * kSfSrc; };
  auto sSfb = [&](int s) { return ring + s * kStageBytes + kOffSfb; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const int T = p.T, E = p.E, k = p.k;

  if (threadIdx.x == 0) {
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&map_gu)) : "memory");
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&map_d)) : "memory");
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&map_xs)) : "memory");
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&map_mid)) : "memory");
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 4);   // weight TMA, two scale converters, token TMA
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kEpiWarps);
    }
    mbar_init(down_ready, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(tmem_holder)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
  }

  // ------------------------------------------ 1. logits and token parts, grid-wide --
  {
    // warp-major across the grid: the dots go one per CTA before any CTA takes a second
    // (a CTA's loads of them queue behind each other), the token blocks from the other end
    const int nw = G * kWarps, gw = warp * G + blockIdx.x;
    const int TE = T * E;
    for (int d = gw; d < TE; d += nw) {
      const int t = d / E, e = d % E;
      const float acc = router_logit_warp(p.x + static_cast<int64_t>(t) * p.H, p.wr + static_cast<int64_t>(e) * p.H, p.H);
      if (lane == 0) p.logits[d] = p.br ? acc + bf16_bits_to_f32(p.br[e]) : acc;
    }
    const int nbx = p.H / 32;
    const int64_t row_stride = p.H / 2;
    for (int it = nw - 1 - gw; it < T * nbx; it += nw) {
      const int t = it / nbx, kb = it % nbx;
      float v = bf16_bits_to_f32(p.x[static_cast<int64_t>(t) * p.H + 32 * kb + lane]);
      if (p.fp8) v = e4m3_to_f32(act_quant_e4m3(v, p.s0));
      uint8_t* sf = p.sfx + static_cast<int64_t>(kb >> 3) * kSfSrc + ((kb >> 2) & 1) * 2048 + (kb & 3);
      split_block(v, p.xs + static_cast<int64_t>(4 * t) * row_stride + 16 * kb, row_stride, sf, 4 * t, lane);
    }
  }
  fence_proxy_async_global();   // the token parts are read by other CTAs' TMA
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    atomicAdd(&p.bar[0], 1u);
    wait_count(&p.bar[0], static_cast<unsigned>(G), abort_flag, p.err);
  }
  __syncthreads();
  const bool run = *abort_flag == 0;

  // ---------------------------------------------------- 2. top-k in every CTA --------
  if (run) {
    float* s_log = reinterpret_cast<float*>(ring);   // the ring is not in use yet
    for (int i = threadIdx.x; i < T * E; i += kThreads) s_log[i] = __ldcg(p.logits + i);
    __syncthreads();
    if (warp < T) topk_warp(s_log + warp * E, E, k, sc.tk_idx[warp], sc.tk_w[warp]);
    __syncthreads();
    if (warp == 0) {
      build_sched(sc, T, E, k, p.err, blockIdx.x == 0 ? p.topk_idx : nullptr, blockIdx.x == 0 ? p.topk_w : nullptr);
      __syncwarp();
      // gate_up's work list now; down's, the token lists and the output's tables are the
      // epilogue warps' first job (they wait for the first accumulator anyway)
      const Phase d = phase_of(p, sc.na, 0);
      if (lane == 0) sc.phs[0] = d;
      build_pieces(sc, d, 0, p.err);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int na = sc.na;
  const int npad = p.npad;
  const int ncol = kParts * T;
  const int nm_gu = (p.I + BM - 1) / BM;
  const int nst_d = (p.I + 255) / 256;

  if (!run) {
    // fall through to the teardown
  } else if (warp == 0) {
    // -------------------------------------------------------- weight producer ------
    if (lane == 0) {
      fence_async_smem();   // the top-k's reads of the ring come before the first copy into it
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int ph = 0; ph < 2 && ok; ++ph) {
        if (ph == 1 && !mbar_wait(down_ready, 0, abort_flag, p.err)) { ok = false; break; }
        for (int ip = 0; ok && ip < sc.npc[ph]; ++ip) {
          const Piece pc = piece_at(sc, ph, ip);
          const int e = sc.act[pc.a];
          for (int kst = pc.k0; kst < pc.k1; ++kst) {
            if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err)) { ok = false; break; }
            mbar_arrive_expect_tx(&full[stage], kABytes);
            if (ph == 0)
              tma_load_3d(sA(stage, 0), &map_gu, &full[stage], kRowBytes * kst, pc.m * BM, 2 * e);
            else
              tma_load_3d(sA(stage, 0), &map_d, &full[stage], kRowBytes * kst, pc.m * 2 * BM, e);

            if (++stage == kStages) { stage = 0; phase ^= 1; }
          }
        }
      }
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------ token producer ---
    if (lane == 0) {
      fence_proxy_async_global();   // other CTAs wrote the token parts before the grid met
      fence_async_smem();           // the top-k's reads of the ring come before the first copy into it
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      const uint32_t tx = static_cast<uint32_t>(npad * kRowBytes + kSfSrc);
      for (int ph = 0; ph < 2 && ok; ++ph) {
        if (ph == 1 && !mbar_wait(down_ready, 0, abort_flag, p.err)) { ok = false; break; }
        for (int ip = 0; ok && ip < sc.npc[ph]; ++ip) {
          const Piece pc = piece_at(sc, ph, ip);
          for (int kst = pc.k0; kst < pc.k1; ++kst) {
            if (ph == 1) {
              // the gate_up warps that write this stage's 256 rows of the intermediate
              const unsigned target = 4u * static_cast<unsigned>(min(2, nm_gu - 2 * kst));
              if (!wait_count(&p.done_gu[pc.a * nst_d + kst], target, abort_flag, p.err)) { ok = false; break; }
              fence_proxy_async_global();
            }
            if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err)) { ok = false; break; }
            mbar_arrive_expect_tx(&full[stage], tx);
            if (ph == 0) {
              tma_load_2d(sB(stage), &map_xs, &full[stage], kRowBytes * kst, 0);
              bulk_g2s(sSfb(stage), p.sfx + static_cast<int64_t>(kst) * kSfSrc, kSfSrc, &full[stage]);
            } else {
              tma_load_2d(sB(stage), &map_mid, &full[stage], kRowBytes * kst, pc.a * npad);
              bulk_g2s(sSfb(stage), p.sf_mid + (static_cast<int64_t>(pc.a) * nst_d + kst) * kSfSrc, kSfSrc,
                       &full[stage]);
            }
            if (++stage == kStages) { stage = 0; phase ^= 1; }
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------------- MMA ----
    int stage = 0;
    uint32_t phase = 0;
    uint32_t use[2] = {0u, 0u};
    int slot = 0;
    bool ok = true;
    const uint32_t id0 = idesc_mxf4(BM, npad);
    for (int ph = 0; ph < 2 && ok; ++ph) {
      if (ph == 1 && !mbar_wait(down_ready, 0, abort_flag, p.err)) { ok = false; break; }
      const Phase& d = sc.phs[ph];
      for (int ip = 0; ok && ip < sc.npc[ph]; ++ip) {
        const Piece pc = piece_at(sc, ph, ip);
        if (!mbar_wait(&acc_empty[slot], (use[slot] & 1u) ^ 1u, abort_flag, p.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d0 = tmem + static_cast<uint32_t>(slot * kSlotCols);
        for (int kst = pc.k0; kst < pc.k1; ++kst) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.err)) { ok = false; break; }
          tc_fence_after();
          if (lane == 0) {
            const int nks = n_ksteps(d.K, kst);
            tc_cp_128x256b(tmem + kSfaCol, smem_desc(smem_u32(sSfa(stage, 0)), 2048, 128, 0));
            tc_cp_128x256b(tmem + kSfaCol + 8, smem_desc(smem_u32(sSfa(stage, 1)), 2048, 128, 0));
            tc_cp_128x256b(tmem + kSfbCol, smem_desc(smem_u32(sSfb(stage)), 2048, 128, 0));
            const uint32_t b0 = smem_u32(sB(stage));
            for (int sk = 0; sk < nks; ++sk) {
              const int t = sk >> 1;
              const uint32_t sfid = static_cast<uint32_t>(sk & 1) * 2u;
              const uint32_t id = id0 | (sfid << 4) | (sfid << 29);
              const uint32_t sel = sfid << 30;
              const uint64_t bd = smem_desc(b0 + 32 * sk, 16, 1024, 2);
              const uint32_t acc = (kst > pc.k0 || sk > 0) ? 1u : 0u;
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const uint64_t ad = smem_desc(smem_u32(sA(stage, h)) + 32 * sk, 16, 1024, 2);
                tc_mma_mxf4(d0 + 32 * h, ad, bd, id, (tmem + kSfaCol + 8 * h + 4 * t) | sel,
                            (tmem + kSfbCol + 4 * t) | sel, acc);
              }
            }
            tc_commit(&empty[stage]);
          }
          __syncwarp();
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        if (lane == 0) tc_commit(&acc_full[slot]);
        __syncwarp();
        ++use[slot];
        slot ^= 1;
      }
    }
  } else if (warp == 2 || warp == 3) {
    // --------------------------------------------------- weight-scale converters ---
    // Lane l owns rows l, l+32, l+64, l+96 of A tile h; a stage's 8 scale bytes of a row
    // are four aligned 16-bit words (K / 32 is even), loaded before the wait for the stage
    // and stored as the tile's 128x256b source (0x7F, a scale of 1, for rows past the end).
    const int h = warp - 2;
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int ph = 0; ph < 2 && ok; ++ph) {
      if (ph == 1 && !mbar_wait(down_ready, 0, abort_flag, p.err)) { ok = false; break; }
      const Phase& d = sc.phs[ph];
      const int nb = d.K / 32;
      for (int ip = 0; ok && ip < sc.npc[ph]; ++ip) {
        const Piece pc = piece_at(sc, ph, ip);
        const int e = sc.act[pc.a];
        int valid;
        const uint8_t* blk;
        if (ph == 0) {
          valid = min(BM, p.I - pc.m * BM);
          blk = p.gu_scales + (static_cast<int64_t>(2 * e + h) * p.I + pc.m * BM) * nb;
        } else {
          const int r0 = pc.m * 2 * BM + h * BM;
          valid = max(0, min(BM, p.H - r0));
          blk = valid > 0 ? p.d_scales + (static_cast<int64_t>(e) * p.H + r0) * nb : p.d_scales;
        }
        const uint16_t* rp[4];
        uint32_t rows_ok = 0u;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = lane + 32 * i;
          rp[i] = reinterpret_cast<const uint16_t*>(blk + static_cast<int64_t>(r < valid ? r : 0) * nb);
          rows_ok |= (r < valid ? 1u : 0u) << i;
        }
        for (int kst = pc.k0; kst < pc.k1; ++kst) {
          uint32_t wv[16];
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const bool have = ((rows_ok >> i) & 1u) && 8 * kst + 2 * q < nb;
              const uint32_t w = __ldg(rp[i] + min(4 * kst + q, nb / 2 - 1));
              wv[4 * i + q] = have ? (w & 0xFFFFu) : 0x7F7Fu;
            }
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err)) { ok = false; break; }
          const uint4 c0 = make_uint4(wv[0] | (wv[1] << 16), wv[4] | (wv[5] << 16), wv[8] | (wv[9] << 16),
                                      wv[12] | (wv[13] << 16));
          const uint4 c1 = make_uint4(wv[2] | (wv[3] << 16), wv[6] | (wv[7] << 16), wv[10] | (wv[11] << 16),
                                      wv[14] | (wv[15] << 16));
          uint8_t* dst = sSfa(stage, h) + 16 * lane;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            *reinterpret_cast<uint4*>(dst + 512 * q) = c0;
            *reinterpret_cast<uint4*>(dst + 2048 + 512 * q) = c1;
          }
          fence_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&full[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue ---
    const int q = warp & 3;
    {
      // the down pieces' layout for the combine (needed only after gate_up; the four
      // epilogue warps work it out while the first weights load)
      const int et = static_cast<int>(threadIdx.x) - 4 * 32;
      if (et < 32) {
        const Phase d1 = phase_of(p, na, 1);
        if (et == 0) sc.phs[1] = d1;
        build_pieces(sc, d1, 1, p.err);
      } else if (et < 64) {
        build_token_lists(sc, T, E, k);
      }
      asm volatile("bar.sync 1, 128;\n" ::: "memory");
      const Phase& dd = sc.phs[1];
      const int nt = na * dd.nm;
      for (int i = et; i < nt; i += 4 * 32) {
        const unsigned s0 = static_cast<unsigned>(i * dd.nst);
        const int cf = cta_of(dd, s0), cl = cta_of(dd, s0 + dd.nst - 1);
        sc.dcf[i] = static_cast<uint8_t>(cf);
        sc.dcn[i] = static_cast<uint8_t>(cl - cf + 1);
      }
      asm volatile("bar.sync 1, 128;\n" ::: "memory");
      if (et < 32) {
        // exclusive prefix of the piece counts: lane l sums a contiguous run of tiles, a
        // shuffle scan adds the runs before it
        const int per_lane = (nt + 31) / 32, i0 = et * per_lane, i1 = min(nt, i0 + per_lane);
        int run = 0;
        for (int i = i0; i < i1; ++i) run += sc.dcn[i];
        int incl = run;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (et >= o) incl += v;
        }
        int acc = incl - run;
        for (int i = i0; i < i1; ++i) {
          sc.poff[i] = static_cast<uint16_t>(acc);
          acc += sc.dcn[i];
        }
      }
      // the routed experts' biases into L2 (the epilogues read them after the flush-cold
      // HBM has gone quiet, one dependent load each otherwise)
      {
        const int gu_lines = 2 * p.I / 32, d_lines = p.H / 32;   // 128-byte lines per expert
        for (int i = et; i < na * (gu_lines + d_lines); i += 4 * 32) {
          const int a = i / (gu_lines + d_lines), l = i - a * (gu_lines + d_lines);
          const float* ptr = l < gu_lines ? p.gu_bias + static_cast<int64_t>(sc.act[a]) * 2 * p.I + 32 * l
                                          : p.d_bias + static_cast<int64_t>(sc.act[a]) * p.H + 32 * (l - gu_lines);
          asm volatile("prefetch.global.L2 [%0];\n" ::"l"(ptr));
        }
      }
      asm volatile("bar.sync 1, 128;\n" ::: "memory");
      if (et == 0) mbar_arrive(down_ready);
      if (et < 32) combine_item(item_args(p, dd.nm), &sc, 0, 0, true);   // the output's code, early
    }
    uint32_t use[2] = {0u, 0u};
    int slot = 0;
    bool ok = true;
    for (int ph = 0; ph < 2 && ok; ++ph) {
      const Phase& d = sc.phs[ph];
      for (int ip = 0; ok && ip < sc.npc[ph]; ++ip) {
        const Piece pc = piece_at(sc, ph, ip);
        if (!mbar_wait(&acc_full[slot], use[slot] & 1u, abort_flag, p.err)) { ok = false; break; }
        tc_fence_after();
        // a token's value is the sum of its four part columns (in part order)
        float g0[kTp], g1[kTp];
        {
          const uint32_t tb = tmem + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(slot * kSlotCols);
          constexpr int kLd = (kTp + 1) / 2;   // 8-column loads: two tokens each
          uint32_t r0[kLd][8] = {}, r1[kLd][8] = {};
#pragma unroll
          for (int i = 0; i < kLd; ++i) {
            if (8 * i < ncol) {
              tc_ld_32x32b_x8(tb + 8 * i, r0[i]);
              tc_ld_32x32b_x8(tb + 32 + 8 * i, r1[i]);
            }
          }
#pragma unroll
          for (int i = 0; i < kLd; ++i) {
            if (8 * i < ncol) tc_wait_ld(r0[i], r1[i]);
          }
#pragma unroll
          for (int t = 0; t < kTp; ++t) {
            float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
            for (int pp = 0; pp < kParts; ++pp) {
              const int n = kParts * t + pp;
              a0 += __uint_as_float(r0[n / 8][n % 8]);
              a1 += __uint_as_float(r1[n / 8][n % 8]);
            }
            g0[t] = a0;
            g1[t] = a1;
          }
        }
        // the slot is free for the piece after next once the values are in registers
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[slot]);
        ++use[slot];
        slot ^= 1;
        if (ph == 0)
          epi_gate_up<kTp>(p, sc, d, pc, g0, g1, q, lane);
        else
          epi_down<kTp>(p, sc, pc, g0, g1, q, lane);
      }
    }
  }

  // --------------------------------------------------- 5. the output, grid-wide ---
  // every CTA has parked its down pieces: meet, then every warp of the grid forms
  // (32-row slice, token) items of the output
  __threadfence();
  tc_fence_before();
  __syncthreads();
  if (run && !*abort_flag) {
    if (threadIdx.x == 0) {
      atomicAdd(&p.bar[2], 1u);
      wait_count(&p.bar[2], static_cast<unsigned>(G), abort_flag, p.err);
    }
    __syncthreads();
    if (!*abort_flag) {
      const int items = p.H / 32 * T;
      // items one per CTA before any CTA takes a second
      const ItemArgs xa = item_args(p, sc.phs[1].nm);
      for (int it = warp * G + blockIdx.x; it < items; it += G * kWarps) combine_item(xa, &sc, it / T, it % T, false);
    }
  }

  // ---------------------------------------------------------------------- teardown ---
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
  // the last CTA out returns the grid-wide counters to zero
  if (threadIdx.x == 0) {
    __threadfence();
    *last_out = atomicAdd(&p.bar[1], 1u) == static_cast<unsigned>(G - 1) ? 1u : 0u;
  }
  __syncthreads();
  if (*last_out) {
    __threadfence();
    const int n = (run ? na : kMaxActive) * nst_d;
    for (int i = threadIdx.x; i < n; i += kThreads) p.done_gu[i] = 0u;
    if (threadIdx.x == 0) {
      p.bar[0] = 0u;
      p.bar[2] = 0u;
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) p.bar[1] = 0u;
  }
}

}  // namespace dl

// ------------------------------------------------------------------------ host side --
namespace {

int npad_for(int T) { return 4 * T <= 16 ? 16 : 32; }

// down pieces at most: every tile is one piece, and each of the G - 1 inner boundaries of
// the CTAs' ranges cuts at most one tile once more
int down_pieces_max(int H, int G) {
  const int nm_d = (H + 2 * dl::BM - 1) / (2 * dl::BM);
  return dl::kMaxActive * nm_d + G;
}

}  // namespace

bool decode_layer_supported(int H, int I, int T, int E, int k, int sms, const void* gu_blocks, const void* d_blocks,
                            const void* gu_scales, const void* d_scales) {
  if (T < 1 || T > dl::kMaxT || E > dl::kMaxE || k > dl::kMaxK) return false;
  if (H % 64 || I % 64 || H < 64 || I < 64 || H > dl::kMaxHI || I > dl::kMaxHI) return false;
  if (sms < 1 || sms > dl::kMaxGrid) return false;
  // a CTA's pieces of one GEMM are at most ceil(tiles / grid) + 2 under every work-list
  // mode (whole tiles, stream-K, hybrid); keep that within the per-CTA list (on a B200's
  // 148 SMs the bound is 30 at the largest shapes)
  const int na_max = std::min(E, T * k);
  const int tiles = na_max * std::max((I + dl::BM - 1) / dl::BM, (H + 2 * dl::BM - 1) / (2 * dl::BM));
  if ((tiles + sms - 1) / sms + 2 > dl::kMaxPieces) return false;
  if ((reinterpret_cast<uintptr_t>(gu_blocks) | reinterpret_cast<uintptr_t>(d_blocks)) & 15u) return false;
  // the weight-scale converters read the e8m0 bytes as 16-bit words
  if ((reinterpret_cast<uintptr_t>(gu_scales) | reinterpret_cast<uintptr_t>(d_scales)) & 1u) return false;
  return tmap_available();
}

cudaError_t decode_layer_prepare() {
  cudaError_t e = cudaFuncSetAttribute(dl::decode_layer_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       dl::kSmemBytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(dl::decode_layer_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, dl::kSmemBytes);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(dl::decode_layer_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, dl::kSmemBytes);
}

DecodeLayerSizes decode_layer_sizes(int T, int H, int I, int sms) {
  DecodeLayerSizes s{};
  const int npad = npad_for(T);
  s.xs = static_cast<size_t>(4 * T) * (H / 2);
  s.sfx = static_cast<size_t>((H + 255) / 256) * dl::kSfSrc;
  s.xs_mid = static_cast<size_t>(dl::kMaxActive) * npad * (I / 2);
  s.sf_mid = static_cast<size_t>(dl::kMaxActive) * ((I + 255) / 256) * dl::kSfSrc;
  s.part = static_cast<size_t>(sms) * 2 * 2 * T * dl::BM * sizeof(float);
  s.dpart = static_cast<size_t>(down_pieces_max(H, sms)) * 2 * T * dl::BM * sizeof(float);
  s.counters = 3 + static_cast<size_t>(dl::kMaxActive) * ((I + 255) / 256) +
               static_cast<size_t>(dl::kMaxActive) * ((I + 127) / 128) * 4;
  return s;
}

cudaError_t launch_decode_layer(const DecodeLayerArgs& a, cudaStream_t st) {
  using namespace dl;
  if (a.T < 1 || a.T > kMaxT || a.E > kMaxE || a.k > kMaxK || a.k > a.E || a.sms < 1 || a.sms > kMaxGrid ||
      a.H > kMaxHI || a.I > kMaxHI)
    return cudaErrorInvalidValue;
  const int npad = npad_for(a.T);
  CUtensorMap m_gu, m_d, m_xs, m_mid;
  {
    const uint64_t rb = static_cast<uint64_t>(a.H) / 2;
    const uint64_t dims[3] = {rb, static_cast<uint64_t>(a.I), 2 * static_cast<uint64_t>(a.E)};
    const uint64_t strides[2] = {rb, rb * a.I};
    const uint32_t box[3] = {kRowBytes, BM, 2};
    if (!tmap_encode(&m_gu, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, a.gu_blocks, dims, strides, box))
      return cudaErrorInvalidValue;
  }
  {
    const uint64_t rb = static_cast<uint64_t>(a.I) / 2;
    const uint64_t dims[3] = {rb, static_cast<uint64_t>(a.H), static_cast<uint64_t>(a.E)};
    const uint64_t strides[2] = {rb, rb * a.H};
    const uint32_t box[3] = {kRowBytes, 2 * BM, 1};
    if (!tmap_encode(&m_d, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, a.d_blocks, dims, strides, box))
      return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(a.H) / 2, static_cast<uint64_t>(4 * a.T)};
    const uint64_t strides[1] = {static_cast<uint64_t>(a.H) / 2};
    const uint32_t box[2] = {kRowBytes, static_cast<uint32_t>(npad)};
    if (!tmap_encode(&m_xs, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, a.xs, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(a.I) / 2, static_cast<uint64_t>(kMaxActive) * npad};
    const uint64_t strides[1] = {static_cast<uint64_t>(a.I) / 2};
    const uint32_t box[2] = {kRowBytes, static_cast<uint32_t>(npad)};
    if (!tmap_encode(&m_mid, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, a.xs_mid, dims, strides, box))
      return cudaErrorInvalidValue;
  }
  Params p{};
  p.x = a.x;
  p.wr = a.router_w;
  p.br = a.router_b;
  p.gu_scales = a.gu_scales;
  p.gu_bias = a.gu_bias;
  p.d_scales = a.d_scales;
  p.d_bias = a.d_bias;
  p.T = a.T;
  p.H = a.H;
  p.I = a.I;
  p.E = a.E;
  p.k = a.k;
  p.npad = npad;
  p.fp8 = a.fp8 ? 1 : 0;
  p.s0 = a.fp8 ? a.s0 : 1.0f;
  p.s1 = a.fp8 ? a.s1 : 1.0f;
  p.logits = a.logits;
  p.xs = a.xs;
  p.sfx = a.sfx;
  p.xs_mid = a.xs_mid;
  p.sf_mid = a.sf_mid;
  p.part = a.part;
  p.dpart = a.dpart;
  p.bar = a.counters;
  p.done_gu = a.counters + 3;
  p.tk_gu = p.done_gu + static_cast<size_t>(kMaxActive) * ((a.I + 255) / 256);
  p.topk_idx = a.topk_idx;
  p.topk_w = a.topk_w;
  p.out = a.out;
  p.err = a.err;
  if (a.T == 1)
    decode_layer_kernel<1><<<a.sms, kThreads, kSmemBytes, st>>>(m_gu, m_d, m_xs, m_mid, p);
  else if (a.T <= 4)
    decode_layer_kernel<4><<<a.sms, kThreads, kSmemBytes, st>>>(m_gu, m_d, m_xs, m_mid, p);
  else
    decode_layer_kernel<8><<<a.sms, kThreads, kSmemBytes, st>>>(m_gu, m_d, m_xs, m_mid, p);
  return cudaGetLastError();
}

}  // namespace mxmoe
