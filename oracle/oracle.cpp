// Plain, slow, obviously-correct CPU oracle for the MXFP4 routed Mixture-of-Experts
// expert layer (W-MXFP4, optional A-FP8-E4M3 static per-tensor activations).
//
// TEST INFRASTRUCTURE ONLY. Nothing in the product library links, includes or calls
// this file; it shares no source, header, table or helper with the CUDA path. Only the
// test suite, the smoke check and the benchmark's CPU-baseline leg load it.
//
// Sources (web pages this follows; cited by page title and section):
//  * "quantization_mxfp4" (KerasFormers), intro: MXFP4 = e2m1 values packed two per
//    byte, one e8m0 power-of-two scale per 32-value block.
//  * same page, "Primitives": dequantize = codebook[nibble] * 2^(scale - 127);
//    quantize picks the block exponent floor(log2(amax)) - 2 and rounds every value to
//    the nearest FP4 grid point.
//  * same page, "As a quantize_model scheme": the contracting dimension must be a
//    multiple of 32, otherwise a clear error.
//  * same page, "As GPT-OSS's native format": experts stored as gate_up_proj (E, 2I, H)
//    and down_proj (E, H, I) packed blocks + scales, biases kept in full precision; on
//    decode only the top-k routed experts are dequantized, with output identical to the
//    dense all-experts path.
//  * "amd/gpt-oss-20b-MoE-Quant-W-MXFP4-A-FP8-KV-FP8", "Quantization schemes": weights
//    OCP MXFP4, activations FP8 symmetric per-tensor, router not quantized.
//  * "gpt-oss-120b-mxfp4-fp8attn-v2", "Model Details" / "Quantization Recipe": FP8 E4M3
//    with static per-tensor scales from min-max calibration; router kept unquantized;
//    attention projections Q/K/V/O as FP8 E4M3 weights with a static per-tensor weight
//    scale and input scale.
//  * "quantization_mxfp4", "Primitives": MXFP4Quantizer quantizes along one arbitrary
//    contracting axis, which it moves to the end; "As a quantize_model scheme": any
//    Dense kernel can be stored MXFP4 (weight-only) and dequantized on the fly.
//
// Readings where the pages are silent (each listed in the design notes):
//  - nibble order: element 2j sits in the low nibble of byte j;
//  - gate rows are [0, I) and up rows are [I, 2I) of gate_up; activation = silu(gate)*up;
//  - top-k ties go to the lower expert id; softmax over the k selected logits;
//  - FP8 quantization is q = e4m3_rne_satfinite(fp32(x / s)), +/-448 saturation;
//  - combine: fp32 accumulation over the selected experts in ascending expert id,
//    one bf16 round-to-nearest-even at the end;
//  - a zero block gets scale byte 0 (2^-127); the sign of every element is kept.
//
// Floating point: long dot products accumulate in double (products of bf16/fp8 by
// MXFP4 values are exact in double) and are rounded to fp32 at the points stated in each
// function. Built with -ffp-contract=off and without fast-math.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>
#include <algorithm>
#include <limits>

extern "C" {

enum { ORC_OK = 0, ORC_EINVAL = -1, ORC_EALIGN = -2, ORC_EUNSUPPORTED = -3 };

// ---------------------------------------------------------------- scalar formats ---

// E2M1 magnitudes for codes 0..7 (sign is bit 3 of the nibble).
static const double kE2M1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

static double e2m1_value(unsigned nib) {
  double v = kE2M1[nib & 7u];
  return (nib & 8u) ? -v : v;
}

static float f32_from_exact_double(double v) {
  // Every dequantized value has at most two significant bits, so it is exactly
  // representable in fp32 unless its magnitude reaches 2^128 (overflow -> inf).
  if (std::fabs(v) >= 0x1p128) return std::copysign(std::numeric_limits<float>::infinity(), v);
  return static_cast<float>(v);
}

static uint16_t bf16_rne(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  if (std::isnan(f)) return static_cast<uint16_t>((u >> 16) | 0x40u);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return static_cast<uint16_t>(u >> 16);
}

static float bf16_to_f32(uint16_t h) {
  uint32_t u = static_cast<uint32_t>(h) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

// FP8 E4M3 ("fn": no infinities, 0x7F/0xFF are NaN, max finite 448).
static double e4m3_value(uint8_t c) {
  int s = c >> 7, ex = (c >> 3) & 15, m = c & 7;
  double v;
  if (ex == 15 && m == 7) return std::numeric_limits<double>::quiet_NaN();
  if (ex == 0) v = std::ldexp(static_cast<double>(m), -9);
  else v = std::ldexp(1.0 + m / 8.0, ex - 7);
  return s ? -v : v;
}

// Round an fp32 value to E4M3 with round-to-nearest-even, saturating to +/-448.
static uint8_t e4m3_rne_satfinite(float q) {
  uint8_t sign = std::signbit(q) ? 0x80 : 0x00;
  if (std::isnan(q)) return static_cast<uint8_t>(sign | 0x7F);
  double a = std::fabs(static_cast<double>(q));
  if (a >= 448.0) return static_cast<uint8_t>(sign | 0x7E);
  if (a < 0x1p-6) {
    // subnormal range: multiples of 2^-9; rounding up to 8 gives the smallest normal.
    double m = std::nearbyint(a * 512.0);  // exact scaling; nearbyint = ties-to-even
    return static_cast<uint8_t>(sign | static_cast<uint8_t>(m));
  }
  int ex;
  std::frexp(a, &ex);  // a = f * 2^ex, f in [0.5, 1)
  int e = ex - 1;      // a in [2^e, 2^(e+1))
  double m = std::nearbyint((std::ldexp(a, -e) - 1.0) * 8.0);
  if (m >= 8.0) { m = 0.0; e += 1; }
  int code = ((e + 7) << 3) | static_cast<int>(m);
  if (code > 0x7E) code = 0x7E;
  return static_cast<uint8_t>(sign | code);
}

// Round |x| / 2^e (already exact in double) onto the E2M1 grid: nearest point, ties to
// the even code, values >= 6 saturate to 6.
static unsigned e2m1_round_code(double r) {
  if (r <= 0.25) return 0;
  if (r < 0.75) return 1;
  if (r <= 1.25) return 2;
  if (r < 1.75) return 3;
  if (r <= 2.5) return 4;
  if (r < 3.5) return 5;
  if (r <= 5.0) return 6;
  return 7;
}

// ------------------------------------------------------------------- MXFP4 codec ---

// Dequantize rows x K packed values. blocks: rows x K/2 bytes (element 2j in the low
// nibble of byte j); scales: rows x K/32 e8m0 bytes. Either output may be null.
int orc_dequantize(const uint8_t* blocks, const uint8_t* scales, int64_t rows, int64_t K,
                   float* out_f32, uint16_t* out_bf16) {
  if (rows < 0 || K < 0) return ORC_EINVAL;
  if (K % 32 != 0) return ORC_EALIGN;
  const int64_t nb = K / 32;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t b = 0; b < nb; ++b) {
      const double scale = std::ldexp(1.0, static_cast<int>(scales[r * nb + b]) - 127);
      for (int i = 0; i < 32; ++i) {
        const int64_t k = b * 32 + i;
        const uint8_t byte = blocks[r * (K / 2) + k / 2];
        const unsigned nib = (k % 2 == 0) ? (byte & 0x0Fu) : (byte >> 4);
        const float v = f32_from_exact_double(e2m1_value(nib) * scale);
        if (out_f32) out_f32[r * K + k] = v;
        if (out_bf16) out_bf16[r * K + k] = bf16_rne(v);  // exact: <= 2 significant bits
      }
    }
  }
  return ORC_OK;
}

// Quantize rows x K fp32 values to MXFP4 (blocks rows x K/2, scales rows x K/32).
int orc_quantize(const float* w, int64_t rows, int64_t K, uint8_t* blocks, uint8_t* scales) {
  if (rows < 0 || K < 0) return ORC_EINVAL;
  if (K % 32 != 0) return ORC_EALIGN;
  const int64_t nb = K / 32;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t b = 0; b < nb; ++b) {
      const float* x = w + r * K + b * 32;
      float amax = 0.0f;
      for (int i = 0; i < 32; ++i) amax = std::max(amax, std::fabs(x[i]));
      int e;
      if (amax == 0.0f) {
        e = -127;  // floor(log2 0) = -inf, clamped
      } else {
        e = std::ilogb(amax) - 2;  // exact floor(log2 amax) from the exponent
        e = std::min(127, std::max(-127, e));
      }
      scales[r * nb + b] = static_cast<uint8_t>(e + 127);
      for (int i = 0; i < 32; i += 2) {
        unsigned nib[2];
        for (int h = 0; h < 2; ++h) {
          const float xi = x[i + h];
          const double rr = std::ldexp(std::fabs(static_cast<double>(xi)), -e);
          nib[h] = e2m1_round_code(rr) | (std::signbit(xi) ? 8u : 0u);
        }
        blocks[r * (K / 2) + (b * 32 + i) / 2] = static_cast<uint8_t>(nib[0] | (nib[1] << 4));
      }
    }
  }
  return ORC_OK;
}

// --------------------------------------------------------------------------- FP8 ---

// q[i] = e4m3_rne_satfinite(fp32(x[i] / s)), IEEE fp32 division.
int orc_fp8_quantize(const float* x, int64_t n, float s, uint8_t* q) {
  if (n < 0) return ORC_EINVAL;
  for (int64_t i = 0; i < n; ++i) {
    volatile float quot = x[i] / s;  // single IEEE fp32 division
    q[i] = e4m3_rne_satfinite(quot);
  }
  return ORC_OK;
}

int orc_fp8_decode(const uint8_t* q, int64_t n, float* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = static_cast<float>(e4m3_value(q[i]));
  return ORC_OK;
}

// bf16 bits -> fp32 (exact), and fp32 -> bf16 bits with round-to-nearest-even.
int orc_bf16_round(const float* x, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = bf16_rne(x[i]);
  return ORC_OK;
}

// ------------------------------------------------------------------------ router ---

// logits[t, e] = fp32( sum_h x[t,h] * Wr[e,h] + br[e] ), the sum taken in double.
// x (T, H), Wr (E, H), br (E) are bf16 bit patterns; br may be null (zero bias).
int orc_router_logits(const uint16_t* x, const uint16_t* wr, const uint16_t* br, int T, int H,
                      int E, float* logits) {
  if (T < 0 || H < 0 || E <= 0) return ORC_EINVAL;
#pragma omp parallel for schedule(static)
  for (int t = 0; t < T; ++t) {
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int h = 0; h < H; ++h)
        acc += static_cast<double>(bf16_to_f32(x[(int64_t)t * H + h])) *
               static_cast<double>(bf16_to_f32(wr[(int64_t)e * H + h]));
      if (br) acc += static_cast<double>(bf16_to_f32(br[e]));
      logits[(int64_t)t * E + e] = static_cast<float>(acc);
    }
  }
  return ORC_OK;
}

// Is logit a ranked before logit b (expert ids ia < ib)? Larger first, NaN last,
// equal values keep the lower id first.
static bool ranks_before(float a, int ia, float b, int ib) {
  bool na = std::isnan(a), nb = std::isnan(b);
  if (na != nb) return nb;       // the non-NaN one first
  if (!na && a != b) return a > b;
  return ia < ib;
}

// Top-k selection (descending logit, ties to the lower id) and a softmax over the k
// selected logits, computed in double and stored as fp32.
int orc_topk_softmax(const float* logits, int T, int E, int k, int32_t* idx, float* wts) {
  if (T < 0 || E <= 0 || k <= 0 || k > E) return ORC_EINVAL;
  for (int t = 0; t < T; ++t) {
    const float* l = logits + (int64_t)t * E;
    std::vector<char> taken(E, 0);
    for (int j = 0; j < k; ++j) {
      int best = -1;
      for (int e = 0; e < E; ++e) {
        if (taken[e]) continue;
        if (best < 0 || ranks_before(l[e], e, l[best], best)) best = e;
      }
      taken[best] = 1;
      idx[(int64_t)t * k + j] = best;
    }
    const double lmax = l[idx[(int64_t)t * k]];
    double z = 0.0;
    std::vector<double> p(k);
    for (int j = 0; j < k; ++j) { p[j] = std::exp(static_cast<double>(l[idx[(int64_t)t * k + j]]) - lmax); z += p[j]; }
    for (int j = 0; j < k; ++j) wts[(int64_t)t * k + j] = static_cast<float>(p[j] / z);
  }
  return ORC_OK;
}

// ---------------------------------------------------------------------- permute ---

// Counting sort of the T*k (token, slot) pairs by expert, stable in the flat pair order
// (ascending token, then slot). offsets has E+1 entries; perm_token / perm_slot have
// T*k entries; inv (T*k, nullable) maps pair t*k+j to its position.
int orc_permute(const int32_t* idx, int T, int E, int k, int32_t* offsets, int32_t* perm_token,
                int32_t* perm_slot, int32_t* inv) {
  if (T < 0 || E <= 0 || k <= 0) return ORC_EINVAL;
  std::vector<int64_t> count(E, 0);
  for (int64_t p = 0; p < (int64_t)T * k; ++p) {
    int e = idx[p];
    if (e < 0 || e >= E) return ORC_EINVAL;
    count[e]++;
  }
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = static_cast<int32_t>(offsets[e] + count[e]);
  std::vector<int64_t> cursor(offsets, offsets + E);
  for (int64_t p = 0; p < (int64_t)T * k; ++p) {
    int e = idx[p];
    int64_t pos = cursor[e]++;
    perm_token[pos] = static_cast<int32_t>(p / k);
    perm_slot[pos] = static_cast<int32_t>(p % k);
    if (inv) inv[p] = static_cast<int32_t>(pos);
  }
  return ORC_OK;
}

// ------------------------------------------------------------------- expert FFN ---

struct LayerArgs {
  const uint16_t* x;         // (T, H) bf16
  const uint16_t* router_w;  // (E, H) bf16
  const uint16_t* router_b;  // (E) bf16 or null
  const uint8_t* gu_blocks;  // (E, 2I, H/2)
  const uint8_t* gu_scales;  // (E, 2I, H/32)
  const float* gu_bias;      // (E, 2I)
  const uint8_t* d_blocks;   // (E, H, I/2)
  const uint8_t* d_scales;   // (E, H, I/32)
  const float* d_bias;       // (E, H)
  int E, k, T, H, I;
  const float* act_scale;    // null: bf16 activations; else {s0, s1}
};

static void dequant_row(const uint8_t* blocks, const uint8_t* scales, int64_t K, double* out) {
  for (int64_t b = 0; b < K / 32; ++b) {
    const double scale = std::ldexp(1.0, static_cast<int>(scales[b]) - 127);
    for (int64_t k = 32 * b; k < 32 * b + 32; ++k) {
      const uint8_t byte = blocks[k / 2];
      const unsigned nib = (k % 2 == 0) ? (byte & 0x0Fu) : (byte >> 4);
      out[k] = e2m1_value(nib) * scale;
    }
  }
}

// One (token, expert) pair: y = down( act( gate_up(x) ) ), fp32 result per output row.
// a_out (nullable, I floats) receives the fp32 gated activation before its rounding.
static void expert_ffn(const LayerArgs& A, int t, int e, float* y, float* a_out) {
  const int H = A.H, I = A.I;
  std::vector<double> xin(H), row(std::max(H, I)), ain(I);
  std::vector<float> g(2 * I);
  double s_in = 1.0, s_mid = 1.0;
  if (A.act_scale) {
    s_in = A.act_scale[0];
    s_mid = A.act_scale[1];
    for (int h = 0; h < H; ++h) {
      volatile float q = bf16_to_f32(A.x[(int64_t)t * H + h]) / A.act_scale[0];
      xin[h] = e4m3_value(e4m3_rne_satfinite(q));
    }
  } else {
    for (int h = 0; h < H; ++h) xin[h] = bf16_to_f32(A.x[(int64_t)t * H + h]);
  }
  // gate_up: g[r] = fp32( fp32(s_in * sum_h xin[h] W[r,h]) + b[r] )
  const int64_t gu_row_bytes = H / 2, gu_row_scales = H / 32;
  for (int r = 0; r < 2 * I; ++r) {
    const int64_t rr = (int64_t)e * 2 * I + r;
    dequant_row(A.gu_blocks + rr * gu_row_bytes, A.gu_scales + rr * gu_row_scales, H, row.data());
    double acc = 0.0;
    for (int h = 0; h < H; ++h) acc += xin[h] * row[h];
    volatile float prod = static_cast<float>(s_in * acc);
    g[r] = prod + A.gu_bias[rr];
  }
  // gated activation: a = silu(gate) * up in double, rounded to fp32, then to the
  // down-projection input precision (bf16, or e4m3 with the static scale s1).
  for (int i = 0; i < I; ++i) {
    const double gate = g[i], up = g[I + i];
    const double silu = gate / (1.0 + std::exp(-gate));
    const float a = static_cast<float>(silu * up);
    if (a_out) a_out[i] = a;
    if (A.act_scale) {
      volatile float q = a / A.act_scale[1];
      ain[i] = e4m3_value(e4m3_rne_satfinite(q));
    } else {
      ain[i] = bf16_to_f32(bf16_rne(a));
    }
  }
  // down: y[r] = fp32( fp32(s_mid * sum_i ain[i] Wd[r,i]) + bd[r] )
  const int64_t d_row_bytes = I / 2, d_row_scales = I / 32;
  for (int r = 0; r < H; ++r) {
    const int64_t rr = (int64_t)e * H + r;
    dequant_row(A.d_blocks + rr * d_row_bytes, A.d_scales + rr * d_row_scales, I, row.data());
    double acc = 0.0;
    for (int i = 0; i < I; ++i) acc += ain[i] * row[i];
    volatile float prod = static_cast<float>(s_mid * acc);
    y[r] = prod + A.d_bias[rr];
  }
}

static int check_layer(const LayerArgs& A) {
  if (!A.x || !A.router_w || !A.gu_blocks || !A.gu_scales || !A.gu_bias || !A.d_blocks ||
      !A.d_scales || !A.d_bias)
    return ORC_EINVAL;
  if (A.T < 0 || A.H <= 0 || A.I <= 0 || A.E <= 0 || A.k <= 0) return ORC_EINVAL;
  if (A.H % 32 != 0 || A.I % 32 != 0) return ORC_EALIGN;
  if (A.k > A.E) return ORC_EUNSUPPORTED;
  return ORC_OK;
}

// The MoE layer. dense == 0: routed-only (each token evaluates its k selected experts);
// dense != 0: every expert is evaluated for every token with gate weight 0 off the
// top-k. Both accumulate gate * y in ascending expert id in fp32 and round once to bf16.
// Outputs: out (T, H) bf16 bits; acc_out (T, H) fp32 (nullable); idx/wts (T, k) nullable.
int orc_moe_forward(const uint16_t* x, const uint16_t* router_w, const uint16_t* router_b,
                    const uint8_t* gu_blocks, const uint8_t* gu_scales, const float* gu_bias,
                    const uint8_t* d_blocks, const uint8_t* d_scales, const float* d_bias,
                    int E, int k, int T, int H, int I, const float* act_scale, int dense,
                    uint16_t* out, float* acc_out, int32_t* idx_out, float* w_out) {
  LayerArgs A{x, router_w, router_b, gu_blocks, gu_scales, gu_bias, d_blocks, d_scales, d_bias,
              E, k, T, H, I, act_scale};
  int rc = check_layer(A);
  if (rc) return rc;
#pragma omp parallel for schedule(dynamic, 1)
  for (int t = 0; t < T; ++t) {
    std::vector<float> logits(E), wts(k), y(H), acc(H, 0.0f), gate_of(E, 0.0f);
    std::vector<int32_t> idx(k);
    std::vector<char> selected(E, 0);
    orc_router_logits(x + (int64_t)t * H, router_w, router_b, 1, H, E, logits.data());
    orc_topk_softmax(logits.data(), 1, E, k, idx.data(), wts.data());
    for (int j = 0; j < k; ++j) { selected[idx[j]] = 1; gate_of[idx[j]] = wts[j]; }
    for (int e = 0; e < E; ++e) {
      if (!dense && !selected[e]) continue;
      expert_ffn(A, t, e, y.data(), nullptr);
      for (int r = 0; r < H; ++r) {
        volatile float term = gate_of[e] * y[r];
        acc[r] = acc[r] + term;
      }
    }
    for (int r = 0; r < H; ++r) {
      out[(int64_t)t * H + r] = bf16_rne(acc[r]);
      if (acc_out) acc_out[(int64_t)t * H + r] = acc[r];
    }
    if (idx_out) for (int j = 0; j < k; ++j) idx_out[(int64_t)t * k + j] = idx[j];
    if (w_out) for (int j = 0; j < k; ++j) w_out[(int64_t)t * k + j] = wts[j];
  }
  return ORC_OK;
}

// The expert FFN of given (row, expert) pairs: y[p] = expert_ffn(x[p], expert[p]) with the
// arithmetic of orc_moe_forward (bf16 or A-FP8 activations). x: (P, H) bf16 rows; expert:
// (P) ids in [0, E); y: (P, H) fp32. The per-pair half of the layer, for checking a
// partition of the experts over several ranks against the whole layer.
int orc_expert_rows(const uint16_t* x, const int32_t* expert, int P, const uint8_t* gu_blocks,
                    const uint8_t* gu_scales, const float* gu_bias, const uint8_t* d_blocks,
                    const uint8_t* d_scales, const float* d_bias, int E, int H, int I,
                    const float* act_scale, float* y) {
  LayerArgs A{x, x, nullptr, gu_blocks, gu_scales, gu_bias, d_blocks, d_scales, d_bias,
              E, 1, P, H, I, act_scale};
  int rc = check_layer(A);
  if (rc) return rc;
  for (int p = 0; p < P; ++p)
    if (expert[p] < 0 || expert[p] >= E) return ORC_EINVAL;
#pragma omp parallel for schedule(dynamic, 1)
  for (int p = 0; p < P; ++p) expert_ffn(A, p, expert[p], y + (int64_t)p * H, nullptr);
  return ORC_OK;
}

// Static per-tensor activation scales from a calibration batch (min-max observer):
// s0 = amax|x| / 448; s1 = amax over routed (token, expert) pairs of the bf16-path gated
// activation (fp32, before rounding) / 448.
int orc_calibrate(const uint16_t* x, const uint16_t* router_w, const uint16_t* router_b,
                  const uint8_t* gu_blocks, const uint8_t* gu_scales, const float* gu_bias,
                  const uint8_t* d_blocks, const uint8_t* d_scales, const float* d_bias,
                  int E, int k, int T, int H, int I, float* act_scale_out) {
  LayerArgs A{x, router_w, router_b, gu_blocks, gu_scales, gu_bias, d_blocks, d_scales, d_bias,
              E, k, T, H, I, nullptr};
  int rc = check_layer(A);
  if (rc) return rc;
  float ax = 0.0f;
  for (int64_t i = 0; i < (int64_t)T * H; ++i) ax = std::max(ax, std::fabs(bf16_to_f32(x[i])));
  std::vector<float> amid(T, 0.0f);
#pragma omp parallel for schedule(dynamic, 1)
  for (int t = 0; t < T; ++t) {
    std::vector<float> logits(E), wts(k), y(H), a(I);
    std::vector<int32_t> idx(k);
    orc_router_logits(x + (int64_t)t * H, router_w, router_b, 1, H, E, logits.data());
    orc_topk_softmax(logits.data(), 1, E, k, idx.data(), wts.data());
    float m = 0.0f;
    for (int j = 0; j < k; ++j) {
      expert_ffn(A, t, idx[j], y.data(), a.data());
      for (int i = 0; i < I; ++i) m = std::max(m, std::fabs(a[i]));
    }
    amid[t] = m;
  }
  float am = 0.0f;
  for (int t = 0; t < T; ++t) am = std::max(am, amid[t]);
  act_scale_out[0] = ax / 448.0f;
  act_scale_out[1] = am / 448.0f;
  return ORC_OK;
}

// --------------------------------------------- quantizer along an arbitrary axis ---

// "quantization_mxfp4", Primitives (MXFP4Quantizer.quantize(w, axis)): the tensor is
// viewed as (outer, K, inner) with the contracting axis (length K) in the middle; that
// axis moves to the end and every resulting row of K values is quantized as orc_quantize
// does. blocks: (outer, inner, K/2); scales: (outer, inner, K/32).
int orc_quantize_axis(const float* w, int64_t outer, int64_t K, int64_t inner, uint8_t* blocks,
                      uint8_t* scales) {
  if (outer < 0 || K < 0 || inner < 0) return ORC_EINVAL;
  if (K % 32 != 0) return ORC_EALIGN;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < outer * inner; ++r) {
    const int64_t o = r / inner, i = r % inner;
    std::vector<float> row(K);
    for (int64_t k = 0; k < K; ++k) row[k] = w[(o * K + k) * inner + i];
    orc_quantize(row.data(), 1, K, blocks + r * (K / 2), scales + r * (K / 32));
  }
  return ORC_OK;
}

// The inverse view: dequantize every (outer, inner) row of K values and put the axis
// back in the middle: out (outer, K, inner). Either output may be null.
int orc_dequantize_axis(const uint8_t* blocks, const uint8_t* scales, int64_t outer, int64_t K,
                        int64_t inner, float* out_f32, uint16_t* out_bf16) {
  if (outer < 0 || K < 0 || inner < 0) return ORC_EINVAL;
  if (K % 32 != 0) return ORC_EALIGN;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < outer * inner; ++r) {
    const int64_t o = r / inner, i = r % inner;
    std::vector<float> f(K);
    std::vector<uint16_t> b(K);
    orc_dequantize(blocks + r * (K / 2), scales + r * (K / 32), 1, K, f.data(), b.data());
    for (int64_t k = 0; k < K; ++k) {
      if (out_f32) out_f32[(o * K + k) * inner + i] = f[k];
      if (out_bf16) out_bf16[(o * K + k) * inner + i] = b[k];
    }
  }
  return ORC_OK;
}

// ------------------------------------------------------------------------ linear ---

// MXFP4 weight-only linear ("quantization_mxfp4", As a quantize_model scheme), with the
// optional FP8 E4M3 static per-tensor activations of the W-MXFP4 / A-FP8 scheme:
// y[t, n] = fp32( fp32(s * sum_k xin[t, k] W[n, k]) + b[n] ), out = bf16(y), where xin is
// the bf16 input (s = 1) or, with act_scale != null, e4m3(fp32(x / s)) with s = *act_scale.
// x: (T, K) bf16; blocks (N, K/2), scales (N, K/32); bias (N) fp32 or null (zero).
int orc_linear(const uint16_t* x, int T, int K, const uint8_t* blocks, const uint8_t* scales, int N,
               const float* bias, const float* act_scale, uint16_t* out, float* acc_out) {
  if (!x || !blocks || !scales || !out || T < 0 || K <= 0 || N <= 0) return ORC_EINVAL;
  if (K % 32 != 0) return ORC_EALIGN;
  const double s = act_scale ? static_cast<double>(*act_scale) : 1.0;
#pragma omp parallel for schedule(dynamic, 1)
  for (int t = 0; t < T; ++t) {
    std::vector<double> xin(K), row(K);
    for (int k = 0; k < K; ++k) {
      const float v = bf16_to_f32(x[(int64_t)t * K + k]);
      if (act_scale) {
        volatile float q = v / *act_scale;
        xin[k] = e4m3_value(e4m3_rne_satfinite(q));
      } else {
        xin[k] = v;
      }
    }
    for (int n = 0; n < N; ++n) {
      dequant_row(blocks + (int64_t)n * (K / 2), scales + (int64_t)n * (K / 32), K, row.data());
      double acc = 0.0;
      for (int k = 0; k < K; ++k) acc += xin[k] * row[k];
      volatile float prod = static_cast<float>(s * acc);
      const float y = prod + (bias ? bias[n] : 0.0f);
      out[(int64_t)t * N + n] = bf16_rne(y);
      if (acc_out) acc_out[(int64_t)t * N + n] = y;
    }
  }
  return ORC_OK;
}

// FP8 E4M3 static per-tensor linear ("gpt-oss-120b-mxfp4-fp8attn-v2", Model Details and
// Quantization Recipe: Q/K/V/O projections with FP8 E4M3 weights, a static per-tensor
// weight_scale and a static per-tensor input_scale). The dequantized operands are
// dec(xq) * s_x and dec(wq) * s_w, so
// y[t, n] = fp32( s_x * s_w * sum_k dec(xq[t, k]) dec(wq[n, k]) ) + b[n], out = bf16(y),
// with xq = e4m3(fp32(x / s_x)). x: (T, K) bf16; wq: (N, K) e4m3 codes; bias null = zero.
int orc_fp8_linear(const uint16_t* x, int T, int K, const uint8_t* wq, int N, float s_x, float s_w,
                   const float* bias, uint16_t* out, float* acc_out) {
  if (!x || !wq || !out || T < 0 || K <= 0 || N <= 0 || !(s_x > 0.0f) || !(s_w > 0.0f)) return ORC_EINVAL;
#pragma omp parallel for schedule(dynamic, 1)
  for (int t = 0; t < T; ++t) {
    std::vector<double> xin(K);
    for (int k = 0; k < K; ++k) {
      volatile float q = bf16_to_f32(x[(int64_t)t * K + k]) / s_x;
      xin[k] = e4m3_value(e4m3_rne_satfinite(q));
    }
    for (int n = 0; n < N; ++n) {
      double acc = 0.0;   // exact: e4m3 products have at most 8 significant bits
      for (int k = 0; k < K; ++k) acc += xin[k] * e4m3_value(wq[(int64_t)n * K + k]);
      volatile float prod = static_cast<float>(static_cast<double>(s_x) * static_cast<double>(s_w) * acc);
      const float y = prod + (bias ? bias[n] : 0.0f);
      out[(int64_t)t * N + n] = bf16_rne(y);
      if (acc_out) acc_out[(int64_t)t * N + n] = y;
    }
  }
  return ORC_OK;
}

}  // extern "C"
