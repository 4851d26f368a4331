// Host-side launchers of the library's kernels (internal; the public ABI is mxfp4_moe.h).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace mxmoe {

cudaError_t launch_quantize(const float* w, int64_t rows, int64_t K, uint8_t* blocks,
                            uint8_t* scales, cudaStream_t st, int sms);
cudaError_t launch_dequantize(const uint8_t* blocks, const uint8_t* scales, int64_t rows,
                              int64_t K, void* out, int out_dtype, cudaStream_t st, int sms);

// the codec along an arbitrary axis: the tensor as (outer, K, inner), packed (outer, inner, K/2)
cudaError_t launch_quantize_axis(const float* w, int64_t outer, int64_t K, int64_t inner, uint8_t* blocks,
                                 uint8_t* scales, cudaStream_t st, int sms);
cudaError_t launch_dequantize_axis(const uint8_t* blocks, const uint8_t* scales, int64_t outer, int64_t K,
                                   int64_t inner, void* out, int out_dtype, cudaStream_t st, int sms);

cudaError_t launch_router(const uint16_t* x, const uint16_t* wr, const uint16_t* br, int T, int H,
                          int E, float* logits, cudaStream_t st);
// rest / n_rest: further K-range partials of the logits (see launch_router_tc), summed into
// logits in range order before the selection; n_rest = 0 for complete logits.
cudaError_t launch_topk(float* logits, const float* rest, int n_rest, int T, int E, int k, int32_t* idx, float* w,
                        cudaStream_t st);
int permute_chunks(int64_t P);
cudaError_t launch_permute(const int32_t* idx, int T, int E, int k, int32_t* counts_ws,
                           int32_t* offsets, int32_t* perm_token, int32_t* perm_slot,
                           int32_t* inv, int32_t* active, int32_t* n_active, int* err,
                           cudaStream_t st, int* launches);
bool route_small_supported(int T, int E, int k);
// Router GEMM on the tensor cores (csrc/router_sm100.cu): H % 64 == 0, 8 <= E <= 256 with
// E % 8 == 0, 16-byte aligned x / router_w / logits. It splits K into ksplit ranges
// (router_tc_ksplit): range 0 (with the bias) goes to logits, range s > 0 to
// logits_rest + (s-1)*T*E; launch_topk adds them.
bool router_tc_supported(int T, int H, int E, const void* x, const void* wr, const void* logits);
int router_tc_ksplit(int T, int H, int sms);
cudaError_t launch_router_tc(const uint16_t* x, const uint16_t* wr, const uint16_t* br, int T, int H, int E,
                             int ksplit, float* logits, float* logits_rest, int* err, cudaStream_t st);
cudaError_t launch_route_small(const uint16_t* x, const uint16_t* wr, const uint16_t* br, int T, int H, int E,
                               int k, float* logits, unsigned* ticket, unsigned* tok_tickets, int32_t* topk_idx,
                               float* topk_w, int32_t* offsets, int32_t* perm_token, int32_t* perm_slot, int32_t* inv,
                               int32_t* active, int32_t* n_active, int* err, cudaStream_t st);
cudaError_t launch_fp8_quant(const uint16_t* x, int64_t n, float s, uint8_t* q, cudaStream_t st,
                             int sms);
cudaError_t launch_fp8_quant_as_bf16(const uint16_t* x, int64_t n, float s, uint16_t* xq,
                                     cudaStream_t st, int sms);
cudaError_t launch_quant_scatter_fp8(const uint16_t* x, const int32_t* topk_idx, const int32_t* inv, int T,
                                    int k, int E, int64_t P, int H, float s, uint8_t* a1, cudaStream_t st,
                                    int sms);
cudaError_t launch_amax_bf16(const uint16_t* x, int64_t n, unsigned* amax_bits, cudaStream_t st,
                             int sms);
cudaError_t launch_finalize_scales(const unsigned* amax_bits, float* out, cudaStream_t st);

struct CombineArgs {      // the combine folded into the down kernel (small batches)
  uint16_t* out;
  const int32_t* topk_idx;
  const float* topk_w;
  const int32_t* inv;
  unsigned* tickets;      // rows_total / 16 counters, zero between calls
  int T, k;
};
cudaError_t launch_expert_mma(const uint8_t* blocks, const uint8_t* scales, const float* bias,
                              int rows_total, int K, const uint16_t* act, const int32_t* act_row,
                              const int32_t* offsets, const int32_t* active,
                              const int32_t* n_active, int max_active, float s_in, int mode, int I,
                              float s_mid, uint16_t* act_out, float* y_out, unsigned* amax_bits,
                              int max_tokens_per_expert, int* err, const CombineArgs* combine,
                              cudaStream_t st);
cudaError_t expert_mma_set_smem_limits(int max_K);

bool tc_gemm_supported(int H, int I, const void* gu_blocks, const void* d_blocks, const void* gu_scales,
                       const void* d_scales);
cudaError_t tc_gemm_prepare(int E);
cudaError_t launch_tc_gemm(bool gate_up, const uint8_t* a, int64_t P_rows, int K, const uint8_t* blocks,
                           const uint8_t* scales, const float* bias, int E, int n_out, const int32_t* offsets,
                           float s_in, float s_out, uint8_t* a_out, float* y_out, int* err, int sms,
                           cudaStream_t st, bool a_shared = false);

// bf16 activations on the tcgen05 grouped GEMM: each activation row as two e4m3 parts with
// e8m0 scales per 32-value block (csrc/gemm_bf16_sm100.cu)
cudaError_t launch_split_parts(const uint16_t* src, const int32_t* perm, int T, int64_t P, int K, uint8_t* parts,
                               uint8_t* scales, int sms, cudaStream_t st);
cudaError_t tc_parts_gemm_prepare(int E);
cudaError_t launch_tc_parts_gemm(bool gate_up, const uint8_t* parts, const uint8_t* a_scales, int64_t P_rows, int K,
                                 const uint8_t* blocks, const uint8_t* scales, const float* bias, int E, int n_out,
                                 const int32_t* offsets, uint16_t* a_out, float* y_out, int* err, int sms,
                                 cudaStream_t st, bool a_shared = false);

struct DecodeGemmArgs {   // tensor-core decode path (kind::mxf4: packed e2m1 weights x e2m1 token parts)
  const uint8_t* gu_blocks;
  const uint8_t* gu_scales;
  const float* gu_bias;
  const uint8_t* d_blocks;
  const uint8_t* d_scales;
  const float* d_bias;
  int E, H, I, T, k;
  int64_t P;
  int max_active;               // bound on the active experts (min(E, P))
  int sms;
  const int32_t* offsets;
  const int32_t* active;
  const int32_t* n_active;
  const uint8_t* xs;            // gate_up B operand: (P*4, H/2) packed e2m1 parts
  const uint8_t* sfb;           // its scale records (decode_tc_sfb_bytes(E, H, T))
  uint8_t* xs_mid;              // down B operand: (P*4, I/2)
  uint8_t* sfb_mid;             // (decode_tc_sfb_bytes(E, I, T))
  float s0;                     // B scale of gate_up (FP8 s0, else 1)
  float s1_quant;               // FP8: scale of a's e4m3 cast; 0: bf16 intermediate
  float s1_in;                  // B scale of down (FP8 s1, else 1)
  float* y;                     // (P, H) fp32
  float* part;                  // split-K partials (decode_tc_part_bytes)
  unsigned* split_tickets_gu;   // zero between calls (decode_tc_ticket_count covers both)
  unsigned* split_tickets_d;
  int* err;
};
constexpr int kDecodeMaxT = 64;      // tokens the tensor-core decode path takes
constexpr int kDecodeMaxGroups = 320;  // row groups (an expert's routed rows, 56 at a time)
// One-launch decode layer (csrc/decode_layer_sm100.cu): routing, token operand, gate_up,
// down and combine of at most kDecodeLayerMaxT tokens in one persistent grid of one CTA
// per SM.
constexpr int kDecodeLayerMaxT = 8;
struct DecodeLayerSizes {   // workspace pieces, bytes (counters: unsigned words, zero between calls)
  size_t xs, sfx, xs_mid, sf_mid, part, dpart, counters;
};
struct DecodeLayerArgs {
  const uint16_t* x;
  const uint16_t* router_w;
  const uint16_t* router_b;     // nullable
  const uint8_t* gu_blocks;
  const uint8_t* gu_scales;
  const float* gu_bias;
  const uint8_t* d_blocks;
  const uint8_t* d_scales;
  const float* d_bias;
  int E, H, I, T, k;
  bool fp8;                     // static per-tensor FP8 activations (s0, s1)
  float s0, s1;
  int sms;                      // grid size: every CTA must be resident at once
  float* logits;                // (T, E)
  uint8_t* xs;
  uint8_t* sfx;
  uint8_t* xs_mid;
  uint8_t* sf_mid;
  float* part;
  float* dpart;
  unsigned* counters;           // decode_layer_sizes().counters words, zero between calls
  int32_t* topk_idx;            // (T, k), nullable
  float* topk_w;
  uint16_t* out;                // (T, H) bf16
  int* err;
};
bool decode_layer_supported(int H, int I, int T, int E, int k, int sms, const void* gu_blocks, const void* d_blocks,
                            const void* gu_scales, const void* d_scales);
cudaError_t decode_layer_prepare();
DecodeLayerSizes decode_layer_sizes(int T, int H, int I, int sms);
cudaError_t launch_decode_layer(const DecodeLayerArgs& a, cudaStream_t st);

bool decode_tc_supported(int H, int I, int T, const void* gu_blocks, const void* d_blocks, const void* gu_scales,
                         const void* d_scales);
cudaError_t decode_tc_prepare();
size_t decode_tc_xs_bytes(int64_t P, int K);
size_t decode_tc_sfb_bytes(int E, int K, int T);       // B scale records, one per 256-deep stage
size_t decode_tc_part_bytes(int64_t P, int H, int I);
size_t decode_tc_ticket_count(int H, int I);
// offsets of the three ticket arrays inside the decode_tc_ticket_count block
inline size_t decode_tc_tickets_d(int I) { return static_cast<size_t>(kDecodeMaxGroups) * ((I + 127) / 128) * 4; }
cudaError_t launch_split_tokens(bool fp8, const uint16_t* x, const int32_t* topk_idx, const int32_t* inv,
                                const int32_t* offsets, int T, int E, int H, int k, float s0, uint8_t* xs, uint8_t* sfb,
                                cudaStream_t st);
cudaError_t launch_decode_gemm(bool gate_up, const DecodeGemmArgs& a, cudaStream_t st);


// dense all-experts path (csrc/dense.cu): gates (T, E) and offsets e * T; the weighted sum
// over all experts of y laid out expert-major (E * T, H)
cudaError_t launch_dense_setup(const int32_t* topk_idx, const float* topk_w, int T, int E, int k, float* gates,
                               int32_t* offsets, cudaStream_t st, int sms);
cudaError_t launch_dense_combine(const float* y, const float* gates, int T, int H, int E, uint16_t* out,
                                 cudaStream_t st, int sms);

// a plain MXFP4 linear as a one-expert grouped GEMM (csrc/dense.cu)
cudaError_t launch_linear_setup(int T, int N, int32_t* offsets, int32_t* active, int32_t* n_active, float* zero_bias,
                                cudaStream_t st, int sms);
cudaError_t launch_f32_to_bf16(const float* y, int64_t n, uint16_t* out, cudaStream_t st, int sms);

cudaError_t launch_combine(const float* y, const int32_t* topk_idx, const float* topk_w,
                           const int32_t* inv, int T, int H, int k, uint16_t* out, cudaStream_t st,
                           int sms);


// FP8 E4M3 static per-tensor linear (csrc/linear_sm100.cu): xq (T, K) e4m3, wq (N, K) e4m3,
// out = bf16(fp32(s * xq.wq^T) + bias); ksplit > 1 needs part = (ksplit, T, N) fp32
int fp8_linear_ksplit(int T, int K, int N, int sms);
bool fp8_linear_supported();
cudaError_t launch_fp8_linear(const uint8_t* xq, int T, int K, const uint8_t* wq, int N, float s, const float* bias,
                              uint16_t* out, float* part, int ksplit, int* err, int sms, cudaStream_t st);

// mxmoe_tc_rate_probe: back-to-back kind::mxf8f6f4 MMAs (M = 128, N = n) on `ctas` CTAs
cudaError_t launch_tc_rate(int n, int with_copy, int random, int iters, int ctas, int* err, cudaStream_t st);

// mxmoe_selftest_wait_timeout: a bounded wait that expires (ETIMEOUT in *err)
cudaError_t launch_wait_selftest(int* err, cudaStream_t st);

}  // namespace mxmoe
