/*
 * mxfp4_moe.h -- C ABI of libmxfp4moe.so: the routed Mixture-of-Experts expert layer
 * with OCP MXFP4 expert weights, for NVIDIA B200 (sm_100a).
 *
 * What the operations compute (web pages, cited by title and section):
 *  - MXFP4: "quantization_mxfp4" (KerasFormers), intro and "Primitives": e2m1 values
 *    packed two per byte, one e8m0 scale per 32 values along the contracting dim;
 *    dequantize = codebook[nibble] * 2^(scale - 127); quantize picks the block exponent
 *    floor(log2(amax)) - 2 and rounds each value to the nearest FP4 grid point.
 *  - The expert layer: same page, "As GPT-OSS's native format": gate_up_proj (E, 2I, H)
 *    and down_proj (E, H, I) as blocks + scales, biases in full precision, only the
 *    top-k routed experts are evaluated on decode.
 *  - W-MXFP4 / A-FP8: "amd/gpt-oss-20b-MoE-Quant-W-MXFP4-A-FP8-KV-FP8", "Quantization
 *    schemes": MoE MLP activations in FP8 with a symmetric per-tensor scale, router not
 *    quantized; "gpt-oss-120b-mxfp4-fp8attn-v2", "Model Details": E4M3 static scales.
 *
 * Conventions shared by every entry point
 *  - Pointers named as device memory must be device (cudaMalloc'd) memory of the current
 *    device, 16-byte aligned, caller-owned. The library never frees caller memory.
 *  - bf16 tensors are passed as arrays of uint16_t holding bf16 bit patterns.
 *  - All tensors are dense row-major with the contracting dimension last.
 *  - Packed MXFP4: a tensor of logical shape (R, K) is `blocks` (R, K/2) uint8, where
 *    element 2j is the low nibble of byte j and 2j+1 the high nibble, plus `scales`
 *    (R, K/32) uint8 e8m0 (value 2^(s-127)). In the expert layer this is
 *    gu_blocks (E, 2I, H/2) [= (E, 2I, H/32, 16)], gu_scales (E, 2I, H/32),
 *    d_blocks (E, H, I/2), d_scales (E, H, I/32). gate_up rows [0, I) are the gate
 *    projection and rows [I, 2I) the up projection.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream). Every
 *    call is asynchronous on it unless stated; the library never synchronizes the
 *    device inside a call.
 *  - Return value: MXMOE_OK (0) or a negative MXMOE_E* code. On error nothing is
 *    launched and mxmoe_last_error() (thread-local) describes the cause.
 *  - T == 0 (or rows == 0) is a no-op returning MXMOE_OK.
 *  - Non-finite inputs give unspecified (but non-faulting) results.
 *  - The library keeps one grow-only workspace per device (device memory it allocates
 *    with cudaMalloc on first use, released by mxmoe_release()). A call that must grow
 *    it allocates, so the first call at a new maximum size must not be inside a CUDA
 *    graph capture. Calls that share a device must not overlap on the GPU (the
 *    workspace is shared): issue them on one stream, or order the streams.
 */
#ifndef MXFP4_MOE_H
#define MXFP4_MOE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MXMOE_OK 0
#define MXMOE_EINVAL (-1)        /* null pointer, negative size, misaligned pointer */
#define MXMOE_EALIGN (-2)        /* contracting dim (K, H or I) not a multiple of 32 */
#define MXMOE_EUNSUPPORTED (-3)  /* k > E, k > 8, E > 256, out_dtype unknown, ... */
#define MXMOE_ECUDA (-4)         /* a CUDA runtime/driver call or a launch failed */
#define MXMOE_ETIMEOUT (-5)      /* a bounded device wait gave up (reported by mxmoe_check) */
#define MXMOE_ENOMEM (-6)        /* workspace allocation failed */
#define MXMOE_EDEVICE (-7)       /* a kernel found bad data, e.g. an expert id out of range */

#define MXMOE_OUT_F32 0
#define MXMOE_OUT_BF16 1

/* mxfp4_quantize -- "quantization_mxfp4", Primitives (quantize_to_mxfp4).
 * w: device fp32 (rows, K). Writes blocks: device (rows, K/2) uint8 and scales: device
 * (rows, K/32) uint8. Per 32-value block: e = clamp(floor(log2(amax)) - 2, -127, 127),
 * scale byte e + 127 (an all-zero block gets byte 0), each value rounded to the nearest
 * of +-{0, 0.5, 1, 1.5, 2, 3, 4, 6} * 2^e with ties to the even code, magnitudes past 6
 * saturating; the sign bit is copied from the input (so -0.0 packs as nibble 8).
 * Errors: MXMOE_EALIGN if K % 32 != 0 ("As a quantize_model scheme": a clear error);
 * MXMOE_EINVAL for null pointers, negative sizes, or w / blocks not 16-byte aligned. */
int mxfp4_quantize(const float* w, int64_t rows, int64_t K, uint8_t* blocks, uint8_t* scales,
                   void* stream);

/* mxfp4_dequantize -- "quantization_mxfp4", Primitives (dequantize_mxfp4).
 * out[r, k] = codebook[nibble] * 2^(scale - 127), written as fp32 (out_dtype
 * MXMOE_OUT_F32) or bf16 bits (MXMOE_OUT_BF16) into device memory out (rows, K).
 * Every finite result is exact in both types (subnormals included); results at or
 * beyond 2^128 are +-inf (scale bytes 253..255). Errors as mxfp4_quantize (with blocks
 * and out the pointers that must be 16-byte aligned), plus MXMOE_EUNSUPPORTED for an
 * unknown out_dtype. */
int mxfp4_dequantize(const uint8_t* blocks, const uint8_t* scales, int64_t rows, int64_t K,
                     void* out, int out_dtype, void* stream);

/* mxfp4_quantize_axis / mxfp4_dequantize_axis -- the codec along an arbitrary contracting
 * axis ("quantization_mxfp4" (KerasFormers), Primitives: MXFP4Quantizer.quantize(w, axis)
 * quantizes along one axis, which it moves to the end). The tensor w is viewed as
 * (outer, K, inner): K is the length of the contracting axis, outer the product of the
 * dims before it, inner the product of the dims after it (inner = 1: the last axis, the
 * same as mxfp4_quantize). The packed result has the axis last: blocks (outer, inner,
 * K/2), scales (outer, inner, K/32), each row of K values quantized exactly as
 * mxfp4_quantize does (same bits). mxfp4_dequantize_axis is the inverse view: it writes
 * (outer, K, inner) fp32 (out_dtype MXMOE_OUT_F32) or bf16 (MXMOE_OUT_BF16) values, the
 * same values as mxfp4_dequantize. All pointers are device memory, caller-owned; w,
 * blocks and out 16-byte aligned. Errors: MXMOE_EALIGN if K % 32 != 0 (the clear error of
 * "As a quantize_model scheme"), MXMOE_EINVAL for a negative size, a null or misaligned
 * pointer, MXMOE_EUNSUPPORTED for an unknown out_dtype, MXMOE_ECUDA on a launch error.
 * Any zero size is a no-op. */
int mxfp4_quantize_axis(const float* w, int64_t outer, int64_t K, int64_t inner, uint8_t* blocks,
                        uint8_t* scales, void* stream);
int mxfp4_dequantize_axis(const uint8_t* blocks, const uint8_t* scales, int64_t outer, int64_t K,
                          int64_t inner, void* out, int out_dtype, void* stream);

/* mxfp4_linear -- a plain MXFP4 weight-only linear layer ("quantization_mxfp4", As a
 * quantize_model scheme: a Dense kernel stored MXFP4 and dequantized on the fly), with the
 * optional FP8 E4M3 static per-tensor activations of the W-MXFP4 / A-FP8 scheme ("amd/gpt-
 * oss-20b-MoE-Quant-W-MXFP4-A-FP8-KV-FP8", Quantization schemes):
 *   out[t, n] = bf16( fp32(s * sum_k xin[t, k] * W[n, k]) + bias[n] ),
 * xin = x (bf16, s = 1) or, with act_scale != NULL, e4m3(fp32(x / s)) with s = *act_scale
 * (a HOST pointer to one float). x: device bf16 (T, K); blocks (N, K/2) and scales
 * (N, K/32) as mxfp4_quantize packs a (N, K) weight; bias: device fp32 (N) or NULL (zero);
 * out: device bf16 (T, N). More than 64 tokens run on the tcgen05 grouped GEMM (one
 * expert) when K and N are multiples of 64 (K <= 4608), else the register-dequant
 * kernel. Errors: MXMOE_EALIGN (K % 32, N % 16), MXMOE_EINVAL (sizes, null or misaligned
 * pointers: x, blocks, out and bias 16-byte aligned), MXMOE_ECUDA. Uses the library
 * workspace; T = 0 is a no-op. */
int mxfp4_linear(const uint16_t* x, int T, int K, const uint8_t* blocks, const uint8_t* scales, int N,
                 const float* bias, const float* act_scale, uint16_t* out, void* stream);

/* fp8_linear -- the FP8 E4M3 static per-tensor linear of the attention projections
 * ("gpt-oss-120b-mxfp4-fp8attn-v2", Model Details and Quantization Recipe: Q/K/V/O with
 * FP8 E4M3 weights, a static per-tensor weight scale and input scale):
 *   out[t, n] = bf16( fp32(fp32(s_x * s_w) * sum_k xq[t, k] * wq[n, k]) + bias[n] ),
 * xq = e4m3(fp32(x / s_x)) (round to nearest even, saturating at +-448). x: device bf16
 * (T, K); wq: device E4M3 codes (N, K) (the checkpoint's FP8 weight); s_x, s_w: the
 * static input and weight scales (> 0); bias: device fp32 (N) or NULL; out: device bf16
 * (T, N). Runs on tcgen05 (kind::f8f6f4) with fp32 accumulation, K split over the SMs
 * when there are few tokens. Errors: MXMOE_EALIGN (K % 32, N % 8), MXMOE_EINVAL (sizes,
 * scales, null or misaligned pointers: x, wq, out, bias 16-byte aligned), MXMOE_ECUDA.
 * Uses the library workspace; T = 0 is a no-op. */
int fp8_linear(const uint16_t* x, int T, int K, const uint8_t* wq, int N, float s_x, float s_w,
               const float* bias, uint16_t* out, void* stream);

/* moe_route_topk -- router + top-k softmax (GPT-OSS top-k routing; router kept in bf16:
 * "gpt-oss-120b-mxfp4-fp8attn-v2", config.json modules_to_not_convert).
 * x: device bf16 (T, H); router_w: device bf16 (E, H); router_b: device bf16 (E) or NULL.
 * logits[t, e] = sum_h x*Wr + br in fp32 arithmetic; logits_out: device fp32 (T, E) or
 * NULL. topk_idx: device int32 (T, k), the k largest logits in descending order, ties to
 * the lower expert id; topk_w: device fp32 (T, k) = softmax over those k logits.
 * Limits: 1 <= k <= 8, k <= E <= 256, H % 32 == 0. */
int moe_route_topk(const uint16_t* x, const uint16_t* router_w, const uint16_t* router_b, int T,
                   int H, int E, int k, float* logits_out, int32_t* topk_idx, float* topk_w,
                   void* stream);

/* moe_topk_from_logits -- the top-k + softmax half of moe_route_topk on given fp32
 * logits (device, (T, E)); same outputs and limits. Lets the selection be checked
 * bit-exactly on identical logits. */
int moe_topk_from_logits(const float* logits, int T, int E, int k, int32_t* topk_idx,
                         float* topk_w, void* stream);

/* moe_permute -- group the T*k (token, slot) pairs by expert (the routed dispatch of
 * "quantization_mxfp4", As GPT-OSS's native format). topk_idx: device int32 (T, k).
 * offsets: device int32 (E+1), offsets[e] = first position of expert e; perm_token,
 * perm_slot: device int32 (T*k): position p holds the pair (perm_token[p], perm_slot[p]).
 * Within an expert, pairs keep ascending token order (a stable counting sort, the same
 * result on every run). An expert id outside [0, E) sets MXMOE_EDEVICE in the device
 * error word (see mxmoe_check) and that pair is dropped. */
int moe_permute(const int32_t* topk_idx, int T, int E, int k, int32_t* offsets,
                int32_t* perm_token, int32_t* perm_slot, void* stream);

/* moe_permute_noalloc -- moe_permute for callers that cannot allocate device memory.
 * The pages have no counterpart to this entry point; it exists for deployments where a
 * library must not call cudaMalloc: a serving runtime that reserves all device memory at
 * start-up (for example handing what is left to a KV cache) and forbids allocation on its
 * hot path, or a latency-bound loop that cannot afford cudaMalloc's implicit device
 * synchronization. moe_permute itself grows the library workspace with cudaMalloc on its
 * first call at a size; this variant allocates nothing and keeps its scratch (per-chunk
 * expert histograms, the list of active experts) in a fixed 132,352-byte array in the
 * library's device image, which every GPU that loads the library holds until the process
 * exits.
 * Same arguments, outputs and ordering as moe_permute. Limits: T*k <= 262144 and
 * E <= 256; larger sizes return MXMOE_EUNSUPPORTED with a message and launch nothing.
 * Differences: a pair with an expert id outside [0, E) is dropped without touching the
 * device error word; offsets[E] then counts only the kept pairs, and perm_token /
 * perm_slot positions from offsets[E] to T*k - 1 are left as they were (unwritten).
 * Every call looks up the array's device address on the current device
 * (cudaGetSymbolAddress; the first lookup in a process may load the library's device
 * image), so make the first call before any stream capture begins. All calls share the
 * one array and each call rewrites what it reads, so calls that overlap on the GPU
 * (different streams, no ordering) race with each other: order them. */
int moe_permute_noalloc(const int32_t* topk_idx, int T, int E, int k, int32_t* offsets,
                        int32_t* perm_token, int32_t* perm_slot, void* stream);

/* moe_fp8_quantize -- the A-FP8 activation cast ("amd/gpt-oss-20b-MoE-Quant-W-MXFP4-A-
 * FP8-KV-FP8", Quantization schemes): q[i] = e4m3(fp32(x[i] / s)), IEEE fp32 division,
 * round-to-nearest-even, saturating to +-448 (E4M3 "fn" has no infinity; NaN stays NaN).
 * x: device bf16 (n); q: device uint8 (n); s: the static per-tensor scale (> 0). */
int moe_fp8_quantize(const uint16_t* x, int64_t n, float s, uint8_t* q, void* stream);

/* moe_mxfp4_forward -- the MoE expert layer ("quantization_mxfp4", As GPT-OSS's native
 * format; A-FP8 option per "amd/gpt-oss-20b-MoE-Quant-W-MXFP4-A-FP8-KV-FP8").
 * For every token t: route (as moe_route_topk), then for each selected expert e with gate
 * w: g = s0 * (xin . Wgu[e]^T) + gu_bias[e];  a = silu(g[:I]) * g[I:];
 * y = s1 * (ain . Wd[e]^T) + d_bias[e];  out[t] = bf16(sum over the k experts of w * y),
 * accumulated in fp32.
 *  - act_scale == NULL: bf16 activations, xin = x, ain = bf16(a), s0 = s1 = 1. (With
 *    T*k >= 1024 the products run on the tensor cores with each activation written as two
 *    e4m3 parts under per-32-value block scales: exact except for elements about 2^14 or
 *    more below their block's largest, which keep an error under ~2^-21 of it. With
 *    T <= 64 the tensor-core decode path expands each activation into four e2m1 parts,
 *    which moves a 2880-long dot product by about 2e-4 of the largest output; at most 8
 *    tokens run as one kernel launch, routing through the combine.)
 *  - act_scale != NULL: HOST pointer to two floats {s0, s1} (static per-tensor scales
 *    read during the call); xin = e4m3(x / s0), ain = e4m3(a / s1).
 * x: device bf16 (T, H); router_w bf16 (E, H); router_b bf16 (E) or NULL; gu_bias fp32
 * (E, 2I); d_bias fp32 (E, H); packed weights as described above; out: device bf16 (T, H).
 * Limits: H, I multiples of 32 (MXMOE_EALIGN), 1 <= k <= 8, k <= E <= 256, T < 2^24.
 * The weights are read in place (no copy, no re-layout). Uses the library workspace. */
int moe_mxfp4_forward(const uint16_t* x, const uint16_t* router_w, const uint16_t* router_b,
                      const uint8_t* gu_blocks, const uint8_t* gu_scales, const float* gu_bias,
                      const uint8_t* d_blocks, const uint8_t* d_scales, const float* d_bias,
                      int E, int k, int T, int H, int I, const float* act_scale, uint16_t* out,
                      void* stream);

/* moe_mxfp4_forward_dense -- the dense all-experts path of the same layer ("quantization_
 * mxfp4" (KerasFormers), As GPT-OSS's native format: long prefills may run all experts on
 * every token instead of the routed ones, with identical output). Same arguments, layouts,
 * activations (act_scale) and result definition as moe_mxfp4_forward: every token is
 * multiplied through all E experts, each expert's output weighted by the token's gate
 * (its softmax weight for the k selected experts, 0 for the others) and summed over all E
 * experts in ascending id, fp32, one bf16 rounding. With finite values that sum equals the
 * routed one term for term, so the output equals moe_mxfp4_forward's wherever both run
 * the same expert kernels (T > 64). The work is E/k times the routed path's. Limits: H and
 * I multiples of 64 in [128, 4608], 32-byte aligned blocks, E*T*max(H, I) < 2^31
 * (MXMOE_EUNSUPPORTED otherwise). Uses the library workspace (E*T*(I + 4H) bytes and more). */
int moe_mxfp4_forward_dense(const uint16_t* x, const uint16_t* router_w, const uint16_t* router_b,
                            const uint8_t* gu_blocks, const uint8_t* gu_scales, const float* gu_bias,
                            const uint8_t* d_blocks, const uint8_t* d_scales, const float* d_bias,
                            int E, int k, int T, int H, int I, const float* act_scale, uint16_t* out,
                            void* stream);

/* moe_mxfp4_experts -- the expert half of the layer on rows already grouped by expert:
 * for every expert e and every row p in [offsets[e], offsets[e+1]),
 *   y[p] = s1 * (ain . Wd[e]^T) + d_bias[e],  ain = the gated activation of
 *   g = s0 * (xin . Wgu[e]^T) + gu_bias[e]  (bf16 or A-FP8 activations as in
 *   moe_mxfp4_forward; act_scale a HOST pointer to {s0, s1} or NULL),
 * fp32 (P, H). "quantization_mxfp4", As GPT-OSS's native format (per-expert gate_up /
 * SwiGLU / down). For a partition of the experts over several ranks (expert parallelism):
 * a rank runs its own experts on the rows the other ranks sent it. x_rows: device bf16
 * (P, H); offsets: device int32 (E + 1), nondecreasing, offsets[E] = P; weights and
 * biases of the E experts as in moe_mxfp4_forward. Runs the tcgen05 grouped GEMMs: H and
 * I multiples of 64 in [128, 4608], blocks 32-byte aligned (MXMOE_EUNSUPPORTED
 * otherwise). Errors as moe_mxfp4_forward. Uses the library workspace. */
int moe_mxfp4_experts(const uint16_t* x_rows, const int32_t* offsets, int E, int P, int H, int I,
                      const uint8_t* gu_blocks, const uint8_t* gu_scales, const float* gu_bias,
                      const uint8_t* d_blocks, const uint8_t* d_scales, const float* d_bias,
                      const float* act_scale, float* y, void* stream);

/* moe_combine -- the weighted combine of the layer: out[t] = bf16( sum over the token's k
 * slots, in ascending expert id, of topk_w[t, j] * y[inv[t*k + j]] ), fp32 with one
 * rounding per multiply and add ("quantization_mxfp4", As GPT-OSS's native format: expert
 * outputs summed with their router gates). y: device fp32 (rows, H); topk_idx / topk_w:
 * device (T, k); inv: device int32 (T*k), the row of y that holds pair (t, j); out:
 * device bf16 (T, H). H % 8 == 0 (MXMOE_EALIGN), 1 <= k <= 8. */
int moe_combine(const float* y, const int32_t* topk_idx, const float* topk_w, const int32_t* inv,
                int T, int H, int k, uint16_t* out, void* stream);

/* moe_mxfp4_calibrate -- static per-tensor FP8 scales from a calibration batch with a
 * min-max observer ("gpt-oss-120b-mxfp4-fp8attn-v2", Quantization Recipe):
 * act_scale_out[0] = amax|x| / 448; act_scale_out[1] = amax over the routed
 * (token, expert) pairs of the bf16-path gated activation a (fp32, before rounding) / 448.
 * Same arguments as moe_mxfp4_forward without act_scale/out; act_scale_out: device fp32 (2). */
int moe_mxfp4_calibrate(const uint16_t* x, const uint16_t* router_w, const uint16_t* router_b,
                        const uint8_t* gu_blocks, const uint8_t* gu_scales, const float* gu_bias,
                        const uint8_t* d_blocks, const uint8_t* d_scales, const float* d_bias,
                        int E, int k, int T, int H, int I, float* act_scale_out, void* stream);

/* mxmoe_check -- synchronize `stream`, then read and clear the device error word.
 * Returns MXMOE_OK, MXMOE_EDEVICE (bad data seen by a kernel), MXMOE_ETIMEOUT (a bounded
 * device wait gave up) or MXMOE_ECUDA (the stream reported an error). */
int mxmoe_check(void* stream);

/* mxmoe_last_error -- message for the last failing call on this host thread ("" if none).
 * The string stays valid until the next library call on the same thread. */
const char* mxmoe_last_error(void);

/* mxmoe_last_launch_count -- number of kernels the last successful moe_mxfp4_forward,
 * mxfp4_quantize or mxfp4_dequantize on this host thread launched (a codec call launches
 * one kernel, none when it fails or has no work). */
int mxmoe_last_launch_count(void);

/* mxmoe_profile_enable -- on != 0: from now on every moe_mxfp4_forward on this host
 * thread records a CUDA event on its stream before its first kernel and after each stage
 * (router, topk, permute, act_quant, gate_up, down, combine, ...); on == 0 stops. Either
 * call discards marks not yet read. Timing only: the results are unchanged. Inside a
 * stream capture the records become event nodes of the graph, so a read after a replay
 * reports that replay. Returns MXMOE_OK. */
int mxmoe_profile_enable(int on);

/* mxmoe_profile_read -- wait for the recorded events and report, per stage name, the
 * summed GPU time in milliseconds and the number of calls since profiling was enabled or
 * last read (then forget them). names: max_entries slots of 32 chars (NUL-terminated);
 * total_ms, calls: max_entries entries. Returns the number of distinct stages (which may
 * exceed max_entries; only the first max_entries are written) or a negative error code. */
int mxmoe_profile_read(char* names, float* total_ms, int* calls, int max_entries);

/* mxmoe_release -- free the workspace of the current device (synchronizes the device).
 * Returns MXMOE_OK or MXMOE_ECUDA. */
int mxmoe_release(void);

/* mxmoe_tc_rate_probe -- measure the tensor pipe's rate for the block-scaled MMA the
 * prefill GEMMs issue (tcgen05.mma kind::mxf8f6f4, E4M3 A with M = 128 against E2M1 B with
 * N = n, K = 32, e8m0 block scales). The pages have no counterpart: the W-MXFP4 / A-FP8
 * GEMMs are judged against the FP8 tensor peak ("amd/gpt-oss-20b-MoE-Quant-W-MXFP4-A-FP8-
 * KV-FP8", Quantization schemes), and this call measures that peak for this instruction.
 * Launches `ctas` CTAs (one per SM for ctas <= the SM count) on `stream`; in each, one
 * thread issues `iters` x 4 MMAs back to back from operands resident in shared memory
 * (with_scale_copy != 0: one tcgen05.cp.128x256b of B scales before every 4, as the
 * prefill GEMM's per-stage scale copy). random_operands: 1 fills the operands with
 * pseudo-random bytes (E4M3 without NaN encodings against E2M1 containers, unit scales),
 * the rate on data like a GEMM's; 0 with zeros, which draw less power and run faster
 * under the power cap. The caller times the launch (CUDA events on `stream`). flops
 * (host, nullable) receives the FLOPs the launch performs, 2 * 128 * n * 32 * 4 * iters
 * * ctas. n: multiple of 16 in [16, 256]; random_operands 0 or 1; iters in [1, 1000000];
 * ctas in [1, 4096]. Returns MXMOE_OK, MXMOE_EINVAL or MXMOE_ECUDA; a bounded wait that
 * expires sets MXMOE_ETIMEOUT for mxmoe_check. */
int mxmoe_tc_rate_probe(int n, int with_scale_copy, int random_operands, int iters, int ctas, double* flops,
                        void* stream);

/* mxmoe_selftest_wait_timeout -- exercise the failure path of the library's bounded
 * device waits. The pages have no counterpart: every mbarrier wait in the tensor-core
 * kernels gives up after about a second (about 2e9 SM cycles), sets MXMOE_ETIMEOUT in the
 * device error word and lets its kernel return instead of hanging. This call launches
 * one CTA on `stream` whose thread waits, through that same bounded wait, on an mbarrier
 * that nothing completes; the wait expires and the next mxmoe_check on the stream
 * returns MXMOE_ETIMEOUT. Nothing faults or traps and the context stays usable.
 * Returns MXMOE_OK (launched) or MXMOE_ECUDA. */
int mxmoe_selftest_wait_timeout(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MXFP4_MOE_H */
