// C ABI of libmxfp4moe: argument checks, the per-device workspace, and the launch
// sequence of the MoE expert layer. Every step of the computation runs in the library's
// own kernels; this file only validates, sizes buffers and launches.
#include <mutex>
#include <string>
#include <vector>
#include <cstdio>
#include <cstdarg>
#include <cstring>
#include <cstdlib>

#include "common.cuh"
#include "launchers.h"

namespace {

thread_local std::string t_last_error;
thread_local int t_last_launches = 0;

// ------------------------------------------------------- optional stage timing -----
// When enabled, run_layer() records a CUDA event on the caller's stream before the first
// launch and after every stage, so a benchmark can time each kernel inside its own timed
// region without a profiler. Events come from a per-thread pool reused after each read.
struct StageMark {
  const char* name;
  cudaEvent_t start, stop;
};
thread_local bool t_profile = false;
thread_local std::vector<cudaEvent_t> t_event_pool;
thread_local size_t t_event_next = 0;
thread_local std::vector<StageMark> t_marks;

cudaEvent_t next_event() {
  if (t_event_next == t_event_pool.size()) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    t_event_pool.push_back(e);
  }
  return t_event_pool[t_event_next++];
}

struct StageTimer {
  cudaStream_t st;
  cudaEvent_t last = nullptr;
  unsigned flags = cudaEventRecordDefault;
  // Inside a stream capture the records are made with cudaEventRecordExternal so that they
  // become event nodes of the graph (timed at every replay); outside, plain records.
  explicit StageTimer(cudaStream_t s) : st(s) {
    if (!t_profile) return;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
      flags = cudaEventRecordExternal;
    if ((last = next_event())) cudaEventRecordWithFlags(last, st, flags);
  }
  void mark(const char* name) {
    if (!t_profile || !last) return;
    cudaEvent_t e = next_event();
    if (!e) return;
    cudaEventRecordWithFlags(e, st, flags);
    t_marks.push_back({name, last, e});
    last = e;
  }
};

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(MXMOE_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr size_t kTicketBytes = 4096;       // 1024 row groups of 16 rows: H <= 16384
constexpr int kFoldCombineMaxT = 64;        // fold the combine into the down kernel up to here
constexpr int kRouteTicket = 1023;          // ticket slot of the fused routing kernel
constexpr int kRouteTokTickets = 959;       // its per-token counters: slots 959 .. 1022 (T <= 64)

// ------------------------------------------------------------------ workspace ------
struct Workspace {
  char* base = nullptr;
  size_t cap = 0;
  int* err = nullptr;  // device error word
  int sms = 0;
  int smem_K = 0;      // largest K the expert kernels were configured for
  bool tc_ready = false;  // tcgen05 GEMM shared-memory limit raised
  bool dtc_ready = false; // tensor-core decode kernels' shared-memory limit raised
  bool dl_ready = false;  // one-launch decode layer's shared-memory limit raised
  bool tcb_ready = false; // two-part (bf16 activation) tcgen05 GEMM's shared-memory limit raised
  size_t tickets_zeroed = 0;  // bytes at the start of the workspace known to be zero
};

// Batches above the tensor-core decode path's size (T > kDecodeMaxT) run on the tcgen05
// grouped GEMMs whenever the shapes allow: FP8 activations directly, bf16 activations as
// two e4m3 parts. The register-dequant kernels (mma.sync) remain for calibration and for
// shapes neither tensor-core path takes.
constexpr int kTcMaxNb = 144;   // K <= 4608: the range the tcgen05 GEMM is tested on

constexpr int kMaxDevices = 64;
std::mutex g_mu;
Workspace g_ws[kMaxDevices];

int current_device_ws(Workspace** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(MXMOE_EUNSUPPORTED, "device %d beyond %d", dev, kMaxDevices);
  std::lock_guard<std::mutex> lk(g_mu);
  Workspace& w = g_ws[dev];
  if (w.err == nullptr) {
    if ((e = cudaMalloc(&w.err, 256)) != cudaSuccess) return fail(MXMOE_ENOMEM, "error word: %s", cudaGetErrorString(e));
    if ((e = cudaMemset(w.err, 0, 256)) != cudaSuccess) return cuda_fail(e, "cudaMemset");
    if ((e = cudaDeviceGetAttribute(&w.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute");
  }
  *out = &w;
  return MXMOE_OK;
}

int ensure_capacity(Workspace* w, size_t bytes) {
  if (bytes <= w->cap) return MXMOE_OK;
  std::lock_guard<std::mutex> lk(g_mu);
  if (bytes <= w->cap) return MXMOE_OK;
  cudaError_t e;
  if (w->base) {
    if ((e = cudaDeviceSynchronize()) != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
    cudaFree(w->base);
    w->base = nullptr;
    w->cap = 0;
  }
  size_t want = bytes + bytes / 8 + (1u << 20);
  if ((e = cudaMalloc(&w->base, want)) != cudaSuccess) {
    cudaGetLastError();
    return fail(MXMOE_ENOMEM, "workspace of %zu bytes: %s", want, cudaGetErrorString(e));
  }
  // the first kTicketBytes hold the down kernel's per-row-group tickets, which must read
  // zero at the start of every call (each call leaves them at zero)
  if ((e = cudaMemset(w->base, 0, kTicketBytes)) != cudaSuccess) return cuda_fail(e, "cudaMemset");
  w->tickets_zeroed = kTicketBytes;
  w->cap = want;
  return MXMOE_OK;
}

// Bump layout over the workspace; every slice is 256-byte aligned. The first slice of
// every layout is the ticket array (kTicketBytes, see ensure_capacity).
struct Carve {
  size_t off = 0;
  template <class T>
  size_t take(int64_t count) {
    size_t o = off;
    off += (static_cast<size_t>(count) * sizeof(T) + 255) & ~static_cast<size_t>(255);
    return o;
  }
};

struct LayerBuffers {
  unsigned* tickets;
  float* logits;
  float* logits_rest;
  int32_t* topk_idx;
  float* topk_w;
  int32_t* counts;
  int32_t* offsets;
  int32_t* active;
  int32_t* n_active;
  int32_t* perm_token;
  int32_t* perm_slot;
  int32_t* inv;
  uint16_t* xq;        // fp8 path: bf16 values of e4m3(x / s0), (T, H)
  uint16_t* act_mid;   // (P, I) bf16 bits of the down-projection input
  float* y;            // (P, H) fp32 expert outputs
  unsigned* amax;      // 2 x fp32 bits (calibration)
  uint8_t* a1;         // tcgen05 path: gate_up input rows grouped by expert, (P, H); two-part
                       // path: their e4m3 parts, (2, P, H)
  uint8_t* a2;         // tcgen05 path: down input rows, (P, I); two-part path: (2, P, I)
  uint8_t* sa1;        // two-part path: the parts' e8m0 scales, (2, P, H/32)
  uint8_t* sa2;        // (2, P, I/32)
  uint8_t* xs;         // tensor-core decode: gate_up B rows (P*4, H/2) packed e2m1 parts
  uint8_t* sfb;        // their scale records
  uint8_t* xs_mid;     // down B rows (P*4, I/2)
  uint8_t* sfb_mid;
  unsigned* dtickets;  // tensor-core decode: split-K and combine tickets (zero between calls)
  size_t tickets_end;  // bytes from the workspace start that hold tickets
  float* part;         // tensor-core decode: split-K partial accumulators
  // one-launch decode layer (T <= kDecodeLayerMaxT)
  unsigned* dl_counters;   // zero between calls
  uint8_t* dl_xs;
  uint8_t* dl_sfx;
  uint8_t* dl_xs_mid;
  uint8_t* dl_sf_mid;
  float* dl_part;
  float* dl_dpart;
};

// n_rest: the tensor-core router's extra K-range partials of the logits (T x E each)
size_t layout(int T, int E, int k, int H, int I, bool fp8, bool tc, bool tcb, bool dtc, bool dlay, int sms,
              int n_rest, LayerBuffers* b, char* base) {
  const int64_t P = static_cast<int64_t>(T) * k;
  const mxmoe::DecodeLayerSizes dls = dlay ? mxmoe::decode_layer_sizes(T, H, I, sms) : mxmoe::DecodeLayerSizes{};
  Carve c;
  size_t o_tickets = c.take<uint8_t>(kTicketBytes);
  size_t o_dtick = c.take<unsigned>(dtc ? static_cast<int64_t>(mxmoe::decode_tc_ticket_count(H, I)) : 0);
  size_t o_dlc = c.take<unsigned>(static_cast<int64_t>(dls.counters));
  const size_t tickets_end = c.off;
  size_t o_logits = c.take<float>(static_cast<int64_t>(T) * E);
  size_t o_lrest = c.take<float>(static_cast<int64_t>(n_rest) * T * E);
  size_t o_idx = c.take<int32_t>(P), o_w = c.take<float>(P);
  size_t o_counts = c.take<int32_t>(static_cast<int64_t>(mxmoe::permute_chunks(P)) * E);
  size_t o_off = c.take<int32_t>(E + 1), o_act = c.take<int32_t>(E), o_nact = c.take<int32_t>(1);
  size_t o_pt = c.take<int32_t>(P), o_ps = c.take<int32_t>(P), o_inv = c.take<int32_t>(P);
  size_t o_xq = c.take<uint16_t>(fp8 ? static_cast<int64_t>(T) * H : 0);
  size_t o_mid = c.take<uint16_t>(tc ? 0 : P * I);
  size_t o_y = c.take<float>(P * H);
  size_t o_amax = c.take<unsigned>(2);
  size_t o_a1 = c.take<uint8_t>(tc ? P * H : tcb ? 2 * P * H : 0);
  size_t o_a2 = c.take<uint8_t>(tc ? P * I : tcb ? 2 * P * I : 0);
  size_t o_sa1 = c.take<uint8_t>(tcb ? 2 * P * (H / 32) : 0);
  size_t o_sa2 = c.take<uint8_t>(tcb ? 2 * P * (I / 32) : 0);
  size_t o_xs = c.take<uint8_t>(dtc ? static_cast<int64_t>(mxmoe::decode_tc_xs_bytes(P, H)) : 0);
  size_t o_sfb = c.take<uint8_t>(dtc ? static_cast<int64_t>(mxmoe::decode_tc_sfb_bytes(E, H, T)) : 0);
  size_t o_xsm = c.take<uint8_t>(dtc ? static_cast<int64_t>(mxmoe::decode_tc_xs_bytes(P, I)) : 0);
  size_t o_sfbm = c.take<uint8_t>(dtc ? static_cast<int64_t>(mxmoe::decode_tc_sfb_bytes(E, I, T)) : 0);
  size_t o_part = c.take<uint8_t>(dtc ? static_cast<int64_t>(mxmoe::decode_tc_part_bytes(P, H, I)) : 0);
  size_t o_dlxs = c.take<uint8_t>(static_cast<int64_t>(dls.xs));
  size_t o_dlsfx = c.take<uint8_t>(static_cast<int64_t>(dls.sfx));
  size_t o_dlmid = c.take<uint8_t>(static_cast<int64_t>(dls.xs_mid));
  size_t o_dlsfm = c.take<uint8_t>(static_cast<int64_t>(dls.sf_mid));
  size_t o_dlp = c.take<uint8_t>(static_cast<int64_t>(dls.part));
  size_t o_dldp = c.take<uint8_t>(static_cast<int64_t>(dls.dpart));
  if (b) {
    b->dl_counters = reinterpret_cast<unsigned*>(base + o_dlc);
    b->dl_xs = reinterpret_cast<uint8_t*>(base + o_dlxs);
    b->dl_sfx = reinterpret_cast<uint8_t*>(base + o_dlsfx);
    b->dl_xs_mid = reinterpret_cast<uint8_t*>(base + o_dlmid);
    b->dl_sf_mid = reinterpret_cast<uint8_t*>(base + o_dlsfm);
    b->dl_part = reinterpret_cast<float*>(base + o_dlp);
    b->dl_dpart = reinterpret_cast<float*>(base + o_dldp);
    b->dtickets = reinterpret_cast<unsigned*>(base + o_dtick);
    b->tickets_end = tickets_end;
    b->part = reinterpret_cast<float*>(base + o_part);
    b->tickets = reinterpret_cast<unsigned*>(base + o_tickets);
    b->logits = reinterpret_cast<float*>(base + o_logits);
    b->logits_rest = n_rest > 0 ? reinterpret_cast<float*>(base + o_lrest) : nullptr;
    b->topk_idx = reinterpret_cast<int32_t*>(base + o_idx);
    b->topk_w = reinterpret_cast<float*>(base + o_w);
    b->counts = reinterpret_cast<int32_t*>(base + o_counts);
    b->offsets = reinterpret_cast<int32_t*>(base + o_off);
    b->active = reinterpret_cast<int32_t*>(base + o_act);
    b->n_active = reinterpret_cast<int32_t*>(base + o_nact);
    b->perm_token = reinterpret_cast<int32_t*>(base + o_pt);
    b->perm_slot = reinterpret_cast<int32_t*>(base + o_ps);
    b->inv = reinterpret_cast<int32_t*>(base + o_inv);
    b->xq = reinterpret_cast<uint16_t*>(base + o_xq);
    b->act_mid = reinterpret_cast<uint16_t*>(base + o_mid);
    b->y = reinterpret_cast<float*>(base + o_y);
    b->amax = reinterpret_cast<unsigned*>(base + o_amax);
    b->a1 = reinterpret_cast<uint8_t*>(base + o_a1);
    b->a2 = reinterpret_cast<uint8_t*>(base + o_a2);
    b->sa1 = reinterpret_cast<uint8_t*>(base + o_sa1);
    b->sa2 = reinterpret_cast<uint8_t*>(base + o_sa2);
    b->xs = reinterpret_cast<uint8_t*>(base + o_xs);
    b->sfb = reinterpret_cast<uint8_t*>(base + o_sfb);
    b->xs_mid = reinterpret_cast<uint8_t*>(base + o_xsm);
    b->sfb_mid = reinterpret_cast<uint8_t*>(base + o_sfbm);
  }
  return c.off;
}

int check_routing_args(int T, int E, int k) {
  if (T < 0) return fail(MXMOE_EINVAL, "T = %d is negative", T);
  if (T >= (1 << 24)) return fail(MXMOE_EUNSUPPORTED, "T = %d exceeds 2^24 - 1", T);
  if (E < 1) return fail(MXMOE_EINVAL, "E = %d must be >= 1", E);
  if (E > 256) return fail(MXMOE_EUNSUPPORTED, "E = %d exceeds 256", E);
  if (k < 1 || k > 8) return fail(MXMOE_EUNSUPPORTED, "k = %d outside [1, 8]", k);
  if (k > E) return fail(MXMOE_EUNSUPPORTED, "k = %d exceeds E = %d", k, E);
  return MXMOE_OK;
}

struct LayerArgs {
  const uint16_t* x;
  const uint16_t* router_w;
  const uint16_t* router_b;
  const uint8_t* gu_blocks;
  const uint8_t* gu_scales;
  const float* gu_bias;
  const uint8_t* d_blocks;
  const uint8_t* d_scales;
  const float* d_bias;
  int E, k, T, H, I;
};

int check_layer_args(const LayerArgs& a) {
  if (int rc = check_routing_args(a.T, a.E, a.k)) return rc;
  if (a.H <= 0 || a.I <= 0) return fail(MXMOE_EINVAL, "H = %d and I = %d must be positive", a.H, a.I);
  if (a.H % 32 || a.I % 32)
    return fail(MXMOE_EALIGN, "H = %d and I = %d must be multiples of 32 (MXFP4 block size)", a.H, a.I);
  const void* ptrs[] = {a.x, a.router_w, a.gu_blocks, a.gu_scales, a.gu_bias,
                        a.d_blocks, a.d_scales, a.d_bias};
  const char* names[] = {"x", "router_w", "gu_blocks", "gu_scales", "gu_bias",
                         "d_blocks", "d_scales", "d_bias"};
  for (int i = 0; i < 8; ++i) {
    if (!ptrs[i]) return fail(MXMOE_EINVAL, "%s is NULL", names[i]);
    if (!aligned16(ptrs[i])) return fail(MXMOE_EINVAL, "%s is not 16-byte aligned", names[i]);
  }
  if (a.router_b && !aligned16(a.router_b)) return fail(MXMOE_EINVAL, "router_b is not 16-byte aligned");
  return MXMOE_OK;
}

// Runs the layer up to the stage that `calib` needs. Returns a status code.
int run_layer(const LayerArgs& a, const float* act_scale, uint16_t* out, float* calib_out,
              cudaStream_t st) {
  using namespace mxmoe;
  Workspace* ws = nullptr;
  if (int rc = current_device_ws(&ws)) return rc;
  const bool fp8 = act_scale != nullptr;
  const int64_t P = static_cast<int64_t>(a.T) * a.k;
  const bool large = a.T > kDecodeMaxT;
  const bool tc = fp8 && !calib_out && large && std::max(a.H, a.I) / 32 <= kTcMaxNb &&
                  tc_gemm_supported(a.H, a.I, a.gu_blocks, a.d_blocks, a.gu_scales, a.d_scales);
  // bf16 activations with many routed pairs: the same GEMMs with each activation as two
  // e4m3 parts (exact for the activations' significant bits)
  const bool tcb = !fp8 && !calib_out && large && std::max(a.H, a.I) / 32 <= kTcMaxNb &&
                   tc_gemm_supported(a.H, a.I, a.gu_blocks, a.d_blocks, a.gu_scales, a.d_scales);
  // a handful of tokens: the whole layer in one launch
  const bool dlay = !tc && !tcb && !calib_out && a.T <= kDecodeLayerMaxT &&
                    decode_layer_supported(a.H, a.I, a.T, a.E, a.k, ws->sms, a.gu_blocks, a.d_blocks, a.gu_scales,
                                           a.d_scales);
  const bool dtc = !tc && !tcb && !dlay && !calib_out &&
                   decode_tc_supported(a.H, a.I, a.T, a.gu_blocks, a.d_blocks, a.gu_scales, a.d_scales);
  // routing: one fused launch for small batches; else the router GEMM (on the tensor cores
  // when the shapes allow, split over K ranges) and a top-k kernel that adds the ranges
  const bool small = !dlay && route_small_supported(a.T, a.E, a.k);
  const int ksplit = !small && router_tc_supported(a.T, a.H, a.E, a.x, a.router_w, nullptr)
                         ? router_tc_ksplit(a.T, a.H, ws->sms)
                         : 0;
  const int n_rest = ksplit > 1 ? ksplit - 1 : 0;
  const size_t need = layout(a.T, a.E, a.k, a.H, a.I, fp8, tc, tcb, dtc, dlay, ws->sms, n_rest, nullptr, nullptr);
  if (int rc = ensure_capacity(ws, need)) return rc;
  if (std::max(a.H, a.I) > ws->smem_K) {
    cudaError_t e = expert_mma_set_smem_limits(std::max(a.H, a.I));
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    ws->smem_K = std::max(a.H, a.I);
  }
  if (tc && !ws->tc_ready) {
    cudaError_t e = tc_gemm_prepare(256);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute (tcgen05 GEMM)");
    ws->tc_ready = true;
  }
  if (tcb && !ws->tcb_ready) {
    cudaError_t e = tc_parts_gemm_prepare(256);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute (two-part tcgen05 GEMM)");
    ws->tcb_ready = true;
  }
  if (dlay && !ws->dl_ready) {
    cudaError_t e = decode_layer_prepare();
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute (decode layer)");
    ws->dl_ready = true;
  }
  if (dtc && !ws->dtc_ready) {
    cudaError_t e = decode_tc_prepare();
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute (tensor-core decode)");
    ws->dtc_ready = true;
  }
  LayerBuffers b;
  layout(a.T, a.E, a.k, a.H, a.I, fp8, tc, tcb, dtc, dlay, ws->sms, n_rest, &b, ws->base);
  // The decode paths' tickets follow the fixed ticket block, where other layouts keep
  // ordinary buffers: they are known to be zero only after a decode-path call, which
  // leaves them at zero. Clear them when that is not known.
  const bool counted = dtc || dlay;
  if (counted && b.tickets_end > ws->tickets_zeroed) {
    cudaError_t e = cudaMemsetAsync(ws->base, 0, b.tickets_end, st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync (tickets)");
  }
  ws->tickets_zeroed = counted ? b.tickets_end : kTicketBytes;
  int launches = 0;
  cudaError_t e;
  const float s0 = fp8 ? act_scale[0] : 1.0f, s1 = fp8 ? act_scale[1] : 1.0f;

  StageTimer tm(st);
  if (dlay) {
    DecodeLayerArgs d{};
    d.x = a.x; d.router_w = a.router_w; d.router_b = a.router_b;
    d.gu_blocks = a.gu_blocks; d.gu_scales = a.gu_scales; d.gu_bias = a.gu_bias;
    d.d_blocks = a.d_blocks; d.d_scales = a.d_scales; d.d_bias = a.d_bias;
    d.E = a.E; d.H = a.H; d.I = a.I; d.T = a.T; d.k = a.k;
    d.fp8 = fp8; d.s0 = s0; d.s1 = s1;
    d.sms = ws->sms;
    d.logits = b.logits;
    d.xs = b.dl_xs; d.sfx = b.dl_sfx; d.xs_mid = b.dl_xs_mid; d.sf_mid = b.dl_sf_mid;
    d.part = b.dl_part; d.dpart = b.dl_dpart; d.counters = b.dl_counters;
    d.topk_idx = b.topk_idx; d.topk_w = b.topk_w;
    d.out = out;
    d.err = ws->err;
    if ((e = launch_decode_layer(d, st))) return cuda_fail(e, "decode layer");
    ++launches;
    tm.mark("layer");
    t_last_launches = launches;
    return MXMOE_OK;
  }
  if (small) {
    // small batch: router, top-k and permutation in one CTA, one launch
    if ((e = launch_route_small(a.x, a.router_w, a.router_b, a.T, a.H, a.E, a.k, b.logits,
                                b.tickets + kRouteTicket, b.tickets + kRouteTokTickets, b.topk_idx, b.topk_w,
                                b.offsets, b.perm_token, b.perm_slot, b.inv, b.active, b.n_active, ws->err, st)))
      return cuda_fail(e, "route");
    ++launches;
    tm.mark("route");
  } else {
    if (ksplit > 0) {
      if ((e = launch_router_tc(a.x, a.router_w, a.router_b, a.T, a.H, a.E, ksplit, b.logits, b.logits_rest, ws->err,
                                st)))
        return cuda_fail(e, "router");
    } else if ((e = launch_router(a.x, a.router_w, a.router_b, a.T, a.H, a.E, b.logits, st))) {
      return cuda_fail(e, "router");
    }
    ++launches;
    tm.mark("router");
    if ((e = launch_topk(b.logits, b.logits_rest, n_rest, a.T, a.E, a.k, b.topk_idx, b.topk_w, st)))
      return cuda_fail(e, "topk");
    ++launches;
    tm.mark("topk");
    if ((e = launch_permute(b.topk_idx, a.T, a.E, a.k, b.counts, b.offsets, b.perm_token, b.perm_slot,
                            b.inv, b.active, b.n_active, ws->err, st, &launches)))
      return cuda_fail(e, "permute");
    tm.mark("permute");
  }
  if (tc) {
    // the A-FP8 cast and the scatter into expert-grouped rows: one pass over x, one cast per token
    if ((e = launch_quant_scatter_fp8(a.x, b.topk_idx, b.inv, a.T, a.k, a.E, P, a.H, s0, b.a1, st, ws->sms)))
      return cuda_fail(e, "fp8 activation cast + scatter");
    ++launches;
    tm.mark("act_quant+scatter");
    if ((e = launch_tc_gemm(true, b.a1, P, a.H, a.gu_blocks, a.gu_scales, a.gu_bias, a.E, a.I, b.offsets, s0, s1,
                            b.a2, nullptr, ws->err, ws->sms, st)))
      return cuda_fail(e, "gate_up (tcgen05)");
    ++launches;
    tm.mark("gate_up");
    if ((e = launch_tc_gemm(false, b.a2, P, a.I, a.d_blocks, a.d_scales, a.d_bias, a.E, a.H, b.offsets, s1, 0.0f,
                            nullptr, b.y, ws->err, ws->sms, st)))
      return cuda_fail(e, "down (tcgen05)");
    ++launches;
    tm.mark("down");
    if ((e = launch_combine(b.y, b.topk_idx, b.topk_w, b.inv, a.T, a.H, a.k, out, st, ws->sms)))
      return cuda_fail(e, "combine");
    ++launches;
    tm.mark("combine");
    t_last_launches = launches;
    return MXMOE_OK;
  }
  if (tcb) {
    // bf16 activations as two e4m3 parts per value (block scales as the MMA's A scales)
    if ((e = launch_split_parts(a.x, b.perm_token, a.T, P, a.H, b.a1, b.sa1, ws->sms, st)))
      return cuda_fail(e, "activation split");
    ++launches;
    tm.mark("act_split");
    if ((e = launch_tc_parts_gemm(true, b.a1, b.sa1, P, a.H, a.gu_blocks, a.gu_scales, a.gu_bias, a.E, a.I,
                                  b.offsets, b.act_mid, nullptr, ws->err, ws->sms, st)))
      return cuda_fail(e, "gate_up (tcgen05, two parts)");
    ++launches;
    tm.mark("gate_up");
    if ((e = launch_split_parts(b.act_mid, nullptr, a.T, P, a.I, b.a2, b.sa2, ws->sms, st)))
      return cuda_fail(e, "intermediate split");
    ++launches;
    tm.mark("mid_split");
    if ((e = launch_tc_parts_gemm(false, b.a2, b.sa2, P, a.I, a.d_blocks, a.d_scales, a.d_bias, a.E, a.H,
                                  b.offsets, nullptr, b.y, ws->err, ws->sms, st)))
      return cuda_fail(e, "down (tcgen05, two parts)");
    ++launches;
    tm.mark("down");
    if ((e = launch_combine(b.y, b.topk_idx, b.topk_w, b.inv, a.T, a.H, a.k, out, st, ws->sms)))
      return cuda_fail(e, "combine");
    ++launches;
    tm.mark("combine");
    t_last_launches = launches;
    return MXMOE_OK;
  }
  if (dtc) {
    // small batch on the tensor cores: tokens as MX-FP8 parts, weights as the A operand
    if ((e = launch_split_tokens(fp8, a.x, b.topk_idx, b.inv, b.offsets, a.T, a.E, a.H, a.k, s0, b.xs, b.sfb, st)))
      return cuda_fail(e, "split");
    ++launches;
    tm.mark("act_split");
    DecodeGemmArgs d{};
    d.gu_blocks = a.gu_blocks; d.gu_scales = a.gu_scales; d.gu_bias = a.gu_bias;
    d.d_blocks = a.d_blocks; d.d_scales = a.d_scales; d.d_bias = a.d_bias;
    d.E = a.E; d.H = a.H; d.I = a.I; d.T = a.T; d.k = a.k; d.P = P;
    d.max_active = static_cast<int>(std::min<int64_t>(a.E, P));
    d.sms = ws->sms;
    d.offsets = b.offsets; d.active = b.active; d.n_active = b.n_active;
    d.xs = b.xs; d.sfb = b.sfb; d.xs_mid = b.xs_mid; d.sfb_mid = b.sfb_mid;
    d.s0 = s0; d.s1_quant = fp8 ? s1 : 0.0f; d.s1_in = s1;
    d.y = b.y;
    d.part = b.part;
    d.split_tickets_gu = b.dtickets;
    d.split_tickets_d = b.dtickets + decode_tc_tickets_d(a.I);
    d.err = ws->err;
    if ((e = launch_decode_gemm(true, d, st))) return cuda_fail(e, "gate_up (tensor-core decode)");
    ++launches;
    tm.mark("gate_up");
    if ((e = launch_decode_gemm(false, d, st))) return cuda_fail(e, "down (tensor-core decode)");
    ++launches;
    tm.mark("down");
    if ((e = launch_combine(b.y, b.topk_idx, b.topk_w, b.inv, a.T, a.H, a.k, out, st, ws->sms)))
      return cuda_fail(e, "combine");
    ++launches;
    tm.mark("combine");
    t_last_launches = launches;
    return MXMOE_OK;
  }
  const uint16_t* act_in = a.x;
  if (fp8) {
    if ((e = launch_fp8_quant_as_bf16(a.x, static_cast<int64_t>(a.T) * a.H, s0, b.xq, st, ws->sms)))
      return cuda_fail(e, "fp8 activation cast");
    ++launches;
    tm.mark("act_quant");
    act_in = b.xq;
  }
  const int max_active = static_cast<int>(std::min<int64_t>(a.E, P));
  if (calib_out) {
    if ((e = cudaMemsetAsync(b.amax, 0, 2 * sizeof(unsigned), st))) return cuda_fail(e, "memset");
    if ((e = launch_amax_bf16(a.x, static_cast<int64_t>(a.T) * a.H, b.amax, st, ws->sms))) return cuda_fail(e, "amax");
    ++launches;
  }
  if ((e = launch_expert_mma(a.gu_blocks, a.gu_scales, a.gu_bias, 2 * a.I, a.H, act_in,
                             b.perm_token, b.offsets, b.active, b.n_active, max_active, s0, 0, a.I,
                             fp8 ? s1 : 0.0f, b.act_mid, nullptr, calib_out ? b.amax + 1 : nullptr,
                             a.T, ws->err, nullptr, st)))
    return cuda_fail(e, "gate_up");
  ++launches;
  tm.mark("gate_up");
  if (calib_out) {
    if ((e = launch_finalize_scales(b.amax, calib_out, st))) return cuda_fail(e, "finalize");
    ++launches;
    t_last_launches = launches;
    return MXMOE_OK;
  }
  const bool fold = a.T <= kFoldCombineMaxT && a.H / 16 <= kRouteTokTickets;
  const CombineArgs cmb{out, b.topk_idx, b.topk_w, b.inv, b.tickets, a.T, a.k};
  if ((e = launch_expert_mma(a.d_blocks, a.d_scales, a.d_bias, a.H, a.I, b.act_mid, nullptr,
                             b.offsets, b.active, b.n_active, max_active, s1, 1, a.I, 0.0f, nullptr,
                             b.y, nullptr, a.T, ws->err, fold ? &cmb : nullptr, st)))
    return cuda_fail(e, "down");
  ++launches;
  tm.mark(fold ? "down+combine" : "down");
  if (!fold) {
    if ((e = launch_combine(b.y, b.topk_idx, b.topk_w, b.inv, a.T, a.H, a.k, out, st, ws->sms)))
      return cuda_fail(e, "combine");
    ++launches;
    tm.mark("combine");
  }
  t_last_launches = launches;
  return MXMOE_OK;
}

// The dense all-experts path: every token through all E experts (expert-major rows
// e * T + t), the gates zero off the top-k, the weighted sum over all experts in ascending
// order. The tcgen05 grouped GEMMs read the T activation rows once per expert (shared A
// rows) instead of a gathered copy per routed pair.
// Shapes the dense path takes: its expert kernels' (tcgen05 grouped GEMMs), with the
// expert-major intermediate indexable in 32 bits.
bool dense_kernels_take(const LayerArgs& a) {
  return std::max(a.H, a.I) / 32 <= kTcMaxNb &&
         mxmoe::tc_gemm_supported(a.H, a.I, a.gu_blocks, a.d_blocks, a.gu_scales, a.d_scales);
}
bool dense_fits(const LayerArgs& a) {
  const int64_t R = static_cast<int64_t>(a.E) * a.T;
  return R * std::max(a.H, a.I) < (int64_t{1} << 31) && R < (int64_t{1} << 24);
}

int run_layer_dense(const LayerArgs& a, const float* act_scale, uint16_t* out, cudaStream_t st) {
  using namespace mxmoe;
  Workspace* ws = nullptr;
  if (int rc = current_device_ws(&ws)) return rc;
  const bool fp8 = act_scale != nullptr;
  const int64_t T = a.T, E = a.E, H = a.H, I = a.I;
  const int64_t R = E * T;   // expert-major rows
  if (!dense_kernels_take(a))
    return fail(MXMOE_EUNSUPPORTED, "the dense path needs H and I multiples of 64 in [128, 4608] and 32-byte "
                                    "aligned blocks (got H = %d, I = %d)", a.H, a.I);
  if (!dense_fits(a))
    return fail(MXMOE_EUNSUPPORTED, "the dense path holds E*T*max(H, I) < 2^31 values (E = %d, T = %d)", a.E, a.T);
  const bool rtc = a.T > 32 && router_tc_supported(a.T, a.H, a.E, a.x, a.router_w, nullptr);
  const int ksplit = rtc ? router_tc_ksplit(a.T, a.H, ws->sms) : 0;
  const int n_rest = ksplit > 1 ? ksplit - 1 : 0;
  Carve c;
  c.take<uint8_t>(kTicketBytes);
  const size_t o_logits = c.take<float>(T * E), o_rest = c.take<float>(n_rest * T * E);
  const size_t o_idx = c.take<int32_t>(T * a.k), o_w = c.take<float>(T * a.k);
  const size_t o_g = c.take<float>(T * E), o_off = c.take<int32_t>(E + 1);
  const size_t o_a1 = c.take<uint8_t>(fp8 ? T * H : 2 * T * H);
  const size_t o_sa1 = c.take<uint8_t>(fp8 ? 0 : 2 * T * (H / 32));
  const size_t o_mid = c.take<uint16_t>(fp8 ? 0 : R * I);
  const size_t o_a2 = c.take<uint8_t>(fp8 ? R * I : 2 * R * I);
  const size_t o_sa2 = c.take<uint8_t>(fp8 ? 0 : 2 * R * (I / 32));
  const size_t o_y = c.take<float>(R * H);
  if (int rc = ensure_capacity(ws, c.off)) return rc;
  if (fp8 && !ws->tc_ready) {
    cudaError_t e = tc_gemm_prepare(256);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute (tcgen05 GEMM)");
    ws->tc_ready = true;
  }
  if (!fp8 && !ws->tcb_ready) {
    cudaError_t e = tc_parts_gemm_prepare(256);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute (two-part tcgen05 GEMM)");
    ws->tcb_ready = true;
  }
  ws->tickets_zeroed = kTicketBytes;
  char* base = ws->base;
  float* logits = reinterpret_cast<float*>(base + o_logits);
  float* rest = n_rest ? reinterpret_cast<float*>(base + o_rest) : nullptr;
  int32_t* idx = reinterpret_cast<int32_t*>(base + o_idx);
  float* w = reinterpret_cast<float*>(base + o_w);
  float* gates = reinterpret_cast<float*>(base + o_g);
  int32_t* offsets = reinterpret_cast<int32_t*>(base + o_off);
  uint8_t* a1 = reinterpret_cast<uint8_t*>(base + o_a1);
  uint8_t* sa1 = reinterpret_cast<uint8_t*>(base + o_sa1);
  uint16_t* mid = reinterpret_cast<uint16_t*>(base + o_mid);
  uint8_t* a2 = reinterpret_cast<uint8_t*>(base + o_a2);
  uint8_t* sa2 = reinterpret_cast<uint8_t*>(base + o_sa2);
  float* y = reinterpret_cast<float*>(base + o_y);
  const float s0 = fp8 ? act_scale[0] : 1.0f, s1 = fp8 ? act_scale[1] : 1.0f;
  int launches = 0;
  cudaError_t e;
  StageTimer tm(st);
  if ((e = rtc ? launch_router_tc(a.x, a.router_w, a.router_b, a.T, a.H, a.E, ksplit, logits, rest, ws->err, st)
               : launch_router(a.x, a.router_w, a.router_b, a.T, a.H, a.E, logits, st)))
    return cuda_fail(e, "router");
  ++launches;
  tm.mark("router");
  if ((e = launch_topk(logits, rest, n_rest, a.T, a.E, a.k, idx, w, st))) return cuda_fail(e, "topk");
  ++launches;
  tm.mark("topk");
  if ((e = launch_dense_setup(idx, w, a.T, a.E, a.k, gates, offsets, st, ws->sms))) return cuda_fail(e, "dense gates");
  ++launches;
  tm.mark("dense_gates");
  if (fp8) {
    if ((e = launch_fp8_quant(a.x, T * H, s0, a1, st, ws->sms))) return cuda_fail(e, "fp8 activation cast");
    ++launches;
    tm.mark("act_quant");
    if ((e = launch_tc_gemm(true, a1, T, a.H, a.gu_blocks, a.gu_scales, a.gu_bias, a.E, a.I, offsets, s0, s1, a2,
                            nullptr, ws->err, ws->sms, st, true)))
      return cuda_fail(e, "gate_up (tcgen05, dense)");
    ++launches;
    tm.mark("gate_up");
    if ((e = launch_tc_gemm(false, a2, R, a.I, a.d_blocks, a.d_scales, a.d_bias, a.E, a.H, offsets, s1, 0.0f,
                            nullptr, y, ws->err, ws->sms, st)))
      return cuda_fail(e, "down (tcgen05, dense)");
    ++launches;
    tm.mark("down");
  } else {
    if ((e = launch_split_parts(a.x, nullptr, a.T, T, a.H, a1, sa1, ws->sms, st)))
      return cuda_fail(e, "activation split");
    ++launches;
    tm.mark("act_split");
    if ((e = launch_tc_parts_gemm(true, a1, sa1, T, a.H, a.gu_blocks, a.gu_scales, a.gu_bias, a.E, a.I, offsets,
                                  mid, nullptr, ws->err, ws->sms, st, true)))
      return cuda_fail(e, "gate_up (tcgen05, two parts, dense)");
    ++launches;
    tm.mark("gate_up");
    if ((e = launch_split_parts(mid, nullptr, a.T, R, a.I, a2, sa2, ws->sms, st)))
      return cuda_fail(e, "intermediate split");
    ++launches;
    tm.mark("mid_split");
    if ((e = launch_tc_parts_gemm(false, a2, sa2, R, a.I, a.d_blocks, a.d_scales, a.d_bias, a.E, a.H, offsets,
                                  nullptr, y, ws->err, ws->sms, st)))
      return cuda_fail(e, "down (tcgen05, two parts, dense)");
    ++launches;
    tm.mark("down");
  }
  if ((e = launch_dense_combine(y, gates, a.T, a.H, a.E, out, st, ws->sms))) return cuda_fail(e, "dense combine");
  ++launches;
  tm.mark("combine");
  t_last_launches = launches;
  return MXMOE_OK;
}

}  // namespace

extern "C" {

int mxfp4_quantize(const float* w, int64_t rows, int64_t K, uint8_t* blocks, uint8_t* scales,
                   void* stream) {
  t_last_error.clear();
  t_last_launches = 0;
  if (rows < 0 || K < 0) return fail(MXMOE_EINVAL, "negative size rows=%lld K=%lld", (long long)rows, (long long)K);
  if (K % 32) return fail(MXMOE_EALIGN, "K = %lld is not a multiple of 32 (MXFP4 block size)", (long long)K);
  if (rows == 0 || K == 0) return MXMOE_OK;
  if (!w || !blocks || !scales) return fail(MXMOE_EINVAL, "null pointer");
  if (!aligned16(w) || !aligned16(blocks)) return fail(MXMOE_EINVAL, "w and blocks must be 16-byte aligned");
  Workspace* ws = nullptr;
  if (int rc = current_device_ws(&ws)) return rc;
  cudaError_t e = mxmoe::launch_quantize(w, rows, K, blocks, scales, static_cast<cudaStream_t>(stream), ws->sms);
  if (e) return cuda_fail(e, "quantize launch");
  t_last_launches = 1;
  return MXMOE_OK;
}

int mxfp4_dequantize(const uint8_t* blocks, const uint8_t* scales, int64_t rows, int64_t K,
                     void* out, int out_dtype, void* stream) {
  t_last_error.clear();
  t_last_launches = 0;
  if (rows < 0 || K < 0) return fail(MXMOE_EINVAL, "negative size rows=%lld K=%lld", (long long)rows, (long long)K);
  if (K % 32) return fail(MXMOE_EALIGN, "K = %lld is not a multiple of 32 (MXFP4 block size)", (long long)K);
  if (out_dtype != MXMOE_OUT_F32 && out_dtype != MXMOE_OUT_BF16)
    return fail(MXMOE_EUNSUPPORTED, "out_dtype %d is neither MXMOE_OUT_F32 nor MXMOE_OUT_BF16", out_dtype);
  if (rows == 0 || K == 0) return MXMOE_OK;
  if (!blocks || !scales || !out) return fail(MXMOE_EINVAL, "null pointer");
  if (!aligned16(blocks) || !aligned16(out)) return fail(MXMOE_EINVAL, "blocks and out must be 16-byte aligned");
  Workspace* ws = nullptr;
  if (int rc = current_device_ws(&ws)) return rc;
  cudaError_t e = mxmoe::launch_dequantize(blocks, scales, rows, K, out, out_dtype,
                                           static_cast<cudaStream_t>(stream), ws->sms);
  if (e) return cuda_fail(e, "dequantize launch");
  t_last_launches = 1;
  return MXMOE_OK;
}

int mxfp4_quantize_axis(const float* w, int64_t outer, int64_t K, int64_t inner, uint8_t* blocks, uint8_t* scales,
                        void* stream) {
  t_last_error.clear();
  t_last_launches = 0;
  if (outer < 0 || K < 0 || inner < 0)
    return fail(MXMOE_EINVAL, "negative size outer=%lld K=%lld inner=%lld", (long long)outer, (long long)K,
                (long long)inner);
  if (K % 32) return fail(MXMOE_EALIGN, "K = %lld is not a multiple of 32 (MXFP4 block size)", (long long)K);
  if (outer == 0 || K == 0 || inner == 0) return MXMOE_OK;
  if (!w || !blocks || !scales) return fail(MXMOE_EINVAL, "null pointer");
  if (!aligned16(w) || !aligned16(blocks)) return fail(MXMOE_EINVAL, "w and blocks must be 16-byte aligned");
  Workspace* ws = nullptr;
  if (int rc = current_device_ws(&ws)) return rc;
  cudaError_t e = mxmoe::launch_quantize_axis(w, outer, K, inner, blocks, scales, static_cast<cudaStream_t>(stream),
                                              ws->sms);
  if (e) return cuda_fail(e, "quantize launch");
  t_last_launches = 1;
  return MXMOE_OK;
}

int mxfp4_dequantize_axis(const uint8_t* blocks, const uint8_t* scales, int64_t outer, int64_t K, int64_t inner,
                          void* out, int out_dtype, void* stream) {
  t_last_error.clear();
  t_last_launches = 0;
  if (outer < 0 || K < 0 || inner < 0)
    return fail(MXMOE_EINVAL, "negative size outer=%lld K=%lld inner=%lld", (long long)outer, (long long)K,
                (long long)inner);
  if (K % 32) return fail(MXMOE_EALIGN, "K = %lld is not a multiple of 32 (MXFP4 block size)", (long long)K);
  if (out_dtype != MXMOE_OUT_F32 && out_dtype != MXMOE_OUT_BF16)
    return fail(MXMOE_EUNSUPPORTED, "out_dtype %d is neither MXMOE_OUT_F32 nor MXMOE_OUT_BF16", out_dtype);
  if (outer == 0 || K == 0 || inner == 0) return MXMOE_OK;
  if (!blocks || !scales || !out) return fail(MXMOE_EINVAL, "null pointer");
  if (!aligned16(blocks) || !aligned16(out)) return fail(MXMOE_EINVAL, "blocks and out must be 16-byte aligned");
  Workspace* ws = nullptr;
  if (int rc = current_device_ws(&ws)) return rc;
  cudaError_t e = mxmoe::launch_dequantize_axis(blocks, scales, outer, K, inner, out, out_dtype,
                                                static_cast<cudaStream_t>(stream), ws->sms);
  if (e) return cuda_fail(e, "dequantize launch");
  t_last_launches = 1;
  return MXMOE_OK;
}

int mxfp4_linear(const uint16_t* x, int T, int K, const uint8_t* blocks, const uint8_t* scales, int N,
                 const float* bias, const float* act_scale, uint16_t* out, void* stream) {
  using namespace mxmoe;
  t_last_error.clear();
  t_last_launches = 0;
  if (T < 0 || K <= 0 || N <= 0) return fail(MXMOE_EINVAL, "T = %d must be >= 0, K = %d and N = %d positive", T, K, N);
  if (K % 32) return fail(MXMOE_EALIGN, "K = %d is not a multiple of 32 (MXFP4 block size)", K);
  if (N % 16) return fail(MXMOE_EALIGN, "N = %d is not a multiple of 16", N);
  if (T >= (1 << 24)) return fail(MXMOE_EUNSUPPORTED, "T = %d exceeds 2^24 - 1", T);
  if (T == 0) return MXMOE_OK;
  if (!x || !blocks || !scales || !out) return fail(MXMOE_EINVAL, "null pointer");
  if (!aligned16(x) || !aligned16(blocks) || !aligned16(out) || (bias && !aligned16(bias)))
    return fail(MXMOE_EINVAL, "x, blocks, out and bias must be 16-byte aligned");
  if (act_scale && !(*act_scale > 0.0f)) return fail(MXMOE_EINVAL, "act_scale must be > 0");
  Workspace* ws = nullptr;
  if (int rc = current_device_ws(&ws)) return rc;
  const bool fp8 = act_scale != nullptr;
  const int64_t TK = static_cast<int64_t>(T) * K;
  // more than a decode batch on the tcgen05 grouped GEMM (one expert), else the
  // register-dequant kernel, which spreads the weight rows over every SM
  const bool tc = T > kDecodeMaxT && K / 32 <= kTcMaxNb && tc_gemm_supported(N, K, blocks, blocks, scales, scales);
  Carve c;
  c.take<uint8_t>(kTicketBytes);
  const size_t o_meta = c.take<int32_t>(8);
  const size_t o_zb = c.take<float>(bias ? 0 : N);
  const size_t o_a = c.take<uint8_t>(tc ? (fp8 ? TK : 2 * TK) : (fp8 ? 2 * TK : 0));
  const size_t o_sa = c.take<uint8_t>(tc && !fp8 ? 2 * (TK / 32) : 0);
  const size_t o_y = c.take<float>(static_cast<int64_t>(T) * N);
  if (int rc = ensure_capacity(ws, c.off)) return rc;
  ws->tickets_zeroed = kTicketBytes;
  if (tc && fp8 && !ws->tc_ready) {
    cudaError_t e = tc_gemm_prepare(256);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute (tcgen05 GEMM)");
    ws->tc_ready = true;
  }
  if (tc && !fp8 && !ws->tcb_ready) {
    cudaError_t e = tc_parts_gemm_prepare(256);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute (two-part tcgen05 GEMM)");
    ws->tcb_ready = true;
  }
  if (!tc && K > ws->smem_K) {
    cudaError_t e = expert_mma_set_smem_limits(K);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    ws->smem_K = K;
  }
  char* base = ws->base;
  int32_t* offsets = reinterpret_cast<int32_t*>(base + o_meta);
  int32_t* active = offsets + 2;
  int32_t* n_active = offsets + 3;
  float* zb = bias ? nullptr : reinterpret_cast<float*>(base + o_zb);
  const float* b = bias ? bias : zb;
  uint8_t* a = reinterpret_cast<uint8_t*>(base + o_a);
  uint8_t* sa = reinterpret_cast<uint8_t*>(base + o_sa);
  float* y = reinterpret_cast<float*>(base + o_y);
  const float s = fp8 ? *act_scale : 1.0f;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int launches = 0;
  cudaError_t e;
  if ((e = launch_linear_setup(T, N, offsets, active, n_active, zb, st, ws->sms))) return cuda_fail(e, "linear set-up");
  ++launches;
  if (tc && fp8) {
    if ((e = launch_fp8_quant(x, TK, s, a, st, ws->sms))) return cuda_fail(e, "fp8 activation cast");
    if ((e = launch_tc_gemm(false, a, T, K, blocks, scales, b, 1, N, offsets, s, 0.0f, nullptr, y, ws->err, ws->sms,
                            st)))
      return cuda_fail(e, "linear (tcgen05)");
    launches += 2;
  } else if (tc) {
    if ((e = launch_split_parts(x, nullptr, T, T, K, a, sa, ws->sms, st))) return cuda_fail(e, "activation split");
    if ((e = launch_tc_parts_gemm(false, a, sa, T, K, blocks, scales, b, 1, N, offsets, nullptr, y, ws->err, ws->sms,
                                  st)))
      return cuda_fail(e, "linear (tcgen05, two parts)");
    launches += 2;
  } else {
    const uint16_t* act = x;
    if (fp8) {
      if ((e = launch_fp8_quant_as_bf16(x, TK, s, reinterpret_cast<uint16_t*>(a), st, ws->sms)))
        return cuda_fail(e, "fp8 activation cast");
      act = reinterpret_cast<uint16_t*>(a);
      ++launches;
    }
    if ((e = launch_expert_mma(blocks, scales, b, N, K, act, nullptr, offsets, active, n_active, 1, s, 1, K, 0.0f,
                               nullptr, y, nullptr, T, ws->err, nullptr, st)))
      return cuda_fail(e, "linear (register dequant)");
    ++launches;
  }
  if ((e = launch_f32_to_bf16(y, static_cast<int64_t>(T) * N, out, st, ws->sms))) return cuda_fail(e, "bf16 output");
  ++launches;
  t_last_launches = launches;
  return MXMOE_OK;
}

int fp8_linear(const uint16_t* x, int T, int K, const uint8_t* wq, int N, float s_x, float s_w, const float* bias,
               uint16_t* out, void* stream) {
  using namespace mxmoe;
  t_last_error.clear();
  t_last_launches = 0;
  if (T < 0 || K <= 0 || N <= 0) return fail(MXMOE_EINVAL, "T = %d must be >= 0, K = %d and N = %d positive", T, K, N);
  if (K % 32) return fail(MXMOE_EALIGN, "K = %d is not a multiple of 32", K);
  if (N % 8) return fail(MXMOE_EALIGN, "N = %d is not a multiple of 8", N);
  if (!(s_x > 0.0f) || !(s_w > 0.0f)) return fail(MXMOE_EINVAL, "s_x and s_w must be > 0");
  if (T >= (1 << 24)) return fail(MXMOE_EUNSUPPORTED, "T = %d exceeds 2^24 - 1", T);
  if (T == 0) return MXMOE_OK;
  if (!x || !wq || !out) return fail(MXMOE_EINVAL, "null pointer");
  if (!aligned16(x) || !aligned16(wq) || !aligned16(out) || (bias && !aligned16(bias)))
    return fail(MXMOE_EINVAL, "x, wq, out and bias must be 16-byte aligned");
  if (!fp8_linear_supported()) return fail(MXMOE_EUNSUPPORTED, "cuTensorMapEncodeTiled is unavailable");
  Workspace* ws = nullptr;
  if (int rc = current_device_ws(&ws)) return rc;
  const int ksplit = fp8_linear_ksplit(T, K, N, ws->sms);
  Carve c;
  c.take<uint8_t>(kTicketBytes);
  const size_t o_xq = c.take<uint8_t>(static_cast<int64_t>(T) * K);
  const size_t o_part = c.take<float>(ksplit > 1 ? static_cast<int64_t>(ksplit) * T * N : 0);
  if (int rc = ensure_capacity(ws, c.off)) return rc;
  ws->tickets_zeroed = kTicketBytes;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* xq = reinterpret_cast<uint8_t*>(ws->base + o_xq);
  float* part = reinterpret_cast<float*>(ws->base + o_part);
  cudaError_t e;
  StageTimer tm(st);
  if ((e = launch_fp8_quant(x, static_cast<int64_t>(T) * K, s_x, xq, st, ws->sms)))
    return cuda_fail(e, "fp8 activation cast");
  tm.mark("act_quant");
  const float s = s_x * s_w;
  if ((e = launch_fp8_linear(xq, T, K, wq, N, s, bias, out, part, ksplit, ws->err, ws->sms, st)))
    return cuda_fail(e, "fp8 linear");
  tm.mark("fp8_gemm");
  t_last_launches = ksplit > 1 ? 3 : 2;
  return MXMOE_OK;
}

int moe_route_topk(const uint16_t* x, const uint16_t* router_w, const uint16_t* router_b, int T,
                   int H, int E, int k, float* logits_out, int32_t* topk_idx, float* topk_w,
                   void* stream) {
  t_last_error.clear();
  if (int rc = check_routing_args(T, E, k)) return rc;
  if (H <= 0) return fail(MXMOE_EINVAL, "H = %d must be positive", H);
  if (H % 32) return fail(MXMOE_EALIGN, "H = %d is not a multiple of 32", H);
  if (T == 0) return MXMOE_OK;
  if (!x || !router_w || !topk_idx || !topk_w) return fail(MXMOE_EINVAL, "null pointer");
  if (!aligned16(x) || !aligned16(router_w)) return fail(MXMOE_EINVAL, "x and router_w must be 16-byte aligned");
  Workspace* ws = nullptr;
  if (int rc = current_device_ws(&ws)) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // workspace: the logits (unless the caller keeps them) and the tensor-core router's extra
  // K-range partials
  const bool rtc = T > 32 && mxmoe::router_tc_supported(T, H, E, x, router_w, logits_out);
  const int ksplit = rtc ? mxmoe::router_tc_ksplit(T, H, ws->sms) : 0;
  const int n_rest = ksplit > 1 ? ksplit - 1 : 0;
  const size_t lbytes = (static_cast<size_t>(T) * E * sizeof(float) + 255) & ~static_cast<size_t>(255);
  if (int rc = ensure_capacity(ws, kTicketBytes + (logits_out ? 0 : lbytes) + n_rest * lbytes)) return rc;
  ws->tickets_zeroed = kTicketBytes;   // the decode path's tickets may lie here
  float* logits = logits_out ? logits_out : reinterpret_cast<float*>(ws->base + kTicketBytes);
  float* rest = reinterpret_cast<float*>(ws->base + kTicketBytes + (logits_out ? 0 : lbytes));
  cudaError_t e = rtc ? mxmoe::launch_router_tc(x, router_w, router_b, T, H, E, ksplit, logits, rest, ws->err, st)
                      : mxmoe::launch_router(x, router_w, router_b, T, H, E, logits, st);
  if (e) return cuda_fail(e, "router launch");
  e = mxmoe::launch_topk(logits, rest, n_rest, T, E, k, topk_idx, topk_w, st);
  return e ? cuda_fail(e, "topk launch") : MXMOE_OK;
}

int moe_topk_from_logits(const float* logits, int T, int E, int k, int32_t* topk_idx,
                         float* topk_w, void* stream) {
  t_last_error.clear();
  if (int rc = check_routing_args(T, E, k)) return rc;
  if (T == 0) return MXMOE_OK;
  if (!logits || !topk_idx || !topk_w) return fail(MXMOE_EINVAL, "null pointer");
  cudaError_t e = mxmoe::launch_topk(const_cast<float*>(logits), nullptr, 0, T, E, k, topk_idx, topk_w,
                                     static_cast<cudaStream_t>(stream));
  return e ? cuda_fail(e, "topk launch") : MXMOE_OK;
}

int moe_permute(const int32_t* topk_idx, int T, int E, int k, int32_t* offsets,
                int32_t* perm_token, int32_t* perm_slot, void* stream) {
  t_last_error.clear();
  if (int rc = check_routing_args(T, E, k)) return rc;
  if (!offsets) return fail(MXMOE_EINVAL, "offsets is NULL");
  if (T > 0 && (!topk_idx || !perm_token || !perm_slot)) return fail(MXMOE_EINVAL, "null pointer");
  Workspace* ws = nullptr;
  if (int rc = current_device_ws(&ws)) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t P = static_cast<int64_t>(T) * k;
  if (T == 0) {
    cudaError_t e = cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), st);
    return e ? cuda_fail(e, "memset") : MXMOE_OK;
  }
  Carve c;
  c.take<uint8_t>(kTicketBytes);
  size_t o_counts = c.take<int32_t>(static_cast<int64_t>(mxmoe::permute_chunks(P)) * E);
  size_t o_act = c.take<int32_t>(E), o_n = c.take<int32_t>(1);
  if (int rc = ensure_capacity(ws, c.off)) return rc;
  ws->tickets_zeroed = kTicketBytes;   // the decode path's tickets may lie here
  int launches = 0;
  cudaError_t e = mxmoe::launch_permute(
      topk_idx, T, E, k, reinterpret_cast<int32_t*>(ws->base + o_counts), offsets, perm_token,
      perm_slot, nullptr, reinterpret_cast<int32_t*>(ws->base + o_act),
      reinterpret_cast<int32_t*>(ws->base + o_n), ws->err, st, &launches);
  return e ? cuda_fail(e, "permute launch") : MXMOE_OK;
}

int moe_fp8_quantize(const uint16_t* x, int64_t n, float s, uint8_t* q, void* stream) {
  t_last_error.clear();
  if (n < 0) return fail(MXMOE_EINVAL, "n = %lld is negative", (long long)n);
  if (n == 0) return MXMOE_OK;
  if (!x || !q) return fail(MXMOE_EINVAL, "null pointer");
  if (!(s > 0.0f)) return fail(MXMOE_EINVAL, "scale must be > 0");
  Workspace* ws = nullptr;
  if (int rc = current_device_ws(&ws)) return rc;
  cudaError_t e = mxmoe::launch_fp8_quant(x, n, s, q, static_cast<cudaStream_t>(stream), ws->sms);
  return e ? cuda_fail(e, "fp8 quant launch") : MXMOE_OK;
}

int moe_mxfp4_forward(const uint16_t* x, const uint16_t* router_w, const uint16_t* router_b,
                      const uint8_t* gu_blocks, const uint8_t* gu_scales, const float* gu_bias,
                      const uint8_t* d_blocks, const uint8_t* d_scales, const float* d_bias,
                      int E, int k, int T, int H, int I, const float* act_scale, uint16_t* out,
                      void* stream) {
  t_last_error.clear();
  LayerArgs a{x, router_w, router_b, gu_blocks, gu_scales, gu_bias, d_blocks, d_scales, d_bias,
              E, k, T, H, I};
  if (T == 0) return check_routing_args(T, E, k);
  if (int rc = check_layer_args(a)) return rc;
  if (!out) return fail(MXMOE_EINVAL, "out is NULL");
  if (!aligned16(out)) return fail(MXMOE_EINVAL, "out is not 16-byte aligned");
  if (act_scale && !(act_scale[0] > 0.0f && act_scale[1] > 0.0f))
    return fail(MXMOE_EINVAL, "act_scale values must be > 0");
  // Routed / dense crossover. With every expert selected (k == E) the dense all-experts
  // path does the same expert work as the routed one, without the permutation, the
  // gather into expert-grouped rows and the ordered combine (measured on B200, FP8, H = I =
  // 2880: k = E = 4 and 8 at T = 128 .. 4096, dense 0.82-0.99x the routed time). With k < E
  // it does E/k times the expert work and was slower at every measured size (top-4 of 32:
  // 1.13x at T = 128 rising to 4.3x at 1024; of 128: 1.4x at T = 64 to 20x at 4096), so the
  // routed path keeps those. Above the decode sizes both run the same expert kernels, so
  // the output is the same bit for bit.
  if (k == E && T > mxmoe::kDecodeMaxT && dense_kernels_take(a) && dense_fits(a))
    return run_layer_dense(a, act_scale, out, static_cast<cudaStream_t>(stream));
  return run_layer(a, act_scale, out, nullptr, static_cast<cudaStream_t>(stream));
}

int moe_mxfp4_forward_dense(const uint16_t* x, const uint16_t* router_w, const uint16_t* router_b,
                            const uint8_t* gu_blocks, const uint8_t* gu_scales, const float* gu_bias,
                            const uint8_t* d_blocks, const uint8_t* d_scales, const float* d_bias,
                            int E, int k, int T, int H, int I, const float* act_scale, uint16_t* out,
                            void* stream) {
  t_last_error.clear();
  t_last_launches = 0;
  LayerArgs a{x, router_w, router_b, gu_blocks, gu_scales, gu_bias, d_blocks, d_scales, d_bias,
              E, k, T, H, I};
  if (T == 0) return check_routing_args(T, E, k);
  if (int rc = check_layer_args(a)) return rc;
  if (!out) return fail(MXMOE_EINVAL, "out is NULL");
  if (!aligned16(out)) return fail(MXMOE_EINVAL, "out is not 16-byte aligned");
  if (act_scale && !(act_scale[0] > 0.0f && act_scale[1] > 0.0f))
    return fail(MXMOE_EINVAL, "act_scale values must be > 0");
  return run_layer_dense(a, act_scale, out, static_cast<cudaStream_t>(stream));
}

int moe_mxfp4_experts(const uint16_t* x_rows, const int32_t* offsets, int E, int P, int H, int I,
                      const uint8_t* gu_blocks, const uint8_t* gu_scales, const float* gu_bias,
                      const uint8_t* d_blocks, const uint8_t* d_scales, const float* d_bias,
                      const float* act_scale, float* y, void* stream) {
  using namespace mxmoe;
  t_last_error.clear();
  t_last_launches = 0;
  if (E < 1 || E > 256) return fail(MXMOE_EUNSUPPORTED, "E = %d outside [1, 256]", E);
  if (P < 0 || H <= 0 || I <= 0) return fail(MXMOE_EINVAL, "P = %d must be >= 0, H = %d and I = %d positive", P, H, I);
  if (H % 32 || I % 32) return fail(MXMOE_EALIGN, "H = %d and I = %d must be multiples of 32", H, I);
  if (P >= (1 << 24)) return fail(MXMOE_EUNSUPPORTED, "P = %d exceeds 2^24 - 1", P);
  if (P == 0) return MXMOE_OK;
  const void* ptrs[] = {x_rows, offsets, gu_blocks, gu_scales, gu_bias, d_blocks, d_scales, d_bias, y};
  for (const void* q : ptrs)
    if (!q) return fail(MXMOE_EINVAL, "null pointer");
  if (!aligned16(x_rows) || !aligned16(y) || !aligned16(gu_blocks) || !aligned16(d_blocks) || !aligned16(gu_bias) ||
      !aligned16(d_bias))
    return fail(MXMOE_EINVAL, "x_rows, y, blocks and biases must be 16-byte aligned");
  if (act_scale && !(act_scale[0] > 0.0f && act_scale[1] > 0.0f))
    return fail(MXMOE_EINVAL, "act_scale values must be > 0");
  if (!(std::max(H, I) / 32 <= kTcMaxNb && tc_gemm_supported(H, I, gu_blocks, d_blocks, gu_scales, d_scales)))
    return fail(MXMOE_EUNSUPPORTED, "the grouped expert GEMMs need H and I multiples of 64 in [128, 4608] and "
                                    "32-byte aligned blocks (got H = %d, I = %d)", H, I);
  Workspace* ws = nullptr;
  if (int rc = current_device_ws(&ws)) return rc;
  const bool fp8 = act_scale != nullptr;
  const int64_t PH = static_cast<int64_t>(P) * H, PI = static_cast<int64_t>(P) * I;
  Carve c;
  c.take<uint8_t>(kTicketBytes);
  const size_t o_a1 = c.take<uint8_t>(fp8 ? PH : 2 * PH);
  const size_t o_sa1 = c.take<uint8_t>(fp8 ? 0 : 2 * (PH / 32));
  const size_t o_mid = c.take<uint16_t>(fp8 ? 0 : PI);
  const size_t o_a2 = c.take<uint8_t>(fp8 ? PI : 2 * PI);
  const size_t o_sa2 = c.take<uint8_t>(fp8 ? 0 : 2 * (PI / 32));
  if (int rc = ensure_capacity(ws, c.off)) return rc;
  ws->tickets_zeroed = kTicketBytes;
  if (fp8 && !ws->tc_ready) {
    cudaError_t e = tc_gemm_prepare(256);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute (tcgen05 GEMM)");
    ws->tc_ready = true;
  }
  if (!fp8 && !ws->tcb_ready) {
    cudaError_t e = tc_parts_gemm_prepare(256);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute (two-part tcgen05 GEMM)");
    ws->tcb_ready = true;
  }
  char* base = ws->base;
  uint8_t* a1 = reinterpret_cast<uint8_t*>(base + o_a1);
  uint8_t* sa1 = reinterpret_cast<uint8_t*>(base + o_sa1);
  uint16_t* mid = reinterpret_cast<uint16_t*>(base + o_mid);
  uint8_t* a2 = reinterpret_cast<uint8_t*>(base + o_a2);
  uint8_t* sa2 = reinterpret_cast<uint8_t*>(base + o_sa2);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (fp8) {
    const float s0 = act_scale[0], s1 = act_scale[1];
    if ((e = launch_fp8_quant(x_rows, PH, s0, a1, st, ws->sms))) return cuda_fail(e, "fp8 activation cast");
    if ((e = launch_tc_gemm(true, a1, P, H, gu_blocks, gu_scales, gu_bias, E, I, offsets, s0, s1, a2, nullptr, ws->err,
                            ws->sms, st)))
      return cuda_fail(e, "gate_up (tcgen05)");
    if ((e = launch_tc_gemm(false, a2, P, I, d_blocks, d_scales, d_bias, E, H, offsets, s1, 0.0f, nullptr, y, ws->err,
                            ws->sms, st)))
      return cuda_fail(e, "down (tcgen05)");
  } else {
    if ((e = launch_split_parts(x_rows, nullptr, P, P, H, a1, sa1, ws->sms, st))) return cuda_fail(e, "activation split");
    if ((e = launch_tc_parts_gemm(true, a1, sa1, P, H, gu_blocks, gu_scales, gu_bias, E, I, offsets, mid, nullptr,
                                  ws->err, ws->sms, st)))
      return cuda_fail(e, "gate_up (tcgen05, two parts)");
    if ((e = launch_split_parts(mid, nullptr, P, P, I, a2, sa2, ws->sms, st))) return cuda_fail(e, "intermediate split");
    if ((e = launch_tc_parts_gemm(false, a2, sa2, P, I, d_blocks, d_scales, d_bias, E, H, offsets, nullptr, y, ws->err,
                                  ws->sms, st)))
      return cuda_fail(e, "down (tcgen05, two parts)");
  }
  t_last_launches = fp8 ? 3 : 4;
  return MXMOE_OK;
}

int moe_combine(const float* y, const int32_t* topk_idx, const float* topk_w, const int32_t* inv, int T, int H, int k,
                uint16_t* out, void* stream) {
  t_last_error.clear();
  t_last_launches = 0;
  if (T < 0 || H <= 0) return fail(MXMOE_EINVAL, "T = %d must be >= 0 and H = %d positive", T, H);
  if (k < 1 || k > 8) return fail(MXMOE_EUNSUPPORTED, "k = %d outside [1, 8]", k);
  if (H % 8) return fail(MXMOE_EALIGN, "H = %d is not a multiple of 8", H);
  if (T == 0) return MXMOE_OK;
  if (!y || !topk_idx || !topk_w || !inv || !out) return fail(MXMOE_EINVAL, "null pointer");
  if (!aligned16(y) || !aligned16(out)) return fail(MXMOE_EINVAL, "y and out must be 16-byte aligned");
  Workspace* ws = nullptr;
  if (int rc = current_device_ws(&ws)) return rc;
  cudaError_t e = mxmoe::launch_combine(y, topk_idx, topk_w, inv, T, H, k, out, static_cast<cudaStream_t>(stream),
                                        ws->sms);
  if (e) return cuda_fail(e, "combine launch");
  t_last_launches = 1;
  return MXMOE_OK;
}

int moe_mxfp4_calibrate(const uint16_t* x, const uint16_t* router_w, const uint16_t* router_b,
                        const uint8_t* gu_blocks, const uint8_t* gu_scales, const float* gu_bias,
                        const uint8_t* d_blocks, const uint8_t* d_scales, const float* d_bias,
                        int E, int k, int T, int H, int I, float* act_scale_out, void* stream) {
  t_last_error.clear();
  LayerArgs a{x, router_w, router_b, gu_blocks, gu_scales, gu_bias, d_blocks, d_scales, d_bias,
              E, k, T, H, I};
  if (T == 0) return fail(MXMOE_EINVAL, "calibration needs T > 0 tokens");
  if (int rc = check_layer_args(a)) return rc;
  if (!act_scale_out) return fail(MXMOE_EINVAL, "act_scale_out is NULL");
  return run_layer(a, nullptr, nullptr, act_scale_out, static_cast<cudaStream_t>(stream));
}

int mxmoe_check(void* stream) {
  t_last_error.clear();
  Workspace* ws = nullptr;
  if (int rc = current_device_ws(&ws)) return rc;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stream");
  int v = 0;
  if ((e = cudaMemcpy(&v, ws->err, sizeof(int), cudaMemcpyDeviceToHost))) return cuda_fail(e, "read error word");
  if (v != 0) {
    if ((e = cudaMemset(ws->err, 0, sizeof(int)))) return cuda_fail(e, "clear error word");
    // a kernel that stopped early may have left its counters short of zero
    ws->tickets_zeroed = 0;
    return fail(v, "device error word = %d", v);
  }
  return MXMOE_OK;
}

int mxmoe_selftest_wait_timeout(void* stream) {
  t_last_error.clear();
  Workspace* ws = nullptr;
  if (int rc = current_device_ws(&ws)) return rc;
  cudaError_t e = mxmoe::launch_wait_selftest(ws->err, static_cast<cudaStream_t>(stream));
  return e ? cuda_fail(e, "wait self-test launch") : MXMOE_OK;
}

int mxmoe_tc_rate_probe(int n, int with_scale_copy, int random_operands, int iters, int ctas, double* flops,
                        void* stream) {
  t_last_error.clear();
  t_last_launches = 0;
  if (n < 16 || n > 256 || n % 16) return fail(MXMOE_EINVAL, "n = %d must be a multiple of 16 in [16, 256]", n);
  if (random_operands != 0 && random_operands != 1)
    return fail(MXMOE_EINVAL, "random_operands = %d must be 0 or 1", random_operands);
  if (iters < 1 || iters > 1000000) return fail(MXMOE_EINVAL, "iters = %d outside [1, 1000000]", iters);
  if (ctas < 1 || ctas > 4096) return fail(MXMOE_EINVAL, "ctas = %d outside [1, 4096]", ctas);
  Workspace* ws = nullptr;
  if (int rc = current_device_ws(&ws)) return rc;
  cudaError_t e = mxmoe::launch_tc_rate(n, with_scale_copy ? 1 : 0, random_operands, iters, ctas, ws->err,
                                        static_cast<cudaStream_t>(stream));
  if (e) return cuda_fail(e, "rate probe launch");
  t_last_launches = 1;
  if (flops) *flops = 2.0 * 128.0 * n * 32.0 * 4.0 * iters * ctas;
  return MXMOE_OK;
}

const char* mxmoe_last_error(void) { return t_last_error.c_str(); }

int mxmoe_last_launch_count(void) { return t_last_launches; }

int mxmoe_profile_enable(int on) {
  t_last_error.clear();
  t_profile = on != 0;
  t_marks.clear();
  t_event_next = 0;
  return MXMOE_OK;
}

int mxmoe_profile_read(char* names, float* total_ms, int* calls, int max_entries) {
  t_last_error.clear();
  if (max_entries < 0 || (max_entries > 0 && (!names || !total_ms || !calls)))
    return fail(MXMOE_EINVAL, "bad output arrays");
  std::vector<std::string> keys;
  std::vector<double> ms;
  std::vector<int> n;
  for (const StageMark& m : t_marks) {
    cudaError_t e = cudaEventSynchronize(m.stop);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventSynchronize");
    float dt = 0.0f;
    if ((e = cudaEventElapsedTime(&dt, m.start, m.stop)) != cudaSuccess) return cuda_fail(e, "cudaEventElapsedTime");
    size_t i = 0;
    while (i < keys.size() && keys[i] != m.name) ++i;
    if (i == keys.size()) { keys.push_back(m.name); ms.push_back(0.0); n.push_back(0); }
    ms[i] += dt;
    n[i] += 1;
  }
  const int cnt = static_cast<int>(keys.size());
  for (int i = 0; i < cnt && i < max_entries; ++i) {
    std::snprintf(names + 32 * i, 32, "%s", keys[i].c_str());
    total_ms[i] = static_cast<float>(ms[i]);
    calls[i] = n[i];
  }
  t_marks.clear();
  t_event_next = 0;
  return cnt;
}

int mxmoe_release(void) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  std::lock_guard<std::mutex> lk(g_mu);
  if (dev >= 0 && dev < kMaxDevices && g_ws[dev].base) {
    if ((e = cudaDeviceSynchronize()) != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
    cudaFree(g_ws[dev].base);
    g_ws[dev].base = nullptr;
    g_ws[dev].cap = 0;
  }
  return MXMOE_OK;
}

}  // extern "C"

// ------------------------------------------------- allocation-free permute -----
// moe_permute_noalloc: the same grouping as moe_permute, for callers that must not
// allocate device memory. The kernels' scratch (per-chunk expert histograms and the
// active-expert list) lives in a fixed array of this library's device image instead of
// the cudaMalloc'd workspace. Host code may not pass `g_noalloc_scratch` itself to a
// kernel (in host code the name stands for a host-side shadow, not a device address),
// so every call looks the current device's address up with cudaGetSymbolAddress (it
// allocates nothing). Looking it up per call rather than caching it keeps the address
// valid after a context teardown (cudaDeviceReset) reloads the library's device image.
namespace {

constexpr int64_t kNoAllocMaxPairs = 262144;   // T * k accepted by the variant
constexpr int kNoAllocMaxExperts = 256;
constexpr int kNoAllocMaxChunks = 128;         // the permute never uses more chunks
constexpr int kNoAllocInts = kNoAllocMaxChunks * kNoAllocMaxExperts + kNoAllocMaxExperts + 64;

// 256-byte aligned, 132,352 bytes; every GPU that loads the library keeps it until exit.
static __device__ __align__(256) int32_t g_noalloc_scratch[kNoAllocInts];

}  // namespace

extern "C" int moe_permute_noalloc(const int32_t* topk_idx, int T, int E, int k, int32_t* offsets,
                                   int32_t* perm_token, int32_t* perm_slot, void* stream) {
  t_last_error.clear();
  if (int rc = check_routing_args(T, E, k)) return rc;
  const int64_t P = static_cast<int64_t>(T) * k;
  if (P > kNoAllocMaxPairs)
    return fail(MXMOE_EUNSUPPORTED, "moe_permute_noalloc: T*k = %lld exceeds its fixed scratch limit of %lld pairs",
                (long long)P, (long long)kNoAllocMaxPairs);
  if (mxmoe::permute_chunks(P) > kNoAllocMaxChunks)
    return fail(MXMOE_EUNSUPPORTED, "moe_permute_noalloc: too many chunks");
  if (!offsets) return fail(MXMOE_EINVAL, "offsets is NULL");
  if (T > 0 && (!topk_idx || !perm_token || !perm_slot)) return fail(MXMOE_EINVAL, "null pointer");
  void* ptr = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);   // the current device's copy
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(scratch)");
  int32_t* scratch = static_cast<int32_t*>(ptr);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (T == 0) {
    e = cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), st);
    return e ? cuda_fail(e, "memset") : MXMOE_OK;
  }
  // Every launch writes all the scratch it reads (each chunk's full histogram row, the
  // active list and its count), so nothing has to be cleared between calls.
  int32_t* counts = scratch;
  int32_t* active = scratch + kNoAllocMaxChunks * kNoAllocMaxExperts;
  int32_t* n_active = active + kNoAllocMaxExperts;
  int launches = 0;
  e = mxmoe::launch_permute(topk_idx, T, E, k, counts, offsets, perm_token, perm_slot, nullptr, active,
                            n_active, nullptr, st, &launches);
  return e ? cuda_fail(e, "permute launch") : MXMOE_OK;
}
