// coli_api.cu -- the extern "C" entry points of libcoli (declared in
// include/coli.h): argument validation, workspace layout, launch order.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

#include "../../include/coli.h"
#include "coli_launch.h"
#include "coli_tc.cuh"

#define COLI_EXPORT extern "C" __attribute__((visibility("default")))

namespace coli {
namespace {

thread_local std::string g_last_error;
thread_local cudaEvent_t g_phase_ev[3] = {nullptr, nullptr, nullptr};
thread_local int32_t* g_capture = nullptr;  // armed partials capture (coli_debug_capture_partials)
thread_local size_t g_capture_words = 0;

coli_status fail(coli_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

coli_status cuda_status(cudaError_t e, const char* where) {
  if (e == cudaSuccess) return COLI_OK;
  return fail(COLI_ECUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define CHECK_PTR(p)                                                                  \
  do {                                                                                \
    if ((p) == nullptr) return fail(COLI_EINVAL, "%s: null pointer '%s'", fn, #p);    \
    if (!aligned16(p)) return fail(COLI_EINVAL, "%s: '%s' is not 16-byte aligned", fn, #p); \
  } while (0)

#define CHECK_LAUNCH(expr)                                  \
  do {                                                      \
    coli_status _s = cuda_status((expr), fn);               \
    if (_s != COLI_OK) return _s;                           \
  } while (0)

coli_status check_cfg(const coli_moe_config* c, const char* fn) {
  if (c == nullptr) return fail(COLI_EINVAL, "%s: null config", fn);
  if (c->hidden <= 0 || c->hidden % 128 != 0)
    return fail(COLI_EINVAL, "%s: hidden=%d must be a positive multiple of 128", fn, c->hidden);
  if (c->inter <= 0 || c->inter % 32 != 0)
    return fail(COLI_EINVAL, "%s: inter=%d must be a positive multiple of 32", fn, c->inter);
  if (c->n_experts < 1 || c->n_experts > kMaxExperts)
    return fail(COLI_EINVAL, "%s: n_experts=%d outside [1, %d]", fn, c->n_experts, kMaxExperts);
  if (c->top_k < 1 || c->top_k > c->n_experts || c->top_k > kMaxTopK)
    return fail(COLI_EINVAL, "%s: top_k=%d outside [1, min(n_experts, %d)]", fn, c->top_k, kMaxTopK);
  if (c->n_shared < 0 || c->n_shared > kMaxShared)
    return fail(COLI_EINVAL, "%s: n_shared=%d outside [0, %d]", fn, c->n_shared, kMaxShared);
  if (c->n_shared > 0 && c->shared_inter != c->inter)
    return fail(COLI_EINVAL, "%s: shared_inter=%d must equal inter=%d", fn, c->shared_inter, c->inter);
  if (c->weight_bits != 0 && c->weight_bits != 4 && c->weight_bits != 8)
    return fail(COLI_EINVAL, "%s: weight_bits=%d (4 or 8)", fn, c->weight_bits);
  if (c->weight_bits == 8 && !prefill_supported(c->hidden, c->inter))
    return fail(COLI_EINVAL, "%s: int8 weights need hidden and inter multiples of 128", fn);
  return COLI_OK;
}

int bits_of(const coli_moe_config& c) { return c.weight_bits == 8 ? 8 : 4; }

coli_status check_expert(const coli_expert* e, const char* fn) {
  if (e == nullptr) return fail(COLI_EINVAL, "%s: null expert", fn);
  CHECK_PTR(e->gate_q);
  CHECK_PTR(e->gate_s);
  CHECK_PTR(e->up_q);
  CHECK_PTR(e->up_s);
  CHECK_PTR(e->down_q);
  CHECK_PTR(e->down_s);
  return COLI_OK;
}

coli_status check_layer(const coli_moe_layer* L, const char* fn) {
  if (L == nullptr) return fail(COLI_EINVAL, "%s: null layer", fn);
  coli_status s = check_cfg(&L->cfg, fn);
  if (s != COLI_OK) return s;
  CHECK_PTR(L->w_router);
  CHECK_PTR(L->bias);
  if (L->experts == nullptr) return fail(COLI_EINVAL, "%s: null experts array", fn);
  if (L->cfg.n_shared > 0 && L->shared == nullptr) return fail(COLI_EINVAL, "%s: null shared array", fn);
  if (L->prepared != nullptr && (reinterpret_cast<uintptr_t>(L->prepared) & 255u) != 0)
    return fail(COLI_EINVAL, "%s: 'prepared' is not 256-byte aligned", fn);
  for (int e = 0; e < L->cfg.n_experts; ++e)
    if ((s = check_expert(&L->experts[e], fn)) != COLI_OK) return s;
  for (int e = 0; e < L->cfg.n_shared; ++e)
    if ((s = check_expert(&L->shared[e], fn)) != COLI_OK) return s;
  return COLI_OK;
}

// ---------------------------------------------------------------------------
// workspace

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

struct Workspace {
  size_t xq, xd, scores, idx, w, counts, offsets, perm, inv, slots, n_slots, status, tiles, n_tiles, hq, hd, xr, hdc,
      xdc, ctr, y, xn, xa, xb, total;
};

Workspace layout(const coli_moe_config& c, int64_t T) {
  Workspace L{};
  const int64_t H = c.hidden, I = c.inter, E = c.n_experts, K = c.top_k, S = c.n_shared;
  const int64_t rows = T * K + T * S;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t at = off;
    off = align256(off + (bytes ? bytes : 1));
    return at;
  };
  L.status = take(4);  // first, at offset 0: coli_sync_status reads it without knowing T
  L.xq = take(T * H);
  L.xd = take(T * (H / 32) * 4);
  L.scores = take(T * E * 4);
  L.idx = take(T * K * 4);
  L.w = take(T * K * 4);
  L.counts = take(E * 4);
  L.offsets = take((E + 1) * 4);
  L.perm = take(T * K * 4);
  L.inv = take(T * K * 4);
  L.slots = take((size_t)kMaxSlots * sizeof(Slot));
  L.n_slots = take(4);
  // the tensor-core prefill path's buffers only when a call of T tokens can take that path
  // (int8 weights: whenever the layer is not prepared or T > kStreamMaxTok)
  const bool tc = (T > kDecodeMaxTok || !decode_supported((int)H, (int)I) || bits_of(c) == 8) &&
                  prefill_supported((int)H, (int)I);
  L.tiles = take(tc ? prefill_tile_bytes((int)T, (int)K, (int)E, (int)S) : 0);
  L.n_tiles = take(4);
  L.hq = take(rows * I);  // h as int8 rows (Q8 of h; the tensor-core path's down operand)
  L.xr = take(tc ? rows * H : 0);
  L.hd = take(rows * (I / 32) * 4);
  // the streaming decode kernel (prepared layers, up to kStreamMaxTok
  // tokens): (d, c16) of every h block of a call, its x planes' (d, c16),
  // and its counters
  const bool sm = T <= kStreamMaxTok;
  L.hdc = take(sm ? T * (K + S) * (I / 32) * 8 : 0);
  L.xdc = take(sm ? T * (H / 32) * 8 : 0);  // with xq: the x planes the router kernel writes for > 2 tokens
  L.ctr = take(sm ? (size_t)kStreamMaxSlots * 4 : 0);
  L.y = take(rows * H * 4);
  L.xn = take(T * H * 4);
  L.xa = take(T * H * 4);
  L.xb = take(T * H * 4);
  L.total = off;
  return L;
}

template <typename P>
P* at(void* ws, size_t off) {
  return reinterpret_cast<P*>(static_cast<char*>(ws) + off);
}

void fill_tables(const coli_moe_layer* L, GateUpTable& gu, DownTable& dn) {
  const int E = L->cfg.n_experts;
  auto put = [&](int i, const coli_expert& e) {
    gu.gate_q[i] = e.gate_q;
    gu.gate_s[i] = e.gate_s;
    gu.up_q[i] = e.up_q;
    gu.up_s[i] = e.up_s;
    dn.down_q[i] = e.down_q;
    dn.down_s[i] = e.down_s;
  };
  for (int e = 0; e < E; ++e) put(e, L->experts[e]);
  for (int s = 0; s < L->cfg.n_shared; ++s) put(E + s, L->shared[s]);
}

// The layer forward on a validated layer, x -> out, scratch in ws.
// clear_status: this call starts the workspace's status word afresh (the
// first layer of a forward call).
coli_status layer_forward(const coli_moe_layer* L, const float* x, int64_t T, float* out, void* ws,
                          const Workspace& W, cudaStream_t st, const char* fn, bool clear_status) {
  const coli_moe_config& c = L->cfg;
  const int H = c.hidden, I = c.inter, E = c.n_experts, K = c.top_k, S = c.n_shared;
  int8_t* xq = at<int8_t>(ws, W.xq);
  float* xd = at<float>(ws, W.xd);
  float* scores = at<float>(ws, W.scores);
  int32_t* idx = at<int32_t>(ws, W.idx);
  float* wts = at<float>(ws, W.w);
  int32_t* perm = at<int32_t>(ws, W.perm);
  int32_t* inv = at<int32_t>(ws, W.inv);
  Slot* slots = at<Slot>(ws, W.slots);
  int32_t* n_slots = at<int32_t>(ws, W.n_slots);
  int8_t* hq = at<int8_t>(ws, W.hq);
  float* hd = at<float>(ws, W.hd);
  float* y = at<float>(ws, W.y);

  static thread_local GateUpTable gu;
  static thread_local DownTable dn;
  fill_tables(L, gu, dn);

  cudaEvent_t ev[3] = {g_phase_ev[0], g_phase_ev[1], g_phase_ev[2]};
  g_phase_ev[0] = g_phase_ev[1] = g_phase_ev[2] = nullptr;
  int32_t* capture = g_capture;
  const size_t capture_words = g_capture_words;
  g_capture = nullptr;
  g_capture_words = 0;
  if (capture != nullptr) {
    const size_t P = 2 * (size_t)I * (H / 32) + (size_t)H * (I / 32);
    const size_t need = (size_t)T * (K + S) * P;
    if (capture_words < need)
      return fail(COLI_EINVAL, "%s: the partials capture needs %zu int32 words, %zu given", fn, need, capture_words);
  }
  auto mark = [&](int i) -> cudaError_t {
    return ev[i] ? cudaEventRecordWithFlags(ev[i], st, cudaEventRecordExternal) : cudaSuccess;
  };

  int32_t* status = at<int32_t>(ws, W.status);
  const int bits = bits_of(c);
  const bool aligned16 = ((uintptr_t)x & 15) == 0;
  if (L->prepared != nullptr && aligned16 && T <= kStreamMaxTok && stream_supported(H, I, bits, (int)T, K, S, E)) {
    // decode on the streaming copy: 2 kernels, the second launched with PDL
    int32_t* ctr = at<int32_t>(ws, W.ctr);
    // up to 2 tokens the streaming kernel quantises x itself (so that the
    // shared expert starts before the router kernel ends); more tokens take
    // the router kernel's planes
    int8_t* xpl = T > 2 ? xq : nullptr;
    float2* xdcp = T > 2 ? at<float2>(ws, W.xdc) : nullptr;
    CHECK_LAUNCH(launch_router_decode(x, L->w_router, (int)T, E, H, scores, nullptr, nullptr,
                                      clear_status ? status : nullptr, ctr, kStreamMaxSlots, st, xpl, xdcp));
    CHECK_LAUNCH(mark(0));
    StreamArgs a{};
    a.prep = static_cast<const unsigned char*>(L->prepared);
    a.g = stream_geom(H, I, bits);
    a.E = E;
    a.K = K;
    a.S = S;
    a.T = (int)T;
    a.norm = c.norm_topk_prob;
    a.rsf = c.routed_scaling_factor;
    a.scores = scores;
    a.bias = L->bias;
    a.x = x;
    a.xpl_g = xpl;
    a.xdc_g = xdcp;
    a.hpl = hq;
    a.hdc = at<float2>(ws, W.hdc);
    a.out = out;
    a.h_ready = ctr;
    a.status = status;
    a.dbg = capture;
    CHECK_LAUNCH(launch_expert_stream(a, st));
    CHECK_LAUNCH(mark(1));
    CHECK_LAUNCH(mark(2));
    return COLI_OK;
  }
  if (bits == 4 && T <= kDecodeMaxTok && decode_supported(H, I)) {
    if (capture != nullptr)
      return fail(COLI_EINVAL, "%s: the partials capture covers the streaming (prepared layer, <= %d tokens) and "
                  "tensor-core kernels, not this call's decode kernels", fn, kStreamMaxTok);
    // decode: 5 kernels, the last four launched with PDL
    CHECK_LAUNCH(launch_router_decode(x, L->w_router, (int)T, E, H, scores, xq, xd, clear_status ? status : nullptr,
                                      nullptr, 0, st));
    CHECK_LAUNCH(launch_topk_bucket_small(scores, L->bias, (int)T, E, K, c.norm_topk_prob, c.routed_scaling_factor,
                                          idx, wts, at<int32_t>(ws, W.counts), at<int32_t>(ws, W.offsets), perm, inv,
                                          slots, n_slots, st));
    CHECK_LAUNCH(mark(0));
    CHECK_LAUNCH(launch_gateup_decode(gu, slots, n_slots, perm, (int)T, K, E, S, x, xq, xd, H, I, hq, hd, status, st));
    CHECK_LAUNCH(mark(1));
    CHECK_LAUNCH(launch_down_decode(dn, slots, n_slots, (int)T, K, E, S, hq, hd, inv, wts, H, I, y, out, status, st));
    CHECK_LAUNCH(mark(2));
    return COLI_OK;
  }

  if (clear_status) CHECK_LAUNCH(cudaMemsetAsync(status, 0, sizeof(int32_t), st));
  CHECK_LAUNCH(launch_quantize_act_q8(x, T, H, xq, xd, st));
  CHECK_LAUNCH(launch_router_scores(x, L->w_router, (int)T, E, H, scores, st));
  CHECK_LAUNCH(launch_topk(scores, L->bias, (int)T, E, K, c.norm_topk_prob, c.routed_scaling_factor, idx, wts, st));
  CHECK_LAUNCH(launch_bucket(idx, (int)T, K, E, S, at<int32_t>(ws, W.counts), at<int32_t>(ws, W.offsets), perm, inv,
                             slots, n_slots, at<int32_t>(ws, W.status), st));
  GemvSlots sl{};
  sl.slots = slots;
  sl.n_slots = n_slots;
  sl.max_slots = (int)((T * K < E ? T * K : E) + S);
  sl.perm = perm;
  sl.top_k = K;
  const int max_tok = (int)T;
  CHECK_LAUNCH(mark(0));
  if (prefill_supported(H, I)) {
    CHECK_LAUNCH(launch_prefill_experts(gu, dn, slots, n_slots, at<void>(ws, W.tiles), at<int32_t>(ws, W.n_tiles),
                                        perm, K, S, bits, xq, xd, (int)T, H, I, at<void>(ws, W.xr), hq, hd, y,
                                        at<int32_t>(ws, W.status), st, ev[1], capture, E));
  } else {
    if (capture != nullptr)
      return fail(COLI_EINVAL, "%s: the partials capture covers the streaming and tensor-core kernels only", fn);
    CHECK_LAUNCH(launch_gateup(gu, sl, xq, xd, H, I, max_tok, hq, hd, st));
    CHECK_LAUNCH(mark(1));
    CHECK_LAUNCH(launch_down(dn, sl, hq, hd, H, I, max_tok, y, st));
  }
  CHECK_LAUNCH(mark(2));
  CHECK_LAUNCH(launch_combine(y, inv, wts, (int)T, K, S, H, out, st));
  return COLI_OK;
}

}  // namespace

void set_error_message(const char* msg) { g_last_error = msg; }

}  // namespace coli

using namespace coli;

COLI_EXPORT const char* coli_last_error(void) { return g_last_error.c_str(); }

COLI_EXPORT coli_status coli_debug_capture_partials(int32_t* isum_out, size_t n_words) {
  const char* fn = "coli_debug_capture_partials";
  if (isum_out == nullptr || (reinterpret_cast<uintptr_t>(isum_out) & 15u) != 0)
    return fail(COLI_EINVAL, "%s: isum_out must be a 16-byte aligned device pointer", fn);
  g_capture = isum_out;
  g_capture_words = n_words;
  return COLI_OK;
}

COLI_EXPORT coli_status coli_debug_phase_events(void* before_experts, void* after_gateup, void* after_down) {
  g_phase_ev[0] = (cudaEvent_t)before_experts;
  g_phase_ev[1] = (cudaEvent_t)after_gateup;
  g_phase_ev[2] = (cudaEvent_t)after_down;
  return COLI_OK;
}

COLI_EXPORT size_t coli_moe_workspace_bytes(const coli_moe_config* cfg, int64_t max_tokens) {
  if (check_cfg(cfg, "coli_moe_workspace_bytes") != COLI_OK || max_tokens < 0) return 0;
  return layout(*cfg, max_tokens).total;
}

COLI_EXPORT size_t coli_moe_prepared_bytes(const coli_moe_config* cfg) {
  if (check_cfg(cfg, "coli_moe_prepared_bytes") != COLI_OK) return 0;
  if (!stream_shape_ok(cfg->hidden, cfg->inter, bits_of(*cfg))) return 0;
  return (size_t)(cfg->n_experts + cfg->n_shared) * stream_expert_bytes(cfg->hidden, cfg->inter, bits_of(*cfg));
}

COLI_EXPORT coli_status coli_moe_prepare(const coli_moe_layer* layer, void* prepared, size_t bytes, void* stream) {
  const char* fn = "coli_moe_prepare";
  coli_status s = check_layer(layer, fn);
  if (s != COLI_OK) return s;
  const coli_moe_config& c = layer->cfg;
  const size_t need = coli_moe_prepared_bytes(&c);
  if (need == 0)
    return fail(COLI_EINVAL, "%s: hidden=%d inter=%d has no streaming layout (both multiples of 128; int4: hidden/32 "
                "a multiple of 16 or 4, 8; inter/32 a multiple of 32 or 4, 8, 16; int8: hidden/32 a multiple of 8 or "
                "4; inter/32 a multiple of 16 or 4, 8)", fn, c.hidden, c.inter);
  if (prepared == nullptr) return fail(COLI_EINVAL, "%s: null pointer 'prepared'", fn);
  if ((reinterpret_cast<uintptr_t>(prepared) & 255u) != 0)
    return fail(COLI_EINVAL, "%s: 'prepared' is not 256-byte aligned", fn);
  if (bytes < need) return fail(COLI_ENOMEM, "%s: %zu bytes < %zu needed", fn, bytes, need);
  const uint64_t eb = stream_expert_bytes(c.hidden, c.inter, bits_of(c));
  cudaStream_t st = (cudaStream_t)stream;
  for (int j = 0; j < c.n_experts + c.n_shared; ++j) {
    const coli_expert& e = j < c.n_experts ? layer->experts[j] : layer->shared[j - c.n_experts];
    CHECK_LAUNCH(launch_prepare_expert(c.hidden, c.inter, bits_of(c), e.gate_q, e.gate_s, e.up_q, e.up_s, e.down_q,
                                       e.down_s, static_cast<unsigned char*>(prepared) + (size_t)j * eb, st));
  }
  return COLI_OK;
}

namespace coli {
namespace {

const char* status_meaning(int32_t code) {
  switch (code) {
    case kStatusBadExpert: return "bucketing met an expert index outside [0, n_experts)";
    case 10: return "prefill producers gave up waiting for an operand stage";
    case 11: return "prefill MMA issuer gave up waiting for operands";
    case 12: return "prefill MMA issuer gave up waiting for accumulator buffers";
    case 13: return "prefill fold gave up waiting for accumulators";
    case 16: return "prefill A-tile loader gave up waiting for an operand stage";
    case 22: return "decode down kernel gave up waiting for h rows";
    case 25: return "streaming decode kernel gave up waiting for a slot's h rows from other CTAs";
    case 26: return "streaming decode kernel gave up waiting for a slot's h rows in shared memory";
    case 27: return "streaming decode kernel gave up waiting for its warp pair's h buffer";
    case 28: return "streaming decode kernel gave up waiting for a weight stage copy";
    case 29: return "streaming decode kernel gave up waiting for the routing of the batch";

    case kStatusWaitProbe: return "test probe: a wait that nothing completes gave up";
    default: return code >= kStatusTimeoutFirst ? "a bounded wait gave up" : "a device-side check failed";
  }
}

// Test probe: one thread waits on an mbarrier that nothing arrives at, for
// at most `cycles` clock cycles, then records kStatusWaitProbe.
__global__ void wait_probe_kernel(int32_t* status, long long cycles) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  tc::mbar_init(&bar, 1);
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  const long long t0 = clock64();
  bool done = false;
  while (!(done = tc::mbar_try_wait_sleep(&bar, 0, 1000)) && clock64() - t0 < cycles) {
  }
  if (!done) atomicExch(status, kStatusWaitProbe);
}

}  // namespace
}  // namespace coli

COLI_EXPORT coli_status coli_sync_status(void* workspace, void* stream) {
  const char* fn = "coli_sync_status";
  void* ws = workspace;
  if (ws == nullptr) {
    coli_status s = cuda_status(noalloc_scratch(&ws), fn);
    if (s != COLI_OK) return s;
  } else {
    CHECK_PTR(workspace);
  }
  CHECK_LAUNCH(cudaStreamSynchronize((cudaStream_t)stream));
  int32_t code = 0;
  CHECK_LAUNCH(cudaMemcpy(&code, ws, sizeof code, cudaMemcpyDeviceToHost));
  if (code == 0) return COLI_OK;
  return fail(code >= kStatusTimeoutFirst ? COLI_ETIMEOUT : COLI_EDEVICE, "%s: device status %d: %s", fn, (int)code,
              status_meaning(code));
}

COLI_EXPORT coli_status coli_debug_wait_probe(void* workspace, int64_t cycles, void* stream) {
  const char* fn = "coli_debug_wait_probe";
  CHECK_PTR(workspace);
  if (cycles < 0 || cycles > (int64_t)4000000000LL)
    return fail(COLI_EINVAL, "%s: cycles=%lld outside [0, 4e9]", fn, (long long)cycles);
  wait_probe_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(static_cast<int32_t*>(workspace), (long long)cycles);
  CHECK_LAUNCH(cudaGetLastError());
  return COLI_OK;
}

COLI_EXPORT coli_status coli_quantize_rows_int4(const float* w, int64_t rows, int64_t cols, uint8_t* q_out,
                                                float* scale_out, void* stream) {
  const char* fn = "coli_quantize_rows_int4";
  if (rows < 0 || cols <= 0 || cols % 32 != 0)
    return fail(COLI_EINVAL, "%s: rows=%lld cols=%lld (cols must be a positive multiple of 32)", fn,
                (long long)rows, (long long)cols);
  if (rows == 0) return COLI_OK;
  CHECK_PTR(w);
  CHECK_PTR(q_out);
  CHECK_PTR(scale_out);
  CHECK_LAUNCH(launch_quantize_rows_int4(w, rows, cols, q_out, scale_out, (cudaStream_t)stream));
  return COLI_OK;
}

COLI_EXPORT coli_status coli_quantize_rows_int8(const float* w, int64_t rows, int64_t cols, int8_t* q_out,
                                                float* scale_out, void* stream) {
  const char* fn = "coli_quantize_rows_int8";
  if (rows < 0 || cols <= 0 || cols % 32 != 0)
    return fail(COLI_EINVAL, "%s: rows=%lld cols=%lld (cols must be a positive multiple of 32)", fn,
                (long long)rows, (long long)cols);
  if (rows == 0) return COLI_OK;
  CHECK_PTR(w);
  CHECK_PTR(q_out);
  CHECK_PTR(scale_out);
  CHECK_LAUNCH(launch_quantize_rows_int8(w, rows, cols, q_out, scale_out, (cudaStream_t)stream));
  return COLI_OK;
}

COLI_EXPORT coli_status coli_requantize_fp8_int4(const uint8_t* w8, const float* block_factors, int64_t rows,
                                                 int64_t cols, int32_t block, uint8_t* q_out, float* scale_out,
                                                 void* stream) {
  const char* fn = "coli_requantize_fp8_int4";
  if (rows < 0 || cols <= 0 || cols % 32 != 0 || rows > (int64_t(1) << 31))
    return fail(COLI_EINVAL, "%s: rows=%lld cols=%lld (cols must be a positive multiple of 32)", fn,
                (long long)rows, (long long)cols);
  if (block < 8 || block % 8 != 0)
    return fail(COLI_EINVAL, "%s: block=%d (must be a positive multiple of 8)", fn, (int)block);
  if (rows == 0) return COLI_OK;
  CHECK_PTR(w8);
  CHECK_PTR(block_factors);
  CHECK_PTR(q_out);
  CHECK_PTR(scale_out);
  CHECK_LAUNCH(launch_requantize_fp8_int4(w8, block_factors, rows, cols, block, q_out, scale_out,
                                          (cudaStream_t)stream));
  return COLI_OK;
}

COLI_EXPORT coli_status coli_quantize_act_q8(const float* x, int64_t n_tok, int64_t dim, int8_t* q_out,
                                             float* scale_out, void* stream) {
  const char* fn = "coli_quantize_act_q8";
  if (n_tok < 0 || dim <= 0 || dim % 32 != 0)
    return fail(COLI_EINVAL, "%s: n_tok=%lld dim=%lld (dim must be a positive multiple of 32)", fn,
                (long long)n_tok, (long long)dim);
  if (n_tok == 0) return COLI_OK;
  CHECK_PTR(x);
  CHECK_PTR(q_out);
  CHECK_PTR(scale_out);
  CHECK_LAUNCH(launch_quantize_act_q8(x, n_tok, dim, q_out, scale_out, (cudaStream_t)stream));
  return COLI_OK;
}

COLI_EXPORT coli_status coli_moe_route(const coli_moe_layer* layer, const float* x, int64_t n_tok, float* scores,
                                       int32_t* topk_idx, float* topk_w, void* stream) {
  const char* fn = "coli_moe_route";
  if (layer == nullptr) return fail(COLI_EINVAL, "%s: null layer", fn);
  coli_status s = check_cfg(&layer->cfg, fn);
  if (s != COLI_OK) return s;
  if (n_tok < 0 || n_tok > (1 << 24)) return fail(COLI_EINVAL, "%s: n_tok=%lld", fn, (long long)n_tok);
  if (n_tok == 0) return COLI_OK;
  CHECK_PTR(layer->w_router);
  CHECK_PTR(layer->bias);
  CHECK_PTR(x);
  CHECK_PTR(topk_idx);
  CHECK_PTR(topk_w);
  const coli_moe_config& c = layer->cfg;
  cudaStream_t st = (cudaStream_t)stream;
  if (scores == nullptr) {  // the scores stay on chip
    CHECK_LAUNCH(launch_route_topk(x, layer->w_router, layer->bias, (int)n_tok, c.n_experts, c.hidden, c.top_k,
                                   c.norm_topk_prob, c.routed_scaling_factor, topk_idx, topk_w, st));
    return COLI_OK;
  }
  CHECK_PTR(scores);
  CHECK_LAUNCH(launch_router_scores(x, layer->w_router, (int)n_tok, c.n_experts, c.hidden, scores, st));
  CHECK_LAUNCH(launch_topk(scores, layer->bias, (int)n_tok, c.n_experts, c.top_k, c.norm_topk_prob,
                           c.routed_scaling_factor, topk_idx, topk_w, st));
  return COLI_OK;
}

COLI_EXPORT coli_status coli_moe_bucket(const int32_t* topk_idx, int64_t n_tok, int32_t top_k, int32_t n_experts,
                                        int32_t* counts, int32_t* offsets, int32_t* perm, void* stream) {
  const char* fn = "coli_moe_bucket";
  if (n_experts < 1 || n_experts > kMaxExperts)
    return fail(COLI_EINVAL, "%s: n_experts=%d outside [1, %d]", fn, n_experts, kMaxExperts);
  if (top_k < 1 || top_k > n_experts) return fail(COLI_EINVAL, "%s: top_k=%d", fn, top_k);
  if (n_tok < 0 || n_tok * top_k > (1ll << 30)) return fail(COLI_EINVAL, "%s: n_tok=%lld", fn, (long long)n_tok);
  CHECK_PTR(counts);
  CHECK_PTR(offsets);
  if (n_tok > 0) {
    CHECK_PTR(topk_idx);
    CHECK_PTR(perm);
  }
  CHECK_LAUNCH(launch_bucket(topk_idx, (int)n_tok, top_k, n_experts, 0, counts, offsets, perm, nullptr, nullptr,
                             nullptr, nullptr, (cudaStream_t)stream));
  return COLI_OK;
}

COLI_EXPORT coli_status coli_moe_expert_ffn(const coli_moe_config* cfg, const coli_expert* expert, const int8_t* xq,
                                            const float* xs, int64_t n_tok, float* y_out, void* workspace,
                                            size_t ws_bytes, void* stream) {
  const char* fn = "coli_moe_expert_ffn";
  coli_status s = check_cfg(cfg, fn);
  if (s != COLI_OK) return s;
  if (bits_of(*cfg) != 4) return fail(COLI_EINVAL, "%s: int4 weights only (weight_bits 4)", fn);
  if (n_tok < 0 || n_tok > (1 << 24)) return fail(COLI_EINVAL, "%s: n_tok=%lld", fn, (long long)n_tok);
  if (n_tok == 0) return COLI_OK;
  if ((s = check_expert(expert, fn)) != COLI_OK) return s;
  CHECK_PTR(xq);
  CHECK_PTR(xs);
  CHECK_PTR(y_out);
  CHECK_PTR(workspace);
  const Workspace W = layout(*cfg, n_tok);
  if (ws_bytes < W.total)
    return fail(COLI_ENOMEM, "%s: workspace %zu bytes < %zu needed", fn, ws_bytes, W.total);
  static thread_local GateUpTable gu;
  static thread_local DownTable dn;
  gu.gate_q[0] = expert->gate_q;
  gu.gate_s[0] = expert->gate_s;
  gu.up_q[0] = expert->up_q;
  gu.up_s[0] = expert->up_s;
  dn.down_q[0] = expert->down_q;
  dn.down_s[0] = expert->down_s;
  GemvSlots sl{};
  sl.slots = nullptr;
  sl.one = Slot{0, 0, (int32_t)n_tok, -1};
  sl.max_slots = 1;
  sl.top_k = 1;
  int8_t* hq = at<int8_t>(workspace, W.hq);
  float* hd = at<float>(workspace, W.hd);
  cudaStream_t st = (cudaStream_t)stream;
  CHECK_LAUNCH(launch_gateup(gu, sl, xq, xs, cfg->hidden, cfg->inter, (int)n_tok, hq, hd, st));
  CHECK_LAUNCH(launch_down(dn, sl, hq, hd, cfg->hidden, cfg->inter, (int)n_tok, y_out, st));
  return COLI_OK;
}

COLI_EXPORT coli_status coli_moe_layer_forward(const coli_moe_layer* layer, const float* x, int64_t n_tok, float* out,
                                               void* workspace, size_t ws_bytes, void* stream) {
  const char* fn = "coli_moe_layer_forward";
  coli_status s = check_layer(layer, fn);
  if (s != COLI_OK) return s;
  if (n_tok < 0 || n_tok > (1 << 24)) return fail(COLI_EINVAL, "%s: n_tok=%lld", fn, (long long)n_tok);
  if (n_tok == 0) return COLI_OK;
  CHECK_PTR(x);
  CHECK_PTR(out);
  CHECK_PTR(workspace);
  if (x == out) return fail(COLI_EINVAL, "%s: x and out must not alias", fn);
  const Workspace W = layout(layer->cfg, n_tok);
  if (ws_bytes < W.total)
    return fail(COLI_ENOMEM, "%s: workspace %zu bytes < %zu needed", fn, ws_bytes, W.total);
  return layer_forward(layer, x, n_tok, out, workspace, W, (cudaStream_t)stream, fn, true);
}

COLI_EXPORT coli_status coli_moe_stack_forward(const coli_moe_layer* layers, int32_t n_layers, const float* x,
                                               int64_t n_tok, float eps, float* out, void* workspace, size_t ws_bytes,
                                               void* stream) {
  const char* fn = "coli_moe_stack_forward";
  if (layers == nullptr || n_layers < 1) return fail(COLI_EINVAL, "%s: no layers", fn);
  coli_status s;
  for (int l = 0; l < n_layers; ++l) {
    if ((s = check_layer(&layers[l], fn)) != COLI_OK) return s;
    if (memcmp(&layers[l].cfg, &layers[0].cfg, sizeof(coli_moe_config)) != 0)
      return fail(COLI_EINVAL, "%s: layer %d has a different cfg", fn, l);
  }
  if (n_tok < 0 || n_tok > (1 << 24)) return fail(COLI_EINVAL, "%s: n_tok=%lld", fn, (long long)n_tok);
  if (n_tok == 0) return COLI_OK;
  CHECK_PTR(x);
  CHECK_PTR(out);
  CHECK_PTR(workspace);
  const Workspace W = layout(layers[0].cfg, n_tok);
  if (ws_bytes < W.total)
    return fail(COLI_ENOMEM, "%s: workspace %zu bytes < %zu needed", fn, ws_bytes, W.total);
  cudaStream_t st = (cudaStream_t)stream;
  const int H = layers[0].cfg.hidden;
  float* xn = at<float>(workspace, W.xn);
  float* ping[2] = {at<float>(workspace, W.xa), at<float>(workspace, W.xb)};
  const float* cur = x;
  for (int l = 0; l < n_layers; ++l) {
    // ping[l % 2] never holds `cur` (which is x or ping[(l - 1) % 2])
    float* m = ping[l % 2];
    CHECK_LAUNCH(launch_rmsnorm(cur, (int)n_tok, H, eps, xn, st));
    if ((s = layer_forward(&layers[l], xn, n_tok, m, workspace, W, st, fn, l == 0)) != COLI_OK) return s;
    float* next = (l == n_layers - 1) ? out : m;  // m = cur + m in place, or the final output
    CHECK_LAUNCH(launch_residual_add(cur, m, n_tok * H, next, st));
    cur = next;
  }
  return COLI_OK;
}

COLI_EXPORT coli_status coli_rmsnorm(const float* x, int64_t n_tok, int64_t dim, float eps, float* y, void* stream) {
  const char* fn = "coli_rmsnorm";
  if (n_tok < 0 || dim <= 0 || dim % 128 != 0 || n_tok > (1 << 24))
    return fail(COLI_EINVAL, "%s: n_tok=%lld dim=%lld (dim must be a positive multiple of 128)", fn,
                (long long)n_tok, (long long)dim);
  if (n_tok == 0) return COLI_OK;
  CHECK_PTR(x);
  CHECK_PTR(y);
  CHECK_LAUNCH(launch_rmsnorm(x, (int)n_tok, (int)dim, eps, y, (cudaStream_t)stream));
  return COLI_OK;
}

COLI_EXPORT coli_status coli_debug_block_partials(const coli_expert* expert, int32_t which, const int8_t* xq,
                                                  int64_t n_tok, int64_t dim_in, int64_t rows, int32_t* isum_out,
                                                  void* stream) {
  const char* fn = "coli_debug_block_partials";
  if (expert == nullptr) return fail(COLI_EINVAL, "%s: null expert", fn);
  if (which < 0 || which > 2) return fail(COLI_EINVAL, "%s: which=%d", fn, which);
  if (n_tok < 0 || rows < 0 || dim_in <= 0 || dim_in % 32 != 0)
    return fail(COLI_EINVAL, "%s: bad shape", fn);
  if (n_tok == 0 || rows == 0) return COLI_OK;
  const uint8_t* wq = which == 0 ? expert->gate_q : (which == 1 ? expert->up_q : expert->down_q);
  CHECK_PTR(wq);
  CHECK_PTR(xq);
  CHECK_PTR(isum_out);
  CHECK_LAUNCH(launch_debug_partials(wq, xq, (int)n_tok, (int)dim_in, (int)rows, isum_out, (cudaStream_t)stream));
  return COLI_OK;
}
