// coli_launch.h -- kernel launchers of libcoli (private to the library).
#pragma once

#include <cstdint>
#include <utility>

#include <cuda_runtime.h>

#include "coli_device.cuh"
#include "coli_expert_stream.cuh"

namespace coli {

// Largest batch that takes the decode path (router_decode, topk_bucket_small,
// gate/up, down, combine in coli_decode.cu).
constexpr int kDecodeMaxTok = 16;

// Launch with programmatic stream serialisation (PDL) when `pdl` is set: the
// kernel may start while its predecessor is still running and must call
// pdl_wait() before it reads anything the predecessor writes.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Raise a kernel's dynamic shared-memory opt-in on the current device to
// `bytes` when the last setting there is lower (the attribute belongs to the
// device's context; `granted` is the caller's per-kernel record for devices
// 0..63).  The opt-in plus the kernel's static shared memory must stay
// within the device's per-block limit, so ask for what the launch needs.
template <typename KernelT>
cudaError_t smem_opt_in(KernelT* kernel, int bytes, int (&granted)[64]) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (granted[dev] >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) granted[dev] = bytes;
  return e;
}

// Quantisers
cudaError_t launch_quantize_rows_int4(const float* w, int64_t rows, int64_t cols, uint8_t* q,
                                      float* s, cudaStream_t st);
// FP8 (e4m3 codes, [rows x cols]) with one F32 factor per block x block tile
// -> packed int4 rows + F32 row scales.  cols % 32 == 0, block % 8 == 0.
cudaError_t launch_requantize_fp8_int4(const uint8_t* w8, const float* factors, int64_t rows, int64_t cols,
                                       int block, uint8_t* q, float* s, cudaStream_t st);
cudaError_t launch_quantize_act_q8(const float* x, int64_t n_tok, int64_t dim, int8_t* q, float* d,
                                   cudaStream_t st);
cudaError_t launch_quantize_rows_int8(const float* w, int64_t rows, int64_t cols, int8_t* q, float* s,
                                      cudaStream_t st);

// Router: scores[t,e] = sigmoid(logit) (contract R), then top-k + weights.
cudaError_t launch_router_scores(const float* x, const float* w_router, int n_tok, int E, int H,
                                 float* scores, cudaStream_t st);
cudaError_t launch_topk(const float* scores, const float* bias, int n_tok, int E, int K, int norm,
                        float rsf, int32_t* idx, float* w, cudaStream_t st);
// Scores and top-k in one kernel (one CTA per token, scores only in shared
// memory): the same idx and w as launch_router_scores + launch_topk.
cudaError_t launch_route_topk(const float* x, const float* w_router, const float* bias, int n_tok, int E, int H, int K,
                              int norm, float rsf, int32_t* idx, float* w, cudaStream_t st);

// Decode batches: router scores with the router rows staged in shared memory
// (plain launch), then top-k + weights + bucketing in one CTA (PDL launch).
// The router kernel also clears n_zero words at `zero` (the streaming
// kernel's counters; may be null).
cudaError_t launch_router_decode(const float* x, const float* w_router, int n_tok, int E, int H, float* scores,
                                 int8_t* xq, float* xd, int32_t* status_clear, int32_t* zero, int n_zero,
                                 cudaStream_t st, int8_t* xpl = nullptr, float2* xdc = nullptr);
cudaError_t launch_topk_bucket_small(const float* scores, const float* bias, int n_tok, int E, int K, int norm,
                                     float rsf, int32_t* idx, float* w, int32_t* counts, int32_t* offsets,
                                     int32_t* perm, int32_t* inv, Slot* slots, int32_t* n_slots, cudaStream_t st);

// Bucketing: counts, offsets, perm; optionally the inverse map (pair ->
// position), the expert slot table (+ shared slots) and its length.
cudaError_t launch_bucket(const int32_t* idx, int n_tok, int K, int E, int n_shared, int32_t* counts,
                          int32_t* offsets, int32_t* perm, int32_t* inv, Slot* slots,
                          int32_t* n_slots, int32_t* status, cudaStream_t st);

// Expert GEMVs over the slot table (slots == nullptr: the single slot `one`).
struct GemvSlots {
  const Slot* slots;      // device table, or nullptr
  const int32_t* n_slots; // device count (when slots != nullptr)
  Slot one;               // used when slots == nullptr
  int max_slots;          // grid.y
  const int32_t* perm;    // token ids of routed slots
  int top_k;
};
cudaError_t launch_gateup(const GateUpTable& tbl, const GemvSlots& sl, const int8_t* xq,
                          const float* xd, int hidden, int inter, int max_tok_per_slot, int8_t* hq,
                          float* hd, cudaStream_t st);
cudaError_t launch_down(const DownTable& tbl, const GemvSlots& sl, const int8_t* hq, const float* hd,
                        int hidden, int inter, int max_tok_per_slot, float* y, cudaStream_t st);

// Decode expert kernels (persistent, PDL launches).  Slot table = the routed
// experts only; shared expert s is implicit (rows n_tok*K + s*n_tok ..).
// gate/up quantises the F32 x itself for the shared experts (which start
// before the routing is done) and reads the router kernel's Q8 of x for the
// routed ones, and writes h as plane rows (per 32-block: 16 even elements,
// then 16 odd); down writes y and a combine kernel reduces it into `out`.
// Needs decode_supported(hidden, inter).
bool decode_supported(int hidden, int inter);
cudaError_t launch_gateup_decode(const GateUpTable& tbl, const Slot* slots, const int32_t* n_slots,
                                 const int32_t* perm, int n_tok, int K, int E, int n_shared, const float* x,
                                 const int8_t* xq, const float* xd, int hidden, int inter, int8_t* hq, float* hd,
                                 int32_t* status, cudaStream_t st);
cudaError_t launch_down_decode(const DownTable& tbl, const Slot* slots, const int32_t* n_slots, int n_tok, int K,
                               int E, int n_shared, const int8_t* hq, const float* hd, const int32_t* inv,
                               const float* w, int hidden, int inter, float* y, float* out, int32_t* status,
                               cudaStream_t st);

// Decode batches of <= kStreamMaxTok tokens on a prepared layer: one
// persistent kernel (PDL launch after router_decode) that routes the batch
// in every CTA, streams the layer's streaming copy stage by stage (gate/up,
// SwiGLU, Q8_0 of h; down; combine) and writes `out`.  Every expert the
// batch chose is read once; an expert with more than kStreamSlotTok of the
// batch's tokens (the shared experts of a batch above that size) is several
// slots over the same weights.
constexpr int kStreamMaxTok = 16;  // tokens of one streaming kernel launch
constexpr int kStreamSlotTok = 8;  // tokens of one slot
constexpr int kStreamMaxSlots =
    ((kStreamMaxTok + kStreamSlotTok - 1) / kStreamSlotTok) * kMaxShared + kStreamMaxTok * kMaxTopK;
struct StreamArgs {
  const unsigned char* prep;  // the layer's streaming copy (coli_moe_prepare)
  StreamGeom g;
  int E, K, S, T, norm;
  float rsf;
  const float* scores;  // [T x E] (router_decode)
  const float* bias;
  const float* x;       // [T x H] the layer input
  const int8_t* xpl_g;  // null (the kernel quantises x itself), or [T x H/32 x 32] planes of Q8(x) (router_decode)
  const float2* xdc_g;  // [T x H/32] (d, -128 * sum of the even plane) with xpl_g
  int8_t* hpl;          // [rows x I/32 x 32]: h of every (slot, token) row as even / odd byte planes
  float2* hdc;          // [rows x I/32]: (d, -128 * sum of the even plane as int bits)
  float* out;           // [T x H]
  int32_t* h_ready;     // [kStreamMaxSlots] gate/up units done per slot (zero at launch)
  int32_t* status;
  int32_t* dbg;         // null, or the partials capture (coli_debug_capture_partials layout)
};
bool stream_supported(int hidden, int inter, int bits, int n_tok, int top_k, int n_shared, int n_experts);

uint64_t stream_expert_bytes(int hidden, int inter, int bits);
cudaError_t launch_prepare_expert(int hidden, int inter, int bits, const uint8_t* gq, const float* gs,
                                  const uint8_t* uq, const float* us, const uint8_t* dq, const float* ds, void* dst,
                                  cudaStream_t st);
cudaError_t launch_expert_stream(const StreamArgs& a, cudaStream_t st);

// Prefill expert kernels on the tensor cores (tcgen05.mma.kind::i8): the
// int8 operand rows of the Q8 activations, one per (slot, token) in slot
// order (xr: n_tok*(K+n_shared) x hidden bytes; with int4 weights per 8
// elements in the order 0,2,4,6,1,3,5,7), the tile list (<= 128 tokens of
// one slot per tile) built from the slot table, then the persistent gate/up
// GEMM (+ SwiGLU + Q8 of h, written as int8 rows hr: rows x inter, scales hd)
// and the persistent down GEMM (-> y).
// `tiles` needs prefill_tile_bytes().
bool prefill_supported(int hidden, int inter);
size_t prefill_tiles_bound(int n_tok, int K, int E, int n_shared);
size_t prefill_tile_bytes(int n_tok, int K, int E, int n_shared);
cudaError_t launch_prefill_experts(const GateUpTable& gu, const DownTable& dn, const Slot* slots,
                                   const int32_t* n_slots, void* tiles, int32_t* n_tiles, const int32_t* perm,
                                   int K, int n_shared, int bits, const int8_t* xq, const float* xd, int n_tok,
                                   int hidden, int inter, void* xr, void* hr, float* hd, float* y, int32_t* err,
                                   cudaStream_t st, cudaEvent_t ev_mid, int32_t* dbg_buf, int n_experts);

// out[t] = sum_k w[t,k] y[inv[t,k]] + sum_s y[n_tok*K + s*n_tok + t]  (contract C)
cudaError_t launch_combine(const float* y, const int32_t* inv, const float* w, int n_tok, int K,
                           int n_shared, int H, float* out, cudaStream_t st);

// RMSNorm (weight 1) and residual add for a pre-norm stack.
cudaError_t launch_rmsnorm(const float* x, int n_tok, int dim, float eps, float* y, cudaStream_t st);
cudaError_t launch_residual_add(const float* x, const float* m, int64_t n, float* out, cudaStream_t st);

// Test hook: per-block isums of rows x tokens.
cudaError_t launch_debug_partials(const uint8_t* wq, const int8_t* xq, int n_tok, int dim_in, int rows,
                                  int32_t* out, cudaStream_t st);

// Sets the message coli_last_error() returns on the calling thread.
void set_error_message(const char* msg);

// Device status word: the first 4 bytes of a workspace.  A forward call
// clears it when it starts; kernels record the first problem they meet.
//   0            no error
//   1 .. 9       a device-side check failed (COLI_EDEVICE):
//                1 = bucketing met an expert index outside [0, E)
//   10 .. 39     a bounded wait gave up (COLI_ETIMEOUT):
//                10 prefill producers (operand stage), 11 prefill MMA (operands),
//                12 prefill MMA (accumulators), 13 prefill fold (accumulators),
//                16 prefill TMA warp (operand stage), 22 decode down (h rows),
//                25 streaming kernel (a slot's h from other CTAs),
//                26 streaming kernel (staged h), 27 streaming kernel (its warp
//                pair's h buffer),
//                30 the test probe coli_debug_wait_probe
constexpr int32_t kStatusBadExpert = 1;
constexpr int32_t kStatusTimeoutFirst = 10;
constexpr int32_t kStatusWaitProbe = 30;

// Device address of the fixed scratch behind coli_moe_layer_forward_noalloc
// on the current device.
cudaError_t noalloc_scratch(void** out);

}  // namespace coli
