// coli_launch.h -- kernel launchers of libcoli (private to the library).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "coli_device.cuh"

namespace coli {

// Quantisers
cudaError_t launch_quantize_rows_int4(const float* w, int64_t rows, int64_t cols, uint8_t* q,
                                      float* s, cudaStream_t st);
cudaError_t launch_quantize_act_q8(const float* x, int64_t n_tok, int64_t dim, int8_t* q, float* d,
                                   cudaStream_t st);

// Router: scores[t,e] = sigmoid(logit) (contract R), then top-k + weights.
cudaError_t launch_router_scores(const float* x, const float* w_router, int n_tok, int E, int H,
                                 float* scores, cudaStream_t st);
cudaError_t launch_topk(const float* scores, const float* bias, int n_tok, int E, int K, int norm,
                        float rsf, int32_t* idx, float* w, cudaStream_t st);

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

}  // namespace coli
