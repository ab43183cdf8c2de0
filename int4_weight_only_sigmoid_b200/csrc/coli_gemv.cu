// coli_gemv.cu -- the expert kernels for few tokens per expert (decode):
// int4 x Q8 block dots (dp4a), the row fold (contract F), SwiGLU + Q8_0 of
// the intermediate, the down projection, and the combine (contract C).
//
// Sources: "Colibri：在笔记本上跑744B参数的AI模型", "关键特性" (integer dot
// kernels, Q8_0 int8 activations, packed int4); "GLM-5.2-colibri-int4架构
// 解析…", "MoE的工作原理" (weighted combine) and "GLM-5.2的MoE实现" (shared
// expert); HN summary, "已实现的功能" (batched MoE: each selected expert's
// weights are streamed once for all of its tokens).
//
// Layout of the work: a CTA owns one expert slot and a tile of weight rows;
// each of its 4 warps owns 16 rows.  Per step a warp reads 32 consecutive
// 16-byte blocks (512 B, coalesced) of each of its rows with streaming loads;
// lane l computes the integer partial sum of block 32s+l for every row and
// token and parks it in shared memory; then lane c folds chain (row c%16,
// token c/16 [+2m]) over the 32 blocks in ascending order.  Integer work is
// spread over all lanes; the float fold stays sequential per output as
// contract F requires.
#include "coli_gemv.cuh"

namespace coli {
namespace {

using namespace gemv;

// Gate/up + SwiGLU + Q8_0 of h.  CTA = (32 intermediate outputs, slot).
// Warp w owns outputs o0+8w .. o0+8w+7: rows 0..7 are their gate rows,
// rows 8..15 their up rows.
template <int TT>
__global__ void __launch_bounds__(kThreads) gateup_kernel(const __grid_constant__ GateUpTable tbl,
                                                          const __grid_constant__ GemvSlots sl,
                                                          const int8_t* __restrict__ xq,
                                                          const float* __restrict__ xd, int hidden, int inter,
                                                          int8_t* __restrict__ hq, float* __restrict__ hd) {
  bool live;
  const Slot slot = load_slot(sl, blockIdx.y, live);
  if (!live) return;
  extern __shared__ __align__(16) unsigned char smem[];
  const int nb = hidden / 32;
  uint4* xe_s = reinterpret_cast<uint4*>(smem);
  uint4* xo_s = xe_s + TT * nb;
  float* xd_s = reinterpret_cast<float*>(xo_s + TT * nb);
  int32_t* S = reinterpret_cast<int32_t*>(xd_s + TT * nb);
  float* Hs = reinterpret_cast<float*>(S + kWarps * TT * kRows * kSPad);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cr = lane & 15, ct = lane >> 4;
  const int o0 = blockIdx.x * 32;
  const int ti = slot.table_idx;
  const size_t rb = (size_t)hidden / 2;
  const uint8_t* gq = tbl.gate_q[ti] + (size_t)(o0 + 8 * warp) * rb;
  const uint8_t* uq = tbl.up_q[ti] + (size_t)(o0 + 8 * warp) * rb;
  auto row_ptr = [&](int r) -> const uint8_t* { return r < 8 ? gq + r * rb : uq + (r - 8) * rb; };
  // this lane's output row for the fold result (gate rows 0..7 / up rows 8..15)
  const int o_lane = o0 + 8 * warp + (cr & 7);
  const float s_lane = cr < 8 ? tbl.gate_s[ti][o_lane] : tbl.up_s[ti][o_lane];
  int32_t* Sw = S + warp * TT * kRows * kSPad;

  for (int g0 = 0; g0 < slot.count; g0 += TT) {
    const int n_valid = min(TT, slot.count - g0);
    stage_acts<TT>(xq, xd, hidden, n_valid, [&](int t) { return (int64_t)token_of(sl, slot, g0 + t); }, xe_s,
                   xo_s, xd_s);
    __syncthreads();
    float facc[(TT + 1) / 2];
    warp_rows_fold<TT>(row_ptr, nb, n_valid, xe_s, xo_s, xd_s, Sw, facc);
#pragma unroll
    for (int m = 0; m < (TT + 1) / 2; ++m) {
      const int t = ct + 2 * m;
      const float val = __fmul_rn(s_lane, facc[m]);
      const float u = __shfl_down_sync(0xffffffffu, val, 8);
      if (cr < 8 && t < n_valid && t < TT) {
        const float g = val;
        Hs[t * 32 + 8 * warp + cr] = __fmul_rn(__fmul_rn(g, sigmoid_cw(g)), u);
      }
    }
    __syncthreads();
    for (int t = warp; t < n_valid; t += kWarps) {
      const float v = Hs[t * 32 + lane];
      const float d = __fdiv_rn(warp_max(fabsf(v)), 127.0f);
      const int64_t row = slot.row_base + g0 + t;
      hq[row * inter + o0 + lane] = (int8_t)q8_of(v, d);
      if (lane == 0) hd[row * (inter / 32) + (o0 / 32)] = d;
    }
    __syncthreads();
  }
}

// Down projection.  CTA = (64 output rows, slot); warp w owns rows
// o0+16w .. o0+16w+15.
template <int TT>
__global__ void __launch_bounds__(kThreads) down_kernel(const __grid_constant__ DownTable tbl,
                                                        const __grid_constant__ GemvSlots sl,
                                                        const int8_t* __restrict__ hq, const float* __restrict__ hd,
                                                        int hidden, int inter, float* __restrict__ y) {
  bool live;
  const Slot slot = load_slot(sl, blockIdx.y, live);
  if (!live) return;
  extern __shared__ __align__(16) unsigned char smem[];
  const int nb = inter / 32;
  uint4* xe_s = reinterpret_cast<uint4*>(smem);
  uint4* xo_s = xe_s + TT * nb;
  float* xd_s = reinterpret_cast<float*>(xo_s + TT * nb);
  int32_t* S = reinterpret_cast<int32_t*>(xd_s + TT * nb);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cr = lane & 15, ct = lane >> 4;
  const int o0 = blockIdx.x * 64 + 16 * warp;
  const int ti = slot.table_idx;
  const size_t rb = (size_t)inter / 2;
  const uint8_t* dq = tbl.down_q[ti] + (size_t)o0 * rb;
  auto row_ptr = [&](int r) -> const uint8_t* { return dq + r * rb; };
  const float s_lane = tbl.down_s[ti][o0 + cr];
  int32_t* Sw = S + warp * TT * kRows * kSPad;

  for (int g0 = 0; g0 < slot.count; g0 += TT) {
    const int n_valid = min(TT, slot.count - g0);
    stage_acts<TT>(hq, hd, inter, n_valid, [&](int t) { return (int64_t)slot.row_base + g0 + t; }, xe_s, xo_s,
                   xd_s);
    __syncthreads();
    float facc[(TT + 1) / 2];
    warp_rows_fold<TT>(row_ptr, nb, n_valid, xe_s, xo_s, xd_s, Sw, facc);
#pragma unroll
    for (int m = 0; m < (TT + 1) / 2; ++m) {
      const int t = ct + 2 * m;
      if (t < n_valid && t < TT) {
        const int64_t row = slot.row_base + g0 + t;
        y[row * hidden + o0 + cr] = __fmul_rn(s_lane, facc[m]);
      }
    }
    __syncthreads();
  }
}

// out[t, o] = (sum_k fmaf(w[t,k], y[inv[t,k], o])) + y_shared_0[t, o] + ...
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ y, const int32_t* __restrict__ inv,
                                                      const float* __restrict__ w, int n_tok, int K, int n_shared,
                                                      int H, float* __restrict__ out) {
  const int t = blockIdx.y;
  const int o = blockIdx.x * blockDim.x + threadIdx.x;
  if (o >= H) return;
  float acc = 0.0f;
  for (int k = 0; k < K; ++k) {
    const int64_t j = inv[(int64_t)t * K + k];
    acc = __fmaf_rn(w[(int64_t)t * K + k], y[j * H + o], acc);
  }
  for (int s = 0; s < n_shared; ++s) acc = __fadd_rn(acc, y[((int64_t)n_tok * K + (int64_t)s * n_tok + t) * H + o]);
  out[(int64_t)t * H + o] = acc;
}

template <int TT>
cudaError_t gateup_tt(const GateUpTable& tbl, const GemvSlots& sl, const int8_t* xq, const float* xd, int hidden,
                      int inter, int8_t* hq, float* hd, cudaStream_t st) {
  const size_t smem = GemvSmem<TT>::bytes(hidden);
  static int granted[64] = {};
  const cudaError_t e = smem_opt_in(gateup_kernel<TT>, 200 * 1024, granted);
  if (e != cudaSuccess) return e;
  dim3 grid(inter / 32, sl.max_slots);
  gateup_kernel<TT><<<grid, kThreads, smem, st>>>(tbl, sl, xq, xd, hidden, inter, hq, hd);
  return cudaGetLastError();
}

template <int TT>
cudaError_t down_tt(const DownTable& tbl, const GemvSlots& sl, const int8_t* hq, const float* hd, int hidden,
                    int inter, float* y, cudaStream_t st) {
  const size_t smem = GemvSmem<TT>::bytes(inter);
  static int granted[64] = {};
  const cudaError_t e = smem_opt_in(down_kernel<TT>, 200 * 1024, granted);
  if (e != cudaSuccess) return e;
  dim3 grid(hidden / 64, sl.max_slots);
  down_kernel<TT><<<grid, kThreads, smem, st>>>(tbl, sl, hq, hd, hidden, inter, y);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gateup(const GateUpTable& tbl, const GemvSlots& sl, const int8_t* xq, const float* xd, int hidden,
                          int inter, int max_tok_per_slot, int8_t* hq, float* hd, cudaStream_t st) {
  if (max_tok_per_slot <= 1) return gateup_tt<1>(tbl, sl, xq, xd, hidden, inter, hq, hd, st);
  if (max_tok_per_slot <= 2) return gateup_tt<2>(tbl, sl, xq, xd, hidden, inter, hq, hd, st);
  return gateup_tt<4>(tbl, sl, xq, xd, hidden, inter, hq, hd, st);
}

cudaError_t launch_down(const DownTable& tbl, const GemvSlots& sl, const int8_t* hq, const float* hd, int hidden,
                        int inter, int max_tok_per_slot, float* y, cudaStream_t st) {
  if (max_tok_per_slot <= 1) return down_tt<1>(tbl, sl, hq, hd, hidden, inter, y, st);
  if (max_tok_per_slot <= 2) return down_tt<2>(tbl, sl, hq, hd, hidden, inter, y, st);
  return down_tt<4>(tbl, sl, hq, hd, hidden, inter, y, st);
}

cudaError_t launch_combine(const float* y, const int32_t* inv, const float* w, int n_tok, int K, int n_shared, int H,
                           float* out, cudaStream_t st) {
  dim3 grid((H + 255) / 256, n_tok);
  combine_kernel<<<grid, 256, 0, st>>>(y, inv, w, n_tok, K, n_shared, H, out);
  return cudaGetLastError();
}

}  // namespace coli
