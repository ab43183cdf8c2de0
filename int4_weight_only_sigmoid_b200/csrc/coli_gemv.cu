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
#include "coli_launch.h"

namespace coli {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;
constexpr int kRows = 16;  // rows per warp
constexpr int kSPad = 33;  // padded row of the isum park: conflict-free fold reads

template <int TT>
struct GemvSmem {
  static size_t bytes(int dim_in) {
    const int nb = dim_in / 32;
    return (size_t)2 * TT * nb * 16        // even / odd activation planes
           + (size_t)TT * nb * 4           // block scales
           + (size_t)kWarps * TT * kRows * kSPad * 4  // isum park
           + (size_t)TT * 32 * 4;          // h tile (gate/up)
  }
};

__device__ __forceinline__ Slot load_slot(const GemvSlots& sl, int y, bool& live) {
  if (sl.slots == nullptr) {
    live = (y == 0);
    return sl.one;
  }
  live = y < *sl.n_slots;
  return live ? sl.slots[y] : Slot{0, 0, 0, -1};
}

__device__ __forceinline__ int token_of(const GemvSlots& sl, const Slot& s, int i) {
  return s.perm_base < 0 ? i : sl.perm[s.perm_base + i] / sl.top_k;
}

// Stage n_valid activation rows (Q8 bytes + block scales) into shared memory
// as even/odd byte planes.  act_row(i) gives the source row of token i.
template <int TT, typename RowFn>
__device__ __forceinline__ void stage_acts(const int8_t* __restrict__ aq, const float* __restrict__ ad, int dim_in,
                                           int n_valid, RowFn act_row, uint4* xe_s, uint4* xo_s, float* xd_s) {
  const int nb = dim_in / 32;
  for (int i = threadIdx.x; i < n_valid * nb; i += kThreads) {
    const int t = i / nb, b = i - t * nb;
    const int64_t row = act_row(t);
    const uint4* src = reinterpret_cast<const uint4*>(aq + row * dim_in + 32 * b);
    const uint4 a0 = src[0], a1 = src[1];
    uint4 e, o;
    split_even_odd(a0.x, a0.y, e.x, o.x);
    split_even_odd(a0.z, a0.w, e.y, o.y);
    split_even_odd(a1.x, a1.y, e.z, o.z);
    split_even_odd(a1.z, a1.w, e.w, o.w);
    xe_s[t * nb + b] = e;
    xo_s[t * nb + b] = o;
    xd_s[t * nb + b] = ad[row * nb + b];
  }
}

// The warp's 16 rows against n_valid staged tokens; facc[m] ends with the
// fold of chain (row = lane % 16, token = lane / 16 + 2m).
template <int TT, typename RowPtrFn>
__device__ __forceinline__ void warp_rows_fold(RowPtrFn row_ptr, int nb, int n_valid, const uint4* xe_s,
                                               const uint4* xo_s, const float* xd_s, int32_t* Sw,
                                               float (&facc)[(TT + 1) / 2]) {
  const int lane = threadIdx.x & 31;
  const int cr = lane & 15, ct = lane >> 4;
#pragma unroll
  for (int m = 0; m < (TT + 1) / 2; ++m) facc[m] = 0.0f;
  const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
  for (int s0 = 0; s0 < nb; s0 += 32) {
    const int b = s0 + lane;
    const bool valid = b < nb;
    uint4 wv[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) wv[r] = valid ? ldg_stream(row_ptr(r) + 16 * b) : zero;
#pragma unroll
    for (int t = 0; t < TT; ++t) {
      if (t < n_valid) {
        const uint4 xe = valid ? xe_s[t * nb + b] : zero;
        const uint4 xo = valid ? xo_s[t * nb + b] : zero;
#pragma unroll
        for (int r = 0; r < kRows; ++r) Sw[(t * kRows + r) * kSPad + lane] = block_isum(wv[r], xe, xo);
      }
    }
    __syncwarp();
    const int nsteps = min(32, nb - s0);
#pragma unroll
    for (int m = 0; m < (TT + 1) / 2; ++m) {
      const int t = ct + 2 * m;
      if (t < n_valid && t < TT) {
        const int32_t* srow = Sw + (t * kRows + cr) * kSPad;
        const float* dsrc = xd_s + t * nb + s0;
        float a = facc[m];
        for (int j = 0; j < nsteps; ++j) a = __fmaf_rn(dsrc[j], (float)srow[j], a);
        facc[m] = a;
      }
    }
    __syncwarp();
  }
}

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
  static int attr_dev_mask = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(attr_dev_mask & (1 << (dev & 31)))) {
    cudaError_t e = cudaFuncSetAttribute(gateup_kernel<TT>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (e != cudaSuccess) return e;
    attr_dev_mask |= 1 << (dev & 31);
  }
  dim3 grid(inter / 32, sl.max_slots);
  gateup_kernel<TT><<<grid, kThreads, smem, st>>>(tbl, sl, xq, xd, hidden, inter, hq, hd);
  return cudaGetLastError();
}

template <int TT>
cudaError_t down_tt(const DownTable& tbl, const GemvSlots& sl, const int8_t* hq, const float* hd, int hidden,
                    int inter, float* y, cudaStream_t st) {
  const size_t smem = GemvSmem<TT>::bytes(inter);
  static int attr_dev_mask = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(attr_dev_mask & (1 << (dev & 31)))) {
    cudaError_t e = cudaFuncSetAttribute(down_kernel<TT>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (e != cudaSuccess) return e;
    attr_dev_mask |= 1 << (dev & 31);
  }
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
