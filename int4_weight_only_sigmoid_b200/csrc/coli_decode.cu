// coli_decode.cu -- the expert kernels of a decode batch (n_tok <= 16),
// launched with programmatic dependent launch so the routing, the gate/up
// sweep and the down sweep overlap at their boundaries:
//
//   router_decode (plain launch)  ->  topk_bucket_small (PDL)
//     -> gateup_decode (PDL): the shared experts' CTAs do not depend on the
//        routing and start streaming at once; the routed CTAs wait for it
//     -> down_combine (PDL): down projection of every slot for 16 output
//        rows per CTA, then the weighted combine of those rows, written
//        straight to `out` (no y buffer, no combine kernel).
//
// The integer and float arithmetic is the same as coli_gemv.cu's (dp4a block
// sums, contract F fold, SwiGLU, Q8_0 of h, contract C combine), so the
// output is bit-identical to the general path.
//
// Sources: "Colibri：在笔记本上跑744B参数的AI模型", "关键特性" (integer dot
// kernels, Q8_0 activations); "GLM-5.2-colibri-int4架构解析…", "MoE的工作原理"
// (weighted combine), "GLM-5.2的MoE实现" (shared expert); HN summary,
// "已实现的功能" (batched MoE).
#include "coli_gemv.cuh"

namespace coli {
namespace {

using namespace gemv;

__device__ __forceinline__ Slot shared_slot(int s, int n_tok, int K, int E) {
  return Slot{E + s, n_tok * K + s * n_tok, n_tok, -1};
}

// Stage n_valid F32 token rows as Q8_0 (the same arithmetic as
// quantize_act_q8_kernel: d = absmax/127, q = rint(x/d) in [-127,127]) into
// even/odd byte planes + block scales.
template <typename TokFn>
__device__ __forceinline__ void stage_quantize_f32(const float* __restrict__ x, int dim, int n_valid, TokFn tok,
                                                   uint4* xe_s, uint4* xo_s, float* xd_s) {
  const int nb = dim / 32;
  for (int i = threadIdx.x; i < n_valid * nb; i += kThreads) {
    const int t = i / nb, b = i - t * nb;
    const float4* src = reinterpret_cast<const float4*>(x + (int64_t)tok(t) * dim + 32 * b);
    float v[32];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float4 f = __ldg(src + j);
      v[4 * j] = f.x;
      v[4 * j + 1] = f.y;
      v[4 * j + 2] = f.z;
      v[4 * j + 3] = f.w;
    }
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 32; ++j) amax = fmaxf(amax, fabsf(v[j]));
    const float d = __fdiv_rn(amax, 127.0f);
    uint32_t w[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      uint32_t word = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) word |= ((uint32_t)q8_of(v[4 * k + j], d) & 0xFFu) << (8 * j);
      w[k] = word;
    }
    uint4 e, o;
    split_even_odd(w[0], w[1], e.x, o.x);
    split_even_odd(w[2], w[3], e.y, o.y);
    split_even_odd(w[4], w[5], e.z, o.z);
    split_even_odd(w[6], w[7], e.w, o.w);
    xe_s[t * nb + b] = e;
    xo_s[t * nb + b] = o;
    xd_s[t * nb + b] = d;
  }
}

// Gate/up + SwiGLU + Q8_0 of h.  CTA = (32 intermediate outputs, slot);
// blockIdx.y < n_shared: shared expert blockIdx.y, else routed slot
// blockIdx.y - n_shared of the table (after the routing is complete).
template <int TT>
__global__ void __launch_bounds__(kThreads) gateup_decode_kernel(
    const __grid_constant__ GateUpTable tbl, const Slot* __restrict__ slots, const int32_t* __restrict__ n_slots,
    const int32_t* __restrict__ perm, int n_tok, int K, int E, int n_shared, const float* __restrict__ x, int hidden,
    int inter, int8_t* __restrict__ hq, float* __restrict__ hd) {
  Slot slot;
  if ((int)blockIdx.y < n_shared) {
    pdl_launch_dependents();
    slot = shared_slot(blockIdx.y, n_tok, K, E);
  } else {
    pdl_wait();
    pdl_launch_dependents();
    const int r = blockIdx.y - n_shared;
    if (r >= *n_slots) return;
    slot = slots[r];
  }
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
  const int o_lane = o0 + 8 * warp + (cr & 7);
  const float s_lane = cr < 8 ? tbl.gate_s[ti][o_lane] : tbl.up_s[ti][o_lane];
  int32_t* Sw = S + warp * TT * kRows * kSPad;

  for (int g0 = 0; g0 < slot.count; g0 += TT) {
    const int n_valid = min(TT, slot.count - g0);
    stage_quantize_f32(x, hidden, n_valid,
                       [&](int t) { return slot.perm_base < 0 ? g0 + t : perm[slot.perm_base + g0 + t] / K; }, xe_s,
                       xo_s, xd_s);
    __syncthreads();
    float facc[(TT + 1) / 2];
    warp_rows_fold<TT>(row_ptr, nb, n_valid, xe_s, xo_s, xd_s, Sw, facc);
#pragma unroll
    for (int m = 0; m < (TT + 1) / 2; ++m) {
      const int t = ct + 2 * m;
      const float val = __fmul_rn(s_lane, facc[m]);
      const float u = __shfl_down_sync(0xffffffffu, val, 8);
      if (cr < 8 && t < n_valid && t < TT) Hs[t * 32 + 8 * warp + cr] = __fmul_rn(__fmul_rn(val, sigmoid_cw(val)), u);
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

// Stage n_valid Q8 rows of h into one warp's even/odd planes (lane-strided).
__device__ __forceinline__ void stage_rows_warp(const int8_t* __restrict__ aq, const float* __restrict__ ad, int dim_in,
                                                int64_t row0, int n_valid, uint4* xe_s, uint4* xo_s, float* xd_s) {
  const int nb = dim_in / 32;
  const int lane = threadIdx.x & 31;
  for (int i = lane; i < n_valid * nb; i += 32) {
    const int t = i / nb, b = i - t * nb;
    const int64_t row = row0 + t;
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

template <int TT>
struct DownCombineSmem {
  __host__ __device__ static size_t warp_bytes(int inter) {  // rounded up to 16 B so every warp region stays uint4-aligned
    const int nb = inter / 32;
    return ((size_t)TT * nb * (16 + 16 + 4) + (size_t)TT * kRows * kSPad * 4 + 15) & ~size_t(15);
  }
  __host__ __device__ static size_t bytes(int inter, int n_tok, int K, int n_shared) {
    return kWarps * warp_bytes(inter) + (size_t)(n_tok * K + n_tok * n_shared) * kRows * 4;
  }
};

// Down projection + combine.  CTA = 16 output rows [o0, o0+16) of every slot;
// warp w takes slots w, w+4, ... (shared experts first).  The y values of
// the CTA's rows land in shared memory by their buffer row (perm position,
// or n_tok*K + s*n_tok + t for shared expert s); then each (token, row) is
// combined in rank order (contract C) and written to out.
template <int TT>
__global__ void __launch_bounds__(kThreads) down_combine_kernel(
    const __grid_constant__ DownTable tbl, const Slot* __restrict__ slots, const int32_t* __restrict__ n_slots,
    int n_tok, int K, int E, int n_shared, const int8_t* __restrict__ hq, const float* __restrict__ hd,
    const int32_t* __restrict__ inv, const float* __restrict__ w, int hidden, int inter, float* __restrict__ out) {
  extern __shared__ __align__(16) unsigned char smem[];
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cr = lane & 15, ct = lane >> 4;
  const int o0 = blockIdx.x * kRows;
  const int nb = inter / 32;
  unsigned char* wbase = smem + warp * DownCombineSmem<TT>::warp_bytes(inter);
  uint4* xe_s = reinterpret_cast<uint4*>(wbase);
  uint4* xo_s = xe_s + TT * nb;
  float* xd_s = reinterpret_cast<float*>(xo_s + TT * nb);
  int32_t* Sw = reinterpret_cast<int32_t*>(xd_s + TT * nb);
  float* ys = reinterpret_cast<float*>(smem + kWarps * DownCombineSmem<TT>::warp_bytes(inter));
  const size_t rb = (size_t)inter / 2;
  const int n_total = n_shared + *n_slots;

  for (int si = warp; si < n_total; si += kWarps) {
    const Slot slot = si < n_shared ? shared_slot(si, n_tok, K, E) : slots[si - n_shared];
    const int ti = slot.table_idx;
    const uint8_t* dq = tbl.down_q[ti] + (size_t)o0 * rb;
    auto row_ptr = [&](int r) -> const uint8_t* { return dq + r * rb; };
    const float s_lane = tbl.down_s[ti][o0 + cr];
    for (int g0 = 0; g0 < slot.count; g0 += TT) {
      const int n_valid = min(TT, slot.count - g0);
      stage_rows_warp(hq, hd, inter, (int64_t)slot.row_base + g0, n_valid, xe_s, xo_s, xd_s);
      __syncwarp();
      float facc[(TT + 1) / 2];
      warp_rows_fold<TT>(row_ptr, nb, n_valid, xe_s, xo_s, xd_s, Sw, facc);
#pragma unroll
      for (int m = 0; m < (TT + 1) / 2; ++m) {
        const int t = ct + 2 * m;
        if (t < n_valid && t < TT) ys[(slot.row_base + g0 + t) * kRows + cr] = __fmul_rn(s_lane, facc[m]);
      }
      __syncwarp();
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < n_tok * kRows; i += kThreads) {
    const int t = i / kRows, r = i - t * kRows;
    float acc = 0.0f;
    for (int k = 0; k < K; ++k) acc = __fmaf_rn(w[t * K + k], ys[inv[t * K + k] * kRows + r], acc);
    for (int s = 0; s < n_shared; ++s) acc = __fadd_rn(acc, ys[(n_tok * K + s * n_tok + t) * kRows + r]);
    out[(int64_t)t * hidden + o0 + r] = acc;
  }
}

template <typename KernelT>
cudaError_t allow_smem(KernelT* k, int& mask) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (mask & (1 << (dev & 31))) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
  if (e == cudaSuccess) mask |= 1 << (dev & 31);
  return e;
}

template <int TT>
cudaError_t gateup_decode_tt(const GateUpTable& tbl, const Slot* slots, const int32_t* n_slots, const int32_t* perm,
                             int n_tok, int K, int E, int n_shared, const float* x, int hidden, int inter, int8_t* hq,
                             float* hd, cudaStream_t st) {
  static int mask = 0;
  cudaError_t e = allow_smem(gateup_decode_kernel<TT>, mask);
  if (e != cudaSuccess) return e;
  const int max_routed = n_tok * K < E ? n_tok * K : E;
  return launch_pdl(gateup_decode_kernel<TT>, dim3(inter / 32, n_shared + max_routed), dim3(kThreads),
                    GemvSmem<TT>::bytes(hidden), st, true, tbl, slots, n_slots, perm, n_tok, K, E, n_shared, x,
                    hidden, inter, hq, hd);
}

template <int TT>
cudaError_t down_combine_tt(const DownTable& tbl, const Slot* slots, const int32_t* n_slots, int n_tok, int K, int E,
                            int n_shared, const int8_t* hq, const float* hd, const int32_t* inv, const float* w,
                            int hidden, int inter, float* out, cudaStream_t st) {
  static int mask = 0;
  cudaError_t e = allow_smem(down_combine_kernel<TT>, mask);
  if (e != cudaSuccess) return e;
  return launch_pdl(down_combine_kernel<TT>, dim3(hidden / kRows), dim3(kThreads),
                    DownCombineSmem<TT>::bytes(inter, n_tok, K, n_shared), st, true, tbl, slots, n_slots, n_tok, K,
                    E, n_shared, hq, hd, inv, w, hidden, inter, out);
}

}  // namespace

cudaError_t launch_gateup_decode(const GateUpTable& tbl, const Slot* slots, const int32_t* n_slots,
                                 const int32_t* perm, int n_tok, int K, int E, int n_shared, const float* x,
                                 int hidden, int inter, int8_t* hq, float* hd, cudaStream_t st) {
  if (n_tok <= 1)
    return gateup_decode_tt<1>(tbl, slots, n_slots, perm, n_tok, K, E, n_shared, x, hidden, inter, hq, hd, st);
  if (n_tok <= 2)
    return gateup_decode_tt<2>(tbl, slots, n_slots, perm, n_tok, K, E, n_shared, x, hidden, inter, hq, hd, st);
  return gateup_decode_tt<4>(tbl, slots, n_slots, perm, n_tok, K, E, n_shared, x, hidden, inter, hq, hd, st);
}

cudaError_t launch_down_combine(const DownTable& tbl, const Slot* slots, const int32_t* n_slots, int n_tok, int K,
                                int E, int n_shared, const int8_t* hq, const float* hd, const int32_t* inv,
                                const float* w, int hidden, int inter, float* out, cudaStream_t st) {
  if (n_tok <= 1)
    return down_combine_tt<1>(tbl, slots, n_slots, n_tok, K, E, n_shared, hq, hd, inv, w, hidden, inter, out, st);
  if (n_tok <= 2)
    return down_combine_tt<2>(tbl, slots, n_slots, n_tok, K, E, n_shared, hq, hd, inv, w, hidden, inter, out, st);
  return down_combine_tt<4>(tbl, slots, n_slots, n_tok, K, E, n_shared, hq, hd, inv, w, hidden, inter, out, st);
}

}  // namespace coli
