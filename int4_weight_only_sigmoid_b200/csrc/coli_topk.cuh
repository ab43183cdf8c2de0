// coli_topk.cuh -- warp-level pieces of the top-k selection and of the
// bucketing scans (coli_route.cu).
//
// Sources: "GLM-5.2-colibri-int4架构解析…" (wmrh.cn), "MoE的工作原理" and
// "路由策略定制" (top-k of the router scores, norm_topk_prob,
// routed_scaling_factor); "Colibri：在笔记本上跑744B参数的AI模型", "关键特性"
// (DeepSeek-V3 style sigmoid router: the correction bias steers the choice,
// the weights come from the unbiased scores).
#pragma once

#include <climits>

#include "coli_device.cuh"

namespace coli {
namespace topk {

// Exclusive scan of v[0..n) in place by one warp; returns the total.
__device__ __forceinline__ int warp_exclusive_scan(int* v, int n, int lane) {
  const int per = (n + 31) / 32;
  const int lo = lane * per;
  int local = 0;
  for (int i = lo; i < lo + per && i < n; ++i) local += v[i];
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  int run = incl - local;
  for (int i = lo; i < lo + per && i < n; ++i) {
    const int c = v[i];
    v[i] = run;
    run += c;
  }
  return __shfl_sync(0xffffffffu, incl, 31);
}

// Warp-wide top-k of one token: K rounds of an argmax over scores + bias
// (ties to the lower expert index).  Every lane returns the same sel[0..K)
// and the selected unbiased scores ssel[0..K).  score(e) gives the token's
// score of expert e.
template <typename ScoreAt>
__device__ __forceinline__ void warp_select_topk_by(ScoreAt score, const float* __restrict__ bias, int E, int K,
                                                    int lane, int (&sel)[kMaxTopK], float (&ssel)[kMaxTopK]) {
  float v[kMaxExperts / 32], sv[kMaxExperts / 32];
#pragma unroll
  for (int i = 0; i < kMaxExperts / 32; ++i) {
    const int e = lane + 32 * i;
    sv[i] = e < E ? score(e) : 0.0f;
    v[i] = e < E ? __fadd_rn(sv[i], bias[e]) : 0.0f;
  }
  uint32_t taken = 0;
#pragma unroll
  for (int k = 0; k < kMaxTopK; ++k) {
    if (k >= K) break;
    float bv = 0.0f, bs = 0.0f;
    int be = INT_MAX;
#pragma unroll
    for (int i = 0; i < kMaxExperts / 32; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !((taken >> i) & 1u)) {
        if (be == INT_MAX || v[i] > bv) {  // ascending e: strict '>' keeps the lower index
          bv = v[i];
          bs = sv[i];
          be = e;
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const float os = __shfl_xor_sync(0xffffffffu, bs, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (oe != INT_MAX && (be == INT_MAX || ov > bv || (ov == bv && oe < be))) {
        bv = ov;
        bs = os;
        be = oe;
      }
    }
    sel[k] = be;
    ssel[k] = bs;
    if ((be & 31) == lane) taken |= 1u << (be >> 5);
  }
}

// The same over a score row in global memory that an earlier kernel of the
// forward wrote (read through L2).
__device__ __forceinline__ void warp_select_topk(const float* st, const float* __restrict__ bias, int E, int K,
                                                 int lane, int (&sel)[kMaxTopK], float (&ssel)[kMaxTopK]) {
  warp_select_topk_by([st](int e) { return ld_dep(st + e); }, bias, E, K, lane, sel, ssel);
}

// Weights of the selected experts (one lane): denom = s_r0 + s_r1 + ...
// left to right; w_k = (s_rk / denom) * rsf, or s_rk * rsf.
__device__ __forceinline__ void topk_weights(const int (&sel)[kMaxTopK], const float (&sk)[kMaxTopK], int K, int norm,
                                             float rsf, int32_t* __restrict__ idx, float* __restrict__ wout) {
  float denom = 0.0f;
#pragma unroll
  for (int k = 0; k < kMaxTopK; ++k) {
    if (k >= K) break;
    denom = (k == 0) ? sk[k] : __fadd_rn(denom, sk[k]);
  }
#pragma unroll
  for (int k = 0; k < kMaxTopK; ++k) {
    if (k >= K) break;
    idx[k] = sel[k];
    wout[k] = norm ? __fmul_rn(__fdiv_rn(sk[k], denom), rsf) : __fmul_rn(sk[k], rsf);
  }
}

}  // namespace topk
}  // namespace coli
