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

// Order key of a selection value: a larger float gives a larger unsigned key
// (-0 and +0 share a key, so that equal floats tie).
__device__ __forceinline__ uint32_t order_key(float v) {
  const uint32_t u = __float_as_uint(v == 0.0f ? 0.0f : v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The top-k of one token and its weights, by one warp.  Lane l holds the
// experts l, l + 32, .. (M per lane, E <= 32 M; bias_r[i] = bias of expert
// l + 32 i, loaded ahead by the caller); each of the K rounds is a warp max
// of the order keys of score + bias and a warp min of the expert ids that
// hold it (ties to the lower expert index), so the selection equals
// warp_select_topk_by's.  Lane k < K writes idx[k] and w[k] (topk_weights'
// arithmetic: the left-to-right sum of the selected unbiased scores, then
// w_k = (s_k / denom) * rsf, or s_k * rsf).
template <int M, int MB, typename ScoreAt>
__device__ __forceinline__ void warp_route_token(ScoreAt score, const float (&bias_r)[MB], int E, int K, int norm,
                                                 float rsf, int lane, int32_t* __restrict__ idx,
                                                 float* __restrict__ w) {
  static_assert(M <= MB, "bias registers");
  float sv[M];
  uint32_t key[M];
#pragma unroll
  for (int i = 0; i < M; ++i) {
    const int e = lane + 32 * i;
    sv[i] = e < E ? score(e) : 0.0f;
    key[i] = e < E ? order_key(__fadd_rn(sv[i], bias_r[i])) : 0u;  // 0: below every real key
  }
  int mine = 0;
  for (int k = 0; k < K; ++k) {
    uint32_t m[M];
#pragma unroll
    for (int i = 0; i < M; ++i) m[i] = key[i];
#pragma unroll
    for (int h = M / 2; h > 0; h >>= 1)
#pragma unroll
      for (int i = 0; i < h; ++i) m[i] = max(m[i], m[i + h]);
    const uint32_t mx = __reduce_max_sync(0xffffffffu, m[0]);
    int ce = INT_MAX;
#pragma unroll
    for (int i = M - 1; i >= 0; --i)
      if (key[i] == mx) ce = lane + 32 * i;
    const int ew = __reduce_min_sync(0xffffffffu, ce);
    if (lane == k) mine = ew;
#pragma unroll
    for (int i = 0; i < M; ++i)
      if (ew == lane + 32 * i) key[i] = 0u;
  }
  // the unbiased score of this lane's pick, from the lane that holds it
  float sk = 0.0f;
#pragma unroll
  for (int i = 0; i < M; ++i) {
    const float v = __shfl_sync(0xffffffffu, sv[i], mine & 31);
    if ((mine >> 5) == i) sk = v;
  }
  if (lane >= K) sk = 0.0f;
  float denom = 0.0f;
  for (int j = 0; j < K; ++j) {
    const float s = __shfl_sync(0xffffffffu, sk, j);
    denom = j == 0 ? s : __fadd_rn(denom, s);
  }
  if (lane < K) {
    idx[lane] = mine;
    w[lane] = norm ? __fmul_rn(__fdiv_rn(sk, denom), rsf) : __fmul_rn(sk, rsf);
  }
}

}  // namespace topk
}  // namespace coli
