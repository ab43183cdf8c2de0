// coli_route.cu -- router scores, top-k selection and bucketing.
//
// Router: "GLM-5.2-colibri-int4架构解析…" (wmrh.cn), sections "MoE的工作原理"
// (router scores pick 8 experts; weighted sum), "路由策略定制"
// (routed_scaling_factor, norm_topk_prob), "量化保留模块" (router kept F32);
// "Colibri：在笔记本上跑744B参数的AI模型", "关键特性" (DeepSeek-V3 style
// sigmoid router).  Bucketing: "如何在普通电脑上运行 7440 亿参数神经网络",
// "引擎是如何工作的" (requests for one expert merged) and the HN summary,
// "已实现的功能" (batched MoE: an expert used by several positions is read
// once).
#include "coli_launch.h"
#include "coli_topk.cuh"

namespace coli {
namespace {

using namespace topk;

// One warp per (token, expert): lane l owns accumulator l of contract R and
// reads float4 number l + 32j of the row, so each warp load is coalesced.
__global__ void __launch_bounds__(256) router_scores_kernel(const float* __restrict__ x,
                                                            const float* __restrict__ wr, int n_tok, int E,
                                                            int H, float* __restrict__ scores) {
  const int lane = threadIdx.x & 31;
  const int64_t gw = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (gw >= (int64_t)n_tok * E) return;
  const int t = (int)(gw / E), e = (int)(gw % E);
  const float4* xp = reinterpret_cast<const float4*>(x + (int64_t)t * H);
  const float4* wp = reinterpret_cast<const float4*>(wr + (int64_t)e * H);
  float acc = 0.0f;
  for (int j = lane; j < H / 4; j += 32) {
    const float4 a = xp[j];
    const float4 b = __ldg(wp + j);
    acc = __fmaf_rn(a.x, b.x, acc);
    acc = __fmaf_rn(a.y, b.y, acc);
    acc = __fmaf_rn(a.z, b.z, acc);
    acc = __fmaf_rn(a.w, b.w, acc);
  }
  const float logit = warp_sum_in_lane_order(acc);
  if (lane == 0) scores[gw] = sigmoid_cw(logit);
}

// Router scores for many tokens: a CTA of 8 warps owns a tile of 16 tokens
// x 16 experts and stages both sets of rows through shared memory in
// chunks of 512 values (cp.async, two chunks in flight), so each row is read
// from L2 once per tile instead of once per dot product.  Warp w folds 4
// tokens x 8 experts (32 accumulators per lane); lane l still owns
// accumulator l of contract R (float4 number l + 32j of the row, ascending
// j), and the 32 lane partials of each dot are summed left to right by one
// lane after a transpose through shared memory.
constexpr int kRtTok = 16, kRtExp = 16, kRtChunk = 64;  // chunk: float4 per row
// the epilogue's per-warp transpose (8 warps x 32 dots x 33 floats) reuses
// the staging buffers, which must hold it
static_assert(2 * (kRtTok + kRtExp) * kRtChunk * 16 >= 8 * 32 * 33 * 4, "router tile staging too small");
__global__ void __launch_bounds__(256) router_tiled_kernel(const float* __restrict__ x,
                                                           const float* __restrict__ wr, int n_tok, int E, int H,
                                                           float* __restrict__ scores) {
  extern __shared__ __align__(16) float4 rsm[];  // [2][(kRtTok + kRtExp) * kRtChunk]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * kRtTok, e0 = blockIdx.y * kRtExp;
  const int nq = H / 4, n_chunks = nq / kRtChunk;
  constexpr int kRows = kRtTok + kRtExp;
  auto load_chunk = [&](int c, int buf) {
    float4* dst = rsm + buf * kRows * kRtChunk;
    for (int i = threadIdx.x; i < kRows * kRtChunk; i += blockDim.x) {
      const int r = i / kRtChunk, j = i - r * kRtChunk;
      const bool is_x = r < kRtTok;
      const int g = is_x ? t0 + r : e0 + (r - kRtTok);
      if (g < (is_x ? n_tok : E)) {
        const float* src = (is_x ? x : wr) + (int64_t)g * H + 4 * (c * kRtChunk + j);
        cp_async16(dst + i, src);
      } else {
        dst[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  const int tw = (warp >> 1) * 4, ew = (warp & 1) * 8;  // this warp's 4 tokens, 8 experts within the tile
  float acc[4][8];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 8; ++b) acc[a][b] = 0.0f;
  load_chunk(0, 0);
  for (int c = 0; c < n_chunks; ++c) {
    if (c + 1 < n_chunks) {
      load_chunk(c + 1, (c + 1) & 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    const float4* xs = rsm + (c & 1) * kRows * kRtChunk;
    const float4* ws = xs + kRtTok * kRtChunk;
#pragma unroll
    for (int k = 0; k < kRtChunk / 32; ++k) {
      const int j = 32 * k + lane;
      float4 xv[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) xv[a] = xs[(tw + a) * kRtChunk + j];
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        const float4 wv = ws[(ew + b) * kRtChunk + j];
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          acc[a][b] = __fmaf_rn(xv[a].x, wv.x, acc[a][b]);
          acc[a][b] = __fmaf_rn(xv[a].y, wv.y, acc[a][b]);
          acc[a][b] = __fmaf_rn(xv[a].z, wv.z, acc[a][b]);
          acc[a][b] = __fmaf_rn(xv[a].w, wv.w, acc[a][b]);
        }
      }
    }
    __syncthreads();  // the buffer is refilled by the next iteration's copies
  }
  // transpose: red[d][l] = lane l's partial of dot d; lane d then sums its row left to right
  float* red = reinterpret_cast<float*>(rsm) + warp * 32 * 33;
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 8; ++b) red[(a * 8 + b) * 33 + lane] = acc[a][b];
  __syncwarp();
  const int t = t0 + tw + (lane >> 3), e = e0 + ew + (lane & 7);
  float logit = red[lane * 33];
#pragma unroll
  for (int l = 1; l < 32; ++l) logit = __fadd_rn(logit, red[lane * 33 + l]);
  if (t < n_tok && e < E) scores[(int64_t)t * E + e] = sigmoid_cw(logit);
}

size_t router_tiled_smem() { return (size_t)2 * (kRtTok + kRtExp) * kRtChunk * sizeof(float4); }

// One warp per token.
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ scores,
                                                   const float* __restrict__ bias, int n_tok, int E, int K,
                                                   int norm, float rsf, int32_t* __restrict__ idx,
                                                   float* __restrict__ wout) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= n_tok) return;
  const float* st = scores + (int64_t)t * E;
  int sel[kMaxTopK];
  float ssel[kMaxTopK];
  warp_select_topk(st, bias, E, K, lane, sel, ssel);
  if (lane == 0) topk_weights(sel, ssel, K, norm, rsf, idx + (int64_t)t * K, wout + (int64_t)t * K);
}

// Router scores and top-k of one token per CTA, the scores kept in shared
// memory only (coli_moe_route called without a scores buffer).  Warp w
// computes experts w, w + 8, ... with the lane mapping and order of
// router_scores_kernel (contract R), so the scores, and hence the choice,
// are the same bits.
constexpr int kRouteThreads = 256;
__global__ void __launch_bounds__(kRouteThreads) route_topk_kernel(const float* __restrict__ x,
                                                                   const float* __restrict__ wr,
                                                                   const float* __restrict__ bias, int E, int H,
                                                                   int K, int norm, float rsf,
                                                                   int32_t* __restrict__ idx,
                                                                   float* __restrict__ wout) {
  __shared__ float s_sc[kMaxExperts];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x;
  const float4* xp = reinterpret_cast<const float4*>(x + (int64_t)t * H);
  for (int e = warp; e < E; e += kRouteThreads / 32) {
    const float4* wp = reinterpret_cast<const float4*>(wr + (int64_t)e * H);
    float acc = 0.0f;
    for (int j = lane; j < H / 4; j += 32) {
      const float4 a = __ldg(xp + j);
      const float4 b = __ldg(wp + j);
      acc = __fmaf_rn(a.x, b.x, acc);
      acc = __fmaf_rn(a.y, b.y, acc);
      acc = __fmaf_rn(a.z, b.z, acc);
      acc = __fmaf_rn(a.w, b.w, acc);
    }
    const float logit = warp_sum_in_lane_order(acc);
    if (lane == 0) s_sc[e] = sigmoid_cw(logit);
  }
  __syncthreads();
  if (warp != 0) return;
  int sel[kMaxTopK];
  float ssel[kMaxTopK];
  warp_select_topk_by([](int e) { return s_sc[e]; }, bias, E, K, lane, sel, ssel);
  if (lane == 0) topk_weights(sel, ssel, K, norm, rsf, idx + (int64_t)t * K, wout + (int64_t)t * K);
}

// ---------------------------------------------------------------------------
// Decode batches (n_tok <= kDecodeMaxTok): two kernels.

// Router scores.  A CTA of 8 warps owns 2 experts; their router rows and
// the token rows (kStageTok tokens at a time) are copied to shared memory
// with cp.async, so the fold loop below reads only shared memory; in each
// pass warp w folds expert (w & 1) for token w/2 of the pass.  The CTAs also
// write the Q8_0 of x for the expert kernels.
constexpr int kStageTok = 4;
__global__ void __launch_bounds__(256) router_decode_kernel(const float* __restrict__ x,
                                                            const float* __restrict__ wr, int n_tok, int E, int H,
                                                            float* __restrict__ scores, int8_t* __restrict__ xq,
                                                            float* __restrict__ xd, int8_t* __restrict__ xpl,
                                                            float2* __restrict__ xdc, int32_t* status_clear,
                                                            int32_t* zero, int n_zero) {
  extern __shared__ __align__(16) float4 wsm[];  // [2][H/4] router rows, then [<= kStageTok][H/4] tokens
  // first kernel of a decode forward (launched without PDL, so everything
  // before it in the stream is complete): start the status word afresh
  if (status_clear && blockIdx.x == 0 && threadIdx.x == 0) *status_clear = 0;
  if (zero && blockIdx.x == 0)
    for (int i = threadIdx.x; i < n_zero; i += blockDim.x) zero[i] = 0;
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e0 = blockIdx.x * 2;
  const int nq = H / 4;
  const int G = n_tok < kStageTok ? n_tok : kStageTok;  // tokens per pass
  {
    // the router rows are read once per forward: first out of L2
    const uint64_t pol = l2_evict_first();
    for (int i = threadIdx.x; i < 2 * nq; i += blockDim.x) {
      const int r = i / nq, j = i - r * nq;
      if (e0 + r < E) cp_async16_hint(wsm + i, wr + (size_t)(e0 + r) * H + 4 * j, pol);
    }
  }
  for (int i = threadIdx.x; i < G * nq; i += blockDim.x) cp_async16(wsm + 2 * nq + i, x + 4 * (size_t)i);
  // the Q8_0 of x for the expert kernels: one warp per 32-element block,
  // as rows (xq, xd) and / or as the streaming kernel's even / odd byte
  // planes with (d, -128 * sum of the even plane) (xpl, xdc)
  for (int j = blockIdx.x * 8 + warp; (xq != nullptr || xpl != nullptr) && j < n_tok * (H / 32);
       j += gridDim.x * 8) {
    const float v = x[(size_t)j * 32 + lane];
    const float d = __fdiv_rn(warp_max(fabsf(v)), 127.0f);
    const int q = q8_of(v, d);
    if (xq != nullptr) {
      xq[(size_t)j * 32 + lane] = (int8_t)q;
      if (lane == 0) xd[j] = d;
    }
    if (xpl != nullptr) {
      xpl[(size_t)j * 32 + (lane & 1) * 16 + (lane >> 1)] = (int8_t)q;
      int se = (lane & 1) ? 0 : q;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) se += __shfl_xor_sync(0xffffffffu, se, o);
      if (lane == 0) xdc[j] = make_float2(d, __int_as_float(-128 * se));
    }
  }
  const int r = warp & 1, e = e0 + r;
  const float4* ws = wsm + r * nq;
  for (int t0 = 0; t0 < n_tok; t0 += G) {
    if (t0 > 0) {
      __syncthreads();  // the previous pass's reads of the staged tokens are done
      const int g = n_tok - t0 < G ? n_tok - t0 : G;
      for (int i = threadIdx.x; i < g * nq; i += blockDim.x)
        cp_async16(wsm + 2 * nq + i, x + (size_t)t0 * H + 4 * (size_t)i);
    }
    cp_async_wait_all();
    __syncthreads();
    for (int tl = warp >> 1; e < E && tl < G && t0 + tl < n_tok; tl += 4) {
      const float4* xp = wsm + (2 + tl) * nq;
      float acc = 0.0f;
#pragma unroll 8
      for (int j = lane; j < nq; j += 32) {
        const float4 a = xp[j];
        const float4 b = ws[j];
        acc = __fmaf_rn(a.x, b.x, acc);
        acc = __fmaf_rn(a.y, b.y, acc);
        acc = __fmaf_rn(a.z, b.z, acc);
        acc = __fmaf_rn(a.w, b.w, acc);
      }
      const float logit = warp_sum_in_lane_order(acc);
      if (lane == 0) scores[(size_t)(t0 + tl) * E + e] = sigmoid_cw(logit);
    }
  }
}

// Top-k, weights and bucketing of a decode batch in one CTA: warp t selects
// token t's experts; counts by shared atomics; offsets and the active-expert
// list by warp scans; a pair's position within its expert group is the
// number of earlier tokens that chose the same expert (stable by token).
// The slot table lists the routed experts in ascending id.
constexpr int kSmallThreads = 512;
__global__ void __launch_bounds__(kSmallThreads) topk_bucket_small_kernel(
    const float* scores, const float* __restrict__ bias, int n_tok, int E, int K, int norm, float rsf,
    int32_t* __restrict__ idx_out, float* __restrict__ w_out, int32_t* __restrict__ counts,
    int32_t* __restrict__ offsets, int32_t* __restrict__ perm, int32_t* __restrict__ inv, Slot* __restrict__ slots,
    int32_t* __restrict__ n_slots) {
  __shared__ int s_idx[kDecodeMaxTok * kMaxTopK];
  __shared__ int cnt[kMaxExperts];
  __shared__ int off[kMaxExperts];
  __shared__ int act[kMaxExperts];
  pdl_wait();
  pdl_launch_dependents();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int e = tid; e < E; e += blockDim.x) cnt[e] = 0;
  if (warp < n_tok) {
    const float* st = scores + (size_t)warp * E;
    int sel[kMaxTopK];
    float ssel[kMaxTopK];
    warp_select_topk(st, bias, E, K, lane, sel, ssel);
    if (lane == 0) {
      topk_weights(sel, ssel, K, norm, rsf, idx_out + (size_t)warp * K, w_out + (size_t)warp * K);
#pragma unroll
      for (int k = 0; k < kMaxTopK; ++k)
        if (k < K) s_idx[warp * K + k] = sel[k];
    }
  }
  __syncthreads();
  const int n_pairs = n_tok * K;
  for (int p = tid; p < n_pairs; p += blockDim.x) atomicAdd(&cnt[s_idx[p]], 1);
  __syncthreads();
  if (warp == 0) {
    for (int e = lane; e < E; e += 32) {
      off[e] = cnt[e];
      act[e] = cnt[e] > 0 ? 1 : 0;
    }
    __syncwarp();
    const int total = warp_exclusive_scan(off, E, lane);
    __syncwarp();
    const int n_active = warp_exclusive_scan(act, E, lane);
    __syncwarp();
    for (int e = lane; e < E; e += 32) {
      counts[e] = cnt[e];
      offsets[e] = off[e];
      if (cnt[e] > 0) slots[act[e]] = Slot{e, off[e], cnt[e], off[e]};
    }
    if (lane == 0) {
      offsets[E] = total;
      *n_slots = n_active;
    }
  }
  __syncthreads();
  for (int p = tid; p < n_pairs; p += blockDim.x) {
    const int t = p / K, e = s_idx[p];
    int rank = 0;
    for (int q = 0; q < t * K; ++q) rank += (s_idx[q] == e);
    const int pos = off[e] + rank;
    perm[pos] = p;
    inv[p] = pos;
  }
}

constexpr int kBucketThreads = 1024;
constexpr int kChunk = 1024;  // tokens per ranking round: one per thread

// Single block.  Counts by shared-memory atomics (order-free), offsets by a
// scan, then a stable scatter: tokens are ranked within each expert through
// a per-chunk bitmap [E x 32 words] and popcounts, so every output position
// is a pure function of the input (deterministic, no ordering races).
__global__ void __launch_bounds__(kBucketThreads) bucket_kernel(const int32_t* __restrict__ idx, int n_tok, int K,
                                                                int E, int n_shared, int32_t* __restrict__ counts,
                                                                int32_t* __restrict__ offsets,
                                                                int32_t* __restrict__ perm, int32_t* __restrict__ inv,
                                                                Slot* __restrict__ slots,
                                                                int32_t* __restrict__ n_slots,
                                                                int32_t* __restrict__ status) {
  extern __shared__ int sm[];
  int* cnt = sm;             // [E]
  int* off = cnt + E;        // [E]
  int* run = off + E;        // [E]
  int* tot = run + E;        // [E]
  int* act = tot + E;        // [E] active-slot index
  uint32_t* bm = reinterpret_cast<uint32_t*>(act + E);  // [E][32]
  int* pre = reinterpret_cast<int*>(bm + 32 * E);        // [E][32]
  const int tid = threadIdx.x, lane = tid & 31;
  const int64_t n_pairs = (int64_t)n_tok * K;

  for (int e = tid; e < E; e += blockDim.x) {
    cnt[e] = 0;
    run[e] = 0;
  }
  __syncthreads();
  for (int64_t i = tid; i < n_pairs; i += blockDim.x) {
    const int e = idx[i];
    if (e >= 0 && e < E) {
      atomicAdd(&cnt[e], 1);
    } else if (status) {
      atomicExch(status, kStatusBadExpert);
    }
  }
  __syncthreads();
  if (tid < 32) {
    for (int e = lane; e < E; e += 32) {
      off[e] = cnt[e];
      act[e] = cnt[e] > 0 ? 1 : 0;
    }
    __syncwarp();
    const int total = warp_exclusive_scan(off, E, lane);
    __syncwarp();
    const int n_active = warp_exclusive_scan(act, E, lane);
    __syncwarp();
    for (int e = lane; e < E; e += 32) {
      counts[e] = cnt[e];
      offsets[e] = off[e];
      if (slots && cnt[e] > 0) slots[act[e]] = Slot{e, off[e], cnt[e], off[e]};
    }
    if (lane == 0) {
      offsets[E] = total;
      if (slots) {
        for (int s = 0; s < n_shared; ++s)
          slots[n_active + s] = Slot{E + s, (int)n_pairs + s * n_tok, n_tok, -1};
        *n_slots = n_active + n_shared;
      }
    }
  }
  __syncthreads();

  for (int base = 0; base < n_tok; base += kChunk) {
    for (int i = tid; i < 32 * E; i += blockDim.x) bm[i] = 0u;
    __syncthreads();
    const int j = tid;
    const int t = base + j;
    if (j < kChunk && t < n_tok) {
      for (int k = 0; k < K; ++k) {
        const int e = idx[(int64_t)t * K + k];
        if (e >= 0 && e < E) atomicOr(&bm[e * 32 + (j >> 5)], 1u << (j & 31));
      }
    }
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x) {
      int r = 0;
      for (int wd = 0; wd < 32; ++wd) {
        pre[e * 32 + wd] = r;
        r += __popc(bm[e * 32 + wd]);
      }
      tot[e] = r;
    }
    __syncthreads();
    if (j < kChunk && t < n_tok) {
      for (int k = 0; k < K; ++k) {
        const int e = idx[(int64_t)t * K + k];
        if (e < 0 || e >= E) continue;
        const uint32_t below = bm[e * 32 + (j >> 5)] & ((1u << (j & 31)) - 1u);
        const int pos = off[e] + run[e] + pre[e * 32 + (j >> 5)] + __popc(below);
        perm[pos] = t * K + k;
        if (inv) inv[(int64_t)t * K + k] = pos;
      }
    }
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x) run[e] += tot[e];
    __syncthreads();
  }
}

size_t bucket_smem_bytes(int E) { return (size_t)E * (5 + 64) * sizeof(int); }

}  // namespace

cudaError_t launch_router_scores(const float* x, const float* w_router, int n_tok, int E, int H, float* scores,
                                 cudaStream_t st) {
  if (n_tok >= 64 && H % (4 * kRtChunk) == 0) {
    static int granted[64] = {};
    const cudaError_t e = smem_opt_in(router_tiled_kernel, (int)router_tiled_smem(), granted);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)((n_tok + kRtTok - 1) / kRtTok), (unsigned)((E + kRtExp - 1) / kRtExp));
    router_tiled_kernel<<<grid, 256, router_tiled_smem(), st>>>(x, w_router, n_tok, E, H, scores);
    return cudaGetLastError();
  }
  const int64_t warps = (int64_t)n_tok * E;
  const int64_t blocks = (warps + 7) / 8;
  router_scores_kernel<<<(unsigned)blocks, 256, 0, st>>>(x, w_router, n_tok, E, H, scores);
  return cudaGetLastError();
}

cudaError_t launch_route_topk(const float* x, const float* w_router, const float* bias, int n_tok, int E, int H, int K,
                              int norm, float rsf, int32_t* idx, float* w, cudaStream_t st) {
  route_topk_kernel<<<n_tok, kRouteThreads, 0, st>>>(x, w_router, bias, E, H, K, norm, rsf, idx, w);
  return cudaGetLastError();
}

cudaError_t launch_topk(const float* scores, const float* bias, int n_tok, int E, int K, int norm, float rsf,
                        int32_t* idx, float* w, cudaStream_t st) {
  topk_kernel<<<(n_tok + 7) / 8, 256, 0, st>>>(scores, bias, n_tok, E, K, norm, rsf, idx, w);
  return cudaGetLastError();
}

cudaError_t launch_router_decode(const float* x, const float* w_router, int n_tok, int E, int H, float* scores,
                                 int8_t* xq, float* xd, int32_t* status_clear, int32_t* zero, int n_zero,
                                 cudaStream_t st, int8_t* xpl, float2* xdc) {
  const size_t smem = (size_t)(2 + (n_tok < kStageTok ? n_tok : kStageTok)) * H * sizeof(float);
  static int granted[64] = {};
  const cudaError_t e = smem_opt_in(router_decode_kernel, 200 * 1024, granted);
  if (e != cudaSuccess) return e;
  router_decode_kernel<<<(E + 1) / 2, 256, smem, st>>>(x, w_router, n_tok, E, H, scores, xq, xd, xpl, xdc,
                                                       status_clear, zero, n_zero);
  return cudaGetLastError();
}

cudaError_t launch_topk_bucket_small(const float* scores, const float* bias, int n_tok, int E, int K, int norm,
                                     float rsf, int32_t* idx, float* w, int32_t* counts, int32_t* offsets,
                                     int32_t* perm, int32_t* inv, Slot* slots, int32_t* n_slots, cudaStream_t st) {
  return launch_pdl(topk_bucket_small_kernel, dim3(1), dim3(kSmallThreads), 0, st, true, scores, bias, n_tok, E, K,
                    norm, rsf, idx, w, counts, offsets, perm, inv, slots, n_slots);
}

cudaError_t launch_bucket(const int32_t* idx, int n_tok, int K, int E, int n_shared, int32_t* counts,
                          int32_t* offsets, int32_t* perm, int32_t* inv, Slot* slots, int32_t* n_slots,
                          int32_t* status, cudaStream_t st) {
  const size_t smem = bucket_smem_bytes(E);
  static int granted[64] = {};  // the opt-in is per device
  const cudaError_t e = smem_opt_in(bucket_kernel, (int)bucket_smem_bytes(kMaxExperts), granted);
  if (e != cudaSuccess) return e;
  bucket_kernel<<<1, kBucketThreads, smem, st>>>(idx, n_tok, K, E, n_shared, counts, offsets, perm, inv, slots,
                                                  n_slots, status);
  return cudaGetLastError();
}

}  // namespace coli
