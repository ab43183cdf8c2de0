// coli_stream.cuh -- device pieces of the decode expert kernels
// (coli_decode.cu): weight-ring geometry, bulk copies and mbarriers,
// token staging (Q8_0 even / odd byte planes) and the rows-on-lanes int4 x
// int8 dot with its contract-F fold.
//
// Sources: "Colibri：在笔记本上跑744B参数的AI模型", "关键特性" (integer dot
// kernels, Q8_0 activations, packed int4).
#pragma once

#include "coli_gemv.cuh"
#include "coli_tc.cuh"

namespace coli {
namespace stream {

using gemv::kThreads;
using gemv::kWarps;

constexpr int kSmemLimit = 227 * 1024;  // dynamic shared memory a CTA may opt in to

constexpr int kBlkStep = 16;                     // packed blocks per row per step
constexpr int kPitchU4 = kBlkStep;               // stage row pitch (16-byte units)
constexpr int kStageBytes = 32 * kPitchU4 * 16;  // 32 rows (one per lane) = 8 KB
constexpr int kStageU4 = kStageBytes / 16;

// Block j of stage row r sits in 16-byte slot j ^ (r & 7) of the row, so the
// 8 lanes of each phase of a rows-on-lanes LDS.128 hit 8 different bank
// groups (the rows are 256 B apart, a multiple of the bank period).
__host__ __device__ constexpr int stage_slot(int r, int j) { return r * kPitchU4 + (j ^ (r & 7)); }

// Ring depth (stages per warp): one stage in flight while one is computed.
// Two stages keep 16 KB per warp, so three 4-warp CTAs fit on an SM.
template <int TT>
__host__ __device__ constexpr int ring_depth() {
  return 2;
}

// ---------------------------------------------------------------------------
// bulk copies and mbarriers

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(tc::smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

// global -> shared bulk copy completing on `bar` (addresses 16-byte aligned,
// size a multiple of 16).
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   tc::smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(tc::smem_u32(bar))
               : "memory");
}

// Orders this thread's earlier (generic-proxy) view of global memory before
// its later async-proxy reads of it (a bulk copy of data that other CTAs
// stored and this thread acquired).
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Hint: bring [src, src + bytes) into L2 (16-byte aligned, a multiple of 16).
__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// bulk_g2s with an L2 cache policy
__device__ __forceinline__ void bulk_g2s_hint(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                              uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          tc::smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(tc::smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

// Wait (bounded, ignoring the abort flag) for a copy the kernel still has in
// flight before it exits.
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!tc::mbar_try_wait(bar, parity))
    if (clock64() - t0 > tc::kSpinCycles) return;
}

// ---------------------------------------------------------------------------
// token staging: xs[2*(t*nb + b)] / [.. + 1] = even / odd byte plane of block b
// of staged token t; xsd[t*nb + b] = its Q8 scale.

__device__ __forceinline__ Slot shared_slot(int s, int n_tok, int K, int E) {
  return Slot{E + s, n_tok * K + s * n_tok, n_tok, -1};
}

// A slot-table entry written by the routing kernel (read through L2).
__device__ __forceinline__ Slot load_slot_dep(const Slot* p) {
  const uint4 v = ld_dep(reinterpret_cast<const uint4*>(p));
  return Slot{(int32_t)v.x, (int32_t)v.y, (int32_t)v.z, (int32_t)v.w};
}

template <int TT>
__device__ __forceinline__ int pick(const int (&tok)[TT], int t) {
  int row = tok[0];
#pragma unroll
  for (int j = 1; j < TT; ++j)
    if (t == j) row = tok[j];
  return row;
}

// Q8_0 of F32 token rows (the arithmetic of quantize_act_q8_kernel:
// d = absmax/127, q = rint(x/d) in [-127,127]).
template <int TT>
__device__ __forceinline__ void stage_x_f32(const float* x, int dim, int n_valid, const int (&tok)[TT], uint4* xs,
                                            float* xsd) {
  const int nb = dim / 32;
  for (int i = threadIdx.x; i < n_valid * nb; i += kThreads) {
    const int t = i / nb, b = i - t * nb;
    const float4* src = reinterpret_cast<const float4*>(x + (int64_t)pick<TT>(tok, t) * dim + 32 * b);
    float v[32];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float4 f = __ldcg(src + j);  // x may be a buffer an earlier kernel rewrote
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
    xs[2 * (t * nb + b)] = e;
    xs[2 * (t * nb + b) + 1] = o;
    xsd[t * nb + b] = d;
  }
}

// The router kernel's Q8_0 rows of x, split into planes.
template <int TT>
__device__ __forceinline__ void stage_x_q8(const int8_t* xq, const float* xd, int dim, int n_valid,
                                           const int (&tok)[TT], uint4* xs, float* xsd) {
  const int nb = dim / 32;
  for (int i = threadIdx.x; i < n_valid * nb; i += kThreads) {
    const int t = i / nb, b = i - t * nb;
    const int64_t row = pick<TT>(tok, t);
    const uint4* src = reinterpret_cast<const uint4*>(xq + row * dim + 32 * b);
    const uint4 a0 = ld_dep(src), a1 = ld_dep(src + 1);
    uint4 e, o;
    split_even_odd(a0.x, a0.y, e.x, o.x);
    split_even_odd(a0.z, a0.w, e.y, o.y);
    split_even_odd(a1.x, a1.y, e.z, o.z);
    split_even_odd(a1.z, a1.w, e.w, o.w);
    xs[2 * (t * nb + b)] = e;
    xs[2 * (t * nb + b) + 1] = o;
    xsd[t * nb + b] = ld_dep(xd + row * nb + b);
  }
}

// ---------------------------------------------------------------------------
// The dot: lane l holds weight row l of the stage and folds its blocks in
// ascending order against every staged token (contract F), so no transpose
// is needed and every lane works whatever the token count.

template <int TT>
__device__ __forceinline__ void block_fold(const uint4 w, int b, int nb, int n_valid, const uint4* xs,
                                           const float (&dx)[TT], float (&acc)[TT]) {
  const int e0 = (int)((w.x << 4) & 0xF0F0F0F0u), o0 = (int)(w.x & 0xF0F0F0F0u);
  const int e1 = (int)((w.y << 4) & 0xF0F0F0F0u), o1 = (int)(w.y & 0xF0F0F0F0u);
  const int e2 = (int)((w.z << 4) & 0xF0F0F0F0u), o2 = (int)(w.z & 0xF0F0F0F0u);
  const int e3 = (int)((w.w << 4) & 0xF0F0F0F0u), o3 = (int)(w.w & 0xF0F0F0F0u);
#pragma unroll
  for (int t = 0; t < TT; ++t) {
    if (t < n_valid) {
      const uint4 xe = xs[2 * (t * nb + b)], xo = xs[2 * (t * nb + b) + 1];
      int se = __dp4a(e0, (int)xe.x, 0);
      int so = __dp4a(o0, (int)xo.x, 0);
      se = __dp4a(e1, (int)xe.y, se);
      so = __dp4a(o1, (int)xo.y, so);
      se = __dp4a(e2, (int)xe.z, se);
      so = __dp4a(o2, (int)xo.z, so);
      se = __dp4a(e3, (int)xe.w, se);
      so = __dp4a(o3, (int)xo.w, so);
      // |isum| <= 32512: the conversion is exact
      acc[t] = __fmaf_rn(dx[t], __int2float_rn((se + so) >> 4), acc[t]);
    }
  }
}

// One ring stage: blocks b0 .. b0 + nblk - 1 of the lane's row.  A full
// stage (16 blocks, b0 and nb multiples of 4) reads the token scales four
// at a time.
template <int TT>
__device__ __forceinline__ void rows_step(const uint4* stage, int b0, int nblk, int nb, int n_valid, const uint4* xs,
                                          const float* xsd, float (&acc)[TT]) {
  const int lane = threadIdx.x & 31;
  const uint4* wrow = stage + lane * kPitchU4;
  const int sw = lane & 7;
  if (nblk == kBlkStep && (nb & 3) == 0) {
#pragma unroll
    for (int j4 = 0; j4 < kBlkStep; j4 += 4) {
      float4 d4[TT];
#pragma unroll
      for (int t = 0; t < TT; ++t)
        if (t < n_valid) d4[t] = *reinterpret_cast<const float4*>(xsd + t * nb + b0 + j4);
      float dx[TT];
#pragma unroll
      for (int t = 0; t < TT; ++t) dx[t] = d4[t].x;
      block_fold<TT>(wrow[(j4 + 0) ^ sw], b0 + j4 + 0, nb, n_valid, xs, dx, acc);
#pragma unroll
      for (int t = 0; t < TT; ++t) dx[t] = d4[t].y;
      block_fold<TT>(wrow[(j4 + 1) ^ sw], b0 + j4 + 1, nb, n_valid, xs, dx, acc);
#pragma unroll
      for (int t = 0; t < TT; ++t) dx[t] = d4[t].z;
      block_fold<TT>(wrow[(j4 + 2) ^ sw], b0 + j4 + 2, nb, n_valid, xs, dx, acc);
#pragma unroll
      for (int t = 0; t < TT; ++t) dx[t] = d4[t].w;
      block_fold<TT>(wrow[(j4 + 3) ^ sw], b0 + j4 + 3, nb, n_valid, xs, dx, acc);
    }
  } else {
    for (int j = 0; j < nblk; ++j) {
      float dx[TT];
#pragma unroll
      for (int t = 0; t < TT; ++t) dx[t] = t < n_valid ? xsd[t * nb + b0 + j] : 0.0f;
      block_fold<TT>(wrow[j ^ sw], b0 + j, nb, n_valid, xs, dx, acc);
    }
  }
}

}  // namespace stream
}  // namespace coli
