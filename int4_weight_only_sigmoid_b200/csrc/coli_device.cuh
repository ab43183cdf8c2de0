// coli_device.cuh -- device helpers shared by the libcoli kernels.
//
// Every float operation that a result depends on is an explicit
// round-to-nearest intrinsic (__fmaf_rn, __fmul_rn, __fadd_rn, __fdiv_rn)
// and the library is compiled with -fmad=false, so the compiler cannot fuse
// or reorder them: the results follow the written evaluation contracts
//   R (router logit, RMSNorm sum of squares): element h feeds accumulator
//     l = (h/4) mod 32, each an fmaf chain in ascending h from +0; then
//     acc_0 + acc_1 + ... + acc_31 left to right;
//   F (row fold): acc = 0; for 32-blocks b ascending:
//     acc = fmaf(d_x[b], (float)isum[b], acc); y = s_w * acc;
//   C (combine): acc = 0; for k in rank order acc = fmaf(w_k, y_k, acc);
//     out = acc + y_shared_0 (+ ...).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace coli {

constexpr int kMaxExperts = 512;
constexpr int kMaxShared = 4;
constexpr int kMaxTopK = 16;
constexpr int kMaxSlots = kMaxExperts + kMaxShared;

// ---------------------------------------------------------------------------
// exp, sigmoid: our own e^x, from Cody & Waite's argument reduction
// ("Software Manual for the Elementary Functions", 1980) and the Taylor
// series of e^r to degree 7.  k = rint(x*log2 e); r = x - k*ln2 with ln 2
// split into a 15-bit head (so k*head is exact) and a binary32 tail;
// p = sum r^n/n! by Horner; result p * 2^k applied as two factors
// 2^(k/2) * 2^(k-k/2) built from exponent bits, so only the last multiply
// rounds.  Constants: log2 e, the split of ln 2 and 1/n!, each rounded to
// binary32.

__device__ __forceinline__ float pow2i(int k) { return __int_as_float((k + 127) << 23); }

__device__ __forceinline__ float exp_cw(float x) {
  if (x != x) return x;
  if (x > 0x1.62e43p+6f) return __int_as_float(0x7f800000);
  if (x < -0x1.9fe36ap+6f) return 0.0f;
  const float k = rintf(__fmul_rn(x, 0x1.715476p+0f));
  float r = __fmaf_rn(-k, 0x1.62e4p-1f, x);
  r = __fmaf_rn(-k, 0x1.7f7d1cp-20f, r);
  float p = 0x1.a01a02p-13f;            // 1/7!
  p = __fmaf_rn(p, r, 0x1.6c16c2p-10f); // 1/6!
  p = __fmaf_rn(p, r, 0x1.111112p-7f);  // 1/5!
  p = __fmaf_rn(p, r, 0x1.555556p-5f);  // 1/4!
  p = __fmaf_rn(p, r, 0x1.555556p-3f);  // 1/3!
  p = __fmaf_rn(p, r, 0.5f);            // 1/2!
  p = __fmaf_rn(p, r, 1.0f);
  p = __fmaf_rn(p, r, 1.0f);
  const int ki = (int)k;
  const int k1 = ki / 2;  // truncates toward zero
  const int k2 = ki - k1;
  return __fmul_rn(__fmul_rn(p, pow2i(k1)), pow2i(k2));
}

__device__ __forceinline__ float sigmoid_cw(float x) {
  return __fdiv_rn(1.0f, __fadd_rn(1.0f, exp_cw(-x)));
}

// ---------------------------------------------------------------------------
// warp helpers

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// acc_0 + acc_1 + ... + acc_31, added left to right (contract R's last step);
// every lane gets the sum.
__device__ __forceinline__ float warp_sum_in_lane_order(float acc) {
  float s = __shfl_sync(0xffffffffu, acc, 0);
#pragma unroll
  for (int l = 1; l < 32; ++l) s = __fadd_rn(s, __shfl_sync(0xffffffffu, acc, l));
  return s;
}

// ---------------------------------------------------------------------------
// int4 x int8 block dot.
//
// A packed 16-byte weight block holds 32 nibbles: word k has elements
// 8k..8k+7, element 8k+2i in the low nibble of byte i.  (w << 4) & 0xF0F0F0F0
// puts the even elements' nibbles in the high half of each byte, i.e. 16*q as
// a signed byte; w & 0xF0F0F0F0 does the same for the odd elements.  Paired
// with activations split into even/odd byte planes, two dp4a per word give
// 16 * sum q_w q_x exactly (|16 * isum| <= 16 * 32512 < 2^31); >> 4 is exact.

// Split two canonical activation words [x0..x3], [x4..x7] into the even
// [x0,x2,x4,x6] and odd [x1,x3,x5,x7] byte planes.
__device__ __forceinline__ void split_even_odd(uint32_t a, uint32_t b, uint32_t& even, uint32_t& odd) {
  even = __byte_perm(a, b, 0x6420);
  odd = __byte_perm(a, b, 0x7531);
}

__device__ __forceinline__ int32_t block_isum(const uint4 w, const uint4 xe, const uint4 xo) {
  int32_t acc = 0;
  acc = __dp4a((int)((w.x << 4) & 0xF0F0F0F0u), (int)xe.x, acc);
  acc = __dp4a((int)(w.x & 0xF0F0F0F0u), (int)xo.x, acc);
  acc = __dp4a((int)((w.y << 4) & 0xF0F0F0F0u), (int)xe.y, acc);
  acc = __dp4a((int)(w.y & 0xF0F0F0F0u), (int)xo.y, acc);
  acc = __dp4a((int)((w.z << 4) & 0xF0F0F0F0u), (int)xe.z, acc);
  acc = __dp4a((int)(w.z & 0xF0F0F0F0u), (int)xo.z, acc);
  acc = __dp4a((int)((w.w << 4) & 0xF0F0F0F0u), (int)xe.w, acc);
  acc = __dp4a((int)(w.w & 0xF0F0F0F0u), (int)xo.w, acc);
  return acc >> 4;
}

// 16-byte streaming load that does not allocate in L1 (weights are read once).
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// 16-byte asynchronous global -> shared copy (cp.async, L2 only) and the wait
// for all of this thread's outstanding copies.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
// An L2 policy whose lines go first when L2 needs room (data read once).
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// cp_async16 under an L2 policy
__device__ __forceinline__ void cp_async16_hint(void* smem, const void* gmem, uint64_t policy) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(
                   (uint32_t)__cvta_generic_to_shared(smem)),
               "l"(gmem), "l"(policy)
               : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Programmatic dependent launch: wait for the grids this one depends on (a
// no-op when launched without the attribute), and let the next grid in the
// stream start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Loads of data that an earlier kernel of the same forward writes.  Kernels
// launched with programmatic dependent launch start while their predecessor
// still runs, so such data must not be declared __restrict__ (the compiler
// may then treat it as invariant and load it before the dependency wait) and
// is read through L2 (ld.global.cg), after pdl_wait().
__device__ __forceinline__ int32_t ld_dep(const int32_t* p) { return __ldcg(p); }
__device__ __forceinline__ float ld_dep(const float* p) { return __ldcg(p); }
__device__ __forceinline__ uint4 ld_dep(const uint4* p) { return __ldcg(p); }

// Q8_0 of one value given its block scale d (d == 0 -> 0).
__device__ __forceinline__ int q8_of(float v, float d) {
  if (d == 0.0f) return 0;
  int q = (int)rintf(__fdiv_rn(v, d));
  return q < -127 ? -127 : (q > 127 ? 127 : q);
}

// v / d rounded to nearest from r = RN(1 / d), by Markstein's theorem (P. W.
// Markstein, "Computation of elementary functions on the IBM RISC System/
// 6000 processor", IBM J. Res. Dev. 34(1), 1990): with q0 = RN(v r) the
// remainder v - q0 d is exact in one FMA, and RN(q0 + (v - q0 d) r) is the
// correctly rounded quotient when nothing overflows or underflows, which
// holds for 2^-100 <= d <= 2^100 and |v| <= 127 d (a quotient below 1/4 in
// magnitude, the only case where the remainder can be subnormal, rounds to
// the integer 0 either way).
__device__ __forceinline__ bool div_by_recip_ok(float d) { return d >= 0x1p-100f && d <= 0x1p100f; }
__device__ __forceinline__ float div_by_recip(float v, float d, float r) {
  const float q0 = __fmul_rn(v, r);
  return __fmaf_rn(__fmaf_rn(-q0, d, v), r, q0);
}

// (kept out of line: one copy of the division, off the common path)
static __device__ __noinline__ float div_rn_outlined(float v, float d) { return __fdiv_rn(v, d); }

// q8_of with one reciprocal per block: r = __frcp_rn(d) (unused unless
// div_by_recip_ok(d)); the same integer as q8_of(v, d).
__device__ __forceinline__ int q8_of_r(float v, float d, float r) {
  if (d == 0.0f) return 0;
  int q = (int)rintf(div_by_recip_ok(d) ? div_by_recip(v, d, r) : div_rn_outlined(v, d));
  return q < -127 ? -127 : (q > 127 ? 127 : q);
}

// ---------------------------------------------------------------------------
// Expert slots.  A slot is one expert applied to a contiguous group of rows
// of the intermediate / output buffers:
//   table index (routed expert e -> e, shared expert s -> n_experts + s),
//   row_base, count, perm_base (-1: tokens are 0..count-1; else token i is
//   perm[perm_base + i] / top_k).
struct Slot {
  int32_t table_idx, row_base, count, perm_base;
};

struct GateUpTable {
  const uint8_t* gate_q[kMaxSlots];
  const float* gate_s[kMaxSlots];
  const uint8_t* up_q[kMaxSlots];
  const float* up_s[kMaxSlots];
};

struct DownTable {
  const uint8_t* down_q[kMaxSlots];
  const float* down_s[kMaxSlots];
};

}  // namespace coli
