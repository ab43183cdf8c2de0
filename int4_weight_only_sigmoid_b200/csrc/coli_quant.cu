// coli_quant.cu -- the quantisers, RMSNorm, residual add and the isum hook.
//
// int4 rows: "GLM-5.2-colibri-int4架构解析…" (wmrh.cn), section
// "GLM-5.2-colibri-int4的量化流程" (rint, one F32 scale per row, packed U8).
// Q8_0 activations: "Colibri：在笔记本上跑744B参数的AI模型", "关键特性".
#include "coli_launch.h"

namespace coli {
namespace {

// One warp per row.  scale = absmax/7; q = rint(w/scale) in [-8,7]; element
// 2j in the low nibble of byte j.  Each lane packs 8 consecutive elements
// into one 32-bit word per step.
__global__ void __launch_bounds__(256) quantize_rows_int4_kernel(const float* __restrict__ w, int64_t rows,
                                                                 int64_t cols, uint8_t* __restrict__ q,
                                                                 float* __restrict__ s) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const float* wr = w + row * cols;
  float amax = 0.0f;
  for (int64_t c = lane * 4; c < cols; c += 128) {
    if (c + 4 <= cols) {
      const float4 v = *reinterpret_cast<const float4*>(wr + c);
      amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    } else {
      for (int64_t i = c; i < cols; ++i) amax = fmaxf(amax, fabsf(wr[i]));
    }
  }
  amax = warp_max(amax);
  const float scale = __fdiv_rn(amax, 7.0f);
  uint32_t* qr = reinterpret_cast<uint32_t*>(q + row * (cols / 2));
  for (int64_t g = lane; g < cols / 8; g += 32) {
    const float4 a = *reinterpret_cast<const float4*>(wr + 8 * g);
    const float4 b = *reinterpret_cast<const float4*>(wr + 8 * g + 4);
    const float e[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t word = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      int qi = 0;
      if (amax != 0.0f) {
        qi = (int)rintf(__fdiv_rn(e[i], scale));
        qi = qi < -8 ? -8 : (qi > 7 ? 7 : qi);
      }
      word |= ((uint32_t)qi & 0xFu) << (4 * i);
    }
    qr[g] = word;
  }
  if (lane == 0) s[row] = scale;
}

// One warp per row.  int8 weights: scale = absmax/127; q = rint(w/scale)
// in [-127,127], one byte per element ("Colibri：在笔记本上跑744B参数的AI
// 模型", "关键特性": the int8 kernel variant).
__global__ void __launch_bounds__(256) quantize_rows_int8_kernel(const float* __restrict__ w, int64_t rows,
                                                                 int64_t cols, int8_t* __restrict__ q,
                                                                 float* __restrict__ s) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const float* wr = w + row * cols;
  float amax = 0.0f;
  for (int64_t c = lane * 4; c < cols; c += 128) {
    const float4 v = *reinterpret_cast<const float4*>(wr + c);
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
  }
  amax = warp_max(amax);
  const float scale = __fdiv_rn(amax, 127.0f);
  uint32_t* qr = reinterpret_cast<uint32_t*>(q + row * cols);
  for (int64_t g = lane; g < cols / 4; g += 32) {
    const float4 a = *reinterpret_cast<const float4*>(wr + 4 * g);
    const float e[4] = {a.x, a.y, a.z, a.w};
    uint32_t word = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      int qi = 0;
      if (amax != 0.0f) {
        qi = (int)rintf(__fdiv_rn(e[i], scale));
        qi = qi < -127 ? -127 : (qi > 127 ? 127 : qi);
      }
      word |= ((uint32_t)qi & 0xFFu) << (8 * i);
    }
    qr[g] = word;
  }
  if (lane == 0) s[row] = scale;
}

// FP8 -> int4 requantiser (the converter: "GLM-5.2-colibri-int4架构解析…",
// "GLM-5.2-colibri-int4的量化流程": FP8 e4m3 source -> F32 -> int4 per
// row; config weight_block_size [128, 128]).  e4m3 code -> F32, exact:
// bit 7 sign, bits 6..3 exponent (bias 7), bits 2..0 mantissa; exponent 0
// is subnormal (m * 2^-9); 0x7F / 0xFF are NaN (no infinities).
__device__ __forceinline__ float e4m3_value(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  float v;
  if (e == 15u && m == 7u)
    v = __int_as_float(0x7fc00000);
  else if (e == 0u)
    v = __fmul_rn((float)m, 0x1p-9f);
  else
    v = __int_as_float((int)(((e + 120u) << 23) | (m << 20)));
  return (b & 0x80u) ? -v : v;
}

// Element value: e4m3 * the factor of its block x block tile (one F32
// multiply); a non-finite product (NaN code, overflow) counts as 0.
__device__ __forceinline__ float fp8_element(uint32_t code, float factor) {
  const float v = __fmul_rn(e4m3_value(code), factor);
  return fabsf(v) <= 3.402823466e38f ? v : 0.0f;
}

// One warp per row, 8 codes (one 8-byte load, one block factor: block is a
// multiple of 8) per lane step; absmax pass, then the int4 row rule of
// quantize_rows_int4_kernel on the same values.
__global__ void __launch_bounds__(256) requantize_fp8_int4_kernel(const uint8_t* __restrict__ w8,
                                                                  const float* __restrict__ factors, int64_t rows,
                                                                  int64_t cols, int block, uint8_t* __restrict__ q,
                                                                  float* __restrict__ s) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int64_t bcols = (cols + block - 1) / block;
  const uint2* wr = reinterpret_cast<const uint2*>(w8 + row * cols);
  const float* fr = factors + (row / block) * bcols;
  float amax = 0.0f;
  for (int64_t g = lane; g < cols / 8; g += 32) {
    const uint2 c = __ldg(wr + g);
    const float f = __ldg(fr + (8 * g) / block);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      amax = fmaxf(amax, fabsf(fp8_element((c.x >> (8 * i)) & 0xFFu, f)));
      amax = fmaxf(amax, fabsf(fp8_element((c.y >> (8 * i)) & 0xFFu, f)));
    }
  }
  amax = warp_max(amax);
  const float scale = __fdiv_rn(amax, 7.0f);
  uint32_t* qr = reinterpret_cast<uint32_t*>(q + row * (cols / 2));
  for (int64_t g = lane; g < cols / 8; g += 32) {
    const uint2 c = __ldg(wr + g);
    const float f = __ldg(fr + (8 * g) / block);
    uint32_t word = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t code = ((i < 4 ? c.x : c.y) >> (8 * (i & 3))) & 0xFFu;
      int qi = 0;
      if (amax != 0.0f) {
        qi = (int)rintf(__fdiv_rn(fp8_element(code, f), scale));
        qi = qi < -8 ? -8 : (qi > 7 ? 7 : qi);
      }
      word |= ((uint32_t)qi & 0xFu) << (4 * i);
    }
    qr[g] = word;
  }
  if (lane == 0) s[row] = scale;
}

// One warp per 32-element block.
__global__ void __launch_bounds__(256) quantize_act_q8_kernel(const float* __restrict__ x, int64_t n_blocks,
                                                              int8_t* __restrict__ q, float* __restrict__ d) {
  const int lane = threadIdx.x & 31;
  const int64_t blk = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (blk >= n_blocks) return;
  const float v = x[blk * 32 + lane];
  const float amax = warp_max(fabsf(v));
  const float dd = __fdiv_rn(amax, 127.0f);
  q[blk * 32 + lane] = (int8_t)q8_of_r(v, dd, __frcp_rn(dd));  // the quotient the streaming kernel uses
  if (lane == 0) d[blk] = dd;
}

// RMSNorm, weight 1, one warp per token; sum of squares under contract R.
__global__ void __launch_bounds__(256) rmsnorm_kernel(const float* __restrict__ x, int n_tok, int dim, float eps,
                                                      float* __restrict__ y) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= n_tok) return;
  const float* xt = x + (int64_t)t * dim;
  float acc = 0.0f;
  for (int h = 4 * lane; h < dim; h += 128) {
    const float4 v = *reinterpret_cast<const float4*>(xt + h);
    acc = __fmaf_rn(v.x, v.x, acc);
    acc = __fmaf_rn(v.y, v.y, acc);
    acc = __fmaf_rn(v.z, v.z, acc);
    acc = __fmaf_rn(v.w, v.w, acc);
  }
  const float ss = warp_sum_in_lane_order(acc);
  const float mean = __fdiv_rn(ss, (float)dim);
  const float r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(mean, eps)));
  float* yt = y + (int64_t)t * dim;
  for (int h = 4 * lane; h < dim; h += 128) {
    const float4 v = *reinterpret_cast<const float4*>(xt + h);
    *reinterpret_cast<float4*>(yt + h) =
        make_float4(__fmul_rn(v.x, r), __fmul_rn(v.y, r), __fmul_rn(v.z, r), __fmul_rn(v.w, r));
  }
}

__global__ void residual_add_kernel(const float* __restrict__ x, const float* __restrict__ m, int64_t n,
                                    float* __restrict__ out) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = __fadd_rn(x[i], m[i]);
}

// isum[t, r, b] through the same block_isum routine as the expert kernels.
__global__ void debug_partials_kernel(const uint8_t* __restrict__ wq, const int8_t* __restrict__ xq, int n_tok,
                                      int dim_in, int rows, int32_t* __restrict__ out) {
  const int nb = dim_in / 32;
  const int64_t total = (int64_t)n_tok * rows * nb;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int b = (int)(i % nb);
    const int r = (int)((i / nb) % rows);
    const int t = (int)(i / ((int64_t)nb * rows));
    const uint4 w = *reinterpret_cast<const uint4*>(wq + (int64_t)r * (dim_in / 2) + 16 * b);
    const uint4* xp = reinterpret_cast<const uint4*>(xq + (int64_t)t * dim_in + 32 * b);
    const uint4 a0 = xp[0], a1 = xp[1];
    uint4 xe, xo;
    split_even_odd(a0.x, a0.y, xe.x, xo.x);
    split_even_odd(a0.z, a0.w, xe.y, xo.y);
    split_even_odd(a1.x, a1.y, xe.z, xo.z);
    split_even_odd(a1.z, a1.w, xe.w, xo.w);
    out[i] = block_isum(w, xe, xo);
  }
}

int blocks_for(int64_t items, int per_block) {
  int64_t g = (items + per_block - 1) / per_block;
  return (int)(g < 1 ? 1 : g);
}

}  // namespace

cudaError_t launch_quantize_rows_int4(const float* w, int64_t rows, int64_t cols, uint8_t* q, float* s,
                                      cudaStream_t st) {
  quantize_rows_int4_kernel<<<blocks_for(rows, 8), 256, 0, st>>>(w, rows, cols, q, s);
  return cudaGetLastError();
}

cudaError_t launch_quantize_rows_int8(const float* w, int64_t rows, int64_t cols, int8_t* q, float* s,
                                      cudaStream_t st) {
  quantize_rows_int8_kernel<<<blocks_for(rows, 8), 256, 0, st>>>(w, rows, cols, q, s);
  return cudaGetLastError();
}

cudaError_t launch_requantize_fp8_int4(const uint8_t* w8, const float* factors, int64_t rows, int64_t cols,
                                       int block, uint8_t* q, float* s, cudaStream_t st) {
  const int64_t blocks = (rows + 7) / 8;
  requantize_fp8_int4_kernel<<<(unsigned)blocks, 256, 0, st>>>(w8, factors, rows, cols, block, q, s);
  return cudaGetLastError();
}

cudaError_t launch_quantize_act_q8(const float* x, int64_t n_tok, int64_t dim, int8_t* q, float* d,
                                   cudaStream_t st) {
  const int64_t nbk = n_tok * (dim / 32);
  quantize_act_q8_kernel<<<blocks_for(nbk, 8), 256, 0, st>>>(x, nbk, q, d);
  return cudaGetLastError();
}

cudaError_t launch_rmsnorm(const float* x, int n_tok, int dim, float eps, float* y, cudaStream_t st) {
  rmsnorm_kernel<<<blocks_for(n_tok, 8), 256, 0, st>>>(x, n_tok, dim, eps, y);
  return cudaGetLastError();
}

cudaError_t launch_residual_add(const float* x, const float* m, int64_t n, float* out, cudaStream_t st) {
  int g = blocks_for(n, 256);
  if (g > 148 * 16) g = 148 * 16;
  residual_add_kernel<<<g, 256, 0, st>>>(x, m, n, out);
  return cudaGetLastError();
}

cudaError_t launch_debug_partials(const uint8_t* wq, const int8_t* xq, int n_tok, int dim_in, int rows,
                                  int32_t* out, cudaStream_t st) {
  const int64_t total = (int64_t)n_tok * rows * (dim_in / 32);
  int g = blocks_for(total, 256);
  if (g > 148 * 32) g = 148 * 32;
  debug_partials_kernel<<<g, 256, 0, st>>>(wq, xq, n_tok, dim_in, rows, out);
  return cudaGetLastError();
}

}  // namespace coli
