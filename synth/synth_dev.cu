// synth_dev.cu -- seeded synthetic inputs, CUDA implementation.
//
// Same definition as synth_host.c (SplitMix64 counters, Irwin-Hall-12
// normals, 24-bit uniforms); written separately for the device so weights of
// any size can be generated in place on the GPU.  Holds none of the MoE
// method's arithmetic.  Every float operation is an explicit round-to-nearest
// intrinsic, so the results are the host's bits.
#include <cstdint>
#include <cuda_runtime.h>

#define SYN_API extern "C" __attribute__((visibility("default")))

namespace {

constexpr uint64_t kG = 0x9E3779B97F4A7C15ull;

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z ^= z >> 30;
  z *= 0xBF58476D1CE4E5B9ull;
  z ^= z >> 27;
  z *= 0x94D049BB133111EBull;
  z ^= z >> 31;
  return z;
}

__device__ __forceinline__ uint64_t draw(uint64_t key, uint64_t c) { return mix64(key + (c + 1) * kG); }

__global__ void normal_kernel(float* __restrict__ out, int64_t n, uint64_t i0, uint64_t key, float sigma) {
  for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < n;
       j += (int64_t)gridDim.x * blockDim.x) {
    const uint64_t i = i0 + (uint64_t)j;
    uint32_t s = 0;
#pragma unroll
    for (int k = 0; k < 6; ++k) {
      const uint64_t z = draw(key, 6 * i + (uint64_t)k);
      s += (uint32_t)(z >> 40) + (uint32_t)((z >> 16) & 0xFFFFFFu);
    }
    const float v = __fmul_rn(__int2float_rn((int32_t)s - (int32_t)(6u << 24)), 0x1p-24f);
    out[j] = __fmul_rn(sigma, v);
  }
}

__global__ void uniform_kernel(float* __restrict__ out, int64_t n, uint64_t i0, uint64_t key, float a,
                               float b) {
  const float range = __fsub_rn(b, a);
  for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < n;
       j += (int64_t)gridDim.x * blockDim.x) {
    const uint32_t u = (uint32_t)(draw(key, i0 + (uint64_t)j) >> 40);
    const float t = __fmul_rn(__uint2float_rn(u), 0x1p-24f);
    out[j] = __fadd_rn(a, __fmul_rn(range, t));
  }
}

__global__ void add_range_kernel(float* out, int64_t n, float v) {
  for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < n;
       j += (int64_t)gridDim.x * blockDim.x)
    out[j] = __fadd_rn(out[j], v);
}

// x[t, h] = base[h] + a * x[t, h]
__global__ void axpy_base_kernel(float* x, const float* base, int64_t T, int64_t H, float a) {
  for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < T * H;
       j += (int64_t)gridDim.x * blockDim.x)
    x[j] = __fadd_rn(base[j % H], __fmul_rn(a, x[j]));
}

int grid_for(int64_t n) {
  int64_t g = (n + 255) / 256;
  if (g > 148 * 64) g = 148 * 64;
  if (g < 1) g = 1;
  return (int)g;
}

}  // namespace

SYN_API int synth_dev_normal(float* out, int64_t n, uint64_t i0, uint64_t key, float sigma, void* stream) {
  if (n <= 0) return 0;
  normal_kernel<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(out, n, i0, key, sigma);
  return (int)cudaGetLastError();
}

SYN_API int synth_dev_uniform(float* out, int64_t n, uint64_t i0, uint64_t key, float a, float b,
                              void* stream) {
  if (n <= 0) return 0;
  uniform_kernel<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(out, n, i0, key, a, b);
  return (int)cudaGetLastError();
}

SYN_API int synth_dev_add_range(float* out, int64_t n, float v, void* stream) {
  if (n <= 0) return 0;
  add_range_kernel<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(out, n, v);
  return (int)cudaGetLastError();
}

SYN_API int synth_dev_axpy_base(float* x, const float* base, int64_t T, int64_t H, float a, void* stream) {
  if (T * H <= 0) return 0;
  axpy_base_kernel<<<grid_for(T * H), 256, 0, (cudaStream_t)stream>>>(x, base, T, H, a);
  return (int)cudaGetLastError();
}
