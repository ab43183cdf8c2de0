// coli_decode.cu -- the expert kernels of a decode batch (n_tok <= 16).
//
//   router_decode (plain launch; also writes the Q8_0 of x)
//     -> topk_bucket_small (PDL)
//     -> gateup_stream (PDL): persistent; the shared experts' items do not
//        depend on the routing and start at once, the routed items wait
//     -> down_stream (PDL): persistent; down projection per (64-row chunk,
//        expert) item, and the last item of each chunk combines the chunk
//        into `out` (no separate combine kernel).
//
// Persistent streaming: a CTA of 4 warps walks a list of items (item i of
// CTA c is c + i * gridDim.x, so the items of all CTAs are spread evenly);
// every warp owns 16 weight rows of the current item and streams them
// through a private ring of kRing steps (a step = 32 consecutive 16-byte
// blocks of each of its 16 rows = 8 KB), filled by cp.async kRing - 1 steps
// ahead, across item boundaries, so the weight stream does not drain between
// items.  A lane copies exactly the 16-byte blocks it later reduces, so a
// lane's own cp.async.wait_group is the only synchronisation the ring needs.
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

constexpr int kRing = 2;
constexpr int kStepU4 = kRows * 32;  // uint4 per ring step of one warp

__device__ __forceinline__ Slot shared_slot(int s, int n_tok, int K, int E) {
  return Slot{E + s, n_tok * K + s * n_tok, n_tok, -1};
}

// A slot-table entry written by the routing kernel (read through L2).
__device__ __forceinline__ Slot load_slot_dep(const Slot* p) {
  const uint4 v = ld_dep(reinterpret_cast<const uint4*>(p));
  return Slot{(int32_t)v.x, (int32_t)v.y, (int32_t)v.z, (int32_t)v.w};
}

// Stage n_valid F32 token rows as Q8_0 (the same arithmetic as
// quantize_act_q8_kernel: d = absmax/127, q = rint(x/d) in [-127,127]) into
// even/odd byte planes + block scales.
template <typename TokFn>
__device__ __forceinline__ void stage_quantize_f32(const float* x, int dim, int n_valid, TokFn tok,
                                                   uint4* xe_s, uint4* xo_s, float* xd_s) {
  const int nb = dim / 32;
  for (int i = threadIdx.x; i < n_valid * nb; i += kThreads) {
    const int t = i / nb, b = i - t * nb;
    const float4* src = reinterpret_cast<const float4*>(x + (int64_t)tok(t) * dim + 32 * b);
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
    xe_s[t * nb + b] = e;
    xo_s[t * nb + b] = o;
    xd_s[t * nb + b] = d;
  }
}

template <int TT>
struct StreamSmem {
  __host__ __device__ static size_t ring_bytes() { return (size_t)kWarps * kRing * kStepU4 * 16; }
  __host__ __device__ static size_t bytes(int dim_in) {
    const int nb = dim_in / 32;
    return ring_bytes() + (size_t)TT * nb * 36 + (size_t)kWarps * TT * kRows * kSPad * 4 + (size_t)TT * 32 * 4;
  }
};

struct Item {
  int it;      // item index
  bool valid;
  Slot slot;
  int r0;      // first output row of the item
  int groups;  // token groups of <= TT tokens
};

// Copy this lane's 16-byte block b of 16 rows (row0.. and row8.., rb bytes
// apart) into ring slot rs; always commits one cp.async group.
__device__ __forceinline__ void ring_fill(uint4* ring, int rs, const uint8_t* row0, const uint8_t* row8, size_t rb,
                                          int b, int nb) {
  const int lane = threadIdx.x & 31;
  if (b < nb) {
    uint4* dst = ring + rs * kStepU4 + lane;
#pragma unroll
    for (int r = 0; r < 8; ++r) cp_async16(dst + r * 32, row0 + r * rb + 16 * b);
#pragma unroll
    for (int r = 0; r < 8; ++r) cp_async16(dst + (8 + r) * 32, row8 + r * rb + 16 * b);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}

// One step of the fold from the ring: isums of 16 rows x n_valid tokens
// parked in shared memory, then each lane's chains (row c % 16, token
// c / 16 + 2m) advance over the step's blocks in ascending order.
template <int TT>
__device__ __forceinline__ void ring_step(const uint4* ring, int rs, int s0, int nb, int n_valid, const uint4* xe_s,
                                          const uint4* xo_s, const float* xd_s, int32_t* Sw,
                                          float (&facc)[(TT + 1) / 2]) {
  const int lane = threadIdx.x & 31;
  const int cr = lane & 15, ct = lane >> 4;
  const int b = s0 + lane;
  const bool valid = b < nb;
  const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
  uint4 wv[kRows];
#pragma unroll
  for (int r = 0; r < kRows; ++r) wv[r] = valid ? ring[rs * kStepU4 + r * 32 + lane] : zero;
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
  const int nst = min(32, nb - s0);
#pragma unroll
  for (int m = 0; m < (TT + 1) / 2; ++m) {
    const int t = ct + 2 * m;
    if (t < n_valid && t < TT) {
      const int32_t* srow = Sw + (t * kRows + cr) * kSPad;
      const float* dsrc = xd_s + t * nb + s0;
      float a = facc[m];
      for (int j = 0; j < nst; ++j) a = __fmaf_rn(dsrc[j], (float)srow[j], a);
      facc[m] = a;
    }
  }
  __syncwarp();
}

// Gate/up + SwiGLU + Q8_0 of h.  Items: (expert slot y, 32 intermediate
// outputs), slot-major, shared experts first (y < n_shared: no dependence on
// the routing); warp w owns gate rows r0+8w..+7 and the matching up rows.
template <int TT>
__global__ void __launch_bounds__(kThreads) gateup_stream_kernel(
    const __grid_constant__ GateUpTable tbl, const Slot* slots, const int32_t* n_slots, const int32_t* perm, int n_tok,
    int K, int E, int n_shared, int max_routed, const float* x, const int8_t* xq, const float* xd,
    int hidden, int inter, int8_t* hq, float* hd) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cr = lane & 15, ct = lane >> 4;
  const int nb = hidden / 32, nsteps = (nb + 31) / 32;
  const int nchunk = inter / 32;
  const int n_items = (n_shared + max_routed) * nchunk;
  const size_t rb = (size_t)hidden / 2;
  uint4* ring = reinterpret_cast<uint4*>(smem) + warp * kRing * kStepU4;
  uint4* xe_s = reinterpret_cast<uint4*>(smem) + kWarps * kRing * kStepU4;
  uint4* xo_s = xe_s + TT * nb;
  float* xd_s = reinterpret_cast<float*>(xo_s + TT * nb);
  int32_t* Sp = reinterpret_cast<int32_t*>(xd_s + TT * nb);
  float* Hs = reinterpret_cast<float*>(Sp + kWarps * TT * kRows * kSPad);
  int32_t* Sw = Sp + warp * TT * kRows * kSPad;

  bool waited = false;
  auto resolve = [&](Item& c) {
    c.valid = false;
    if (c.it >= n_items) return;
    const int yy = c.it / nchunk;
    c.r0 = (c.it - yy * nchunk) * 32;
    if (yy < n_shared) {
      c.slot = shared_slot(yy, n_tok, K, E);
    } else {
      if (!waited) {
        pdl_wait();  // the routing (and the Q8 of x) is complete and visible
        pdl_launch_dependents();
        waited = true;
      }
      const int r = yy - n_shared;
      if (r >= ld_dep(n_slots)) return;
      c.slot = load_slot_dep(slots + r);
    }
    c.groups = (c.slot.count + TT - 1) / TT;
    c.valid = true;
  };

  Item cur;
  cur.it = blockIdx.x;
  resolve(cur);
  Item pf = cur;
  int pf_step = 0, g_pf = 0, g = 0;
  auto prefetch = [&]() {
    if (pf.valid) {
      const int st = pf_step % nsteps;
      const int ti = pf.slot.table_idx;
      ring_fill(ring, g_pf % kRing, tbl.gate_q[ti] + (size_t)(pf.r0 + 8 * warp) * rb,
                tbl.up_q[ti] + (size_t)(pf.r0 + 8 * warp) * rb, rb, 32 * st + lane, nb);
    } else {
      asm volatile("cp.async.commit_group;" ::: "memory");
    }
    ++g_pf;
    if (pf.valid && ++pf_step == pf.groups * nsteps) {
      pf_step = 0;
      pf.it += gridDim.x;
      resolve(pf);
    }
  };
#pragma unroll
  for (int i = 0; i < kRing - 1; ++i) prefetch();

  while (cur.valid) {
    const int ti = cur.slot.table_idx;
    const int o_lane = cur.r0 + 8 * warp + (cr & 7);
    const float s_lane = cr < 8 ? tbl.gate_s[ti][o_lane] : tbl.up_s[ti][o_lane];
    const bool is_shared = cur.slot.perm_base < 0;
    for (int grp = 0; grp < cur.groups; ++grp) {
      const int g0 = grp * TT;
      const int n_valid = min(TT, cur.slot.count - g0);
      __syncthreads();  // the previous group's staging and Hs are consumed
      if (is_shared) {
        stage_quantize_f32(x, hidden, n_valid, [=](int t) { return g0 + t; }, xe_s, xo_s, xd_s);
      } else {
        const int pb = cur.slot.perm_base;
        stage_acts<TT>(xq, xd, hidden, n_valid, [=](int t) { return (int64_t)(ld_dep(perm + pb + g0 + t) / K); },
                       xe_s, xo_s, xd_s);
      }
      __syncthreads();
      float facc[(TT + 1) / 2];
#pragma unroll
      for (int m = 0; m < (TT + 1) / 2; ++m) facc[m] = 0.0f;
      for (int st = 0; st < nsteps; ++st, ++g) {
        prefetch();
        asm volatile("cp.async.wait_group %0;" ::"n"(kRing - 1) : "memory");
        ring_step<TT>(ring, g % kRing, 32 * st, nb, n_valid, xe_s, xo_s, xd_s, Sw, facc);
      }
#pragma unroll
      for (int m = 0; m < (TT + 1) / 2; ++m) {
        const int t = ct + 2 * m;
        const float val = __fmul_rn(s_lane, facc[m]);
        const float u = __shfl_down_sync(0xffffffffu, val, 8);
        if (cr < 8 && t < n_valid && t < TT)
          Hs[t * 32 + 8 * warp + cr] = __fmul_rn(__fmul_rn(val, sigmoid_cw(val)), u);
      }
      __syncthreads();
      for (int t = warp; t < n_valid; t += kWarps) {
        const float v = Hs[t * 32 + lane];
        const float d = __fdiv_rn(warp_max(fabsf(v)), 127.0f);
        const int64_t row = cur.slot.row_base + g0 + t;
        hq[row * inter + cur.r0 + lane] = (int8_t)q8_of(v, d);
        if (lane == 0) hd[row * (inter / 32) + (cur.r0 / 32)] = d;
      }
    }
    cur.it += gridDim.x;
    resolve(cur);
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// Stage n_valid Q8 rows of h into one warp's even/odd planes (lane-strided,
// warp-private staging).
__device__ __forceinline__ void stage_rows_warp(const int8_t* aq, const float* ad, int dim_in, int64_t row0,
                                                int n_valid, uint4* xe_s, uint4* xo_s, float* xd_s) {
  const int nb = dim_in / 32;
  const int lane = threadIdx.x & 31;
  for (int i = lane; i < n_valid * nb; i += 32) {
    const int t = i / nb, b = i - t * nb;
    const int64_t row = row0 + t;
    const uint4* src = reinterpret_cast<const uint4*>(aq + row * dim_in + 32 * b);
    const uint4 a0 = ld_dep(src), a1 = ld_dep(src + 1);
    uint4 e, o;
    split_even_odd(a0.x, a0.y, e.x, o.x);
    split_even_odd(a0.z, a0.w, e.y, o.y);
    split_even_odd(a1.x, a1.y, e.z, o.z);
    split_even_odd(a1.z, a1.w, e.w, o.w);
    xe_s[t * nb + b] = e;
    xo_s[t * nb + b] = o;
    xd_s[t * nb + b] = ld_dep(ad + row * nb + b);
  }
}

template <int TT>
struct DownSmem {
  __host__ __device__ static size_t warp_bytes(int inter) {  // multiple of 16 B
    const int nb = inter / 32;
    return ((size_t)kRing * kStepU4 * 16 + (size_t)TT * nb * 36 + (size_t)TT * kRows * kSPad * 4 + 15) & ~size_t(15);
  }
  __host__ __device__ static size_t bytes(int inter, int n_tok, int K, int n_shared) {
    return kWarps * warp_bytes(inter) + (size_t)(n_tok * K + n_tok * n_shared) * kRows * 4;
  }
};

// Down projection + combine.  Items: 16-row chunks of the output; for its
// item a warp takes expert slots w, w+4, ... (shared experts first) and
// streams their 16 down rows through its ring; the y values of the chunk
// land in shared memory by buffer row (perm position, or n_tok*K + s*n_tok
// + t for shared expert s); then each (token, row) is combined in rank order
// (contract C) and written to out.
template <int TT>
__global__ void __launch_bounds__(kThreads) down_stream_kernel(
    const __grid_constant__ DownTable tbl, const Slot* slots, const int32_t* n_slots, int n_tok, int K, int E,
    int n_shared, const int8_t* hq, const float* hd, const int32_t* inv, const float* w, int hidden, int inter,
    float* __restrict__ out) {
  extern __shared__ __align__(16) unsigned char smem[];
  pdl_wait();  // h (gate/up kernel) and the slot table are complete
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cr = lane & 15, ct = lane >> 4;
  const int nb = inter / 32, nsteps = (nb + 31) / 32;
  const int n_total = n_shared + ld_dep(n_slots);
  const int n_items = hidden / kRows;
  const size_t rb = (size_t)inter / 2;
  unsigned char* wbase = smem + warp * DownSmem<TT>::warp_bytes(inter);
  uint4* ring = reinterpret_cast<uint4*>(wbase);
  uint4* xe_s = ring + kRing * kStepU4;
  uint4* xo_s = xe_s + TT * nb;
  float* xd_s = reinterpret_cast<float*>(xo_s + TT * nb);
  int32_t* Sw = reinterpret_cast<int32_t*>(xd_s + TT * nb);
  float* ys = reinterpret_cast<float*>(smem + kWarps * DownSmem<TT>::warp_bytes(inter));

  auto slot_of = [&](int si) -> Slot {
    return si < n_shared ? shared_slot(si, n_tok, K, E) : load_slot_dep(slots + si - n_shared);
  };
  // the warp's stream: items it = blockIdx.x + k*gridDim.x; in each, slots
  // si = warp + 4j < n_total; in each, groups x steps
  int pf_it = blockIdx.x, pf_si = warp, pf_step = 0, g_pf = 0;
  Slot pf_slot = (pf_it < n_items && pf_si < n_total) ? slot_of(pf_si) : Slot{0, 0, 0, -1};
  auto advance_pf = [&]() {  // to the next (slot, item) with work for this warp
    pf_step = 0;
    pf_si += kWarps;
    while (pf_it < n_items && pf_si >= n_total) {
      pf_it += gridDim.x;
      pf_si = warp;
    }
    if (pf_it < n_items) pf_slot = slot_of(pf_si);
  };
  if (pf_it < n_items && pf_si >= n_total) advance_pf();
  auto prefetch = [&]() {
    if (pf_it < n_items) {
      const int st = pf_step % nsteps;
      const uint8_t* base = tbl.down_q[pf_slot.table_idx] + (size_t)(pf_it * kRows) * rb;
      ring_fill(ring, g_pf % kRing, base, base + 8 * rb, rb, 32 * st + lane, nb);
      if (++pf_step == ((pf_slot.count + TT - 1) / TT) * nsteps) advance_pf();
    } else {
      asm volatile("cp.async.commit_group;" ::: "memory");
    }
    ++g_pf;
  };
#pragma unroll
  for (int i = 0; i < kRing - 1; ++i) prefetch();

  int g = 0;
  for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
    const int o0 = it * kRows;
    for (int si = warp; si < n_total; si += kWarps) {
      const Slot slot = slot_of(si);
      const float s_lane = tbl.down_s[slot.table_idx][o0 + cr];
      for (int g0 = 0; g0 < slot.count; g0 += TT) {
        const int n_valid = min(TT, slot.count - g0);
        stage_rows_warp(hq, hd, inter, (int64_t)slot.row_base + g0, n_valid, xe_s, xo_s, xd_s);
        __syncwarp();
        float facc[(TT + 1) / 2];
#pragma unroll
        for (int m = 0; m < (TT + 1) / 2; ++m) facc[m] = 0.0f;
        for (int st = 0; st < nsteps; ++st, ++g) {
          prefetch();
          asm volatile("cp.async.wait_group %0;" ::"n"(kRing - 1) : "memory");
          ring_step<TT>(ring, g % kRing, 32 * st, nb, n_valid, xe_s, xo_s, xd_s, Sw, facc);
        }
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
      for (int k = 0; k < K; ++k) acc = __fmaf_rn(ld_dep(w + t * K + k), ys[ld_dep(inv + t * K + k) * kRows + r], acc);
      for (int s2 = 0; s2 < n_shared; ++s2) acc = __fadd_rn(acc, ys[(n_tok * K + s2 * n_tok + t) * kRows + r]);
      out[(int64_t)t * hidden + o0 + r] = acc;
    }
    __syncthreads();
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
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

// Resident CTAs of a persistent kernel on the current device (cached per
// kernel instance and device).
template <typename KernelT>
cudaError_t persistent_grid(KernelT* k, size_t smem, int (&cache)[64], int& ctas) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (cache[dev] == 0) {
    int sms = 0, per = 0;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, k, kThreads, smem)) != cudaSuccess) return e;
    cache[dev] = sms * (per > 0 ? per : 1);
  }
  ctas = cache[dev];
  return cudaSuccess;
}

template <int TT>
cudaError_t gateup_stream_tt(const GateUpTable& tbl, const Slot* slots, const int32_t* n_slots, const int32_t* perm,
                             int n_tok, int K, int E, int n_shared, const float* x, const int8_t* xq, const float* xd,
                             int hidden, int inter, int8_t* hq, float* hd, cudaStream_t st) {
  static int mask = 0;
  static int cache[64] = {};
  cudaError_t e = allow_smem(gateup_stream_kernel<TT>, mask);
  if (e != cudaSuccess) return e;
  const size_t smem = StreamSmem<TT>::bytes(hidden);
  int ctas = 0;
  if ((e = persistent_grid(gateup_stream_kernel<TT>, smem, cache, ctas)) != cudaSuccess) return e;
  const int max_routed = n_tok * K < E ? n_tok * K : E;
  const int items = (n_shared + max_routed) * (inter / 32);
  return launch_pdl(gateup_stream_kernel<TT>, dim3(items < ctas ? items : ctas), dim3(kThreads), smem, st, true,
                    tbl, slots, n_slots, perm, n_tok, K, E, n_shared, max_routed, x, xq, xd, hidden, inter, hq, hd);
}

template <int TT>
cudaError_t down_stream_tt(const DownTable& tbl, const Slot* slots, const int32_t* n_slots, int n_tok, int K, int E,
                           int n_shared, const int8_t* hq, const float* hd, const int32_t* inv, const float* w,
                           int hidden, int inter, float* out, cudaStream_t st) {
  static int mask = 0;
  static int cache[64] = {};
  cudaError_t e = allow_smem(down_stream_kernel<TT>, mask);
  if (e != cudaSuccess) return e;
  const size_t smem = DownSmem<TT>::bytes(inter, n_tok, K, n_shared);
  int ctas = 0;
  if ((e = persistent_grid(down_stream_kernel<TT>, DownSmem<TT>::bytes(inter, kDecodeMaxTok, kMaxTopK, kMaxShared), cache,
                           ctas)) != cudaSuccess)
    return e;
  const int items = hidden / kRows;
  return launch_pdl(down_stream_kernel<TT>, dim3(items < ctas ? items : ctas), dim3(kThreads), smem, st, true, tbl,
                    slots, n_slots, n_tok, K, E, n_shared, hq, hd, inv, w, hidden, inter, out);
}

}  // namespace

cudaError_t launch_gateup_decode(const GateUpTable& tbl, const Slot* slots, const int32_t* n_slots,
                                 const int32_t* perm, int n_tok, int K, int E, int n_shared, const float* x,
                                 const int8_t* xq, const float* xd, int hidden, int inter, int8_t* hq, float* hd,
                                 cudaStream_t st) {
  if (n_tok <= 1)
    return gateup_stream_tt<1>(tbl, slots, n_slots, perm, n_tok, K, E, n_shared, x, xq, xd, hidden, inter, hq, hd, st);
  if (n_tok <= 2)
    return gateup_stream_tt<2>(tbl, slots, n_slots, perm, n_tok, K, E, n_shared, x, xq, xd, hidden, inter, hq, hd, st);
  return gateup_stream_tt<4>(tbl, slots, n_slots, perm, n_tok, K, E, n_shared, x, xq, xd, hidden, inter, hq, hd, st);
}

cudaError_t launch_down_combine(const DownTable& tbl, const Slot* slots, const int32_t* n_slots, int n_tok, int K,
                                int E, int n_shared, const int8_t* hq, const float* hd, const int32_t* inv,
                                const float* w, int hidden, int inter, float* out, cudaStream_t st) {
  if (n_tok <= 1) return down_stream_tt<1>(tbl, slots, n_slots, n_tok, K, E, n_shared, hq, hd, inv, w, hidden, inter, out, st);
  if (n_tok <= 2) return down_stream_tt<2>(tbl, slots, n_slots, n_tok, K, E, n_shared, hq, hd, inv, w, hidden, inter, out, st);
  return down_stream_tt<4>(tbl, slots, n_slots, n_tok, K, E, n_shared, hq, hd, inv, w, hidden, inter, out, st);
}

}  // namespace coli
