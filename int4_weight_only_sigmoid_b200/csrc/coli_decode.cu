// coli_decode.cu -- the expert kernels of a decode batch (n_tok <= 16).
//
//   router_decode (plain launch; also writes the Q8_0 of x)
//     -> topk_bucket_small (PDL)
//     -> gateup_ring (PDL): persistent 4-warp CTAs; items (expert slot, 64
//        intermediate outputs), shared experts first: those do not depend on
//        the routing and start while it runs
//     -> down_cta (PDL): persistent; items (expert slot, 32*W output rows)
//        for a W-warp CTA, token groups of <= TT -> y
//     -> combine_decode (PDL): out = contract C over y
//
// Weight streaming.  Every warp owns a ring of stages of 32 weight rows x 16
// packed blocks (8 KB; one row per lane, blocks XOR-swizzled within a row so
// the lanes' reads do not conflict).  The warp fills the stages with cp.async (each
// instruction copies 256-byte pieces of two rows) one or two steps ahead of
// the step it computes, across item boundaries, so the stream does not drain
// between items.  The down kernel fetches a group's h rows once per CTA with
// bulk copies on an mbarrier; that wait is bounded (about a second): on
// expiry the CTA raises its abort flag, records the error in the status
// word, runs on without waiting (the output is then garbage) and, before it
// exits, waits (bounded again) for the copies it still has in flight.
//
// Arithmetic: lane l holds weight row l; for each block in ascending order it
// unpacks the 16 bytes once ((w << 4) & 0xF0F0F0F0 and w & 0xF0F0F0F0 are
// 16*q of the even and odd elements as signed bytes), takes the dp4a block
// sum against every staged token (even / odd byte planes, read as
// broadcasts) and folds it into that token's chain (contract F).  SwiGLU,
// the Q8_0 of h and the combine follow the same contracts as coli_gemv.cu,
// so the output is bit-identical to the general path.
//
// The decode path stores h as "plane" rows: within every 32-element block the
// 16 even elements come first, then the 16 odd ones, which is the layout the
// down kernel's dot wants; only the decode kernels read it.
//
// Sources: "Colibri：在笔记本上跑744B参数的AI模型", "关键特性" (integer dot
// kernels, Q8_0 activations); "GLM-5.2-colibri-int4架构解析…", "MoE的工作原理"
// (weighted combine), "GLM-5.2的MoE实现" (shared expert); HN summary,
// "已实现的功能" (batched MoE).
#include "coli_stream.cuh"

namespace coli {
namespace {

using namespace gemv;
using namespace stream;

constexpr int kMaxWarpsDown = 12;
constexpr int kErrDownH = 22;  // status word: the down kernel gave up waiting for h rows

// ---------------------------------------------------------------------------
// gate/up + SwiGLU + Q8_0 of h

template <int TT>
struct GateUpSmem {
  static constexpr int R = ring_depth<TT>();
  __host__ __device__ static size_t ring() { return (size_t)kWarps * R * kStageBytes; }
  __host__ __device__ static size_t xs(int nb) { return (size_t)TT * nb * 32; }
  __host__ __device__ static size_t xsd(int nb) { return (size_t)TT * nb * 4; }
  __host__ __device__ static size_t bytes(int hidden) {
    const int nb = hidden / 32;
    return ring() + xs(nb) + xsd(nb) + (size_t)TT * 64 * 4;
  }
};

struct Item {
  int it;  // item index
  bool valid;
  Slot slot;
  int r0;      // first intermediate output of the item
  int groups;  // token groups of <= TT tokens
};

// Items: (expert slot y, 64 intermediate outputs), slot-major, shared experts
// first; warp w holds gate rows r0+16w..+15 on lanes 0..15 and the matching
// up rows on lanes 16..31.  The staged tokens are kept while consecutive
// groups use the same token list (a 1-token batch stages x once per CTA).
template <int TT>
__global__ void __launch_bounds__(kThreads, 3) gateup_ring_kernel(
    const __grid_constant__ GateUpTable tbl, const Slot* slots, const int32_t* n_slots, const int32_t* perm, int n_tok,
    int K, int E, int n_shared, int max_routed, const float* x, const int8_t* xq, const float* xd, int hidden,
    int inter, int8_t* hq, float* hd) {
  extern __shared__ __align__(1024) unsigned char smem[];
  using SM = GateUpSmem<TT>;
  constexpr int R = SM::R;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nb = hidden / 32, nsteps = (nb + kBlkStep - 1) / kBlkStep;
  const int nchunk = inter / 64;
  const int n_items = (n_shared + max_routed) * nchunk;
  const size_t rb = (size_t)hidden / 2;
  uint4* ring = reinterpret_cast<uint4*>(smem) + warp * R * kStageU4;
  uint4* xs = reinterpret_cast<uint4*>(smem + SM::ring());
  float* xsd = reinterpret_cast<float*>(smem + SM::ring() + SM::xs(nb));
  float* Hs = reinterpret_cast<float*>(smem + SM::ring() + SM::xs(nb) + SM::xsd(nb));

  bool waited = false;
  auto resolve = [&](Item& c) {
    c.valid = false;
    if (c.it >= n_items) return;
    const int yy = c.it / nchunk;
    c.r0 = (c.it - yy * nchunk) * 64;
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
  // Copy the next step into ring slot g_pf % R: lane l copies block l & 15 of
  // rows 2k + (l >> 4), k = 0..15 (two 256-byte row pieces per instruction);
  // every call commits one cp.async group, empty at the end of the work.
  auto prefetch = [&]() {
    if (!pf.valid) {
      asm volatile("cp.async.commit_group;" ::: "memory");
      return;
    }
    const int st = pf_step % nsteps;
    const int s = g_pf % R;
    const int ti = pf.slot.table_idx;
    const int j = lane & 15, rsub = lane >> 4;
    const size_t off = (size_t)(pf.r0 + 16 * warp) * rb + (size_t)kBlkStep * 16 * st + 16 * j;
    const uint8_t* gb = tbl.gate_q[ti] + off;
    const uint8_t* ub = tbl.up_q[ti] + off;
    uint4* dst = ring + s * kStageU4;
    if (j < min(kBlkStep, nb - kBlkStep * st)) {
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const int r = 2 * k + rsub;
        cp_async16(dst + stage_slot(r, j), (k < 8 ? gb : ub) + (size_t)(r & 15) * rb);
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    ++g_pf;
    if (++pf_step == pf.groups * nsteps) {
      pf_step = 0;
      pf.it += gridDim.x;
      resolve(pf);
    }
  };
#pragma unroll
  for (int i = 0; i < R - 1; ++i) prefetch();

  int staged_n = -1;
  int staged_tok[TT];
#pragma unroll
  for (int t = 0; t < TT; ++t) staged_tok[t] = -1;

  while (cur.valid) {
    const int ti = cur.slot.table_idx;
    const int o_lane = cur.r0 + 16 * warp + (lane & 15);
    const float s_lane = lane < 16 ? tbl.gate_s[ti][o_lane] : tbl.up_s[ti][o_lane];
    const bool is_shared = cur.slot.perm_base < 0;
    for (int grp = 0; grp < cur.groups; ++grp) {
      const int g0 = grp * TT;
      const int n_valid = min(TT, cur.slot.count - g0);
      int tok[TT];
      bool same = n_valid == staged_n;
#pragma unroll
      for (int t = 0; t < TT; ++t) {
        tok[t] = 0;
        if (t < n_valid) {
          tok[t] = is_shared ? g0 + t : (n_tok == 1 ? 0 : ld_dep(perm + cur.slot.perm_base + g0 + t) / K);
          if (tok[t] != staged_tok[t]) same = false;
        }
      }
      if (!same) {  // uniform over the CTA
        __syncthreads();
        if (is_shared)
          stage_x_f32<TT>(x, hidden, n_valid, tok, xs, xsd);
        else
          stage_x_q8<TT>(xq, xd, hidden, n_valid, tok, xs, xsd);
        __syncthreads();
        staged_n = n_valid;
#pragma unroll
        for (int t = 0; t < TT; ++t) staged_tok[t] = tok[t];
      }
      float acc[TT];
#pragma unroll
      for (int t = 0; t < TT; ++t) acc[t] = 0.0f;
      for (int st = 0; st < nsteps; ++st, ++g) {
        prefetch();
        const int s = g % R;
        asm volatile("cp.async.wait_group %0;" ::"n"(R - 1) : "memory");  // this lane's copies of step g
        __syncwarp();                                                        // ... and every other lane's
        rows_step<TT>(ring + s * kStageU4, kBlkStep * st, min(kBlkStep, nb - kBlkStep * st), nb, n_valid, xs, xsd,
                      acc);
      }
#pragma unroll
      for (int t = 0; t < TT; ++t) {
        const float val = __fmul_rn(s_lane, acc[t]);
        const float u = __shfl_down_sync(0xffffffffu, val, 16);
        if (lane < 16 && t < n_valid) Hs[t * 64 + 16 * warp + lane] = __fmul_rn(__fmul_rn(val, sigmoid_cw(val)), u);
      }
      __syncthreads();
      for (int p = warp; p < 2 * n_valid; p += kWarps) {
        const int t = p >> 1, blk = p & 1;
        const float v = Hs[t * 64 + 32 * blk + lane];
        const float d = __fdiv_rn(warp_max(fabsf(v)), 127.0f);
        const int64_t row = cur.slot.row_base + g0 + t;
        hq[row * inter + cur.r0 + 32 * blk + (lane & 1) * 16 + (lane >> 1)] = (int8_t)q8_of(v, d);
        if (lane == 0) hd[row * (inter / 32) + (cur.r0 / 32) + blk] = d;
      }
      __syncthreads();
    }
    cur.it += gridDim.x;
    resolve(cur);
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// ---------------------------------------------------------------------------
// down projection -> y

// Shared memory of the down kernel: a 128-byte header (abort flag, two h
// mbarriers), two h buffers of one token group each, then one ring per warp.
constexpr int kDownHeader = 128;
template <int TT>
__host__ __device__ inline size_t down_hbuf_bytes(int inter) {
  return (size_t)TT * (inter + (inter / 32) * 4);
}
template <int TT>
__host__ __device__ inline size_t down_cta_bytes(int inter, int W) {
  return kDownHeader + 2 * down_hbuf_bytes<TT>(inter) + (size_t)W * ring_depth<TT>() * kStageBytes;
}

// Items: (expert slot, 32*W consecutive output rows), slot-major, shared
// experts first; the W warps of a CTA take 32 rows each of the same slot, so
// the slot's h rows are fetched once per CTA (bulk copies on an mbarrier,
// double-buffered by token group).  Lane l computes output row o0 + l.  A
// CTA walks its units (item, token group) in order; thread 0 fetches the
// next unit's h rows while the current one computes, and a CTA barrier ends
// every unit, so a buffer is refilled only after all warps are done with it.
template <int TT>
__global__ void __launch_bounds__(kMaxWarpsDown * 32, 1) down_cta_kernel(
    const __grid_constant__ DownTable tbl, const Slot* slots, const int32_t* n_slots, int n_tok, int K, int E,
    int n_shared, const int8_t* hq, const float* hd, int hidden, int inter, float* y, int32_t* status) {
  extern __shared__ __align__(1024) unsigned char smem[];
  constexpr int R = ring_depth<TT>();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int W = blockDim.x >> 5;
  const int nb = inter / 32, nsteps = (nb + kBlkStep - 1) / kBlkStep;
  const int per_slot = hidden / (32 * W);
  const size_t rb = (size_t)inter / 2;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem);
  uint64_t* hbar = reinterpret_cast<uint64_t*>(smem + 64);
  unsigned char* hbuf = smem + kDownHeader;
  const size_t hb_bytes = down_hbuf_bytes<TT>(inter);
  uint4* ring = reinterpret_cast<uint4*>(smem + kDownHeader + 2 * hb_bytes) + (size_t)warp * R * kStageU4;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    tc::mbar_init(hbar, 1);
    tc::mbar_init(hbar + 1, 1);
    fence_mbar_init();
  }
  __syncthreads();
  pdl_wait();  // h (gate/up kernel) and the slot table are complete
  pdl_launch_dependents();
  const int n_total = n_shared + ld_dep(n_slots);
  const int n_items = n_total * per_slot;

  // a unit iterator (item, group); every thread walks the same sequence
  struct Unit {
    int it, grp, ngrp;
    Slot slot;
    bool valid;
  };
  auto resolve = [&](Unit& u) {
    u.valid = u.it < n_items;
    if (!u.valid) return;
    const int si = u.it / per_slot;
    u.slot = si < n_shared ? shared_slot(si, n_tok, K, E) : load_slot_dep(slots + si - n_shared);
    u.ngrp = (u.slot.count + TT - 1) / TT;
    u.grp = 0;
  };
  auto advance = [&](Unit& u) {
    if (++u.grp == u.ngrp) {
      u.it += gridDim.x;
      resolve(u);
    }
  };
  // thread 0: the h rows of unit k into buffer k & 1
  auto fetch_h = [&](const Unit& u, int k) {
    const int nv = min(TT, u.slot.count - u.grp * TT);
    const int64_t row0 = u.slot.row_base + u.grp * TT;
    unsigned char* dst = hbuf + (size_t)(k & 1) * hb_bytes;
    mbar_expect_tx(hbar + (k & 1), (uint32_t)(nv * (inter + nb * 4)));
    bulk_g2s(dst, hq + row0 * inter, (uint32_t)(nv * inter), hbar + (k & 1));
    bulk_g2s(dst + (size_t)TT * inter, hd + row0 * nb, (uint32_t)(nv * nb * 4), hbar + (k & 1));
  };

  // producer (per warp): the weights of the warp's 32 rows, step by step
  Unit pu;
  pu.it = blockIdx.x;
  resolve(pu);
  int pstep = 0, g_pf = 0;
  auto prefetch = [&]() {
    if (!pu.valid || *abort_flag) {
      asm volatile("cp.async.commit_group;" ::: "memory");
      return;
    }
    const int o0 = (pu.it % per_slot) * 32 * W + 32 * warp;
    const int j = lane & 15, rsub = lane >> 4;
    const uint8_t* b0p = tbl.down_q[pu.slot.table_idx] + (size_t)o0 * rb + (size_t)kBlkStep * 16 * pstep + 16 * j;
    uint4* dst = ring + (g_pf % R) * kStageU4;
    if (j < min(kBlkStep, nb - kBlkStep * pstep)) {
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const int r = 2 * k + rsub;
        cp_async16(dst + stage_slot(r, j), b0p + (size_t)r * rb);
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    ++g_pf;
    if (++pstep == nsteps) {
      pstep = 0;
      advance(pu);
    }
  };

  Unit cu;
  cu.it = blockIdx.x;
  resolve(cu);
  Unit hu = cu;  // thread 0's fetch iterator, one unit ahead of cu
  if (threadIdx.x == 0 && hu.valid) fetch_h(hu, 0);
#pragma unroll
  for (int i = 0; i < R - 1; ++i) prefetch();

  int g = 0, k = 0, first_fail = -1;
  for (; cu.valid; ++k) {
    if (threadIdx.x == 0) {  // the next unit's h rows into the other buffer (free since the last barrier)
      advance(hu);
      if (hu.valid) fetch_h(hu, k + 1);
    }
    if (!tc::mbar_wait(hbar + (k & 1), (uint32_t)((k >> 1) & 1), abort_flag, status, kErrDownH) && first_fail < 0)
      first_fail = k;
    const int nv = min(TT, cu.slot.count - cu.grp * TT);
    const int64_t row0 = cu.slot.row_base + cu.grp * TT;
    const int o = (cu.it % per_slot) * 32 * W + 32 * warp + lane;
    const float s_lane = tbl.down_s[cu.slot.table_idx][o];
    const uint4* xs = reinterpret_cast<const uint4*>(hbuf + (size_t)(k & 1) * hb_bytes);
    const float* xsd = reinterpret_cast<const float*>(hbuf + (size_t)(k & 1) * hb_bytes + (size_t)TT * inter);
    float acc[TT];
#pragma unroll
    for (int t = 0; t < TT; ++t) acc[t] = 0.0f;
    for (int st = 0; st < nsteps; ++st, ++g) {
      prefetch();
      asm volatile("cp.async.wait_group %0;" ::"n"(R - 1) : "memory");  // this lane's copies of step g
      __syncwarp();                                                        // ... and every other lane's
      rows_step<TT>(ring + (g % R) * kStageU4, kBlkStep * st, min(kBlkStep, nb - kBlkStep * st), nb, nv, xs, xsd,
                    acc);
    }
#pragma unroll
    for (int t = 0; t < TT; ++t)
      if (t < nv) y[(row0 + t) * hidden + o] = __fmul_rn(s_lane, acc[t]);
    advance(cu);
    __syncthreads();  // every warp is done with h buffer k & 1
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  if (threadIdx.x == 0 && first_fail >= 0)  // h copies that may still be in flight
    for (int kk = first_fail; kk <= k; ++kk) mbar_drain(hbar + (kk & 1), (uint32_t)((kk >> 1) & 1));
}

// out[t] = sum_k w[t,k] y[inv[t,k]] + sum_s y[shared row s of t] (contract C).
__global__ void __launch_bounds__(256) combine_decode_kernel(const float* y, const int32_t* inv, const float* w,
                                                             int n_tok, int K, int n_shared, int H,
                                                             float* __restrict__ out) {
  pdl_wait();
  const int t = blockIdx.y;
  const int o = blockIdx.x * blockDim.x + threadIdx.x;
  if (o >= H) return;
  float acc = 0.0f;
  for (int k = 0; k < K; ++k) {
    const int64_t j = ld_dep(inv + t * K + k);
    acc = __fmaf_rn(ld_dep(w + t * K + k), ld_dep(y + j * H + o), acc);
  }
  for (int s = 0; s < n_shared; ++s)
    acc = __fadd_rn(acc, ld_dep(y + ((int64_t)n_tok * K + (int64_t)s * n_tok + t) * H + o));
  out[(int64_t)t * H + o] = acc;
}

// ---------------------------------------------------------------------------
// launchers

template <typename KernelT>
cudaError_t allow_smem(KernelT* k, size_t bytes, size_t (&granted)[64]) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (granted[dev] >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) granted[dev] = bytes;
  return e;
}

cudaError_t sm_count(int& sms) {
  static int cache[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (cache[dev] == 0 && (e = cudaDeviceGetAttribute(&cache[dev], cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  sms = cache[dev];
  return cudaSuccess;
}

template <int TT>
cudaError_t gateup_ring_tt(const GateUpTable& tbl, const Slot* slots, const int32_t* n_slots, const int32_t* perm,
                           int n_tok, int K, int E, int n_shared, const float* x, const int8_t* xq, const float* xd,
                           int hidden, int inter, int8_t* hq, float* hd, int32_t* status, cudaStream_t st) {
  static size_t granted[64] = {};
  static int per_sm[64] = {};
  const size_t smem = GateUpSmem<TT>::bytes(hidden);
  cudaError_t e = allow_smem(gateup_ring_kernel<TT>, smem, granted);
  if (e != cudaSuccess) return e;
  int sms = 0, dev = 0;
  if ((e = sm_count(sms)) != cudaSuccess || (e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if (per_sm[dev] == 0) {
    int per = 0;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, gateup_ring_kernel<TT>, kThreads, smem)) !=
        cudaSuccess)
      return e;
    per_sm[dev] = per > 0 ? per : 1;
  }
  const int ctas = sms * per_sm[dev];
  const int max_routed = n_tok * K < E ? n_tok * K : E;
  const int items = (n_shared + max_routed) * (inter / 64);
  return launch_pdl(gateup_ring_kernel<TT>, dim3(items < ctas ? items : ctas), dim3(kThreads), smem, st, true, tbl,
                    slots, n_slots, perm, n_tok, K, E, n_shared, max_routed, x, xq, xd, hidden, inter, hq, hd);
}

// Warps per down CTA: the largest W <= kMaxWarpsDown that fits shared
// memory and divides hidden into 32*W-row items.
template <int TT>
int down_warps(int hidden, int inter) {
  for (int W = kMaxWarpsDown; W >= 1; --W)
    if (hidden % (32 * W) == 0 && down_cta_bytes<TT>(inter, W) <= (size_t)kSmemLimit) return W;
  return 0;
}

template <int TT>
cudaError_t down_cta_tt(const DownTable& tbl, const Slot* slots, const int32_t* n_slots, int n_tok, int K, int E,
                        int n_shared, const int8_t* hq, const float* hd, int hidden, int inter, float* y,
                        int32_t* status, cudaStream_t st) {
  static size_t granted[64] = {};
  int sms = 0;
  cudaError_t e = sm_count(sms);
  if (e != cudaSuccess) return e;
  const int W = down_warps<TT>(hidden, inter);
  if (W < 1) return cudaErrorInvalidConfiguration;
  const size_t smem = down_cta_bytes<TT>(inter, W);
  if ((e = allow_smem(down_cta_kernel<TT>, smem, granted)) != cudaSuccess) return e;
  const int max_items = (n_shared + (n_tok * K < E ? n_tok * K : E)) * (hidden / (32 * W));
  const int ctas = max_items < sms ? max_items : sms;
  return launch_pdl(down_cta_kernel<TT>, dim3(ctas), dim3(32 * W), smem, st, true, tbl, slots, n_slots, n_tok, K, E,
                    n_shared, hq, hd, hidden, inter, y, status);
}

}  // namespace

bool decode_supported(int hidden, int inter) {
  if (hidden % 128 != 0 || inter % 128 != 0) return false;
  return GateUpSmem<4>::bytes(hidden) <= (size_t)kSmemLimit && down_warps<4>(hidden, inter) >= 1;
}

cudaError_t launch_gateup_decode(const GateUpTable& tbl, const Slot* slots, const int32_t* n_slots,
                                 const int32_t* perm, int n_tok, int K, int E, int n_shared, const float* x,
                                 const int8_t* xq, const float* xd, int hidden, int inter, int8_t* hq, float* hd,
                                 int32_t* status, cudaStream_t st) {
  if (n_tok <= 1)
    return gateup_ring_tt<1>(tbl, slots, n_slots, perm, n_tok, K, E, n_shared, x, xq, xd, hidden, inter, hq, hd,
                             status, st);
  if (n_tok <= 2)
    return gateup_ring_tt<2>(tbl, slots, n_slots, perm, n_tok, K, E, n_shared, x, xq, xd, hidden, inter, hq, hd,
                             status, st);
  return gateup_ring_tt<4>(tbl, slots, n_slots, perm, n_tok, K, E, n_shared, x, xq, xd, hidden, inter, hq, hd,
                           status, st);
}

cudaError_t launch_down_decode(const DownTable& tbl, const Slot* slots, const int32_t* n_slots, int n_tok, int K,
                               int E, int n_shared, const int8_t* hq, const float* hd, const int32_t* inv,
                               const float* w, int hidden, int inter, float* y, float* out, int32_t* status,
                               cudaStream_t st) {
  cudaError_t e;
  if (n_tok <= 1)
    e = down_cta_tt<1>(tbl, slots, n_slots, n_tok, K, E, n_shared, hq, hd, hidden, inter, y, status, st);
  else if (n_tok <= 2)
    e = down_cta_tt<2>(tbl, slots, n_slots, n_tok, K, E, n_shared, hq, hd, hidden, inter, y, status, st);
  else
    e = down_cta_tt<4>(tbl, slots, n_slots, n_tok, K, E, n_shared, hq, hd, hidden, inter, y, status, st);
  if (e != cudaSuccess) return e;
  return launch_pdl(combine_decode_kernel, dim3((hidden + 255) / 256, n_tok), dim3(256), 0, st, true, y, inv, w,
                    n_tok, K, n_shared, hidden, out);
}

}  // namespace coli
