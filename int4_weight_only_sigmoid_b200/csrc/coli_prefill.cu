// coli_prefill.cu -- the expert kernels for many tokens per expert (prefill):
// a grouped GEMM on the 5th-generation tensor cores (tcgen05.mma, F32
// accumulators in tensor memory).  Work items are (tile of <= 64 of one
// slot's tokens, 128 output rows); one persistent CTA per SM walks items
// c, c + G, ... and keeps its pipeline (producers -> MMA -> fold) running
// from one item to the next.
//
// Exactness.  Each Q8 block's partial sum must come out exactly, because the
// row fold (contract F: acc = fmaf(d_x[b], (float)isum[b], acc), b
// ascending) needs it per block.  The operands are therefore fp16, in which
// every int4 weight (-8..7) and every Q8 activation (-127..127) is exact;
// the MMA of one 32-element block (two K=16 steps) accumulates products of
// at most 8*127 into an F32 sum of magnitude at most 32512 < 2^24, so every
// partial sum is an exact integer in F32 whatever the tensor core's internal
// order.  The MMA of block b writes a fresh accumulator; the fold warps then
// fold it with d_x[b] in ascending b.  The results equal the dp4a path's bit
// for bit.
//
// Why fp16 operands and not kind::i8: the fold costs one F32 FMA per
// (row, token, block) whatever the MMA kind; with kind::i8 each of those
// also needs an int32 -> F32 conversion, and the CUDA-core fold, not the
// tensor pipe, is the limit of this layer (one FMA per 32 MACs).  fp16
// operands give F32 sums directly.
//
// Operands.  The activations are converted to fp16 once per forward
// (act_f16_kernel; the gate/up fold writes h straight as fp16 for the down
// kernel), in the element order [0,2,4,6,1,3,5,7] of every 8 that the int4
// expansion produces; a tile's B operand is then a gather of 16-byte pieces
// by cp.async.  The packed weights of a block are copied by the producer
// thread that later expands them (each thread owns one row of each matrix),
// so no producer thread waits for another.
//
// Roles (416 threads): warps 0-3 producers, warp 4 the MMA issuer (lane 0)
// and TMEM owner, warps 5-12 the fold (warp w reads TMEM lanes
// 32(w%4).. = 32 of the item's rows, columns [32h, 32h+32) with
// h = (w-5)/4 = half of the tokens).  Per block g: the producers copy (kLook
// blocks ahead, all by cp.async) into operand stage g % kStages (after
// `empty`, raised by the MMA's commit) and the block's token scales into
// scale stage g % kStages (after `dempty`, raised by the fold warps), expand
// the weights and arrive on `full`; the MMA writes TMEM buffer g % kTBufs
// (after `tempty`) and commits `empty` and `tfull`.  All waits are
// bounded (coli_tc.cuh).
//
// Sources: "Colibri：在笔记本上跑744B参数的AI模型", "关键特性" (integer dot
// kernels, Q8_0 activations, packed int4); HN summary (hn.213312.xyz),
// "已实现的功能" (batched MoE: in prefill, an expert used by several
// positions is read once and shared).
#include <cuda_fp16.h>

#include "coli_launch.h"
#include "coli_tc.cuh"

namespace coli {
namespace {

using namespace tc;

constexpr int kM = 128;        // rows per item (TMEM lanes)
constexpr int kN = 64;         // tokens per tile (max)
constexpr int kStages = 8;     // operand / scale ring depth (blocks)
constexpr int kLook = 6;       // blocks the producers' copies run ahead
constexpr int kTBufs = 4;      // TMEM accumulator buffers (blocks the MMA may run ahead of the fold)
constexpr int kProdWarps = 4;
constexpr int kEpiWarps = 8;   // 2 per TMEM lane quadrant, each half of the columns
constexpr int kMmaWarp = kProdWarps;
constexpr int kEpi0 = kProdWarps + 1;                          // first fold warp
constexpr int kThreadsP = 32 * (kProdWarps + 1 + kEpiWarps);  // 416
constexpr int kNProd = 32 * kProdWarps;                        // 128 producer threads
constexpr int kNEpi = 32 * kEpiWarps;                          // 256 fold threads

template <bool GU>
struct PSmem {
  static constexpr int kMats = GU ? 2 : 1;
  static constexpr int kOpA = kM * 64;                 // one matrix: 128 rows x 32 fp16
  static constexpr int kOpB = kN * 64;                 // 64 tokens x 32 fp16
  static constexpr int kOpStage = kMats * kOpA + kOpB;
  static constexpr int kPk = kMats * kM * 16;          // packed weights of one block
  static constexpr int kTmemCols = kTBufs * kMats * kN;  // 4 buffers x (gate, up | down) x 64
  __host__ __device__ static constexpr size_t bytes() {
    return 1024 + (size_t)kStages * kOpStage + (size_t)(kLook + 1) * kPk + (size_t)kStages * kN * 4;
  }
};

struct Tile {
  int32_t slot, n0;
};

// fp16 operands from packed int4: 8 nibbles of one 32-bit word -> 8 fp16 in
// the order [0,2,4,6,1,3,5,7] (the activations use the same order, so the
// dot product is unchanged).  fp16 bits 0x6400 | u are 1024 + u exactly; with
// u = q + 8 (offset nibble), subtracting 1032 leaves q exactly.
__device__ __forceinline__ uint4 expand_int4_word(uint32_t w) {
  const uint32_t u = w ^ 0x88888888u;
  const uint32_t lo = u & 0x0F0F0F0Fu;
  const uint32_t hi = (u >> 4) & 0x0F0F0F0Fu;
  const uint32_t c = 0x64646464u;
  const __half2 off = __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408));  // 1032, 1032
  uint32_t r[4] = {__byte_perm(lo, c, 0x4140), __byte_perm(lo, c, 0x4342), __byte_perm(hi, c, 0x4140),
                   __byte_perm(hi, c, 0x4342)};
  uint4 o;
  __half2 h;
  h = __hsub2(*reinterpret_cast<__half2*>(&r[0]), off);
  o.x = *reinterpret_cast<uint32_t*>(&h);
  h = __hsub2(*reinterpret_cast<__half2*>(&r[1]), off);
  o.y = *reinterpret_cast<uint32_t*>(&h);
  h = __hsub2(*reinterpret_cast<__half2*>(&r[2]), off);
  o.z = *reinterpret_cast<uint32_t*>(&h);
  h = __hsub2(*reinterpret_cast<__half2*>(&r[3]), off);
  o.w = *reinterpret_cast<uint32_t*>(&h);
  return o;
}

// fp16 operands from 8 int8 values (words a = x0..x3, b = x4..x7), same
// element order: with u = x + 128, 0x6400 | u is 1024 + u; minus 1152 is x.
__device__ __forceinline__ uint4 expand_int8_pair(uint32_t a, uint32_t b) {
  const uint32_t ua = a ^ 0x80808080u, ub = b ^ 0x80808080u;
  const uint32_t c = 0x64646464u;
  const __half2 off = __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480));  // 1152, 1152
  uint32_t r[4] = {__byte_perm(ua, c, 0x4240), __byte_perm(ub, c, 0x4240), __byte_perm(ua, c, 0x4341),
                   __byte_perm(ub, c, 0x4341)};
  uint4 o;
  __half2 h;
  h = __hsub2(*reinterpret_cast<__half2*>(&r[0]), off);
  o.x = *reinterpret_cast<uint32_t*>(&h);
  h = __hsub2(*reinterpret_cast<__half2*>(&r[1]), off);
  o.y = *reinterpret_cast<uint32_t*>(&h);
  h = __hsub2(*reinterpret_cast<__half2*>(&r[2]), off);
  o.z = *reinterpret_cast<uint32_t*>(&h);
  h = __hsub2(*reinterpret_cast<__half2*>(&r[3]), off);
  o.w = *reinterpret_cast<uint32_t*>(&h);
  return o;
}

// Position of element e (0..7) of an 8-group in the operand order.
__device__ __forceinline__ int op_pos8(int e) { return (e & 1) ? 4 + (e >> 1) : (e >> 1); }

// Byte offset of 16-byte chunk c (0..3) of row r in a K-major, no-swizzle
// operand tile of 32 fp16 per row: 8-row x 16-byte core matrices, the four
// K chunks of an 8-row group 128 B apart (LBO), groups 512 B apart (SBO).
__device__ __forceinline__ uint32_t op_off(int r, int c) { return (r >> 3) * 512 + c * 128 + (r & 7) * 16; }

// Q8 rows (int8) -> fp16 operand rows, 8 values per thread.
__global__ void __launch_bounds__(256) act_f16_kernel(const int8_t* __restrict__ q, int64_t n8,
                                                      uint4* __restrict__ out) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const uint2 v = reinterpret_cast<const uint2*>(q)[i];
  out[i] = expand_int8_pair(v.x, v.y);
}

// fma on two F32 lanes at once (two IEEE fmas, each rounded once).
__device__ __forceinline__ void fma2(float& a0, float& a1, float d0, float d1, float x0, float x1) {
  unsigned long long acc, dd, xx;
  asm("mov.b64 %0, {%1,%2};" : "=l"(acc) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1,%2};" : "=l"(dd) : "f"(d0), "f"(d1));
  asm("mov.b64 %0, {%1,%2};" : "=l"(xx) : "f"(x0), "f"(x1));
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(dd), "l"(xx));
  asm("mov.b64 {%0,%1}, %2;" : "=f"(a0), "=f"(a1) : "l"(acc));
}

struct ItemInfo {
  Slot slot;
  int n0, n_valid, n_pad, m0;
};

__device__ __forceinline__ ItemInfo item_info(const Slot* slots, const Tile* tiles, int item, int nm) {
  ItemInfo f;
  const int t = item / nm;
  const Tile tile = tiles[t];
  f.slot = slots[tile.slot];
  f.n0 = tile.n0;
  f.n_valid = min(kN, f.slot.count - tile.n0);
  f.n_pad = (f.n_valid + 15) & ~15;
  f.m0 = (item - t * nm) * kM;
  return f;
}

// GU: gate/up (+ SwiGLU + Q8 of h -> hf fp16 rows + hd); !GU: down (-> y).
template <bool GU, typename Tab>
__global__ void __launch_bounds__(kThreadsP, 1) prefill_kernel(
    const __grid_constant__ Tab tab, const Slot* __restrict__ slots, const Tile* __restrict__ tiles,
    const int32_t* __restrict__ n_tiles, const int32_t* __restrict__ perm, int top_k, const __half* act,
    const float* ad, int hidden, int inter, __half* hf, float* hd, float* __restrict__ y,
    int32_t* __restrict__ err) {
  using L = PSmem<GU>;
  __shared__ uint64_t full_bar[kStages], empty_bar[kStages], dempty_bar[kStages], tfull_bar[kTBufs],
      tempty_bar[kTBufs], done_bar;
  __shared__ uint32_t tmem_s;
  __shared__ int abort_s;
  extern __shared__ unsigned char smem_raw[];

  const int dim_in = GU ? hidden : inter;
  const int dim_out = GU ? inter : hidden;
  const int nb = dim_in / 32;
  const int nm = dim_out / kM;
  const int n_items = *n_tiles * nm;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);  // 1 KB aligned
  unsigned char* op_ring = smem;
  unsigned char* pk_ring = op_ring + kStages * L::kOpStage;
  float* d_ring = reinterpret_cast<float*>(pk_ring + (kLook + 1) * L::kPk);  // [kStages][kN]

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], kNProd);
      mbar_init(&empty_bar[s], 1);
      mbar_init(&dempty_bar[s], kNEpi);
    }
    for (int b = 0; b < kTBufs; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], kNEpi);
    }
    mbar_init(&done_bar, 1);
    abort_s = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kMmaWarp) tmem_alloc(&tmem_s, L::kTmemCols);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = tmem_s;
  volatile int* abort = &abort_s;

  if (warp < kProdWarps) {
    // ------------------------------------------------------------ producers
    const int p = threadIdx.x;  // row p of each matrix; B pieces of token row p >> 1
    const size_t rb = (size_t)dim_in / 2;
    int g = 0;  // global block counter
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
      const ItemInfo f = item_info(slots, tiles, item, nm);
      auto tok_of = [&](int n) -> int64_t {
        if (!GU) return (int64_t)f.slot.row_base + f.n0 + n;
        return f.slot.perm_base < 0 ? (int64_t)(f.n0 + n) : (int64_t)(perm[f.slot.perm_base + f.n0 + n] / top_k);
      };
      const int nB = p >> 1;
      const bool vB = nB < f.n_valid;
      const int64_t tokB = vB ? tok_of(nB) : 0;
      const bool vD = p < f.n_valid;
      const int64_t tokD = vD ? tok_of(p) : 0;
      const uint8_t* qa0;
      const uint8_t* qa1;
      if constexpr (GU) {
        qa0 = tab.gate_q[f.slot.table_idx] + (size_t)(f.m0 + p) * rb;
        qa1 = tab.up_q[f.slot.table_idx] + (size_t)(f.m0 + p) * rb;
      } else {
        qa0 = tab.down_q[f.slot.table_idx] + (size_t)(f.m0 + p) * rb;
        qa1 = qa0;
      }
      const __half* arow = act + tokB * dim_in;
      // copies of block kb (global block gk): this thread's packed rows into
      // pk slot kb % (kLook+1), its two B pieces into operand stage
      // gk % kStages and (p < 64) its token's scale into scale stage
      // gk % kStages, once the MMA and the fold warps are done with them
      auto issue = [&](int kb, int gk) {
        const int s = gk % kStages;
        const bool free_op = mbar_wait(&empty_bar[s], ((gk / kStages) & 1) ^ 1, abort, err, 10);
        const bool free_d = mbar_wait(&dempty_bar[s], ((gk / kStages) & 1) ^ 1, abort, err, 14);
        if (free_op && free_d) {
          unsigned char* pk = pk_ring + (kb % (kLook + 1)) * L::kPk;
          cp_async16(pk + p * 16, qa0 + (size_t)kb * 16);
          if constexpr (GU) cp_async16(pk + kM * 16 + p * 16, qa1 + (size_t)kb * 16);
          if (vB) {
            unsigned char* ob = op_ring + s * L::kOpStage + L::kMats * L::kOpA;
            const int c0 = 2 * (p & 1);
            cp_async16(ob + op_off(nB, c0), arow + (size_t)kb * 32 + c0 * 8);
            cp_async16(ob + op_off(nB, c0 + 1), arow + (size_t)kb * 32 + (c0 + 1) * 8);
          }
          if (p < kN) {
            float* dd = d_ring + s * kN + p;
            if (vD) {
              asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dd)), "l"(ad + tokD * nb + kb)
                           : "memory");
            } else {
              *dd = 0.0f;
            }
          }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
      };
#pragma unroll
      for (int i = 0; i < kLook; ++i) {
        if (i < nb) {
          issue(i, g + i);
        } else {
          asm volatile("cp.async.commit_group;" ::: "memory");
        }
      }
      for (int kb = 0; kb < nb; ++kb, ++g) {
        if (kb + kLook < nb) {
          issue(kb + kLook, g + kLook);
        } else {
          asm volatile("cp.async.commit_group;" ::: "memory");
        }
        asm volatile("cp.async.wait_group %0;" ::"n"(kLook) : "memory");  // block kb's copies are in
        const int s = g % kStages;
        if (!*abort) {
          const unsigned char* pk = pk_ring + (kb % (kLook + 1)) * L::kPk;
          unsigned char* op = op_ring + s * L::kOpStage;
#pragma unroll
          for (int m = 0; m < L::kMats; ++m) {
            const uint4 w = *reinterpret_cast<const uint4*>(pk + m * kM * 16 + p * 16);
            unsigned char* dst = op + m * L::kOpA;
            *reinterpret_cast<uint4*>(dst + op_off(p, 0)) = expand_int4_word(w.x);
            *reinterpret_cast<uint4*>(dst + op_off(p, 1)) = expand_int4_word(w.y);
            *reinterpret_cast<uint4*>(dst + op_off(p, 2)) = expand_int4_word(w.z);
            *reinterpret_cast<uint4*>(dst + op_off(p, 3)) = expand_int4_word(w.w);
          }
        }
        fence_async_smem();  // this thread's operand writes (stores and cp.async) -> the tensor core
        mbar_arrive(&full_bar[s]);
      }
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int g = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        const ItemInfo f = item_info(slots, tiles, item, nm);
        const uint32_t idesc = idesc_f16_f32(kM, f.n_pad);
        for (int kb = 0; kb < nb; ++kb, ++g) {
          const int s = g % kStages, b = g % kTBufs;
          if (!mbar_wait(&full_bar[s], (g / kStages) & 1, abort, err, 11)) {
            ok = false;
            break;
          }
          if (!mbar_wait(&tempty_bar[b], ((g / kTBufs) & 1) ^ 1, abort, err, 12)) {
            ok = false;
            break;
          }
          fence_after_sync();
          const uint32_t op = smem_u32(op_ring + s * L::kOpStage);
          const uint32_t opb = op + L::kMats * L::kOpA;
#pragma unroll
          for (int m = 0; m < L::kMats; ++m) {
            const uint32_t d = tmem + b * (L::kMats * kN) + m * kN;
#pragma unroll
            for (int k = 0; k < 2; ++k) {  // two K=16 steps = one Q8 block
              const uint64_t da = smem_desc_k_noswizzle(op + m * L::kOpA + k * 256, 128, 512);
              const uint64_t db = smem_desc_k_noswizzle(opb + k * 256, 128, 512);
              mma_f16(d, da, db, idesc, k);
            }
          }
          mma_commit(&empty_bar[s]);
          mma_commit(&tfull_bar[b]);
        }
      }
      // every MMA this thread issued has finished before TMEM is released
      mma_commit(&done_bar);
      const long long t0 = clock64();
      while (!mbar_try_wait(&done_bar, 0) && clock64() - t0 < kSpinCycles) {
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ fold
    // warp w: TMEM lanes 32*(w%4).. (rows), columns [cb, cb + 32) (tokens)
    constexpr int kC = kN / 2;
    const int quad = warp & 3, cb = ((warp - kEpi0) >> 2) * kC;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    int g = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
      const ItemInfo f = item_info(slots, tiles, item, nm);
      const bool active = cb < f.n_pad;  // warp-uniform
      float acc0[kC], acc1[kC];
#pragma unroll
      for (int n = 0; n < kC; ++n) {
        acc0[n] = 0.0f;
        acc1[n] = 0.0f;
      }
      for (int kb = 0; kb < nb; ++kb, ++g) {
        const int b = g % kTBufs, s = g % kStages;
        // warp-uniform: tcgen05.ld is a warp-wide instruction
        const bool ok = __all_sync(0xffffffffu, mbar_wait(&tfull_bar[b], (g / kTBufs) & 1, abort, err, 13));
        fence_after_sync();
        if (active && ok) {
          // two passes of 16 columns each, so that only 16 TMEM values per
          // matrix and 16 scales are live at a time
          const uint32_t col = tmem + lane_base + b * (L::kMats * kN) + cb;
          mbar_wait(&full_bar[s], (g / kStages) & 1, abort, err, 15);  // the stage's scales are in
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const bool live = cb + 16 * h < f.n_pad;  // warp-uniform
            uint32_t r0[16], r1[16];
            if (live) {
              tmem_ld16(col + 16 * h, r0);
              if constexpr (GU) tmem_ld16(col + kN + 16 * h, r1);
              tmem_ld_wait();
            }
            if (h == 1) {
              fence_before_sync();
              mbar_arrive(&tempty_bar[b]);  // TMEM buffer b may be rewritten now
            }
            float dv[16];
            if (live) {
              const float4* d4p = reinterpret_cast<const float4*>(d_ring + s * kN + cb + 16 * h);
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const float4 d4 = d4p[j];
                dv[4 * j] = d4.x;
                dv[4 * j + 1] = d4.y;
                dv[4 * j + 2] = d4.z;
                dv[4 * j + 3] = d4.w;
              }
            }
            if (h == 1) mbar_arrive(&dempty_bar[s]);
            if (live) {
#pragma unroll
              for (int j = 0; j < 16; j += 2) {
                const int jj = 16 * h + j;
                fma2(acc0[jj], acc0[jj + 1], dv[j], dv[j + 1], __uint_as_float(r0[j]), __uint_as_float(r0[j + 1]));
                if constexpr (GU)
                  fma2(acc1[jj], acc1[jj + 1], dv[j], dv[j + 1], __uint_as_float(r1[j]),
                       __uint_as_float(r1[j + 1]));
              }
            }
          }
        } else {
          fence_before_sync();
          mbar_arrive(&tempty_bar[b]);
          mbar_arrive(&dempty_bar[s]);
        }
      }
      const bool go = __all_sync(0xffffffffu, !*abort) && active;  // warp-uniform (warp_max below)
      if (go) {
        const int o = f.m0 + quad * 32 + lane;
        if constexpr (GU) {
          const float sg = tab.gate_s[f.slot.table_idx][o];
          const float su = tab.up_s[f.slot.table_idx][o];
          const int pos = (lane & ~7) + op_pos8(lane & 7);
#pragma unroll
          for (int j = 0; j < kC; ++j) {
            const int n = cb + j;
            if (n < f.n_valid) {
              const float gv = __fmul_rn(sg, acc0[j]);
              const float u = __fmul_rn(su, acc1[j]);
              const float h = __fmul_rn(__fmul_rn(gv, sigmoid_cw(gv)), u);
              const float d = __fdiv_rn(warp_max(fabsf(h)), 127.0f);
              const int64_t row = (int64_t)f.slot.row_base + f.n0 + n;
              hf[row * inter + (o - lane) + pos] = __int2half_rn(q8_of(h, d));
              if (lane == 0) hd[row * (inter / 32) + (o >> 5)] = d;
            }
          }
        } else {
          const float sd = tab.down_s[f.slot.table_idx][o];
#pragma unroll
          for (int j = 0; j < kC; ++j) {
            const int n = cb + j;
            if (n < f.n_valid) y[((int64_t)f.slot.row_base + f.n0 + n) * hidden + o] = __fmul_rn(sd, acc0[j]);
          }
        }
      }
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    fence_after_sync();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// Tiles of <= kN tokens over the slot table, in slot order.
__global__ void build_tiles_kernel(const Slot* __restrict__ slots, const int32_t* __restrict__ n_slots,
                                   Tile* __restrict__ tiles, int32_t* __restrict__ n_tiles) {
  if (threadIdx.x != 0) return;
  int j = 0;
  const int ns = *n_slots;
  for (int s = 0; s < ns; ++s)
    for (int n0 = 0; n0 < slots[s].count; n0 += kN) tiles[j++] = Tile{s, n0};
  *n_tiles = j;
}

// Opt the kernel in to `bytes` of dynamic shared memory on the current
// device (raised when a larger shape needs more than the last setting).
template <typename KernelT>
cudaError_t allow_smem(KernelT* k, size_t (&granted)[64], size_t bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (granted[dev] >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) granted[dev] = bytes;
  return e;
}

}  // namespace

size_t prefill_tiles_bound(int n_tok, int K, int E, int n_shared) {
  const int64_t pairs = (int64_t)n_tok * (K + n_shared);
  const int64_t slots = (n_tok * (int64_t)K < E ? n_tok * (int64_t)K : E) + n_shared;
  return (size_t)((pairs + kN - 1) / kN + slots);
}

size_t prefill_tile_bytes(int n_tok, int K, int E, int n_shared) {
  return prefill_tiles_bound(n_tok, K, E, n_shared) * sizeof(Tile);
}

bool prefill_supported(int hidden, int inter) {
  return hidden % kM == 0 && inter % kM == 0 && PSmem<true>::bytes() <= 227 * 1024;
}

cudaError_t launch_prefill_experts(const GateUpTable& gu, const DownTable& dn, const Slot* slots,
                                   const int32_t* n_slots, void* tiles, int32_t* n_tiles, const int32_t* perm,
                                   int K, const int8_t* xq, const float* xd, int n_tok, int hidden, int inter,
                                   void* xf, void* hf, float* hd, float* y, int32_t* err, cudaStream_t st,
                                   cudaEvent_t ev_mid) {
  Tile* t = reinterpret_cast<Tile*>(tiles);
  const int64_t n8 = (int64_t)n_tok * hidden / 8;
  act_f16_kernel<<<(unsigned)((n8 + 255) / 256), 256, 0, st>>>(xq, n8, reinterpret_cast<uint4*>(xf));
  build_tiles_kernel<<<1, 32, 0, st>>>(slots, n_slots, t, n_tiles);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  static size_t granted_gu[64] = {}, granted_dn[64] = {};
  static int sms_cache[64] = {};
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (sms_cache[dev] == 0 &&
      (e = cudaDeviceGetAttribute(&sms_cache[dev], cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  const size_t sm_gu = PSmem<true>::bytes(), sm_dn = PSmem<false>::bytes();
  if ((e = allow_smem(prefill_kernel<true, GateUpTable>, granted_gu, sm_gu)) != cudaSuccess) return e;
  if ((e = allow_smem(prefill_kernel<false, DownTable>, granted_dn, sm_dn)) != cudaSuccess) return e;
  const int grid = sms_cache[dev];
  __half* hfh = reinterpret_cast<__half*>(hf);
  prefill_kernel<true, GateUpTable><<<grid, kThreadsP, sm_gu, st>>>(
      gu, slots, t, n_tiles, perm, K, reinterpret_cast<const __half*>(xf), xd, hidden, inter, hfh, hd, y, err);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (ev_mid && (e = cudaEventRecordWithFlags(ev_mid, st, cudaEventRecordExternal)) != cudaSuccess) return e;
  prefill_kernel<false, DownTable><<<grid, kThreadsP, sm_dn, st>>>(dn, slots, t, n_tiles, perm, K, hfh, hd, hidden,
                                                                     inter, hfh, hd, y, err);
  return cudaGetLastError();
}

}  // namespace coli
