// coli_prefill.cu -- the expert kernels for many tokens per expert (prefill):
// a grouped GEMM on the 5th-generation tensor cores (tcgen05.mma, F32
// accumulators in tensor memory), one CTA per (128 output rows, expert slot,
// tile of up to 64 of the slot's tokens).
//
// Exactness.  Each Q8 block's partial sum must come out exactly, because the
// row fold (contract F: acc = fmaf(d_x[b], (float)isum[b], acc), b
// ascending) needs it per block.  The operands are therefore expanded to
// fp16, in which every int4 weight (-8..7) and every Q8 activation
// (-127..127) is exact; the MMA of one 32-element block (two K=16 steps)
// accumulates products of at most 8*127 into an F32 sum of magnitude at most
// 32512 < 2^24, so every partial sum is an exact integer in F32 whatever
// the tensor core's internal order.  The MMA of block b writes a fresh
// accumulator; the epilogue warps then fold it with d_x[b] in ascending b.
// The results equal the dp4a path's bit for bit.
//
// Why fp16 operands and not kind::i8: the fold costs one F32 FMA per
// (row, token, block) whatever the MMA kind; with kind::i8 each of those
// also needs an int32 -> F32 conversion, and the FMA pipe, not the tensor
// pipe, is the limit of this layer (one FMA per 32 MACs).  fp16 operands
// give F32 sums directly.
//
// Roles (384 threads): warps 0-7 epilogue (warp w reads TMEM lanes
// 32(w%4).. = 32 of the tile's rows, columns [32(w/4), 32(w/4)+32) = half of
// the tokens), warps 8-10 producers (cp.async of packed weights and Q8
// activations into a staging ring, expansion to fp16 into the operand ring),
// warp 11 the MMA issuer (lane 0) and TMEM owner.  All waits are bounded
// (coli_tc.cuh).
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

constexpr int kM = 128;       // rows per tile (TMEM lanes)
constexpr int kN = 64;        // tokens per tile (max)
constexpr int kSB = 4;        // Q8 blocks per packed super-stage
constexpr int kStages = 3;    // operand ring depth
constexpr int kEpiWarps = 8;              // 2 per TMEM lane quadrant, each half of the columns
constexpr int kProdWarps = 3;
constexpr int kThreadsP = 32 * (kEpiWarps + kProdWarps + 1);  // 384
constexpr int kProd = 32 * kEpiWarps;                         // first producer thread
constexpr int kNProd = 32 * kProdWarps;                       // producer threads
constexpr int kMma = kProd + kNProd;                          // the MMA warp

template <bool GU>
struct PSmem {
  static constexpr int kMats = GU ? 2 : 1;
  static constexpr int kOpA = kM * 64;                 // one matrix: 128 rows x 32 fp16
  static constexpr int kOpB = kN * 64;                 // 64 tokens x 32 fp16
  static constexpr int kOpStage = kMats * kOpA + kOpB;
  static constexpr int kPkA = kM * kSB * 16;           // packed: 128 rows x kSB blocks x 16 B
  static constexpr int kPkB = kN * kSB * 32;           // Q8: 64 tokens x kSB blocks x 32 B
  static constexpr int kPkStage = kMats * kPkA + kPkB;
  static constexpr int kTmemCols = GU ? 256 : 128;     // 2 buffers x (gate, up | down) x 64
  __host__ __device__ static size_t bytes(int nb) {
    return 1024 + (size_t)kStages * kOpStage + 2 * (size_t)kPkStage + (size_t)nb * kN * 4;
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

// Byte offset of 16-byte chunk c (0..3) of row r in a K-major, no-swizzle
// operand tile of 32 fp16 per row: 8-row x 16-byte core matrices, the four
// K chunks of an 8-row group 128 B apart (LBO), groups 512 B apart (SBO).
__device__ __forceinline__ uint32_t op_off(int r, int c) { return (r >> 3) * 512 + c * 128 + (r & 7) * 16; }

template <bool GU, typename Tab>
__global__ void __launch_bounds__(kThreadsP, 1) prefill_kernel(
    const __grid_constant__ Tab tab, const Slot* __restrict__ slots, const Tile* __restrict__ tiles,
    const int32_t* __restrict__ n_tiles, const int32_t* __restrict__ perm, int top_k, const int8_t* __restrict__ aq,
    const float* __restrict__ ad, int hidden, int inter, int8_t* __restrict__ hq, float* __restrict__ hd,
    float* __restrict__ y, int32_t* __restrict__ err) {
  using L = PSmem<GU>;
  __shared__ uint64_t full_bar[kStages], empty_bar[kStages], tfull_bar[2], tempty_bar[2], done_bar;
  __shared__ uint32_t tmem_s;
  __shared__ int abort_s;
  extern __shared__ unsigned char smem_raw[];

  if ((int)blockIdx.y >= *n_tiles) return;  // uniform per CTA, before any barrier
  const Tile tile = tiles[blockIdx.y];
  const Slot slot = slots[tile.slot];
  const int n_valid = min(kN, slot.count - tile.n0);
  const int n_pad = (n_valid + 15) & ~15;
  const int m0 = blockIdx.x * kM;
  const int dim_in = GU ? hidden : inter;
  const int nb = dim_in / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);  // 1 KB aligned
  unsigned char* op_ring = smem;
  unsigned char* pk_ring = op_ring + kStages * L::kOpStage;
  float* xd_s = reinterpret_cast<float*>(pk_ring + 2 * L::kPkStage);

  const int row_base = slot.row_base, perm_base = slot.perm_base, n0 = tile.n0;
  auto act_row = [=](int n) -> int64_t {
    if (!GU) return (int64_t)row_base + n0 + n;
    return perm_base < 0 ? (int64_t)(n0 + n) : (int64_t)(perm[perm_base + n0 + n] / top_k);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], kNProd);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], 32 * kEpiWarps);
    }
    mbar_init(&done_bar, 1);
    abort_s = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kMma / 32) tmem_alloc(&tmem_s, L::kTmemCols);
  // block scales of the tile's tokens, [kb][64] with the 4-float groups of
  // each row XOR-permuted by (kb & 3) to spread the transposing stores
  for (int i = threadIdx.x; i < kN * nb; i += kThreadsP) {
    const int n = i / nb, kb = i - n * nb;
    xd_s[kb * kN + (n ^ ((kb & 3) << 2))] = n < n_valid ? ad[act_row(n) * nb + kb] : 0.0f;
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = tmem_s;
  volatile int* abort = &abort_s;

  if (threadIdx.x >= kProd && threadIdx.x < kMma) {
    // ------------------------------------------------------------ producers
    const int p = threadIdx.x - kProd;
    const size_t rb = (size_t)dim_in / 2;
    const uint8_t* qa0;
    const uint8_t* qa1;
    if constexpr (GU) {
      qa0 = tab.gate_q[slot.table_idx] + (size_t)m0 * rb;
      qa1 = tab.up_q[slot.table_idx] + (size_t)m0 * rb;
    } else {
      qa0 = tab.down_q[slot.table_idx] + (size_t)m0 * rb;
      qa1 = qa0;
    }
    const int n_super = nb / kSB;
    // copy super-stage ss into packed buffer ss & 1
    auto issue = [=](int ss) {
      unsigned char* pk = pk_ring + (ss & 1) * L::kPkStage;
#pragma unroll
      for (int m = 0; m < L::kMats; ++m) {
        for (int i = p; i < kM * kSB; i += kNProd) {  // 128 rows x kSB 16-byte chunks
          const int r = i / kSB, c = i % kSB;
          cp_async16(pk + m * L::kPkA + r * (kSB * 16) + ((c ^ ((r >> 1) & 3)) * 16),
                     (m == 0 ? qa0 : qa1) + (size_t)r * rb + (size_t)(ss * kSB + c) * 16);
        }
      }
      unsigned char* pb = pk + L::kMats * L::kPkA;
      for (int i = p; i < kN * kSB * 2; i += kNProd) {  // 64 tokens x 2*kSB 16-byte chunks
        const int n = i / (kSB * 2), c = i % (kSB * 2);
        if (n < n_valid)
          cp_async16(pb + n * (kSB * 32) + ((c ^ (n & 7)) * 16), aq + act_row(n) * dim_in + ss * kSB * 32 + c * 16);
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
    };
    // Every producer thread runs the same sequence of named barriers even
    // after an abort (it then only skips work), so none can be left waiting.
    bool alive = true;
    issue(0);
    for (int ss = 0; ss < n_super; ++ss) {
      if (ss + 1 < n_super && alive) issue(ss + 1);
      if (ss + 1 < n_super) {
        asm volatile("cp.async.wait_group 1;" ::: "memory");
      } else {
        asm volatile("cp.async.wait_group 0;" ::: "memory");
      }
      named_bar(1, kNProd);  // every producer's copies of super-stage ss are in
      const unsigned char* pk = pk_ring + (ss & 1) * L::kPkStage;
      for (int kl = 0; kl < kSB; ++kl) {
        const int kb = ss * kSB + kl;
        const int s = kb % kStages;
        alive = alive && mbar_wait(&empty_bar[s], ((kb / kStages) & 1) ^ 1, abort, err, 10);
        if (!alive) continue;
        unsigned char* op = op_ring + s * L::kOpStage;
        // work items of this K-block: (matrix m, row r) expansions of A, then
        // (token n, half h) expansions of B
        for (int i = p; i < L::kMats * kM + 2 * kN; i += kNProd) {
          if (i < L::kMats * kM) {
            const int m = i / kM, r = i % kM;
            const uint4 w = *reinterpret_cast<const uint4*>(pk + m * L::kPkA + r * (kSB * 16) +
                                                            ((kl ^ ((r >> 1) & 3)) * 16));
            unsigned char* dst = op + m * L::kOpA;
            *reinterpret_cast<uint4*>(dst + op_off(r, 0)) = expand_int4_word(w.x);
            *reinterpret_cast<uint4*>(dst + op_off(r, 1)) = expand_int4_word(w.y);
            *reinterpret_cast<uint4*>(dst + op_off(r, 2)) = expand_int4_word(w.z);
            *reinterpret_cast<uint4*>(dst + op_off(r, 3)) = expand_int4_word(w.w);
          } else {
            const int j = i - L::kMats * kM;
            const int n = j >> 1, h = j & 1;
            unsigned char* dst = op + L::kMats * L::kOpA;
            uint4 e0 = make_uint4(0, 0, 0, 0), e1 = e0;
            if (n < n_valid) {
              const int c = 2 * kl + h;
              const uint4 v = *reinterpret_cast<const uint4*>(pk + L::kMats * L::kPkA + n * (kSB * 32) +
                                                              ((c ^ (n & 7)) * 16));
              e0 = expand_int8_pair(v.x, v.y);
              e1 = expand_int8_pair(v.z, v.w);
            }
            *reinterpret_cast<uint4*>(dst + op_off(n, 2 * h)) = e0;
            *reinterpret_cast<uint4*>(dst + op_off(n, 2 * h + 1)) = e1;
          }
        }
        fence_async_smem();
        mbar_arrive(&full_bar[s]);
      }
      named_bar(1, kNProd);  // packed buffer ss & 1 may be refilled after this
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
  } else if (threadIdx.x >= kMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_f16_f32(kM, n_pad);
      for (int kb = 0; kb < nb; ++kb) {
        const int s = kb % kStages, b = kb & 1;
        if (!mbar_wait(&full_bar[s], (kb / kStages) & 1, abort, err, 11)) break;
        if (!mbar_wait(&tempty_bar[b], ((kb >> 1) & 1) ^ 1, abort, err, 12)) break;
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
      // every MMA this thread issued has finished before TMEM is released
      mma_commit(&done_bar);
      const long long t0 = clock64();
      while (!mbar_try_wait(&done_bar, 0) && clock64() - t0 < kSpinCycles) {
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    // warp w: TMEM lanes 32*(w%4).. (rows), columns [cb, cb + 32) (tokens)
    constexpr int kC = kN / 2;
    const int quad = warp & 3, cb = (warp >> 2) * kC;
    float acc0[kC], acc1[kC];
#pragma unroll
    for (int n = 0; n < kC; ++n) {
      acc0[n] = 0.0f;
      acc1[n] = 0.0f;
    }
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const bool active = cb < n_pad;  // warp-uniform
    for (int kb = 0; kb < nb; ++kb) {
      const int b = kb & 1;
      if (!mbar_wait(&tfull_bar[b], (kb >> 1) & 1, abort, err, 13)) break;
      fence_after_sync();
      if (active) {
        const uint32_t col = tmem + lane_base + b * (L::kMats * kN) + cb;
        uint32_t r0[kC], r1[kC];
        // issue every load of the block, then one wait
        tmem_ld16(col, *reinterpret_cast<uint32_t(*)[16]>(&r0[0]));
        if (cb + 16 < n_pad) tmem_ld16(col + 16, *reinterpret_cast<uint32_t(*)[16]>(&r0[16]));
        if constexpr (GU) {
          tmem_ld16(col + kN, *reinterpret_cast<uint32_t(*)[16]>(&r1[0]));
          if (cb + 16 < n_pad) tmem_ld16(col + kN + 16, *reinterpret_cast<uint32_t(*)[16]>(&r1[16]));
        }
        tmem_ld_wait();
        fence_before_sync();
        mbar_arrive(&tempty_bar[b]);  // TMEM buffer b may be rewritten now
        const float* dxk = xd_s + kb * kN;
        const int g_x = kb & 3;
#pragma unroll
        for (int gl = 0; gl < kC / 4; ++gl) {
          const int g = cb / 4 + gl;  // absolute group of 4 columns
          if (4 * g < n_pad) {
            const float4 d4 = *reinterpret_cast<const float4*>(dxk + (g & ~3) * 4 + 4 * ((g & 3) ^ g_x));
            const float dv[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              acc0[4 * gl + i] = __fmaf_rn(dv[i], __uint_as_float(r0[4 * gl + i]), acc0[4 * gl + i]);
              if constexpr (GU) acc1[4 * gl + i] = __fmaf_rn(dv[i], __uint_as_float(r1[4 * gl + i]), acc1[4 * gl + i]);
            }
          }
        }
      } else {
        fence_before_sync();
        mbar_arrive(&tempty_bar[b]);
      }
    }
    if (!*abort && active) {
      const int o = m0 + quad * 32 + lane;
      if constexpr (GU) {
        const float sg = tab.gate_s[slot.table_idx][o];
        const float su = tab.up_s[slot.table_idx][o];
#pragma unroll
        for (int j = 0; j < kC; ++j) {
          const int n = cb + j;
          if (n < n_valid) {
            const float g = __fmul_rn(sg, acc0[j]);
            const float u = __fmul_rn(su, acc1[j]);
            const float h = __fmul_rn(__fmul_rn(g, sigmoid_cw(g)), u);
            const float d = __fdiv_rn(warp_max(fabsf(h)), 127.0f);
            const int64_t row = (int64_t)slot.row_base + tile.n0 + n;
            hq[row * inter + o] = (int8_t)q8_of(h, d);
            if (lane == 0) hd[row * (inter / 32) + (o >> 5)] = d;
          }
        }
      } else {
        const float sd = tab.down_s[slot.table_idx][o];
#pragma unroll
        for (int j = 0; j < kC; ++j) {
          const int n = cb + j;
          if (n < n_valid) y[((int64_t)slot.row_base + tile.n0 + n) * hidden + o] = __fmul_rn(sd, acc0[j]);
        }
      }
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == kMma / 32) {
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
  return hidden % kM == 0 && inter % kM == 0 && (hidden / 32) % kSB == 0 && (inter / 32) % kSB == 0 &&
         PSmem<true>::bytes(hidden / 32) <= 227 * 1024 && PSmem<false>::bytes(inter / 32) <= 227 * 1024;
}

cudaError_t launch_prefill_experts(const GateUpTable& gu, const DownTable& dn, const Slot* slots,
                                   const int32_t* n_slots, void* tiles, int32_t* n_tiles, int max_tiles,
                                   const int32_t* perm, int K, const int8_t* xq, const float* xd, int hidden,
                                   int inter, int8_t* hq, float* hd, float* y, int32_t* err, cudaStream_t st,
                                   cudaEvent_t ev_mid) {
  Tile* t = reinterpret_cast<Tile*>(tiles);
  build_tiles_kernel<<<1, 32, 0, st>>>(slots, n_slots, t, n_tiles);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  static size_t granted_gu[64] = {}, granted_dn[64] = {};
  const size_t sm_gu = PSmem<true>::bytes(hidden / 32), sm_dn = PSmem<false>::bytes(inter / 32);
  if ((e = allow_smem(prefill_kernel<true, GateUpTable>, granted_gu, sm_gu)) != cudaSuccess) return e;
  if ((e = allow_smem(prefill_kernel<false, DownTable>, granted_dn, sm_dn)) != cudaSuccess) return e;
  prefill_kernel<true, GateUpTable><<<dim3(inter / kM, max_tiles), kThreadsP, sm_gu, st>>>(
      gu, slots, t, n_tiles, perm, K, xq, xd, hidden, inter, hq, hd, y, err);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (ev_mid && (e = cudaEventRecordWithFlags(ev_mid, st, cudaEventRecordExternal)) != cudaSuccess) return e;
  prefill_kernel<false, DownTable><<<dim3(hidden / kM, max_tiles), kThreadsP, sm_dn, st>>>(
      dn, slots, t, n_tiles, perm, K, hq, hd, hidden, inter, hq, hd, y, err);
  return cudaGetLastError();
}

}  // namespace coli
