// coli_expert_stream.cu -- the expert part of a decode batch (n_tok <= 8)
// in one persistent kernel, reading the layer's streaming copy
// (coli_expert_stream.cuh, made by coli_moe_prepare):
//
//   router_decode (plain launch: scores, Q8_0 of x, counters cleared)
//   -> expert_stream_kernel (PDL):
//        every CTA takes the top-k and the bucketing of the batch itself
//        (a few hundred scores; no global round trip), then
//        gate/up units (32 intermediate outputs of one expert slot: SiLU(g)*u
//        and the Q8_0 block of h, published with a per-slot counter),
//        then down units (32 output rows of one slot, waiting for the slot's
//        h), and the unit that completes a 32-row chunk for every slot
//        combines it into `out` (contract C).
//
// Streaming.  Every warp owns a ring of R 16 KB stages; lane 0 fills a
// stage with ONE bulk copy (cp.async.bulk, mbarrier completion) of a stage
// image from the streaming copy, R stages ahead of the one the warp
// computes, across unit boundaries and from the gate/up phase into the
// down phase (down weights do not depend on h, so they stream while the
// last gate/up units finish).  The weights of a warp's gate/up unit
// (192 KB at GLM-5.2 shapes) are one contiguous range of HBM.
//
// Arithmetic (contract F, bit-identical to the oracle).  Lane l holds one
// weight row (gate/up: gate row l and up row l of the unit); int8 weights
// (stored as even / odd element planes) take 8 dp4a per block and staged
// token against the token's planes; per 16-byte packed int4 block and
// staged token: (w & 0x0F0F0F0F) ^ 0x08080808 is q + 8 of
// the even elements (unsigned bytes) and w & 0xF0F0F0F0 is 16 q of the odd
// ones (signed bytes); with the token's even / odd byte planes xe, xo and
// c16 = -128 * sum(xe):
//   A = dp4a.u32.s32(q_e + 8, xe) = sum q_e x_e + 8 sum(xe)
//   B = dp4a.s32.s32(16 q_o, xo) starting from c16 = 16 sum q_o x_o - 128 sum(xe)
//   isum = A + (B >> 4)            (B is a multiple of 16: exact)
// then acc = fmaf(d_x[b], (float)isum, acc) in ascending b.
//
// Every wait is bounded (about a second): on expiry the CTA records a
// status code, stops issuing and computing, drains its copies in flight
// (bounded again) and exits.
//
// Sources: "Colibri：在笔记本上跑744B参数的AI模型", "关键特性" (integer dot
// kernels, Q8_0 activations, packed int4); "GLM-5.2-colibri-int4架构解析…",
// "MoE的工作原理" (top-k and the weighted combine), "GLM-5.2的MoE实现" (the
// shared expert); HN summary, "已实现的功能" (batched MoE: one read of an
// expert for all of its tokens).
#include "coli_expert_stream.cuh"
#include "coli_launch.h"
#include "coli_stream.cuh"
#include "coli_topk.cuh"

namespace coli {
namespace {

constexpr int kSW = 8;                               // warps per CTA (all compute; lane 0 also copies)
// Tokens, (token, k) pairs and slots of a launch of the instance for slots
// of TT tokens: batches of up to TT tokens, except the largest TT, which
// takes every batch up to kStreamMaxTok.
template <int TT>
struct StreamTables {
  static constexpr int kTok = TT < kStreamSlotTok ? TT : kStreamMaxTok;
  static constexpr int kPairs = kTok * kMaxTopK;
  static constexpr int kSlots = ((kTok + TT - 1) / TT) * kMaxShared + kTok * kMaxTopK;
};
static_assert(StreamTables<kStreamSlotTok>::kSlots == kStreamMaxSlots, "the counters cover every slot");
constexpr int kErrHReady = 25;                       // status: gave up waiting for a slot's h
constexpr int kErrHStaged = 26;                      // status: gave up waiting for a slot's staged h
constexpr int kErrHPair = 27;                        // status: gave up waiting for a pair's h buffer
constexpr int kErrStage = 28;                        // status: gave up waiting for a weight stage
constexpr int kErrRouting = 29;                      // status: gave up waiting for the routing of the batch
constexpr int kR = 2;                                // ring stages per warp (8 KB each)
constexpr int kQ = 4;                                // a warp's queue of down units (> kR)

// y rows of a CTA's down chunks in shared memory: rows = T * (K + S) of the
// batch (slot order), rpu floats per (chunk, row)
__host__ __device__ inline size_t stream_y_bytes(const StreamGeom& g, int n_sms, int n_rows) {
  const int nch = (g.cpu_dn + n_sms - 1) / n_sms;
  return (size_t)nch * n_rows * g.rpu_dn * 4;
}

// Batches of up to two tokens stage each slot's h rows in shared memory
// (one bulk copy per slot, made by the first warp that needs it); larger
// batches read them through L1.
template <int TT>
struct StreamHStaged {
  static constexpr bool value = TT <= 2;
};
// Batches of 3-4 tokens stage each slot's h rows too, in a ring of kHRing
// slot buffers (the slots of a CTA's down units come in ascending order).
constexpr int kHRing = 4;
template <int TT>
struct StreamHRing {
  static constexpr bool value = TT == 4;
};

// Batches of more than kStreamSlotTok tokens read the x planes (the router
// kernel's) from global memory through L1 instead of shared memory.
template <int TT>
__host__ __device__ inline int stream_x_staged(int n_tok) {
  return n_tok <= kStreamSlotTok ? TT : 0;
}

template <int TT>
__host__ __device__ inline size_t stream_smem_bytes(const StreamGeom& g, int n_sms, int n_tok, int n_rows) {
  const size_t ring = (size_t)kSW * kR * kStreamStageMax;  // 8 KB stages
  const size_t xs = (size_t)stream_x_staged<TT>(n_tok) * g.nbh * 40;  // x planes (32 B) + (d, c16) per block
  const size_t hs = StreamHStaged<TT>::value ? (size_t)n_rows * g.nbi * 40              // h planes + (d, c16)
                    : StreamHRing<TT>::value  ? (size_t)kHRing * TT * g.nbi * 40 : 0;  // per slot buffer
  return 1024 + ring + xs + stream_y_bytes(g, n_sms, n_rows) + hs;
}

__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// isum of one packed weight block (ue = q_e + 8, so = 16 q_o) against one
// token's block (planes xe, xo; c16 = -128 * sum of xe's bytes).
__device__ __forceinline__ int blk_isum(const uint4& ue, const uint4& so, const uint4& xe, const uint4& xo, int c16) {
  int A = dp4a_us(ue.x, xe.x, 0);
  int B = __dp4a((int)so.x, (int)xo.x, c16);
  A = dp4a_us(ue.y, xe.y, A);
  B = __dp4a((int)so.y, (int)xo.y, B);
  A = dp4a_us(ue.z, xe.z, A);
  B = __dp4a((int)so.z, (int)xo.z, B);
  A = dp4a_us(ue.w, xe.w, A);
  B = __dp4a((int)so.w, (int)xo.w, B);
  return A + (B >> 4);
}

__device__ __forceinline__ void unpack_blk(const uint4& w, uint4& ue, uint4& so) {
  ue.x = (w.x & 0x0F0F0F0Fu) ^ 0x08080808u;
  ue.y = (w.y & 0x0F0F0F0Fu) ^ 0x08080808u;
  ue.z = (w.z & 0x0F0F0F0Fu) ^ 0x08080808u;
  ue.w = (w.w & 0x0F0F0F0Fu) ^ 0x08080808u;
  so.x = w.x & 0xF0F0F0F0u;
  so.y = w.y & 0xF0F0F0F0u;
  so.z = w.z & 0xF0F0F0F0u;
  so.w = w.w & 0xF0F0F0F0u;
}

__device__ __forceinline__ int warp_sum_int(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ int ld_acquire_gpu(const int32_t* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// isum of one int8 weight block (even / odd element planes we, wo) against
// one token's block (planes xe, xo).
__device__ __forceinline__ int blk_isum8(const uint4& we, const uint4& wo, const uint4& xe, const uint4& xo) {
  int A = __dp4a((int)we.x, (int)xe.x, 0);
  int B = __dp4a((int)wo.x, (int)xo.x, 0);
  A = __dp4a((int)we.y, (int)xe.y, A);
  B = __dp4a((int)wo.y, (int)xo.y, B);
  A = __dp4a((int)we.z, (int)xe.z, A);
  B = __dp4a((int)wo.z, (int)xo.z, B);
  A = __dp4a((int)we.w, (int)xe.w, A);
  B = __dp4a((int)wo.w, (int)xo.w, B);
  return A + B;
}

template <int BITS>
__device__ __forceinline__ int isum_of(const uint4& a, const uint4& b, const uint4& xe, const uint4& xo, int c16) {
  if constexpr (BITS == 4) return blk_isum(a, b, xe, xo, c16);
  return blk_isum8(a, b, xe, xo);
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ float2 lds64f(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
  return v;
}

// One stage of rows on lanes: blocks b0 .. b0+G-1 of the lane's weight row
// (gate/up halves: lanes 0-15 gate rows, 16-31 the matching up rows; down:
// 32 output rows) against the activation planes of the tokens tok[t] (row
// tok[t] of the plane arrays xpl / xdc, nb blocks per row: shared memory
// when XS, else global memory read through L1).  The stage sits in shared
// memory; the row's chunk c is at (row base | rotation) ^ (c << 4) (the row
// is aligned to its length).  GC > 0 is a compile-time stage width
// (straight-line code); GC == 0 takes G at run time.  pair (GC > 0 only):
// lanes l and l + 16 hold the two pieces of one row (blocks b0 .. of lane l,
// then those of lane l + 16): lanes 16-31 fold their blocks again from lane
// l - 16's result, and both lanes keep the row's sum.
template <int TT, int BITS, bool DBG, int GC, bool XS>
__device__ __forceinline__ void rows_stage(int Grt, const unsigned char* st, int swz, int b0, int nb, int nv,
                                           bool pair, const int (&tok)[TT], const uint4* xpl, const float2* xdc,
                                           float (&acc)[TT], int32_t* const (&dbg)[TT]) {
  const int lane = threadIdx.x & 31;
  constexpr int cpb = BITS / 4;  // 16-byte chunks per block
  const int G = GC > 0 ? GC : Grt;
  const uint32_t rb = (tc::smem_u32(st) + (uint32_t)(lane * (G * cpb * 16))) | (uint32_t)((lane & swz) << 4);
  const uint4* xp[TT];
  const float2* xd[TT];
  uint32_t xps[TT], xds[TT];
#pragma unroll
  for (int t = 0; t < TT; ++t) {
    xp[t] = xpl + 2 * (tok[t] * nb + b0);
    xd[t] = xdc + tok[t] * nb + b0;
    if constexpr (XS) {
      xps[t] = tc::smem_u32(xp[t]);
      xds[t] = tc::smem_u32(xd[t]);
    }
  }
  auto xload = [&](int t, int j, uint4& xe, uint4& xo, float2& dc) {
    if constexpr (XS) {
      xe = lds128(xps[t] + 32 * j);
      xo = lds128(xps[t] + 32 * j + 16);
      dc = lds64f(xds[t] + 8 * j);
    } else {
      xe = xp[t][2 * j];
      xo = xp[t][2 * j + 1];
      dc = xd[t][j];
    }
  };
  float fis[TT][GC > 0 ? GC : 1];  // the blocks' sums, for the second piece of a lane pair
  auto block = [&](int j) {
    uint4 wa, wb;
    if constexpr (BITS == 4) {
      unpack_blk(lds128(rb ^ (uint32_t)(j << 4)), wa, wb);
    } else {
      wa = lds128(rb ^ (uint32_t)((2 * j) << 4));
      wb = lds128(rb ^ (uint32_t)((2 * j + 1) << 4));
    }
#pragma unroll
    for (int t = 0; t < TT; ++t) {
      if (TT == 1 || t < nv) {
        uint4 xe, xo;
        float2 dc;
        xload(t, j, xe, xo, dc);
        const int is = isum_of<BITS>(wa, wb, xe, xo, __float_as_int(dc.y));
        if constexpr (DBG) dbg[t][b0 + j] = is;
        const float f = __int2float_rn(is);
        if constexpr (GC > 0) fis[t][j] = f;
        acc[t] = __fmaf_rn(dc.x, f, acc[t]);
      }
    }
  };
  if constexpr (GC > 0) {
#pragma unroll
    for (int j = 0; j < GC; ++j) block(j);
    if (pair) {
#pragma unroll
      for (int t = 0; t < TT; ++t) {
        if (TT == 1 || t < nv) {
          float a2 = __shfl_xor_sync(0xffffffffu, acc[t], 16);
#pragma unroll
          for (int j = 0; j < GC; ++j) {
            const float d = XS ? lds64f(xds[t] + 8 * j).x : xd[t][j].x;
            a2 = __fmaf_rn(d, fis[t][j], a2);
          }
          const float o2 = __shfl_xor_sync(0xffffffffu, a2, 16);
          acc[t] = lane >= 16 ? a2 : o2;
        }
      }
    }
  } else {
#pragma unroll 4
    for (int j = 0; j < G; ++j) block(j);
  }
}

// Batches of more than two tokens fold on the tensor cores: mma.sync
// m16n8k32 (s8 x s8 -> s32) over 16 weight rows x one Q8 block x 8 token
// columns.  Lane (g, c) = (lane / 4, lane % 4) supplies word c of rows g and
// g + 8 of the block: for int4 its even nibbles as 16 q (a0, a1: the k slots
// 4c .. 4c + 3 are elements 8c, 8c + 2, 8c + 4, 8c + 6) and its odd nibbles
// (a2, a3: k slots 16 + 4c .. are elements 8c + 1, ..); for int8 the words
// c of the block's even and odd planes.  The activation columns in the same
// k order are word c of the token's even and odd byte planes, i.e. the
// staged planes as they are.  The accumulators start at 0x4B400000, so that
// D read as a float is 1.5 2^23 + 16 isum (int4) or + isum (int8), exact.
template <int TT>
struct StreamMma {
  static constexpr bool value = TT >= 4;
};

__device__ __forceinline__ void mma_s8_16x8x32(uint32_t (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  constexpr uint32_t m = 0x4B400000u;
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%10, %11, %12, %13};"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(m), "r"(m), "r"(m), "r"(m));
}

template <int BITS>
__device__ __forceinline__ float isum_of_acc(uint32_t d) {
  if constexpr (BITS == 4) return __fmaf_rn(__uint_as_float(d), 0.0625f, -786432.0f);  // (1.5 2^23 + 16 s) / 16 - 1.5 2^19
  return __fadd_rn(__uint_as_float(d), -12582912.0f);
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

// One stage of the tensor-core fold.  Stage rows 16 rg + g and 16 rg + g + 8
// (rg = 0, 1) of block j against token columns; acc[rg][i]: i = 0 (row g,
// column 2c), 1 (g, 2c + 1), 2 (g + 8, 2c), 3 (g + 8, 2c + 1).  mode 0: the
// two row groups are separate rows (gate / up, or 32 down rows); mode 1:
// they are the two pieces of the same 16 rows (blocks b0 .. b0 + G - 1, then
// b0 + G ..), folded in that order into acc[0].  Activations: row rB of the
// plane array for the lane's B column (g), rows rF0, rF1 for its fold
// columns (2c, 2c + 1); XS: shared memory, else global through L1.
template <int BITS, bool DBG, int GC, bool XS>
__device__ __forceinline__ void rows_stage_mma(int Grt, const unsigned char* st, int swz, int b0, int nb, int mode,
                                               int rB, int rF0, int rF1, const uint4* xpl, const float2* xdc,
                                               float (&acc)[2][4], int32_t* const (&dbg)[2][4]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  constexpr int cpb = BITS / 4;
  const int G = GC > 0 ? GC : Grt;
  const uint32_t sbase = tc::smem_u32(st);
  const uint32_t rowb = (uint32_t)(G * cpb * 16);  // bytes of a stage row
  auto wload = [&](int r, int chunk) -> uint32_t {   // word c of 16-byte chunk `chunk` of stage row r
    return lds32(sbase + (uint32_t)r * rowb + (uint32_t)((chunk ^ (r & swz)) << 4) + 4u * c);
  };
  auto xw = [&](int row, int b, int h) -> uint32_t {  // word c of plane h of block b of activation row `row`
    const uint4* p = xpl + 2 * ((size_t)row * nb + b) + h;
    if constexpr (XS) return lds32(tc::smem_u32(p) + 4u * c);
    return reinterpret_cast<const uint32_t*>(p)[c];
  };
  auto xd = [&](int row, int b) -> float {
    const float2* p = xdc + (size_t)row * nb + b;
    if constexpr (XS) return lds64f(tc::smem_u32(p)).x;
    return p->x;
  };
  auto step = [&](int rg, int j, int b, float (&ac)[4], int32_t* const (&db)[4]) {
    uint32_t a0, a1, a2, a3;
    const int r0 = 16 * rg + g, r1 = r0 + 8;
    if constexpr (BITS == 4) {
      const uint32_t w0 = wload(r0, j), w1 = wload(r1, j);
      a0 = (w0 << 4) & 0xF0F0F0F0u;
      a1 = (w1 << 4) & 0xF0F0F0F0u;
      a2 = w0 & 0xF0F0F0F0u;
      a3 = w1 & 0xF0F0F0F0u;
    } else {
      a0 = wload(r0, 2 * j);
      a1 = wload(r1, 2 * j);
      a2 = wload(r0, 2 * j + 1);
      a3 = wload(r1, 2 * j + 1);
    }
    uint32_t d[4];
    mma_s8_16x8x32(d, a0, a1, a2, a3, xw(rB, b, 0), xw(rB, b, 1));
    const float dx0 = xd(rF0, b), dx1 = xd(rF1, b);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float s = isum_of_acc<BITS>(d[i]);
      if constexpr (DBG)
        if (db[i] != nullptr) db[i][b] = (int32_t)s;
      ac[i] = __fmaf_rn((i & 1) ? dx1 : dx0, s, ac[i]);
    }
  };
  if (mode == 0) {
    if constexpr (GC > 0) {
#pragma unroll
      for (int j = 0; j < GC; ++j) {
        step(0, j, b0 + j, acc[0], dbg[0]);
        step(1, j, b0 + j, acc[1], dbg[1]);
      }
    } else {
#pragma unroll 2
      for (int j = 0; j < G; ++j) {
        step(0, j, b0 + j, acc[0], dbg[0]);
        step(1, j, b0 + j, acc[1], dbg[1]);
      }
    }
  } else {
#pragma unroll 4
    for (int j = 0; j < G; ++j) step(0, j, b0 + j, acc[0], dbg[0]);
#pragma unroll 4
    for (int j = 0; j < G; ++j) step(1, j, b0 + G + j, acc[0], dbg[0]);
  }
}

template <int TT, int BITS, bool DBG, int GC>
__global__ void __launch_bounds__(kSW * 32, 1) expert_stream_kernel(const __grid_constant__ StreamArgs a) {
  constexpr int R = kR;
  constexpr int kPairs = kSW / 2;
  constexpr int kMaxPairsS = StreamTables<TT>::kPairs;
  constexpr int kMaxSlotsS = StreamTables<TT>::kSlots;
  extern __shared__ unsigned char smem_raw[];
  __shared__ uint64_t s_full[kSW][kR];  // one mbarrier per ring slot of each warp
  __shared__ int abort_s;
  __shared__ int s_idx[kMaxPairsS], s_row[kMaxPairsS];
  __shared__ float s_w[kMaxPairsS];
  // per slot: expert (table index), first y / h row, tokens, and the tokens
  // (narrow types: the tables are sized for kStreamMaxSlots slots)
  __shared__ short s_exp[kMaxSlotsS], s_base[kMaxSlotsS];
  __shared__ unsigned char s_cnt[kMaxSlotsS], s_tok[kMaxSlotsS][TT];
  __shared__ uint32_t s_bits[kMaxExperts / 32], s_tm[kMaxExperts / 2];
  __shared__ short s_eslot[kMaxExperts];  // a chosen expert's first slot
  __shared__ int s_nslots;
  __shared__ int s_routed;      // the routing tables below are complete
  __shared__ int s_xready;      // the x planes are complete
  __shared__ uint64_t s_xbar;   // the x planes' bulk copies (from the router kernel) have landed
  __shared__ int s_dn_next;     // the next of this CTA's down units to hand out
  __shared__ int s_q[kSW][kQ];  // per warp: the down units its cursor took, in order (-1: no more)
  __shared__ float s_h[kPairs][2][TT][32];  // a warp pair's h block, double-buffered by unit
  // per unit parity (unit k uses k & 1, like s_h): halves of the pair's
  // units finished, and 1 + the last unit whose Q8 block of h is published
  __shared__ int s_arrive[kPairs][2];
  __shared__ int s_qdone[kPairs][2];
  __shared__ short s_drow[DBG ? kMaxSlotsS : 1][TT];  // capture row of (slot, position): token * (K + S) + rank
  constexpr bool HS = StreamHStaged<TT>::value;
  constexpr bool MMA = StreamMma<TT>::value;
  constexpr bool HR = StreamHRing<TT>::value;
  __shared__ int s_hclaim[HS || HR ? kMaxSlotsS : 1];   // a warp has taken the staging of the slot's h
  __shared__ int s_hissued[HR ? kMaxSlotsS : 1];        // ... and issued its copy (ring: the buffer's phase is set)
  __shared__ uint64_t s_hbar[HS ? kMaxSlotsS : (HR ? kHRing : 1)];  // the slot's (ring: the buffer's) h rows landed
  __shared__ int s_hused[HR ? kHRing : 1];              // ring: down units finished on each buffer, in total

  const StreamGeom& g = a.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = a.E, K = a.K, S = a.S, T = a.T;
  const int n_rows = T * (K + S);  // y rows of the batch (slot order)
  // A slot holds at most TT of the batch's tokens: the shared experts (and
  // any routed expert chosen by more than TT tokens) of a larger batch are
  // several slots over the same weights, TT tokens each.
  const int nsp = (T + TT - 1) / TT;  // slots of a shared expert
  const int S2 = S * nsp;             // shared slots
  const int XT = stream_x_staged<TT>(T);  // tokens of staged x planes (0: read from global)
  unsigned char* smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  unsigned char* ring = smem + (size_t)warp * R * kStreamStageMax;
  uint4* xpl = reinterpret_cast<uint4*>(smem + (size_t)kSW * R * kStreamStageMax);
  float2* xdc = reinterpret_cast<float2*>(xpl + 2 * XT * g.nbh);
  float* s_y = reinterpret_cast<float*>(xdc + XT * g.nbh);  // [chunk of this CTA][y row][rpu_dn]
  // staged h (HS): the batch's rows in global order, planes then (d, c16)
  unsigned char* hst = reinterpret_cast<unsigned char*>(s_y) + stream_y_bytes(g, gridDim.x, n_rows);
  unsigned char* hst_dc = hst + (size_t)n_rows * g.nbi * 32;
  volatile int* abort_f = &abort_s;

  for (int i = threadIdx.x; i < kMaxExperts / 2; i += blockDim.x) {
    if (i < kMaxExperts / 32) s_bits[i] = 0u;
    s_tm[i] = 0u;
  }
  if (threadIdx.x < 2 * kPairs) {
    s_arrive[threadIdx.x >> 1][threadIdx.x & 1] = 0;
    s_qdone[threadIdx.x >> 1][threadIdx.x & 1] = 0;
  }
  if constexpr (HS || HR)
    for (int i = threadIdx.x; i < kMaxSlotsS; i += blockDim.x) {
      s_hclaim[i] = 0;
      if constexpr (HR) s_hissued[i] = 0;
    }
  if constexpr (HR)
    if (threadIdx.x < kHRing) s_hused[threadIdx.x] = 0;
  // the shared slots come first and need no routing: slot s2 < S2 is shared
  // expert s2 / nsp with tokens TT j .. of the batch (j = s2 % nsp); shared
  // expert s has rows s T .. s T + T - 1
  for (int s2 = threadIdx.x; s2 < S2; s2 += blockDim.x) {
    const int s = s2 / nsp, j = s2 - s * nsp;
    s_exp[s2] = E + s;
    s_cnt[s2] = min(TT, T - j * TT);
    s_base[s2] = s * T + j * TT;
    for (int t = 0; t < TT; ++t) {
      s_tok[s2][t] = j * TT + t;
      if constexpr (DBG) s_drow[s2][t] = (j * TT + t) * (K + S) + K + s;
    }
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < kSW * kR; ++i) tc::mbar_init(&s_full[i / kR][i % kR], 1);
    tc::mbar_init(&s_xbar, 1);
    if constexpr (HS)
      for (int i = 0; i < kMaxSlotsS; ++i) tc::mbar_init(&s_hbar[i], 1);
    if constexpr (HR)
      for (int i = 0; i < kHRing; ++i) tc::mbar_init(&s_hbar[i], 1);
    abort_s = 0;
    s_dn_next = 0;
    s_routed = 0;
    s_xready = 0;
    stream::fence_mbar_init();
  }
  __syncthreads();

  // The first T warps route the batch (one token each; warp 0 also
  // buckets) while the others quantise x and start: a warp whose first unit
  // is a shared expert's computes that unit before the routing is known.
  // (The routing is a short serial chain on the critical path: the low warp
  // ids, which the schedulers favour, take it.)
  const int n_router = T < 4 ? T : 4;  // router warps: token warp, warp + 4
  const bool router = warp < n_router;
  // Gate/up work goes to warp pairs: pair p of this CTA takes units
  // gp, gp + NP, ... (gp = p * G + blockIdx.x), warp 2p the first half of
  // each unit, warp 2p + 1 the second.  Down work: this CTA owns the output
  // chunks [c0, c1) (rpu_dn rows each) of every slot, i.e. the units
  // id = slot * nch + (chunk - c0), handed out in that order (slot by slot)
  // to whichever warp's cursor asks next; their y rows stay in shared memory
  // and the CTA combines its own chunks at the end.
  const int G = gridDim.x, NP = G * kPairs;
  // pairs from the top warp down, so that the router warps form the last pairs
  const int pw = kSW - 1 - warp;
  const int pair = pw >> 1, half = pw & 1, gp = pair * G + blockIdx.x;
  const int n_shared_gu = S2 * g.cpu_gu;
  const int c0 = (int)((int64_t)blockIdx.x * g.cpu_dn / G), c1 = (int)((int64_t)(blockIdx.x + 1) * g.cpu_dn / G);
  const int nch = c1 - c0;
  const bool shared_first = !router && gp < n_shared_gu;

  // The warp's stage sequence: its gate/up half units, then the down units
  // it takes.  A cursor walks it R stages ahead of the compute: (phase, unit
  // index k, stage s, the unit's base address); the divisions happen once
  // per unit.  Until the routing is known a shared-first warp's cursor stops
  // at the end of its first unit (phase 3) and owes the stages it skipped.
  int n_gu_mine = shared_first ? 1 : 0, n_dn_cta = 0;  // shared-first: the shared unit, until the routing
  bool routed = false;
  struct Cursor {
    int phase, k, s;  // phase 0 gate/up, 1 down, 2 done, 3 waiting for the routing
    const unsigned char* base;
  };
  auto unit_base = [&](Cursor& c) {
    if (c.phase == 0 && c.k >= n_gu_mine) {
      c.phase = 1;
      c.k = 0;
    }
    if (c.phase == 0) {
      const int u = gp + c.k * NP;
      const int slot = u / g.cpu_gu;
      const int e = s_exp[slot];
      c.base = a.prep + (uint64_t)e * g.expert_bytes + (uint64_t)((u - slot * g.cpu_gu) * 2 + half) * g.ub_gu;
    } else if (c.phase == 1) {
      int id = 0;
      if (lane == 0) id = atomicAdd(&s_dn_next, 1);
      id = __shfl_sync(0xffffffffu, id, 0);
      if (id >= n_dn_cta) {
        id = -1;
        c.phase = 2;
      }
      s_q[warp][c.k & (kQ - 1)] = id;
      if (id >= 0) {
        const int slot = id / nch, chunk = c0 + (id - slot * nch);
        const int e = s_exp[slot];
        c.base = a.prep + (uint64_t)e * g.expert_bytes + g.dn_off + (uint64_t)chunk * g.ub_dn;
      }
    }
  };
  Cursor pc{0, 0, 0, nullptr};
  const uint64_t l2pol = l2_evict_first();  // the weights are read once per forward: first out of L2
  int issued = 0, n_real = 0, owed = 0;  // stages issued (past the end: empty), real copies, stages owed
  // lane 0: the cursor's stage into ring slot issued % R, one bulk copy
  // completing on the slot's mbarrier
  auto copy_stage = [&]() {
    if (pc.phase < 2) {
      const uint32_t bytes = pc.phase == 0 ? g.sb_gu : g.sb_dn;
      if (lane == 0) {
        uint64_t* bar = &s_full[warp][issued % R];
        stream::mbar_expect_tx(bar, bytes);
        stream::bulk_g2s_hint(ring + (size_t)(issued % R) * kStreamStageMax, pc.base + (uint64_t)pc.s * bytes, bytes,
                              bar, l2pol);
      }
      ++n_real;
    }
    ++issued;
  };
  auto issue = [&]() {  // copy, then move the cursor on
    if (pc.phase == 3) {
      ++owed;
      return;
    }
    copy_stage();
    if (pc.phase < 2 && ++pc.s == (pc.phase == 0 ? g.st_gu : g.st_dn)) {
      pc.s = 0;
      ++pc.k;
      if (!routed)
        pc.phase = 3;  // the routing is not known yet
      else
        unit_base(pc);
    }
  };

  if (!router && XT == 0) {
    // the x planes stay in global memory (the router kernel's): every
    // thread that reads them waits for that kernel first
    pdl_wait();
    asm volatile("bar.sync 2, %0;" ::"r"((kSW - n_router) * 32) : "memory");  // the non-router warps
    if (threadIdx.x == n_router * 32) {
      __threadfence_block();
      *(volatile int*)&s_xready = 1;
    }
  } else if (!router && a.xpl_g != nullptr) {
    // the x planes from the router kernel: two bulk copies after the PDL wait
    if (threadIdx.x == n_router * 32) {
      pdl_wait();
      const uint32_t pb = (uint32_t)(T * g.nbh * 32), db = (uint32_t)(T * g.nbh * 8);
      stream::fence_proxy_async_global();
      stream::mbar_expect_tx(&s_xbar, pb + db);
      stream::bulk_g2s(xpl, a.xpl_g, pb, &s_xbar);
      stream::bulk_g2s(xdc, a.xdc_g, db, &s_xbar);
    }
    tc::mbar_wait(&s_xbar, 0, abort_f, a.status, kErrRouting);
    asm volatile("bar.sync 2, %0;" ::"r"((kSW - n_router) * 32) : "memory");  // the non-router warps
    if (threadIdx.x == n_router * 32) {
      __threadfence_block();
      *(volatile int*)&s_xready = 1;
    }
  } else if (!router) {
    // x planes, from the layer input (the Q8_0 of the router kernel,
    // quotients from one reciprocal per block): block b of token t ->
    // even / odd byte planes and (d, c16 = -128 * sum of the even plane)
    // eight lanes per block (lane m: elements 4m .. 4m + 3), four blocks per
    // warp and step; lane m writes bytes 2m, 2m + 1 of both planes
    // (the loads of eight steps go out together: the loop is bound by their latency)
    const int sub = lane >> 3, m = lane & 7, nblk = T * g.nbh, stride = (kSW - n_router) * 4;
    for (int i0 = (warp - n_router) * 4 + sub; i0 < nblk; i0 += 8 * stride) {
      float4 fv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * stride;
        fv[u] = i < nblk ? __ldg(reinterpret_cast<const float4*>(a.x + (size_t)i * 32) + m)
                         : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      }
      // (eight independent chains: unrolled, so that they overlap)
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * stride;
        const float4 f = fv[u];
        float amax = fmaxf(fmaxf(fabsf(f.x), fabsf(f.y)), fmaxf(fabsf(f.z), fabsf(f.w)));
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float d = __fdiv_rn(amax, 127.0f), r = __frcp_rn(d);
        const int q0 = q8_of_r(f.x, d, r), q1 = q8_of_r(f.y, d, r), q2 = q8_of_r(f.z, d, r), q3 = q8_of_r(f.w, d, r);
        int se = q0 + q2;
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) se += __shfl_xor_sync(0xffffffffu, se, o);
        if (i < nblk) {
          unsigned short* pl = reinterpret_cast<unsigned short*>(xpl + 2 * i);
          pl[m] = (unsigned short)((q0 & 0xFF) | (q2 & 0xFF) << 8);      // even plane
          pl[8 + m] = (unsigned short)((q1 & 0xFF) | (q3 & 0xFF) << 8);  // odd plane
          if (m == 0) xdc[i] = make_float2(d, __int_as_float(-128 * se));
        }
      }
    }
    asm volatile("bar.sync 2, %0;" ::"r"((kSW - n_router) * 32) : "memory");  // the non-router warps
    if (threadIdx.x == n_router * 32) {
      __threadfence_block();
      *(volatile int*)&s_xready = 1;
    }
  }


  if (shared_first) {
    unit_base(pc);  // k = 0: the warp's shared unit
    for (int i = 0; i < R; ++i) issue();
  }

  // ---- routing of the batch (every CTA, identical results) -------------
  if (router) {
    // the correction bias is a layer constant: into registers before the wait
    float bias_r[kMaxExperts / 32];
#pragma unroll
    for (int i = 0; i < kMaxExperts / 32; ++i) {
      const int e = lane + 32 * i;
      bias_r[i] = e < E ? __ldg(a.bias + e) : 0.0f;
    }
    pdl_wait();  // the scores and the cleared counters are complete
    for (int tr = warp; tr < T; tr += n_router) {  // this warp's tokens
      const float* st = a.scores + (size_t)tr * E;
      auto sc = [st](int e) { return ld_dep(st + e); };
      if (E <= 256)
        topk::warp_route_token<8>(sc, bias_r, E, K, a.norm, a.rsf, lane, s_idx + tr * K, s_w + tr * K);
      else
        topk::warp_route_token<kMaxExperts / 32>(sc, bias_r, E, K, a.norm, a.rsf, lane, s_idx + tr * K,
                                                 s_w + tr * K);
      __syncwarp();
      // the chosen experts (bit e of s_bits) and, per expert, the tokens that
      // chose it (half e & 1 of s_tm[e >> 1], bit t)
      if (lane < K) {
        const int e = s_idx[tr * K + lane];
        atomicOr(&s_bits[e >> 5], 1u << (e & 31));
        atomicOr(&s_tm[e >> 1], 1u << ((e & 1) * 16 + tr));
      }
    }
    if (n_router > 1) asm volatile("bar.sync 1, %0;" ::"r"(n_router * 32) : "memory");  // the router warps
    if (warp == 0 && T == 1) {
      // one token: every chosen expert is a slot of one row; slot of rank k
      // = S + the number of chosen experts with a lower id
      const int e = lane < K ? s_idx[lane] : INT_MAX;
      int below = 0;
      for (int j = 0; j < K; ++j) below += __shfl_sync(0xffffffffu, e, j) < e;
      if (lane < K) {
        const int r = S + below;
        s_exp[r] = e;
        s_cnt[r] = 1;
        s_base[r] = r;
        s_tok[r][0] = 0;
        s_row[lane] = r;
        if constexpr (DBG) s_drow[r][0] = lane;  // token 0, rank lane
      }
      if (lane == 0) s_nslots = S + K;
      __syncwarp();
      if (lane == 0) {
        __threadfence_block();
        *(volatile int*)&s_routed = 1;
      }
    } else if (warp == 0) {
      __syncwarp();
      auto tm_of = [&](int e) { return (s_tm[e >> 1] >> ((e & 1) * 16)) & 0xFFFFu; };
      // lane l: the experts 32l .. 32l+31; slots in ascending expert id after
      // the shared ones (an expert of more than TT tokens: one slot per TT of
      // them), rows in slot order, a slot's rows in token order
      const int nw = (E + 31) / 32;
      const uint32_t bits = lane < nw ? s_bits[lane] : 0u;
      int rows = 0, c = 0;
      for (uint32_t bb = bits; bb; bb &= bb - 1) {
        const int n = __popc(tm_of(32 * lane + __ffs(bb) - 1));
        rows += n;
        c += (n + TT - 1) / TT;
      }
      int ci = c, ri = rows;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int yc = __shfl_up_sync(0xffffffffu, ci, o), yr = __shfl_up_sync(0xffffffffu, ri, o);
        if (lane >= o) {
          ci += yc;
          ri += yr;
        }
      }
      if (lane == 31) s_nslots = S2 + ci;
      int r = S2 + ci - c, base = S * T + ri - rows;
      for (uint32_t bb = bits; bb; bb &= bb - 1) {
        const int e = 32 * lane + __ffs(bb) - 1;
        const uint32_t m = tm_of(e);
        s_eslot[e] = r;
        int pos = 0;
        for (int t = 0; t < kStreamMaxTok; ++t)
          if ((m >> t) & 1u) {
            if (pos % TT == 0) {  // the next slot of this expert
              if (pos > 0) ++r;
              s_exp[r] = e;
              s_cnt[r] = 0;
              s_base[r] = base + pos;
            }
            s_tok[r][pos % TT] = t;
            ++s_cnt[r];
            ++pos;
          }
        base += pos;
        ++r;
      }
      __syncwarp();
      // each (token, rank) pair: the row of its expert's output (an expert's
      // rows are contiguous over its slots)
      for (int p = lane; p < T * K; p += 32) {
        const int e = s_idx[p], t = p / K;
        const int pos = __popc(tm_of(e) & ((1u << t) - 1u));
        s_row[p] = s_base[s_eslot[e]] + pos;
        if constexpr (DBG) s_drow[s_eslot[e] + pos / TT][pos % TT] = t * (K + S) + (p - t * K);  // rank p - tK of token t
      }
      __syncwarp();
      if (lane == 0) {
        __threadfence_block();
        *(volatile int*)&s_routed = 1;
      }
    }
  }
  // The routing is known to this warp once s_routed is set (bounded wait);
  // then the counts, and the cursor's next unit.
  auto await_routing = [&]() -> bool {
    pdl_wait();
    pdl_launch_dependents();
    int got = 0;
    if (lane == 0) {
      const long long t0 = clock64();
      while (!*abort_f) {
        if (*(volatile int*)&s_routed && *(volatile int*)&s_xready) {
          got = 1;
          break;
        }
        if (clock64() - t0 > tc::kSpinCycles) {
          *abort_f = 1;
          atomicExch(a.status, kErrRouting);
          break;
        }
        __nanosleep(32);
      }
      __threadfence_block();
    }
    if (!__shfl_sync(0xffffffffu, got, 0)) return false;
    const int n_slots = s_nslots;
    const int n_gu = n_slots * g.cpu_gu;
    n_gu_mine = gp < n_gu ? (n_gu - gp + NP - 1) / NP : 0;
    n_dn_cta = n_slots * nch;
    routed = true;
    if (!shared_first) {
      unit_base(pc);  // the cursor's first unit
      for (int i = 0; i < R; ++i) issue();
    } else if (pc.phase == 3) {
      pc.phase = 0;  // past the shared unit: on to the next
      unit_base(pc);
      for (; owed > 0; --owed) issue();
    }
    return true;
  };

  int consumed = 0;
  bool ok = true;
  auto wait_stage = [&]() -> bool {
    const bool got = tc::mbar_wait(&s_full[warp][consumed % R], (uint32_t)((consumed / R) & 1), abort_f, a.status,
                                   kErrStage);
    return __all_sync(0xffffffffu, got);
  };
  // the ring slot of the stage just computed is free again: copy the stage R ahead into it
  auto next_stage = [&]() {
    ++consumed;
    __syncwarp();
    issue();
  };
  const int64_t P = 2 * (int64_t)g.I * g.nbh + (int64_t)g.H * g.nbi;  // capture words per (token, expert)

  // ---- the warp's units: gate/up halves, then down units --------------
  // One loop with one stage-compute call, so that the kernel holds a single
  // copy of the unrolled block loop.
  int acq_slot = -1;  // the last slot whose h this warp has acquired
  for (int k = 0; ok; ++k) {
    if (!routed && (k > 0 || !shared_first) && !await_routing()) {
      ok = false;
      break;
    }
    const bool gu = k < n_gu_mine;
    int slot, chunk, nv, nst, Gs, swz, nb, lpr = 1;
    const uint4* ap;
    const float2* adc;
    int tok[TT];
    int32_t* dbg[TT];
    if (gu) {
      const int u = gp + k * NP;
      slot = u / g.cpu_gu;
      chunk = u - slot * g.cpu_gu;
      nv = s_cnt[slot];
      nst = g.st_gu;
      Gs = g.g_gu;
      swz = g.swz_gu;
      nb = g.nbh;
      ap = XT > 0 ? xpl : reinterpret_cast<const uint4*>(a.xpl_g);
      adc = XT > 0 ? xdc : a.xdc_g;
      const int orow = chunk * 32 + 16 * half + (lane & 15);
#pragma unroll
      for (int t = 0; t < TT; ++t) {
        tok[t] = t < nv ? s_tok[slot][t] : 0;
        dbg[t] = nullptr;
        if constexpr (DBG)
          if (t < nv)
            dbg[t] = a.dbg + s_drow[slot][t] * P + (int64_t)(lane < 16 ? 0 : g.I) * g.nbh + (int64_t)orow * g.nbh;
      }
    } else {
      const int id = s_q[warp][(k - n_gu_mine) & (kQ - 1)];
      if (id < 0) break;  // the CTA's down units are all taken
      slot = id / nch;
      chunk = c0 + (id - slot * nch);
      nv = s_cnt[slot];
      nst = g.st_dn;
      Gs = g.g_dn;
      swz = g.swz_dn;
      nb = g.nbi;
      lpr = g.lpr_dn;
      if (slot != acq_slot) {
        // every gate/up unit of the slot is counted: its h rows are complete,
        // and the acquire orders the reads of them after their stores.  HS:
        // the first warp of the CTA to get here copies the rows into shared
        // memory (one bulk copy for the planes, one for (d, c16)); every
        // warp waits for that copy.
        bool claim = true;
        if constexpr (HS || HR) {
          int c = 0;
          if (lane == 0) c = atomicCAS(&s_hclaim[slot], 0, 1) == 0;
          claim = __shfl_sync(0xffffffffu, c, 0) != 0;
        }
        bool ready = !claim;
        if (claim) {
          const long long t0 = clock64();
          while (!*abort_f) {
            if (ld_acquire_gpu(a.h_ready + slot) >= g.cpu_gu) {
              ready = true;
              break;
            }
            if (clock64() - t0 > tc::kSpinCycles) {
              *abort_f = 1;
              atomicExch(a.status, kErrHReady);
              break;
            }
            __nanosleep(64);
          }
          if constexpr (HS) {
            if (lane == 0 && ready) {
              const size_t r0 = s_base[slot];
              const uint32_t pl = (uint32_t)(nv * g.nbi * 32), dc = (uint32_t)(nv * g.nbi * 8);
              stream::fence_proxy_async_global();
              stream::mbar_expect_tx(&s_hbar[slot], pl + dc);
              stream::bulk_g2s(hst + r0 * g.nbi * 32, a.hpl + r0 * g.nbi * 32, pl, &s_hbar[slot]);
              stream::bulk_g2s(hst_dc + r0 * g.nbi * 8, a.hdc + r0 * g.nbi, dc, &s_hbar[slot]);
            }
          }
          if constexpr (HR) {
            // ring buffer slot % kHRing: free once every down unit of its
            // previous slot (slot - kHRing) has finished here
            if (lane == 0 && ready) {
              const int b = slot % kHRing;
              const int need = (slot / kHRing) * nch;
              const long long t1 = clock64();
              while (*(volatile int*)&s_hused[b] < need && !*abort_f)
                if (clock64() - t1 > tc::kSpinCycles) {
                  *abort_f = 1;
                  atomicExch(a.status, kErrHStaged);
                }
              if (!*abort_f) {
                const size_t r0 = s_base[slot];
                unsigned char* hb = hst + (size_t)b * TT * g.nbi * 40;
                const uint32_t pl = (uint32_t)(nv * g.nbi * 32), dc = (uint32_t)(nv * g.nbi * 8);
                stream::fence_proxy_async_global();
                stream::mbar_expect_tx(&s_hbar[b], pl + dc);
                stream::bulk_g2s(hb, a.hpl + r0 * g.nbi * 32, pl, &s_hbar[b]);
                stream::bulk_g2s(hb + (size_t)TT * g.nbi * 32, a.hdc + r0 * g.nbi, dc, &s_hbar[b]);
                __threadfence_block();
                *(volatile int*)&s_hissued[slot] = 1;
              }
            }
          }
        }
        if constexpr (HS) ready = tc::mbar_wait(&s_hbar[slot], 0, abort_f, a.status, kErrHStaged);
        if constexpr (HR) {
          // the copy is issued (so the buffer's phase is this slot's), then landed
          int is = 1;
          if (lane == 0) {
            const long long t1 = clock64();
            while (!*(volatile int*)&s_hissued[slot] && !*abort_f)
              if (clock64() - t1 > tc::kSpinCycles) {
                *abort_f = 1;
                atomicExch(a.status, kErrHStaged);
              }
            is = !*abort_f;
          }
          is = __shfl_sync(0xffffffffu, is, 0);
          ready = is && tc::mbar_wait(&s_hbar[slot % kHRing], (uint32_t)((slot / kHRing) & 1), abort_f, a.status,
                                      kErrHStaged);
        }
        if (!__all_sync(0xffffffffu, ready)) {
          ok = false;
          break;
        }
        acq_slot = slot;
      }
      if constexpr (HS) {
        ap = reinterpret_cast<const uint4*>(hst + (size_t)s_base[slot] * g.nbi * 32);
        adc = reinterpret_cast<const float2*>(hst_dc + (size_t)s_base[slot] * g.nbi * 8);
      } else if constexpr (HR) {
        const unsigned char* hb = hst + (size_t)(slot % kHRing) * TT * g.nbi * 40;
        ap = reinterpret_cast<const uint4*>(hb);
        adc = reinterpret_cast<const float2*>(hb + (size_t)TT * g.nbi * 32);
      } else {
        // the slot's h rows are read through L1 (every lane loads the same block)
        ap = reinterpret_cast<const uint4*>(a.hpl + (size_t)s_base[slot] * g.nbi * 32);
        adc = a.hdc + (size_t)s_base[slot] * g.nbi;
      }
      const int o = chunk * g.rpu_dn + (lane & (g.rpu_dn - 1));
#pragma unroll
      for (int t = 0; t < TT; ++t) {
        tok[t] = t;  // the slot's h rows are its tokens in order
        dbg[t] = nullptr;
        if constexpr (DBG)
          if (t < nv) dbg[t] = a.dbg + s_drow[slot][t] * P + 2 * (int64_t)g.I * g.nbh + (int64_t)o * g.nbi;
      }
    }
    // tensor-core fold (batches of more than two tokens): lane (gq, cq) =
    // (lane / 4, lane % 4) feeds token column gq and folds columns 2cq,
    // 2cq + 1 of rows gq, gq + 8 (and 16 + .. of the second row group);
    // mode 0: the row groups are separate rows, 1: the two pieces of the
    // same 16 down rows
    const int gq = lane >> 2, cq = lane & 3;
    const int mmode = gu ? 0 : (lpr == 2 ? 1 : 0);
    int rB = 0, rF0 = 0, rF1 = 0;
    float accm[2][4] = {{0.0f, 0.0f, 0.0f, 0.0f}, {0.0f, 0.0f, 0.0f, 0.0f}};
    float rsm[2][2] = {{0.0f, 0.0f}, {0.0f, 0.0f}};
    int32_t* dbgm[2][4] = {{nullptr, nullptr, nullptr, nullptr}, {nullptr, nullptr, nullptr, nullptr}};
    if constexpr (MMA) {
      const int last = nv - 1;
      const int cB = gq < nv ? gq : last, cF0 = 2 * cq < nv ? 2 * cq : last, cF1 = 2 * cq + 1 < nv ? 2 * cq + 1 : last;
      rB = gu ? s_tok[slot][cB] : cB;
      rF0 = gu ? s_tok[slot][cF0] : cF0;
      rF1 = gu ? s_tok[slot][cF1] : cF1;
      const float* scm = reinterpret_cast<const float*>(a.prep + (uint64_t)s_exp[slot] * g.expert_bytes + g.sc_off);
#pragma unroll
      for (int rg = 0; rg < 2; ++rg)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          // the output row of (rg, h) within the unit, and its scale
          const int orow = gu ? chunk * 32 + 16 * half + gq + 8 * h
                              : chunk * g.rpu_dn + (mmode == 1 ? 0 : 16 * rg) + gq + 8 * h;
          if (gu || mmode == 0 || rg == 0)
            rsm[rg][h] = __ldg(scm + (gu ? (rg == 0 ? 0 : g.I) : 2 * g.I) + orow);
          if constexpr (DBG) {
#pragma unroll
            for (int ti = 0; ti < 2; ++ti) {
              const int t = 2 * cq + ti;
              if (t < nv)
                dbgm[rg][2 * h + ti] = gu ? a.dbg + s_drow[slot][t] * P + (int64_t)(rg == 0 ? 0 : g.I) * g.nbh +
                                                (int64_t)orow * g.nbh
                                          : a.dbg + s_drow[slot][t] * P + 2 * (int64_t)g.I * g.nbh +
                                                (int64_t)orow * g.nbi;
            }
          }
        }
    }
    // the row scale of this lane's output, loaded ahead of the stages
    const float* sc = reinterpret_cast<const float*>(a.prep + (uint64_t)s_exp[slot] * g.expert_bytes + g.sc_off);
    const float rs =
        gu ? __ldg(sc + (lane < 16 ? 0 : g.I) + chunk * 32 + 16 * half + (lane & 15))
           : __ldg(sc + 2 * g.I + chunk * g.rpu_dn + (lane & (g.rpu_dn - 1)));
    float acc[TT];
#pragma unroll
    for (int t = 0; t < TT; ++t) acc[t] = 0.0f;
    // a lane's first block in stage s (lane pairs: lanes 16-31 the second piece)
    const int span = lpr * Gs, piece0 = lpr == 2 ? (lane >> 4) * Gs : 0;
    for (int s = 0; s < nst && ok; ++s) {
      ok = wait_stage();
      if (!ok) break;
      const unsigned char* stg = ring + (size_t)(consumed % R) * kStreamStageMax;
      if constexpr (MMA) {
        if (HS || HR || (gu && XT > 0))
          rows_stage_mma<BITS, DBG, GC, true>(Gs, stg, swz, s * span, nb, mmode, rB, rF0, rF1, ap, adc, accm, dbgm);
        else
          rows_stage_mma<BITS, DBG, GC, false>(Gs, stg, swz, s * span, nb, mmode, rB, rF0, rF1, ap, adc, accm, dbgm);
      } else {
        if (HS || HR || (gu && XT > 0))
          rows_stage<TT, BITS, DBG, GC, true>(Gs, stg, swz, s * span + piece0, nb, nv, lpr == 2, tok, ap, adc, acc,
                                              dbg);
        else
          rows_stage<TT, BITS, DBG, GC, false>(Gs, stg, swz, s * span + piece0, nb, nv, lpr == 2, tok, ap, adc, acc,
                                               dbg);
      }
      next_stage();
    }
    if (!ok) break;
    if constexpr (HR) {
      if (!gu) {  // this unit's reads of its ring buffer are done
        __syncwarp();
        if (lane == 0) atomicAdd(&s_hused[slot % kHRing], 1);
      }
    }
    if (gu) {
      // SwiGLU of the half's 16 outputs into shared memory; the second warp
      // of the pair to finish quantises the whole Q8_0 block of h and
      // publishes it (no warp waits for the other)
      float* hbuf = &s_h[pair][k & 1][0][0];
      // the buffer was last used by unit k - 2: its block must be published
      if (k >= 2) {
        const long long t0 = clock64();
        while (*(volatile int*)&s_qdone[pair][k & 1] < k - 1 && !*abort_f) {
          if (clock64() - t0 > tc::kSpinCycles) {
            *abort_f = 1;
            atomicExch(a.status, kErrHPair);
          }
        }
      }
      if constexpr (MMA) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int t = 2 * cq + (i & 1), o = gq + 8 * (i >> 1);
          const float v = __fmul_rn(rsm[0][i >> 1], accm[0][i]), uv = __fmul_rn(rsm[1][i >> 1], accm[1][i]);
          if (t < nv) hbuf[t * 32 + 16 * half + o] = __fmul_rn(__fmul_rn(v, sigmoid_cw(v)), uv);
        }
      } else {
#pragma unroll
        for (int t = 0; t < TT; ++t) {
          const float v = __fmul_rn(rs, acc[t]);
          const float uv = __shfl_down_sync(0xffffffffu, v, 16);
          if (lane < 16 && t < nv) hbuf[t * 32 + 16 * half + lane] = __fmul_rn(__fmul_rn(v, sigmoid_cw(v)), uv);
        }
      }
      __syncwarp();
      int second = 0;
      if (lane == 0) {
        __threadfence_block();
        second = atomicAdd(&s_arrive[pair][k & 1], 1) & 1;
        if (second) __threadfence_block();
      }
      second = __shfl_sync(0xffffffffu, second, 0);
      if (second && !*abort_f) {
#pragma unroll
        for (int t = 0; t < TT; ++t) {
          if (t < nv) {
            const float h = *(volatile float*)&hbuf[t * 32 + lane];
            const float d = __fdiv_rn(warp_max(fabsf(h)), 127.0f);
            const int q = q8_of(h, d);
            const int64_t hrow = s_base[slot] + t;
            a.hpl[(hrow * g.nbi + chunk) * 32 + (lane & 1) * 16 + (lane >> 1)] = (int8_t)q;
            const int se = warp_sum_int((lane & 1) ? 0 : q);
            if (lane == 0) a.hdc[hrow * g.nbi + chunk] = make_float2(d, __int_as_float(-128 * se));
          }
        }
        __threadfence();  // every lane: its h stores are visible before the count moves
        __syncwarp();
        pdl_wait();  // (a shared unit done before the routing) the router kernel has cleared the counts
        if (lane == 0) {
          *(volatile int*)&s_qdone[pair][k & 1] = k + 1;
          atomicAdd(a.h_ready + slot, 1);
        }
      }
      ok = !*abort_f;
    } else {
      // lanes 0 .. rpu_dn - 1: the unit's rows (lane pairs hold the same sum)
      const int rpu = g.rpu_dn;
      if constexpr (MMA) {
        float* yc = s_y + ((size_t)(chunk - c0) * n_rows + s_base[slot]) * rpu;
#pragma unroll
        for (int rg = 0; rg < 2; ++rg)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int t = 2 * cq + (i & 1), rr = (mmode == 1 ? 0 : 16 * rg) + gq + 8 * (i >> 1);
            if (t < nv && (rg == 0 || mmode == 0)) yc[(size_t)t * rpu + rr] = __fmul_rn(rsm[rg][i >> 1], accm[rg][i]);
          }
      } else if (lane < rpu) {
        float* yc = s_y + ((size_t)(chunk - c0) * n_rows + s_base[slot]) * rpu + lane;
#pragma unroll
        for (int t = 0; t < TT; ++t)
          if (t < nv) yc[(size_t)t * rpu] = __fmul_rn(rs, acc[t]);
      }
    }
  }

  // copies still in flight (after an abort, the stages never computed)
  for (int i = consumed; i < n_real; ++i) stream::mbar_drain(&s_full[warp][i % R], (uint32_t)((i / R) & 1));
  __syncthreads();
  if constexpr (HS) {
    if (*abort_f && threadIdx.x == 0)  // h copies issued, perhaps never waited for
      for (int i = 0; i < kMaxSlotsS; ++i)
        if (s_hclaim[i]) stream::mbar_drain(&s_hbar[i], 0);
  }
  if constexpr (HR) {
    if (*abort_f && threadIdx.x == 0)
      for (int i = 0; i < kMaxSlotsS; ++i)
        if (s_hissued[i]) stream::mbar_drain(&s_hbar[i % kHRing], (uint32_t)((i / kHRing) & 1));
  }

  // ---- combine of this CTA's output chunks (contract C): every slot's y
  // rows of them are in shared memory
  if (!*abort_f) {
    const int rpu = g.rpu_dn, n = T * nch * rpu;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      const int t = i / (nch * rpu), rem = i - t * nch * rpu, cl = rem / rpu, rr = rem - cl * rpu;
      const float* yc = s_y + (size_t)cl * n_rows * rpu + rr;
      float accc = 0.0f;
      for (int kk = 0; kk < K; ++kk) accc = __fmaf_rn(s_w[t * K + kk], yc[(size_t)s_row[t * K + kk] * rpu], accc);
      for (int s = 0; s < S; ++s) accc = __fadd_rn(accc, yc[(size_t)(s * T + t) * rpu]);
      a.out[(size_t)t * g.H + (size_t)(c0 + cl) * rpu + rr] = accc;
    }
  }
}

// Streaming copy of one expert: one thread per weight block (16 bytes of
// int4, or 32 bytes of int8 split into its even / odd element planes), then
// the scales.
__global__ void prepare_expert_kernel(StreamGeom g, const uint8_t* __restrict__ gq, const uint8_t* __restrict__ uq,
                                      const uint8_t* __restrict__ dq, const float* __restrict__ gs,
                                      const float* __restrict__ us, const float* __restrict__ ds,
                                      unsigned char* __restrict__ dst) {
  const int64_t n_gu = (int64_t)g.I * g.nbh, n_dn = (int64_t)g.H * g.nbi;
  const int64_t total = 2 * n_gu + n_dn;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    int m, r, b;
    const uint8_t* src;
    if (i < 2 * n_gu) {
      m = (int)(i / n_gu);
      const int64_t j = i - m * n_gu;
      r = (int)(j / g.nbh);
      b = (int)(j - (int64_t)r * g.nbh);
      src = (m == 0 ? gq : uq) + (int64_t)r * (g.H / 32) * g.bpb + (int64_t)g.bpb * b;
    } else {
      m = 2;
      const int64_t j = i - 2 * n_gu;
      r = (int)(j / g.nbi);
      b = (int)(j - (int64_t)r * g.nbi);
      src = dq + (int64_t)r * (g.I / 32) * g.bpb + (int64_t)g.bpb * b;
    }
    const uint4 w0 = *reinterpret_cast<const uint4*>(src);
    if (g.bits == 4) {
      *reinterpret_cast<uint4*>(dst + stream_chunk_offset(g, m, r, b, 0)) = w0;
    } else {
      const uint4 w1 = *reinterpret_cast<const uint4*>(src + 16);
      uint4 e, o;
      split_even_odd(w0.x, w0.y, e.x, o.x);
      split_even_odd(w0.z, w0.w, e.y, o.y);
      split_even_odd(w1.x, w1.y, e.z, o.z);
      split_even_odd(w1.z, w1.w, e.w, o.w);
      *reinterpret_cast<uint4*>(dst + stream_chunk_offset(g, m, r, b, 0)) = e;
      *reinterpret_cast<uint4*>(dst + stream_chunk_offset(g, m, r, b, 1)) = o;
    }
  }
  float* sc = reinterpret_cast<float*>(dst + g.sc_off);
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < 2 * g.I + g.H;
       i += (int64_t)gridDim.x * blockDim.x)
    sc[i] = i < g.I ? gs[i] : (i < 2 * g.I ? us[i - g.I] : ds[i - 2 * g.I]);
}

// SMs of the current device (cached per device)
cudaError_t device_sms(int* n) {
  static int sms[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (sms[dev] == 0 && (e = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  *n = sms[dev];
  return cudaSuccess;
}

constexpr size_t kStreamDynMax = 224 * 1024;  // 227 KB per block, less the kernel's static shared memory

template <int TT, int BITS, bool DBG, int GC>
cudaError_t stream_tt(const StreamArgs& a, cudaStream_t st) {
  static int granted[64] = {};
  int n_sms = 0;
  cudaError_t e = device_sms(&n_sms);
  if (e != cudaSuccess) return e;
  const size_t smem = stream_smem_bytes<TT>(a.g, n_sms, a.T, a.T * (a.K + a.S));
  if (smem > kStreamDynMax) return cudaErrorInvalidConfiguration;
  if ((e = smem_opt_in(expert_stream_kernel<TT, BITS, DBG, GC>, (int)smem, granted)) != cudaSuccess) return e;
  // one CTA per SM, all resident at once (down units wait for gate/up units
  // of other CTAs)
  return launch_pdl(expert_stream_kernel<TT, BITS, DBG, GC>, dim3(n_sms), dim3(kSW * 32), smem, st, true, a);
}

}  // namespace

// The instance's dynamic shared memory for this batch plus its static
// shared memory (the capture instance's, the larger) within the device's
// per-block limit.
template <int TT>
bool stream_fits(const StreamGeom& g, int n_sms, int n_tok, int rows) {
  const size_t need = stream_smem_bytes<TT>(g, n_sms, n_tok, rows);
  if (need > kStreamDynMax) return false;
  cudaFuncAttributes fa{};
  if (cudaFuncGetAttributes(&fa, expert_stream_kernel<TT, 4, true, 0>) != cudaSuccess) return false;
  int dev = 0, optin = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    return false;
  return need + fa.sharedSizeBytes <= (size_t)optin;
}

bool stream_supported(int hidden, int inter, int bits, int n_tok, int top_k, int n_shared, int n_experts) {
  if (n_tok < 1 || n_tok > kStreamMaxTok || !stream_shape_ok(hidden, inter, bits)) return false;
  if (top_k < 1 || top_k > kMaxTopK || n_shared < 0 || n_shared > kMaxShared) return false;
  int n_sms = 0;
  if (device_sms(&n_sms) != cudaSuccess) return false;
  const StreamGeom g = stream_geom(hidden, inter, bits);
  const int rows = n_tok * (top_k + n_shared);  // y (and h) rows of the batch
  (void)n_experts;
  return n_tok <= 1   ? stream_fits<1>(g, n_sms, n_tok, rows)
         : n_tok <= 2 ? stream_fits<2>(g, n_sms, n_tok, rows)
         : n_tok <= 4 ? stream_fits<4>(g, n_sms, n_tok, rows)
                      : stream_fits<8>(g, n_sms, n_tok, rows);
}

uint64_t stream_expert_bytes(int hidden, int inter, int bits) { return stream_geom(hidden, inter, bits).expert_bytes; }

cudaError_t launch_prepare_expert(int hidden, int inter, int bits, const uint8_t* gq, const float* gs,
                                  const uint8_t* uq, const float* us, const uint8_t* dq, const float* ds, void* dst,
                                  cudaStream_t st) {
  const StreamGeom g = stream_geom(hidden, inter, bits);
  prepare_expert_kernel<<<592, 256, 0, st>>>(g, gq, uq, dq, gs, us, ds, static_cast<unsigned char*>(dst));
  return cudaGetLastError();
}

template <int BITS, bool DBG, int GC>
cudaError_t stream_g(const StreamArgs& a, cudaStream_t st) {
  if (a.T <= 1) return stream_tt<1, BITS, DBG, GC>(a, st);
  if (a.T <= 2) return stream_tt<2, BITS, DBG, GC>(a, st);
  if (a.T <= 4) return stream_tt<4, BITS, DBG, GC>(a, st);
  return stream_tt<8, BITS, DBG, GC>(a, st);
}

// Full stages (256-byte rows for gate/up and down) take the compile-time
// width; other shapes the run-time loop.
template <int BITS, bool DBG>
cudaError_t stream_bits(const StreamArgs& a, cudaStream_t st) {
  constexpr int kFull = BITS == 4 ? 16 : 8;
  if (a.g.g_gu == kFull && a.g.g_dn == kFull) return stream_g<BITS, DBG, kFull>(a, st);
  return stream_g<BITS, DBG, 0>(a, st);
}

cudaError_t launch_expert_stream(const StreamArgs& a, cudaStream_t st) {
  // the capture is the same kernel with the partial sums also stored
  if (a.dbg != nullptr) return a.g.bits == 8 ? stream_bits<8, true>(a, st) : stream_bits<4, true>(a, st);
  return a.g.bits == 8 ? stream_bits<8, false>(a, st) : stream_bits<4, false>(a, st);
}

}  // namespace coli
