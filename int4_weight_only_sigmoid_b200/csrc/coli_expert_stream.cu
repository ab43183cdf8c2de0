// coli_expert_stream.cu -- the expert part of a decode batch (n_tok <= 4)
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
constexpr int kMaxPairsS = kStreamMaxTok * kMaxTopK;  // (token, k) pairs of a batch
constexpr int kMaxSlotsS = kStreamMaxSlots;          // slots: shared + distinct routed experts
constexpr int kErrHReady = 25;                       // status: gave up waiting for a slot's h
constexpr int kErrHStaged = 26;                      // status: gave up waiting for staged h
constexpr int kErrHPair = 27;                        // status: gave up waiting for a pair's h buffer

template <int TT>
struct StreamRing {
  static constexpr int R = TT <= 2 ? 3 : 2;  // stages per warp
};

template <int TT>
__host__ __device__ inline size_t stream_smem_bytes(const StreamGeom& g) {
  const size_t ring = (size_t)kSW * StreamRing<TT>::R * kStreamStageMax;  // 8 KB stages
  const size_t xs = (size_t)TT * g.nbh * 40;        // x planes (32 B) + (d, c16) per block
  const size_t hs = 2 * (size_t)TT * g.nbi * 40;    // two slots' h rows
  return 1024 + ring + xs + hs;
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

__device__ __forceinline__ int even_plane_sum(const uint4& e) {
  int s = __dp4a((int)e.x, 0x01010101, 0);
  s = __dp4a((int)e.y, 0x01010101, s);
  s = __dp4a((int)e.z, 0x01010101, s);
  return __dp4a((int)e.w, 0x01010101, s);
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

// One stage of rows on lanes: blocks b0 .. b0+G-1 of the lane's weight row
// (gate/up halves: lanes 0-15 gate rows, 16-31 the matching up rows; down:
// 32 output rows) against the staged activation planes of the tokens tok[t]
// (row tok[t] of the plane arrays xpl / xdc, nb blocks per row).  The row's
// chunk c sits at (row base | rotation) ^ (c << 4) (the row is aligned to its
// length) and the activation loads are offsets from per-stage bases.  GC > 0
// is a compile-time stage width (straight-line code); GC == 0 takes G at run
// time.
template <int TT, int BITS, bool DBG, int GC>
__device__ __forceinline__ void rows_stage(int Grt, const unsigned char* st, int swz, int b0, int nb, int nv,
                                           const int (&tok)[TT], const uint4* xpl, const float2* xdc,
                                           float (&acc)[TT], int32_t* const (&dbg)[TT]) {
  const int lane = threadIdx.x & 31;
  constexpr int cpb = BITS / 4;  // 16-byte chunks per block
  const int G = GC > 0 ? GC : Grt;
  const uintptr_t rb = reinterpret_cast<uintptr_t>(st + lane * (G * cpb * 16)) | (uintptr_t)((lane & swz) << 4);
  const uint4* xp[TT];
  const float2* xd[TT];
#pragma unroll
  for (int t = 0; t < TT; ++t) {
    xp[t] = xpl + 2 * (tok[t] * nb + b0);
    xd[t] = xdc + tok[t] * nb + b0;
  }
  auto block = [&](int j) {
    uint4 wa, wb;
    if constexpr (BITS == 4) {
      unpack_blk(*reinterpret_cast<const uint4*>(rb ^ (uintptr_t)(j << 4)), wa, wb);
    } else {
      wa = *reinterpret_cast<const uint4*>(rb ^ (uintptr_t)((2 * j) << 4));
      wb = *reinterpret_cast<const uint4*>(rb ^ (uintptr_t)((2 * j + 1) << 4));
    }
#pragma unroll
    for (int t = 0; t < TT; ++t) {
      if (TT == 1 || t < nv) {
        const uint4 xe = xp[t][2 * j], xo = xp[t][2 * j + 1];
        const float2 dc = xd[t][j];
        const int is = isum_of<BITS>(wa, wb, xe, xo, __float_as_int(dc.y));
        if constexpr (DBG) dbg[t][b0 + j] = is;
        acc[t] = __fmaf_rn(dc.x, __int2float_rn(is), acc[t]);
      }
    }
  };
  if constexpr (GC > 0) {
#pragma unroll
    for (int j = 0; j < GC; ++j) block(j);
  } else {
#pragma unroll 4
    for (int j = 0; j < G; ++j) block(j);
  }
}

template <int TT, int BITS, bool DBG, int GC>
__global__ void __launch_bounds__(kSW * 32, 1) expert_stream_kernel(const __grid_constant__ StreamArgs a) {
  constexpr int R = StreamRing<TT>::R;
  constexpr int kPairs = kSW / 2;
  extern __shared__ unsigned char smem_raw[];
  __shared__ uint64_t hbar[2];
  __shared__ int abort_s;
  __shared__ int s_idx[kMaxPairsS], s_row[kMaxPairsS];
  __shared__ float s_w[kMaxPairsS];
  __shared__ int s_exp[kMaxSlotsS], s_cnt[kMaxSlotsS], s_base[kMaxSlotsS], s_tok[kMaxSlotsS][TT];
  __shared__ uint32_t s_bits[kMaxExperts / 32];
  __shared__ int s_nslots;
  __shared__ float s_h[kPairs][2][TT][32];  // a warp pair's h block, double-buffered by unit
  // per unit parity (unit k uses k & 1, like s_h): halves of the pair's
  // units finished, and 1 + the last unit whose Q8 block of h is published
  __shared__ int s_arrive[kPairs][2];
  __shared__ int s_qdone[kPairs][2];
  __shared__ int s_drow[DBG ? kMaxSlotsS : 1][TT];  // capture row of (slot, position): token * (K + S) + rank

  const StreamGeom& g = a.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = a.E, K = a.K, S = a.S, T = a.T;
  unsigned char* smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  unsigned char* ring = smem + (size_t)warp * R * kStreamStageMax;
  uint4* xpl = reinterpret_cast<uint4*>(smem + (size_t)kSW * R * kStreamStageMax);
  float2* xdc = reinterpret_cast<float2*>(xpl + 2 * TT * g.nbh);
  unsigned char* hst = reinterpret_cast<unsigned char*>(xdc + TT * g.nbh);
  const size_t hbuf_bytes = (size_t)TT * g.nbi * 40;
  volatile int* abort_f = &abort_s;

  for (int i = threadIdx.x; i < kMaxExperts / 32; i += blockDim.x) s_bits[i] = 0u;
  if (threadIdx.x < 2 * kPairs) {
    s_arrive[threadIdx.x >> 1][threadIdx.x & 1] = 0;
    s_qdone[threadIdx.x >> 1][threadIdx.x & 1] = 0;
  }
  if (threadIdx.x == 0) {
    tc::mbar_init(&hbar[0], 32);
    tc::mbar_init(&hbar[1], 32);
    abort_s = 0;
    stream::fence_mbar_init();
  }
  __syncthreads();

  // Gate/up work goes to warp pairs: pair p of this CTA takes units
  // gp, gp + NP, ... (gp = p * G + blockIdx.x), warp 2p the first half of
  // each unit, warp 2p + 1 the second.  Down units: this CTA's contiguous
  // range [d0, d1), warp w takes d0 + w, d0 + w + kSW, ...
  const int G = gridDim.x, NP = G * kPairs;
  const int pair = warp >> 1, half = warp & 1, gp = pair * G + blockIdx.x;
  const int n_shared_gu = S * g.cpu_gu;

  // The warp's stage sequence: its gate/up half units, then its down units.
  // A cursor walks it R stages ahead of the compute: (phase, unit index k,
  // stage s, the unit's base address); the divisions happen once per unit.
  // Before the routing is known only the first unit, if it is a shared
  // expert's, can stream.
  int n_gu_mine = 0, n_dn_mine = 0, d0 = 0;
  struct Cursor {
    int phase, k, s;  // phase 0 gate/up, 1 down, 2 done
    const unsigned char* base;
  };
  auto unit_base = [&](Cursor& c) {
    if (c.phase == 0 && c.k >= n_gu_mine) {
      c.phase = 1;
      c.k = 0;
    }
    if (c.phase == 1 && c.k >= n_dn_mine) c.phase = 2;
    if (c.phase == 0) {
      const int u = gp + c.k * NP;
      const int slot = u / g.cpu_gu;
      const int e = slot < S ? E + slot : s_exp[slot];
      c.base = a.prep + (uint64_t)e * g.expert_bytes + (uint64_t)((u - slot * g.cpu_gu) * 2 + half) * g.ub_gu;
    } else if (c.phase == 1) {
      const int v = d0 + warp + c.k * kSW;
      const int slot = v / g.cpu_dn;
      const int e = slot < S ? E + slot : s_exp[slot];
      c.base = a.prep + (uint64_t)e * g.expert_bytes + g.dn_off + (uint64_t)(v - slot * g.cpu_dn) * g.ub_dn;
    }
  };
  Cursor pc{0, 0, 0, nullptr};
  int issued = 0;
  // all lanes: the cursor's stage into ring slot issued % R with cp.async
  // (lane l copies 16-byte chunks l, l + 32, ...: each instruction moves 512
  // contiguous bytes), one commit group per stage (empty past the end)
  auto copy_stage = [&]() {
    if (pc.phase < 2) {
      const uint32_t bytes = pc.phase == 0 ? g.sb_gu : g.sb_dn;
      const unsigned char* src = pc.base + (uint64_t)pc.s * bytes;
      unsigned char* dst = ring + (size_t)(issued % R) * kStreamStageMax;
      for (uint32_t off = 16 * lane; off < bytes; off += 512) cp_async16(dst + off, src + off);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    ++issued;
  };
  auto issue = [&]() {  // copy, then move the cursor on
    copy_stage();
    if (pc.phase < 2 && ++pc.s == (pc.phase == 0 ? g.st_gu : g.st_dn)) {
      pc.s = 0;
      ++pc.k;
      unit_base(pc);
    }
  };

  // shared experts' first stages stream while the router finishes (within
  // the warp's first unit: what follows depends on the routing)
  int pre = 0;
  if (gp < n_shared_gu) {
    n_gu_mine = 1;  // provisional: the first unit
    unit_base(pc);
    for (; pre < R && pre < g.st_gu; ++pre) {
      copy_stage();
      ++pc.s;
    }
  }

  pdl_wait();  // scores, the Q8_0 of x and the cleared counters are complete
  pdl_launch_dependents();

  // ---- routing of the batch (every CTA, identical results) -------------
  if (warp < T) {
    int sel[kMaxTopK];
    float ssel[kMaxTopK];
    topk::warp_select_topk(a.scores + (size_t)warp * E, a.bias, E, K, lane, sel, ssel);
    if (lane == 0) topk::topk_weights(sel, ssel, K, a.norm, a.rsf, s_idx + warp * K, s_w + warp * K);
  }
  // x planes: block b of token t -> even / odd byte planes and (d, c16)
  for (int i = threadIdx.x; i < T * g.nbh; i += blockDim.x) {
    const int t = i / g.nbh, b = i - t * g.nbh;
    const uint4* src = reinterpret_cast<const uint4*>(a.xq + (size_t)t * g.H + 32 * b);
    const uint4 a0 = ld_dep(src), a1 = ld_dep(src + 1);
    uint4 e, o;
    split_even_odd(a0.x, a0.y, e.x, o.x);
    split_even_odd(a0.z, a0.w, e.y, o.y);
    split_even_odd(a1.x, a1.y, e.z, o.z);
    split_even_odd(a1.z, a1.w, e.w, o.w);
    xpl[2 * i] = e;
    xpl[2 * i + 1] = o;
    xdc[i] = make_float2(ld_dep(a.xd + i), __int_as_float(-128 * even_plane_sum(e)));
  }
  __syncthreads();
  const int n_pairs = T * K;
  if (warp == 0) {
    for (int p = lane; p < n_pairs; p += 32) atomicOr(&s_bits[s_idx[p] >> 5], 1u << (s_idx[p] & 31));
    __syncwarp();
    // slot of routed expert e: S + (set bits below e); slots in ascending expert id
    const int nw = (E + 31) / 32;
    const int c = lane < nw ? __popc(s_bits[lane]) : 0;
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const int below_word = incl - c;
    const int n_routed = __shfl_sync(0xffffffffu, incl, 31);
    if (lane < nw) {
      uint32_t bits = s_bits[lane];
      int r = S + below_word;
      while (bits) {
        const int bit = __ffs(bits) - 1;
        bits &= bits - 1;
        s_exp[r] = 32 * lane + bit;
        s_cnt[r] = 0;
        ++r;
      }
    }
    for (int s = lane; s < S; s += 32) {
      s_exp[s] = E + s;
      s_cnt[s] = T;
      for (int t = 0; t < TT; ++t) {
        s_tok[s][t] = t;
        if constexpr (DBG) s_drow[s][t] = t * (K + S) + K + s;
      }
    }
    __syncwarp();
    // each pair: its slot, and its position = earlier tokens on the same expert
    int pslot[2] = {0, 0}, ppos[2] = {0, 0};
    for (int h = 0; h < 2; ++h) {
      const int p = lane + 32 * h;
      if (p < n_pairs) {
        const int e = s_idx[p], t = p / K;
        const int w32 = e >> 5;
        const int lo = __popc(s_bits[w32] & ((1u << (e & 31)) - 1u));
        int below = 0;  // set bits in the words below w32
        for (int q = 0; q < w32; ++q) below += __popc(s_bits[q]);
        pslot[h] = S + below + lo;
        int pos = 0;
        for (int q = 0; q < t * K; ++q) pos += (s_idx[q] == e);
        ppos[h] = pos;
        atomicAdd(&s_cnt[pslot[h]], 1);
        s_tok[pslot[h]][pos] = t;
        if constexpr (DBG) s_drow[pslot[h]][pos] = t * (K + S) + (p - t * K);  // rank p - tK of token t
      }
    }
    __syncwarp();
    if (lane == 0) {
      int base = 0;
      for (int s = 0; s < S + n_routed; ++s) {
        s_base[s] = base;
        base += s_cnt[s];
      }
      s_nslots = S + n_routed;
    }
    __syncwarp();
    for (int h = 0; h < 2; ++h) {
      const int p = lane + 32 * h;
      if (p < n_pairs) s_row[p] = s_base[pslot[h]] + ppos[h];
    }
  }
  __syncthreads();

  const int n_slots = s_nslots;
  const int n_gu = n_slots * g.cpu_gu, n_dn = n_slots * g.cpu_dn;
  n_gu_mine = gp < n_gu ? (n_gu - gp + NP - 1) / NP : 0;
  d0 = (int)((int64_t)blockIdx.x * n_dn / G);
  const int d1 = (int)((int64_t)(blockIdx.x + 1) * n_dn / G);
  n_dn_mine = d0 + warp < d1 ? (d1 - d0 - warp + kSW - 1) / kSW : 0;
  // the down slots of this CTA's range (at most two: a range never spans
  // more, since there are at least as many CTAs as slots)
  const int slotA = d0 / g.cpu_dn;
  const int slotB = d1 > d0 ? (d1 - 1) / g.cpu_dn : slotA;
  const int ownerB = slotB != slotA ? ((slotB * g.cpu_dn - d0) % kSW) : -1;

  if (pre == 0) {
    unit_base(pc);  // the cursor's first unit, now that the counts are known
  } else if (pc.s == g.st_gu) {
    pc.s = 0;  // the first unit was streamed whole before the routing: on to the next
    pc.k = 1;
    unit_base(pc);
  }
  for (int i = pre; i < R; ++i) issue();

  int consumed = 0;
  bool ok = true;
  // this lane's copies of the oldest stage are in (R - 1 newer groups may
  // still be in flight), then every lane's
  auto wait_stage = [&]() {
    asm volatile("cp.async.wait_group %0;" ::"n"(R - 1) : "memory");
    __syncwarp();
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
  int staged_slot = -1;
  const int n_units = n_gu_mine + n_dn_mine;
  for (int k = 0; k < n_units && ok; ++k) {
    const bool gu = k < n_gu_mine;
    int slot, chunk, nv, nst, Gs, swz, nb;
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
      ap = xpl;
      adc = xdc;
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
      const int v = d0 + warp + (k - n_gu_mine) * kSW;
      slot = v / g.cpu_dn;
      chunk = v - slot * g.cpu_dn;
      nv = s_cnt[slot];
      nst = g.st_dn;
      Gs = g.g_dn;
      swz = g.swz_dn;
      nb = g.nbi;
      const int buf = slot == slotA ? 0 : 1;
      unsigned char* hb = hst + (size_t)buf * hbuf_bytes;
      if (slot != staged_slot) {
        const bool owner = buf == 0 ? warp == 0 : warp == ownerB;
        if (owner) {
          // wait for every gate/up unit of the slot, then copy its h rows
          int ready = 0;
          if (lane == 0) {
            const long long t0 = clock64();
            while (!*abort_f) {
              if (ld_acquire_gpu(a.h_ready + slot) >= g.cpu_gu) {
                ready = 1;
                break;
              }
              if (clock64() - t0 > tc::kSpinCycles) {
                *abort_f = 1;
                atomicExch(a.status, kErrHReady);
                break;
              }
              __nanosleep(128);
            }
          }
          ready = __shfl_sync(0xffffffffu, ready, 0);
          if (ready) {
            const uint4* sp = reinterpret_cast<const uint4*>(a.hpl + (size_t)s_base[slot] * g.nbi * 32);
            uint4* dp = reinterpret_cast<uint4*>(hb);
            const int n16 = nv * g.nbi * 2;
            for (int i = lane; i < n16; i += 32) dp[i] = __ldcg(sp + i);
            const float4* sd = reinterpret_cast<const float4*>(a.hdc + (size_t)s_base[slot] * g.nbi);
            float4* dd = reinterpret_cast<float4*>(hb + (size_t)TT * g.nbi * 32);
            for (int i = lane; i < nv * g.nbi / 2; i += 32) dd[i] = __ldcg(sd + i);
          }
          tc::mbar_arrive(&hbar[buf]);  // all 32 lanes: the stores above are released to the CTA
        }
        const bool got = tc::mbar_wait(&hbar[buf], 0, abort_f, a.status, kErrHStaged);
        if (!__all_sync(0xffffffffu, got && !*abort_f)) {  // warp-uniform
          ok = false;
          break;
        }
        staged_slot = slot;
      }
      ap = reinterpret_cast<const uint4*>(hb);
      adc = reinterpret_cast<const float2*>(hb + (size_t)TT * g.nbi * 32);
      const int o = chunk * 32 + lane;
#pragma unroll
      for (int t = 0; t < TT; ++t) {
        tok[t] = t;  // the staged h rows are the slot's tokens in order
        dbg[t] = nullptr;
        if constexpr (DBG)
          if (t < nv) dbg[t] = a.dbg + s_drow[slot][t] * P + 2 * (int64_t)g.I * g.nbh + (int64_t)o * g.nbi;
      }
    }
    float acc[TT];
#pragma unroll
    for (int t = 0; t < TT; ++t) acc[t] = 0.0f;
    for (int s = 0; s < nst; ++s) {
      wait_stage();
      rows_stage<TT, BITS, DBG, GC>(Gs, ring + (size_t)(consumed % R) * kStreamStageMax, swz, s * Gs, nb, nv, tok,
                                    ap, adc, acc, dbg);
      next_stage();
    }
    const float* sc = reinterpret_cast<const float*>(a.prep + (uint64_t)s_exp[slot] * g.expert_bytes + g.sc_off);
    if (gu) {
      // SwiGLU of the half's 16 outputs into shared memory; the second warp
      // of the pair to finish quantises the whole Q8_0 block of h and
      // publishes it (no warp waits for the other)
      const int orow = chunk * 32 + 16 * half + (lane & 15);
      const float sv = __ldg(sc + (lane < 16 ? 0 : g.I) + orow);
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
#pragma unroll
      for (int t = 0; t < TT; ++t) {
        const float v = __fmul_rn(sv, acc[t]);
        const float uv = __shfl_down_sync(0xffffffffu, v, 16);
        if (lane < 16 && t < nv) hbuf[t * 32 + 16 * half + lane] = __fmul_rn(__fmul_rn(v, sigmoid_cw(v)), uv);
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
        __syncwarp();
        if (lane == 0) {
          *(volatile int*)&s_qdone[pair][k & 1] = k + 1;
          __threadfence();
          atomicAdd(a.h_ready + slot, 1);
        }
      }
      ok = !*abort_f;
    } else {
      const int o = chunk * 32 + lane;
      const float sd = __ldg(sc + 2 * g.I + o);
#pragma unroll
      for (int t = 0; t < TT; ++t)
        if (t < nv) a.y[((size_t)s_base[slot] + t) * g.H + o] = __fmul_rn(sd, acc[t]);
      __syncwarp();
      int last = 0;
      if (lane == 0) {
        __threadfence();
        last = atomicAdd(a.dn_done + chunk, 1) == n_slots - 1;
        if (last) __threadfence();
      }
      last = __shfl_sync(0xffffffffu, last, 0);
      if (last) {
        // every slot's y rows of this chunk are written: combine (contract C)
        for (int t = 0; t < T; ++t) {
          float accc = 0.0f;
          for (int kk = 0; kk < K; ++kk)
            accc = __fmaf_rn(s_w[t * K + kk], __ldcg(a.y + (size_t)s_row[t * K + kk] * g.H + o), accc);
          for (int s = 0; s < S; ++s) accc = __fadd_rn(accc, __ldcg(a.y + ((size_t)s_base[s] + t) * g.H + o));
          a.out[(size_t)t * g.H + o] = accc;
        }
      }
    }
  }

  // copies still in flight (after an abort, the stages never computed)
  asm volatile("cp.async.wait_all;" ::: "memory");
  // an owner that gave up before arriving leaves hbar incomplete: waiters give up too (bounded)
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

template <int TT, int BITS, bool DBG, int GC>
cudaError_t stream_tt(const StreamArgs& a, cudaStream_t st) {
  static int granted[64] = {};
  static int sms[64] = {};
  const size_t smem = stream_smem_bytes<TT>(a.g);
  if (smem > 224 * 1024) return cudaErrorInvalidConfiguration;
  cudaError_t e = smem_opt_in(expert_stream_kernel<TT, BITS, DBG, GC>, (int)smem, granted);
  if (e != cudaSuccess) return e;
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if (sms[dev] == 0 && (e = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  // one CTA per SM, all resident at once (the down units wait for gate/up
  // units of other CTAs); at least as many CTAs as slots, so that a CTA's
  // range of down units spans at most two slots
  if (sms[dev] < kMaxSlotsS) return cudaErrorInvalidConfiguration;
  return launch_pdl(expert_stream_kernel<TT, BITS, DBG, GC>, dim3(sms[dev]), dim3(kSW * 32), smem, st, true, a);
}

}  // namespace

bool stream_supported(int hidden, int inter, int bits, int n_tok) {
  if (n_tok < 1 || n_tok > kStreamMaxTok || !stream_shape_ok(hidden, inter, bits)) return false;
  const StreamGeom g = stream_geom(hidden, inter, bits);
  constexpr size_t kDyn = 224 * 1024;  // 227 KB per block, less the kernel's static shared memory
  return stream_smem_bytes<4>(g) <= kDyn && stream_smem_bytes<1>(g) <= kDyn && stream_smem_bytes<2>(g) <= kDyn;
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
  return stream_tt<4, BITS, DBG, GC>(a, st);
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
