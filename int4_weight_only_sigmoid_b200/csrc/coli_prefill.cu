// coli_prefill.cu -- the expert kernels for many tokens per expert (prefill):
// a grouped GEMM on the 5th-generation tensor cores (tcgen05.mma, F32
// accumulators in tensor memory).  Work items are (tile of <= 128 of one
// slot's tokens, 128 output columns); one persistent CTA per SM walks items
// c, c + G, ... and keeps its pipeline (producers -> MMA -> fold) running
// from one item to the next.
//
// Orientation.  The tokens are the MMA's M dimension (TMEM lanes) and the
// weight rows its N dimension (TMEM columns), so a fold thread owns one
// token: the token's Q8 scale d_x[b] is one register per block, and in the
// gate/up kernel a thread holds its token's 32 consecutive gate rows and the
// matching up rows, so SwiGLU and the Q8 block of h are thread-local.  The
// gate/up item's 128 columns are 64 gate rows and the same 64 up rows.
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
// also needs an int32 -> F32 conversion, and the CUDA cores (weight
// expansion and the fold), not the tensor pipe, are the limit of this layer.
// fp16 operands give F32 sums directly.
//
// Operands.  The activations are converted to fp16 once per forward, one
// row per (slot, token) in slot order (act_rows_f16_kernel; the gate/up fold
// writes h straight as fp16 rows in the same order for the down kernel), in
// the element order [0,4,1,5,2,6,3,7] of every 8 that the int4 expansion
// produces; a tile's A operand is then 128 consecutive rows, loaded by TMA
// (128-byte swizzle).  The packed weights are copied by the producer warps
// with cp.async and expanded into the B operand (K-major, no swizzle).
//
// Roles (448 threads): warps 0-3 producers (packed-weight copies; thread p
// expands weight row p), warp 4 the A-tile TMA loads, warps 5-12 the fold
// (warp w reads TMEM lanes 32(w%4).. = 32 of the tile's tokens, and half of
// the item's columns), warp 13 the MMA issuer (lane 0) and TMEM owner.
// An operand stage holds 4 Q8 blocks (K = 128).  Per stage g: the TMA warp
// loads its A tile into operand stage g % kStages once `empty` (the MMA's
// commit) says the stage is free; the producers copy its packed weights
// kLookS stages ahead (cp.async), expand them into the stage's B part and
// arrive on `full`; the MMA issues two K=16 steps per block into a fresh
// TMEM accumulator per block (4 of them, handed to the fold kHalf blocks at
// a time through `tfull` / `tempty`) and commits `empty`.  All waits are
// bounded (coli_tc.cuh).
//
// Sources: "Colibri：在笔记本上跑744B参数的AI模型", "关键特性" (integer dot
// kernels, Q8_0 activations, packed int4); HN summary (hn.213312.xyz),
// "已实现的功能" (batched MoE: in prefill, an expert used by several
// positions is read once and shared).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <type_traits>
#include <cuda_fp16.h>

#include "coli_launch.h"
#include "coli_tc.cuh"

namespace coli {
namespace {

using namespace tc;

constexpr int kM = 128;        // tokens per tile (MMA M, TMEM lanes)
constexpr int kN = 128;        // output columns per item (MMA N): 64 gate + 64 up rows, or 128 down rows
constexpr int kBS = 4;         // Q8 blocks per operand stage (K = 128)
constexpr int kStages = 3;     // operand stages
constexpr int kLookS = 2;      // stages the producers' copies run ahead
constexpr int kPkSlots = kLookS + 2;  // packed-weight slots: a slot is rewritten only after every producer expanded it
constexpr int kHalf = 2;       // Q8 blocks per accumulator hand-off (MMA -> fold)
constexpr int kTBufs = 4;      // TMEM accumulators (one per block), handed off in pairs
constexpr int kProdWarps = 4;
constexpr int kEpiWarps = 8;   // 2 per TMEM lane quadrant, each half of the columns
// Warp w runs on scheduler w % 4 and, as a fold warp, reads TMEM lanes
// 32 (w % 4)..; the MMA issuer is kept off scheduler 0, which carries the
// fold of tiles with at most 32 tokens.
constexpr int kTmaWarp = kProdWarps;                           // A-tile loads
constexpr int kEpi0 = kProdWarps + 1;                          // first fold warp
constexpr int kMmaWarp = kEpi0 + kEpiWarps;                    // MMA issuer, TMEM owner
constexpr int kThreadsP = 32 * (kMmaWarp + 1);                 // 448
constexpr int kNProd = 32 * kProdWarps;                        // 128 producer threads
constexpr int kTmemCols = kTBufs * kN;                         // 512

struct PSmem {
  static constexpr int kAtomA = kM * 128;           // A: 128 token rows x 64 fp16 (two blocks), 128B-swizzled
  static constexpr int kStageA = 2 * kAtomA;        // a stage's 4 blocks
  static constexpr int kSubB = kN * 64;             // B, one block: 128 weight rows x 32 fp16
  static constexpr int kOpStage = kStageA + kBS * kSubB;
  static constexpr int kPk = kN * kBS * 16;         // packed weights of one stage (row-major, 64 B per row)
  __host__ __device__ static constexpr size_t bytes() {
    return 1024 + (size_t)kStages * kOpStage + (size_t)kPkSlots * kPk;
  }
};

struct Tile {
  int32_t slot, n0;
};

// fp16 operands from packed int4: the 8 nibbles of one 32-bit word (element
// e in bits 4e..4e+3, two's complement) -> 8 fp16 in the order
// [0,4,1,5,2,6,3,7] (the activations use the same order, so the dot product
// is unchanged).  (w & 0x000F000F) ^ 0x64086408 is the fp16 pair
// 1024 + (q + 8) for elements 0 and 4 exactly; the nibbles one position up
// give 1024 + 16 (q + 8), which x 1/16 - 72 maps to q exactly.
__device__ __forceinline__ uint4 expand_int4_word(uint32_t w) {
  const uint32_t w8 = w >> 8;
  uint32_t r[4] = {(w & 0x000F000Fu) ^ 0x64086408u, (w & 0x00F000F0u) ^ 0x64806480u,
                   (w8 & 0x000F000Fu) ^ 0x64086408u, (w8 & 0x00F000F0u) ^ 0x64806480u};
  const __half2 off = __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408));        // 1032
  const __half2 sixteenth = __halves2half2(__ushort_as_half(0x2C00), __ushort_as_half(0x2C00));  // 1/16
  const __half2 m72 = __halves2half2(__ushort_as_half(0xD480), __ushort_as_half(0xD480));        // -72
  uint4 o;
  __half2 h;
  h = __hsub2(*reinterpret_cast<__half2*>(&r[0]), off);
  o.x = *reinterpret_cast<uint32_t*>(&h);
  h = __hfma2(*reinterpret_cast<__half2*>(&r[1]), sixteenth, m72);
  o.y = *reinterpret_cast<uint32_t*>(&h);
  h = __hsub2(*reinterpret_cast<__half2*>(&r[2]), off);
  o.z = *reinterpret_cast<uint32_t*>(&h);
  h = __hfma2(*reinterpret_cast<__half2*>(&r[3]), sixteenth, m72);
  o.w = *reinterpret_cast<uint32_t*>(&h);
  return o;
}

// fp16 operands from 8 int8 values (words a = x0..x3, b = x4..x7), same
// element order: with u = x + 128, 0x6400 | u is 1024 + u; minus 1152 is x.
__device__ __forceinline__ uint4 expand_int8_pair(uint32_t a, uint32_t b) {
  const uint32_t ua = a ^ 0x80808080u, ub = b ^ 0x80808080u;
  const uint32_t t0 = __byte_perm(ua, ub, 0x5140), t1 = __byte_perm(ua, ub, 0x7362);  // u0 u4 u1 u5 | u2 u6 u3 u7
  const uint32_t c = 0x64646464u;
  const __half2 off = __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480));  // 1152, 1152
  uint32_t r[4] = {__byte_perm(t0, c, 0x4140), __byte_perm(t0, c, 0x4342), __byte_perm(t1, c, 0x4140),
                   __byte_perm(t1, c, 0x4342)};
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

// Byte offset of packed block c (0..3) of weight row r in a stage's packed
// copy: 64 B per row, blocks rotated by (r >> 1) & 3 so that 8 consecutive
// rows reading the same block hit 8 different bank groups.
__device__ __forceinline__ uint32_t pk_off(int r, int c) { return r * 64 + ((c ^ ((r >> 1) & 3)) << 4); }

// Byte offset of 16-byte chunk c (0..3) of row r in a K-major, no-swizzle
// operand tile of 32 fp16 per row: 8-row x 16-byte core matrices, the four
// K chunks of an 8-row group 128 B apart (LBO), groups 512 B apart (SBO).
__device__ __forceinline__ uint32_t op_off(int r, int c) { return (r >> 3) * 512 + c * 128 + (r & 7) * 16; }

// fp16 operand rows of the Q8 activations in row order: row r < n_tok*K is
// token perm[r] / K (the routed slots' rows), row n_tok*K + s*n_tok + t is
// token t (shared expert s).  8 values per thread.
__global__ void __launch_bounds__(256) act_rows_f16_kernel(const int8_t* __restrict__ q, const int32_t* perm,
                                                           int n_tok, int top_k, int64_t rows, int hidden,
                                                           uint4* __restrict__ out) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int per_row = hidden / 8;
  if (i >= rows * per_row) return;
  const int64_t r = i / per_row;
  const int c = (int)(i - r * per_row);
  const int64_t routed = (int64_t)n_tok * top_k;
  const int64_t tok = r < routed ? (int64_t)(__ldg(perm + r) / top_k) : (r - routed) % n_tok;
  const uint2 v = __ldg(reinterpret_cast<const uint2*>(q + tok * hidden) + c);
  out[i] = expand_int8_pair(v.x, v.y);
}

// 2D tiled bulk-tensor load (TMA) of box (x, y) into shared memory,
// completing `bytes` on the mbarrier.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

// Shared-memory matrix descriptor, K-major, 128-byte swizzle (the layout a
// TMA load with CU_TENSOR_MAP_SWIZZLE_128B writes): 8-row x 128-byte atoms,
// consecutive 8-row groups 1024 B apart; a K step inside the atom advances
// the start address.
__device__ __forceinline__ uint64_t smem_desc_k_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1 << 16;             // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024 >> 4) << 32;   // stride byte offset
  d |= (uint64_t)1 << 46;             // descriptor version for tcgen05
  d |= (uint64_t)2 << 61;             // SWIZZLE_128B
  return d;
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

// A fold thread's token scales for one hand-off (kHalf blocks).
using DVec = std::conditional_t<kHalf == 2, float2, float>;
[[maybe_unused]] __device__ __forceinline__ float dvec_at(const float2& v, int i) { return i == 0 ? v.x : v.y; }
[[maybe_unused]] __device__ __forceinline__ float dvec_at(float v, int) { return v; }

struct ItemInfo {
  Slot slot;
  int n0, n_valid, m0;
};

// Item i: tile i / nm, column group i % nm (rows [m0, m0 + group_rows) of
// each output matrix).
__device__ __forceinline__ ItemInfo item_info(const Slot* slots, const Tile* tiles, int item, int nm, int group_rows) {
  ItemInfo f;
  const int t = item / nm;
  const Tile tile = tiles[t];
  f.slot = slots[tile.slot];
  f.n0 = tile.n0;
  f.n_valid = min(kM, f.slot.count - tile.n0);
  f.m0 = (item - t * nm) * group_rows;
  return f;
}

// Source row (into the activation / h rows) of token n of the item's tile.
__device__ __forceinline__ int64_t item_token_row(const ItemInfo& f, bool gu, const int32_t* perm, int top_k, int n) {
  if (!gu) return (int64_t)f.slot.row_base + f.n0 + n;
  return f.slot.perm_base < 0 ? (int64_t)(f.n0 + n) : (int64_t)(perm[f.slot.perm_base + f.n0 + n] / top_k);
}

// GU: gate/up (+ SwiGLU + Q8 of h -> hf fp16 rows + hd); !GU: down (-> y).
template <bool GU, typename Tab>
__global__ void __launch_bounds__(kThreadsP, 1) prefill_kernel(
    const __grid_constant__ Tab tab, const __grid_constant__ CUtensorMap amap, const Slot* __restrict__ slots,
    const Tile* __restrict__ tiles,
    const int32_t* __restrict__ n_tiles, const int32_t* __restrict__ perm, int top_k, const float* ad, int hidden,
    int inter, __half* hf, float* hd, float* __restrict__ y, int32_t* __restrict__ err) {
  using L = PSmem;
  constexpr int kGroupRows = GU ? kN / 2 : kN;  // output rows of one matrix per item
  __shared__ uint64_t full_bar[kStages], empty_bar[kStages], tfull_bar[kTBufs / kHalf], tempty_bar[kTBufs / kHalf],
      done_bar;
  __shared__ uint32_t tmem_s;
  __shared__ int abort_s;
  extern __shared__ unsigned char smem_raw[];

  const int dim_in = GU ? hidden : inter;
  const int dim_out = GU ? inter : hidden;
  const int nb = dim_in / 32;
  const int nst = nb / kBS;  // stages per item
  const int nm = dim_out / kGroupRows;
  const int n_items = *n_tiles * nm;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);  // 1 KB aligned
  unsigned char* op_ring = smem;                                  // [kStages][A: 2 atoms | B: kBS x kSubB]
  unsigned char* pk_ring = op_ring + kStages * L::kOpStage;       // [kPkSlots][128 rows][64 B]

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], kProdWarps + 1);  // + the TMA warp's expect_tx
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < kTBufs / kHalf; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], kEpiWarps);
    }
    mbar_init(&done_bar, 1);
    abort_s = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kMmaWarp) tmem_alloc(&tmem_s, kTmemCols);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = tmem_s;
  volatile int* abort = &abort_s;

  if (warp < kProdWarps) {
    // ------------------------------------------------------------ producers
    // A stage's packed weights (128 rows x 64 B) are copied 4 lanes per
    // row, so that each warp instruction touches few cache lines; thread p
    // then expands weight row p of the stage's 4 blocks into the B operand.
    // The copies run kLookS stages ahead across item boundaries: the issue
    // cursor (item ii, stage ji) moves ahead of the expansion.  (The A tiles
    // come from the TMA warp.)
    const int p = threadIdx.x;
    const size_t rb = (size_t)dim_in / 2;
    const int n_mine = blockIdx.x < n_items ? (n_items - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
    const int total = n_mine * nst;
    int ii = blockIdx.x, ji = 0;
    ItemInfo fi{};
    auto enter_item = [&]() {
      if (ii < n_items) fi = item_info(slots, tiles, ii, nm, kGroupRows);
    };
    // weight row r of the issue item: GU rows 0..63 gate, 64..127 up
    auto wrow = [&](int r) -> const uint8_t* {
      if constexpr (GU)
        return (r < kGroupRows ? tab.gate_q[fi.slot.table_idx] : tab.up_q[fi.slot.table_idx]) +
               (size_t)(fi.m0 + (r & (kGroupRows - 1))) * rb;
      else
        return tab.down_q[fi.slot.table_idx] + (size_t)(fi.m0 + r) * rb;
    };
    // packed-weight copies of the cursor's stage (global stage gj) into pk
    // slot gj % kPkSlots; then the cursor moves on
    auto issue = [&](int gj) {
      if (gj < total) {
        const int kb0 = ji * kBS;
        unsigned char* pk = pk_ring + (gj % kPkSlots) * L::kPk;
#pragma unroll
        for (int it = 0; it < 4; ++it) {  // W: row it*32 + p/4, chunk p%4 (= block kb0 + p%4)
          const int q = it * kNProd + p;
          const int r = q >> 2, c = q & 3;
          cp_async16(pk + pk_off(r, c), wrow(r) + (size_t)(kb0 + c) * 16);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
        if (++ji == nst) {
          ji = 0;
          ii += gridDim.x;
          enter_item();
        }
      } else {
        asm volatile("cp.async.commit_group;" ::: "memory");
      }
    };
    enter_item();
#pragma unroll
    for (int i = 0; i < kLookS; ++i) issue(i);
    for (int gs = 0; gs < total; ++gs) {
      issue(gs + kLookS);
      asm volatile("cp.async.wait_group %0;" ::"n"(kLookS) : "memory");  // stage gs's copies (this thread's) are in
      named_bar(1, kNProd);                                              // ... and every producer's
      const int s = gs % kStages;
      // the MMA is done with the operand stage's previous contents
      if (mbar_wait(&empty_bar[s], ((gs / kStages) & 1) ^ 1, abort, err, 10) && !*abort) {
        const unsigned char* pk = pk_ring + (gs % kPkSlots) * L::kPk;
        unsigned char* ob = op_ring + s * L::kOpStage + L::kStageA;
#pragma unroll
        for (int c = 0; c < kBS; ++c) {
          const uint4 w = *reinterpret_cast<const uint4*>(pk + pk_off(p, c));
          unsigned char* dst = ob + c * L::kSubB;
          *reinterpret_cast<uint4*>(dst + op_off(p, 0)) = expand_int4_word(w.x);
          *reinterpret_cast<uint4*>(dst + op_off(p, 1)) = expand_int4_word(w.y);
          *reinterpret_cast<uint4*>(dst + op_off(p, 2)) = expand_int4_word(w.z);
          *reinterpret_cast<uint4*>(dst + op_off(p, 3)) = expand_int4_word(w.w);
        }
      }
      fence_async_smem();  // this thread's operand writes (stores and cp.async) -> the tensor core
      __syncwarp();
      if (lane == 0) mbar_arrive(&full_bar[s]);
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int gs = 0, gh = 0;
      bool ok = true;
      constexpr uint32_t idesc = idesc_f16_f32(kM, kN);
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        for (int j = 0; j < nst && ok; ++j, ++gs) {
          const int s = gs % kStages;
          if (!mbar_wait(&full_bar[s], (gs / kStages) & 1, abort, err, 11)) {
            ok = false;
            break;
          }
          fence_after_sync();
          const uint32_t opa = smem_u32(op_ring + s * L::kOpStage);
          const uint32_t opb = opa + L::kStageA;
#pragma unroll
          for (int hh = 0; hh < kBS / kHalf; ++hh, ++gh) {
            const int hb = gh % (kTBufs / kHalf);
            if (!mbar_wait(&tempty_bar[hb], ((gh / (kTBufs / kHalf)) & 1) ^ 1, abort, err, 12)) {
              ok = false;
              break;
            }
            fence_after_sync();
#pragma unroll
            for (int i = 0; i < kHalf; ++i) {
              const int c = hh * kHalf + i;  // block within the stage
              const uint32_t d = tmem + (hb * kHalf + i) * kN;
#pragma unroll
              for (int k = 0; k < 2; ++k) {  // two K=16 steps = one Q8 block
                const uint64_t da = smem_desc_k_sw128(opa + (c >> 1) * L::kAtomA + (c & 1) * 64 + k * 32);
                const uint64_t db = smem_desc_k_noswizzle(opb + c * L::kSubB + k * 256, 128, 512);
                mma_f16(d, da, db, idesc, k);
              }
            }
            mma_commit(&tfull_bar[hb]);
          }
          if (ok) mma_commit(&empty_bar[s]);
        }
      }
      // every MMA this thread issued has finished before TMEM is released
      mma_commit(&done_bar);
      const long long t0 = clock64();
      while (!mbar_try_wait(&done_bar, 0) && clock64() - t0 < kSpinCycles) {
      }
    }
    __syncwarp();
  } else if (warp == kTmaWarp) {
    // ------------------------------------------------------------ A tiles
    // For each stage: once the MMA is done with the operand stage, one
    // expect_tx arrival on `full` and two TMA loads of 128 rows x 64 fp16
    // (128-byte swizzle) of the row-ordered activations (gate/up) or h
    // (down), rows [row_base + n0, +128) of the item's slot.
    if (lane == 0) {
      int gs = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        const ItemInfo f = item_info(slots, tiles, item, nm, kGroupRows);
        const int row0 = f.slot.row_base + f.n0;
        for (int j = 0; j < nst; ++j, ++gs) {
          const int s = gs % kStages;
          if (!mbar_wait(&empty_bar[s], ((gs / kStages) & 1) ^ 1, abort, err, 16)) {
            ok = false;
            break;
          }
          unsigned char* oa = op_ring + s * L::kOpStage;
          mbar_arrive_expect_tx(&full_bar[s], L::kStageA);
          tma_load_2d(oa, &amap, j * kBS * 32, row0, &full_bar[s]);
          tma_load_2d(oa + L::kAtomA, &amap, j * kBS * 32 + 64, row0, &full_bar[s]);
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ fold
    // warp w: TMEM lanes 32*(w%4).. (tokens); columns c0.. and c1.. (32 each):
    // gate/up: the gate rows [32 hh, 32 hh + 32) of the group and the same
    // up rows (64 columns on); down: columns [64 hh, 64 hh + 64)
    const int quad = warp & 3, hh = (warp - kEpi0) >> 2;
    const int c0 = GU ? 32 * hh : 64 * hh;
    const int c1 = GU ? kGroupRows + 32 * hh : 64 * hh + 32;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const int n = quad * 32 + lane;  // this thread's token within the tile
    int gh = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
      const ItemInfo f = item_info(slots, tiles, item, nm, kGroupRows);
      const bool active = quad * 32 < f.n_valid;  // warp-uniform
      const bool valid = n < f.n_valid;
      const float* drow = ad + (valid ? item_token_row(f, GU, perm, top_k, n) : 0) * nb;
      float acc0[32], acc1[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        acc0[j] = 0.0f;
        acc1[j] = 0.0f;
      }
      // this token's scales, one hand-off (kHalf blocks) per load, one hand-off ahead
      const DVec* dp = reinterpret_cast<const DVec*>(drow);
      DVec dnext = valid ? __ldg(dp) : DVec{};
      for (int j = 0; j < nst; ++j) {
#pragma unroll
        for (int hs = 0; hs < kBS / kHalf; ++hs, ++gh) {
          const DVec dcur = dnext;
          const int hn = j * (kBS / kHalf) + hs + 1;  // next hand-off of this item
          if (valid && hn < nst * (kBS / kHalf)) dnext = __ldg(dp + hn);
          const int hb = gh % (kTBufs / kHalf);
          // warp-uniform: tcgen05.ld is a warp-wide instruction
          const bool ok =
              __all_sync(0xffffffffu, mbar_wait(&tfull_bar[hb], (gh / (kTBufs / kHalf)) & 1, abort, err, 13));
          fence_after_sync();
          if (active && ok) {
#pragma unroll
            for (int i = 0; i < kHalf; ++i) {
              const float dx = dvec_at(dcur, i);
              const uint32_t col = tmem + lane_base + (hb * kHalf + i) * kN;
              // 8 columns of each range at a time (one wait per pair of
              // loads), so that only 16 TMEM values are live
#pragma unroll
              for (int h = 0; h < 4; ++h) {
                uint32_t r0[8], r1[8];
                tmem_ld8(col + c0 + 8 * h, r0);
                tmem_ld8(col + c1 + 8 * h, r1);
                tmem_ld_wait();
#pragma unroll
                for (int jj = 0; jj < 8; jj += 2) {
                  fma2(acc0[8 * h + jj], acc0[8 * h + jj + 1], dx, dx, __uint_as_float(r0[jj]),
                       __uint_as_float(r0[jj + 1]));
                  fma2(acc1[8 * h + jj], acc1[8 * h + jj + 1], dx, dx, __uint_as_float(r1[jj]),
                       __uint_as_float(r1[jj + 1]));
                }
              }
            }
          }
          fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty_bar[hb]);  // the pair of TMEM buffers may be rewritten now
        }
      }
      const bool go = __all_sync(0xffffffffu, !*abort) && active;  // warp-uniform
      if (go && valid) {
        const int64_t row = (int64_t)f.slot.row_base + f.n0 + n;
        if constexpr (GU) {
          const int o = f.m0 + 32 * hh;  // first intermediate row of this thread's Q8 block of h
          const float* sgp = tab.gate_s[f.slot.table_idx] + o;
          const float* sup = tab.up_s[f.slot.table_idx] + o;
          float amax = 0.0f;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float gv = __fmul_rn(__ldg(sgp + j), acc0[j]);
            const float u = __fmul_rn(__ldg(sup + j), acc1[j]);
            acc0[j] = __fmul_rn(__fmul_rn(gv, sigmoid_cw(gv)), u);
            amax = fmaxf(amax, fabsf(acc0[j]));
          }
          const float d = __fdiv_rn(amax, 127.0f);
          // fp16 of q in the operand order: position 2(e&3) + (e>>2) of each 8
          uint32_t pk[16];
#pragma unroll
          for (int e8 = 0; e8 < 4; ++e8) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const __half lo = __int2half_rn(q8_of(acc0[8 * e8 + i], d));
              const __half hi = __int2half_rn(q8_of(acc0[8 * e8 + 4 + i], d));
              pk[4 * e8 + i] = (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
            }
          }
          uint4* dst = reinterpret_cast<uint4*>(hf + row * inter + o);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          hd[row * (inter / 32) + (o >> 5)] = d;
        } else {
          const float* sdp = tab.down_s[f.slot.table_idx] + f.m0;
          float4* dst0 = reinterpret_cast<float4*>(y + row * hidden + f.m0 + c0);
          float4* dst1 = reinterpret_cast<float4*>(y + row * hidden + f.m0 + c1);
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            const float4 s0 = __ldg(reinterpret_cast<const float4*>(sdp + c0 + j));
            const float4 s1 = __ldg(reinterpret_cast<const float4*>(sdp + c1 + j));
            dst0[j / 4] = make_float4(__fmul_rn(s0.x, acc0[j]), __fmul_rn(s0.y, acc0[j + 1]),
                                      __fmul_rn(s0.z, acc0[j + 2]), __fmul_rn(s0.w, acc0[j + 3]));
            dst1[j / 4] = make_float4(__fmul_rn(s1.x, acc1[j]), __fmul_rn(s1.y, acc1[j + 1]),
                                      __fmul_rn(s1.z, acc1[j + 2]), __fmul_rn(s1.w, acc1[j + 3]));
          }
        }
      }
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Tiles of <= kM tokens over the slot table, in slot order.  One warp:
// rounds of 32 slots, a shuffle scan of their tile counts gives each lane
// where its slot's tiles go.
__global__ void build_tiles_kernel(const Slot* __restrict__ slots, const int32_t* __restrict__ n_slots,
                                   Tile* __restrict__ tiles, int32_t* __restrict__ n_tiles) {
  const int lane = threadIdx.x;
  if (lane >= 32) return;
  const int ns = *n_slots;
  int base = 0;
  for (int s0 = 0; s0 < ns; s0 += 32) {
    const int s = s0 + lane;
    const int cnt = s < ns ? slots[s].count : 0;
    const int nt = (cnt + kM - 1) / kM;
    int incl = nt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    for (int i = 0; i < nt; ++i) tiles[base + incl - nt + i] = Tile{s, i * kM};
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) *n_tiles = base;
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
  return (size_t)((pairs + kM - 1) / kM + slots);
}

size_t prefill_tile_bytes(int n_tok, int K, int E, int n_shared) {
  return prefill_tiles_bound(n_tok, K, E, n_shared) * sizeof(Tile);
}

bool prefill_supported(int hidden, int inter) {
  // K a whole number of stages (kBS blocks of 32) for both GEMMs; whole column groups
  return hidden % (32 * kBS) == 0 && inter % (32 * kBS) == 0 && hidden % kN == 0 && inter % (kN / 2) == 0 &&
         PSmem::bytes() <= 227 * 1024;
}

namespace {

// A 2D tensor map over `rows` fp16 rows of `cols` values (row-major), box
// 64 values x kM rows, 128-byte swizzle: the A operand tiles.
cudaError_t make_rows_map(CUtensorMap* m, const void* base, int64_t rows, int cols) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  if (!encode) {
    cudaDriverEntryPointQueryResult q{};
    void* fn = nullptr;
    const cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess) return e;
    if (q != cudaDriverEntryPointSuccess || !fn) return cudaErrorNotSupported;
    encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)kM};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_prefill_experts(const GateUpTable& gu, const DownTable& dn, const Slot* slots,
                                   const int32_t* n_slots, void* tiles, int32_t* n_tiles, const int32_t* perm,
                                   int K, int n_shared, const int8_t* xq, const float* xd, int n_tok, int hidden,
                                   int inter, void* xf, void* hf, float* hd, float* y, int32_t* err,
                                   cudaStream_t st, cudaEvent_t ev_mid) {
  Tile* t = reinterpret_cast<Tile*>(tiles);
  const int64_t rows = (int64_t)n_tok * (K + n_shared);
  const int64_t n8 = rows * hidden / 8;
  act_rows_f16_kernel<<<(unsigned)((n8 + 255) / 256), 256, 0, st>>>(xq, perm, n_tok, K, rows, hidden,
                                                                    reinterpret_cast<uint4*>(xf));
  build_tiles_kernel<<<1, 32, 0, st>>>(slots, n_slots, t, n_tiles);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap map_x, map_h;
  if ((e = make_rows_map(&map_x, xf, rows, hidden)) != cudaSuccess) return e;
  if ((e = make_rows_map(&map_h, hf, rows, inter)) != cudaSuccess) return e;
  static size_t granted_gu[64] = {}, granted_dn[64] = {};
  static int sms_cache[64] = {};
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (sms_cache[dev] == 0 &&
      (e = cudaDeviceGetAttribute(&sms_cache[dev], cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  const size_t smem = PSmem::bytes();
  if ((e = allow_smem(prefill_kernel<true, GateUpTable>, granted_gu, smem)) != cudaSuccess) return e;
  if ((e = allow_smem(prefill_kernel<false, DownTable>, granted_dn, smem)) != cudaSuccess) return e;
  const int grid = sms_cache[dev];
  __half* hfh = reinterpret_cast<__half*>(hf);
  prefill_kernel<true, GateUpTable><<<grid, kThreadsP, smem, st>>>(gu, map_x, slots, t, n_tiles, perm, K, xd, hidden,
                                                                     inter, hfh, hd, y, err);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (ev_mid && (e = cudaEventRecordWithFlags(ev_mid, st, cudaEventRecordExternal)) != cudaSuccess) return e;
  prefill_kernel<false, DownTable><<<grid, kThreadsP, smem, st>>>(dn, map_h, slots, t, n_tiles, perm, K, hd, hidden,
                                                                    inter, hfh, hd, y, err);
  return cudaGetLastError();
}

}  // namespace coli
