// coli_prefill.cu -- the expert kernels for many tokens per expert (prefill):
// a grouped int8 GEMM on the 5th-generation tensor cores
// (tcgen05.mma.kind::i8, int32 accumulators in tensor memory).  Work items
// are (tile of <= 128 of one slot's tokens, 128 output columns); one
// persistent CTA per SM walks items c, c + G, ... and keeps its pipeline
// (producers -> MMA -> fold) running from one item to the next.
//
// Orientation.  The tokens are the MMA's M dimension (TMEM lanes) and the
// weight rows its N dimension (TMEM columns), so a fold thread owns one
// token: the token's Q8 scale d_x[b] is one register per block, and in the
// gate/up kernel a thread holds its token's 32 consecutive gate rows and the
// matching up rows, so SwiGLU and the Q8 block of h are thread-local.  The
// gate/up item's 128 columns are 64 gate rows and the same 64 up rows.
//
// int8 expert weights (the pages' int8 variant) take the same kernel with
// B = q copied as it is and A in the elements' own order.
//
// Operands.  A = the Q8 activations as signed bytes (one row per (slot,
// token) in slot order, loaded by TMA, 128-byte swizzle); B = the weights as
// signed bytes 16 q, expanded from the packed nibbles by the producer warps:
// for a packed word w, (w << 4) & 0xF0F0F0F0 holds 16 q of elements
// 0, 2, 4, 6 and w & 0xF0F0F0F0 of elements 1, 3, 5, 7 -- two logic ops per
// 8 weights, and the A rows are stored in the same order (per 8 elements:
// 0,2,4,6,1,3,5,7), so the dot product is 16 times the block's.  One MMA
// (K = 32) is exactly one Q8 block.
//
// Exactness.  Each Q8 block's partial sum must come out exactly, because the
// row fold (contract F: acc = fmaf(d_x[b], (float)isum[b], acc), b
// ascending) needs it per block.  The MMA of block b writes S = 16 isum
// (int8 weights: isum) into a fresh int32 accumulator (the previous contents
// are not read).  |S| < 2^22, so S + 0x4B400000 read as a binary32 is
// 1.5 * 2^23 + S exactly: one integer add and one FMA (x 1/16, - 1.5 * 2^19)
// give (float)isum with no integer-to-float conversion.  The fold then
// applies contract F per block, so prefill equals the dp4a paths bit for
// bit.
//
// Roles (640 threads): warps 0-1 producers (each makes every other operand
// stage on its own: packed-weight copies and the expansion of the stage's
// 128 weight rows), warp 2 the A-tile TMA loads, warps 3-18 the fold, warp
// 19 the MMA issuer (lane 0) and TMEM owner.  (20 warps, 5 per scheduler,
// leave 96 registers per thread.)  Fold of an item of more than 32 tokens:
// warp w reads TMEM lanes 32(w%4).. = 32 of the tile's tokens, and a quarter
// of the item's columns (gate/up 16 gate rows and the same 16 up rows, down
// 32 rows); the two warps that hold one Q8 block of h (32 intermediate rows)
// meet at a named barrier to share the block's absmax.  An item of at most
// 32 tokens is computed with the weights as the MMA's M (128 TMEM lanes) and
// the tokens as its N (32 columns per block): warp w folds weight rows
// 32(w%4).. for 8 of the tokens.
// An operand stage holds 4 Q8 blocks (K = 128).  Per stage g: the TMA warp
// loads its A tile into operand stage g % kStages once `empty` (the MMA's
// commit) says the stage is free; a producer warp copies its packed weights
// a few stages ahead (cp.async), expands them into the stage's B part and
// arrives on `full`; the MMA issues one K=32 step per block onto a TMEM
// accumulator per block (handed to the fold through `tfull` / `tempty`, two
// blocks at a time, or eight for an item of at most 32 tokens) and commits
// `empty`.  The fold reads a buffer and releases it.  All waits are bounded
// (coli_tc.cuh).
//
// Sources: "Colibri：在笔记本上跑744B参数的AI模型", "关键特性" (integer dot
// kernels, Q8_0 activations, packed int4); HN summary (hn.213312.xyz),
// "已实现的功能" (batched MoE: in prefill, an expert used by several
// positions is read once and shared).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <type_traits>

#include "coli_launch.h"
#include "coli_tc.cuh"

namespace coli {
namespace {

using namespace tc;

constexpr int kM = 128;        // tokens per tile (MMA M, TMEM lanes)
constexpr int kN = 128;        // output columns per item (MMA N): 64 gate + 64 up rows, or 128 down rows
constexpr int kBS = 4;         // Q8 blocks per operand stage (K = 128)
constexpr int kStages = 4;     // operand stages
// The producers' packed-weight copies: kPkSlots slots of kPk bytes, int4
// rows (64 B per stage) in 8 slots of 8 KB, int8 rows (128 B) in 4 slots of
// 16 KB -- the same 64 KB.  Stage gs uses slot gs % kPkSlots; a producer
// warp's stages are every kProdWarps-th, so a slot is reused only by the warp
// that expanded its previous stage.
template <int BITS>
struct PkRing {
  static constexpr int kPkSlots = BITS == 4 ? 8 : 4;
  static constexpr int kPk = 128 * 4 * BITS * 4;
};
static_assert(PkRing<4>::kPkSlots * PkRing<4>::kPk == PkRing<8>::kPkSlots * PkRing<8>::kPk, "one ring size");
constexpr int kHalf = 2;       // Q8 blocks per accumulator hand-off (MMA -> fold): 1 or 2
constexpr int kTBufs = 4;      // TMEM accumulators (one per block), handed off in pairs
constexpr int kNL = 32;        // light items (<= kNL tokens): the tokens are the MMA's N
constexpr int kProdWarps = 2;
constexpr int kEpiWarps = 16;  // 4 per TMEM lane quadrant, each a quarter of the columns
// Warp w runs on scheduler w % 4 and, as a fold warp, reads TMEM lanes
// 32 (w % 4)..; the MMA issuer is kept off scheduler 0, which carries the
// fold of tiles with at most 32 tokens.
constexpr int kTmaWarp = kProdWarps;                           // A-tile loads
constexpr int kEpi0 = kProdWarps + 1;                          // first fold warp
constexpr int kMmaWarp = kEpi0 + kEpiWarps;                    // MMA issuer, TMEM owner
constexpr int kThreadsP = 32 * (kMmaWarp + 1);                 // 640
constexpr int kTmemCols = kTBufs * kN;                         // 512
constexpr uint32_t kMagic = 0x4B400000u;                       // binary32 1.5 * 2^23
constexpr float kMagicF = 12582912.0f;

struct PSmem {
  static constexpr int kStageA = kM * 128;          // A: 128 token rows x 128 int8 (4 blocks), 128B-swizzled
  static constexpr int kSubB = kN * 32;             // B, one block: 128 weight rows x 32 bytes
  static constexpr int kOpStage = kStageA + kBS * kSubB;
  static constexpr int kPkRing = PkRing<8>::kPkSlots * PkRing<8>::kPk;  // packed-weight copies (either width)
  __host__ __device__ static constexpr size_t bytes() {
    return 1024 + (size_t)kStages * kOpStage + (size_t)kPkRing;
  }
};

struct Tile {
  int32_t slot, n0;
};

// Byte offset of 16-byte chunk c of weight row r in a stage's copy of the
// weights: int4 rows are 64 B (4 chunks, one per block), rotated by
// (r >> 1) & 3; int8 rows are 128 B (8 chunks, two per block), rotated by
// r & 7; either way 8 consecutive rows reading the same chunk hit 8
// different bank groups.
template <int BITS>
__device__ __forceinline__ uint32_t pk_off(int r, int c) {
  if constexpr (BITS == 4) return r * 64 + ((c ^ ((r >> 1) & 3)) << 4);
  return r * 128 + ((c ^ (r & 7)) << 4);
}

// Byte offset of 16-byte chunk c (0..1) of row r in a K-major, no-swizzle
// operand tile of 32 bytes per row: 8-row x 16-byte core matrices, the two
// K chunks of an 8-row group 128 B apart (LBO), groups 256 B apart (SBO).
__device__ __forceinline__ uint32_t op_off(int r, int c) { return (r >> 3) * 256 + c * 128 + (r & 7) * 16; }

// 16 q of the 8 nibbles of a packed word, as signed bytes in the order
// 0,2,4,6 (lo) then 1,3,5,7 (hi): each nibble moved to the high half of its
// byte.
__device__ __forceinline__ void expand_word(uint32_t w, uint32_t& lo, uint32_t& hi) {
  lo = (w << 4) & 0xF0F0F0F0u;
  hi = w & 0xF0F0F0F0u;
}

// Operand rows of the Q8 activations in row order: row r < n_tok*K is
// token perm[r] / K (the routed slots' rows), row n_tok*K + s*n_tok + t is
// token t (shared expert s).  With int4 weights, within every 8 elements the
// order 0,2,4,6,1,3,5,7 (the order of the expanded weights); with int8
// weights the elements' own order.  16 values per thread.
template <int BITS>
__global__ void __launch_bounds__(256) act_rows_i8_kernel(const int8_t* __restrict__ q, const int32_t* perm,
                                                          int n_tok, int top_k, int64_t rows, int hidden,
                                                          uint4* __restrict__ out) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int per_row = hidden / 16;
  if (i >= rows * per_row) return;
  const int64_t r = i / per_row;
  const int c = (int)(i - r * per_row);
  const int64_t routed = (int64_t)n_tok * top_k;
  const int64_t tok = r < routed ? (int64_t)(__ldg(perm + r) / top_k) : (r - routed) % n_tok;
  const uint4 v = __ldg(reinterpret_cast<const uint4*>(q + tok * hidden) + c);
  if constexpr (BITS == 8) {
    out[i] = v;
  } else {
    uint4 o;
    split_even_odd(v.x, v.y, o.x, o.y);
    split_even_odd(v.z, v.w, o.z, o.w);
    out[i] = o;
  }
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

// Instruction descriptor of kind::i8: signed A (activations) and B
// (weights: 16 q for int4, q for int8), int32 accumulator, shape M x N,
// both K-major.
__host__ __device__ constexpr uint32_t idesc_i8_s32(int M, int N) {
  return (2u << 4)                       // D format: S32
         | (1u << 7)                     // A format: S8
         | (1u << 10)                    // B format: S8
         | ((uint32_t)(N >> 3) << 17)    // N / 8
         | ((uint32_t)(M >> 4) << 24);   // M / 16
}

// D[tmem] = A[smem] * B[smem]^T (int8 operands, int32 result; the
// accumulator's previous contents are not read), issued by one thread.
__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, 0, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc)
      : "memory");
}


// fma / add on two F32 lanes at once (each lane one IEEE operation, rounded once).
__device__ __forceinline__ void fma2(float& a0, float& a1, float d0, float d1, float x0, float x1) {
  unsigned long long acc, dd, xx;
  asm("mov.b64 %0, {%1,%2};" : "=l"(acc) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1,%2};" : "=l"(dd) : "f"(d0), "f"(d1));
  asm("mov.b64 %0, {%1,%2};" : "=l"(xx) : "f"(x0), "f"(x1));
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(dd), "l"(xx));
  asm("mov.b64 {%0,%1}, %2;" : "=f"(a0), "=f"(a1) : "l"(acc));
}
// x = fma(x, a, c) on two F32 lanes with the same a and c.
__device__ __forceinline__ void fma2c(float& x0, float& x1, float a, float c) {
  unsigned long long xx, aa, cc;
  asm("mov.b64 %0, {%1,%2};" : "=l"(xx) : "f"(x0), "f"(x1));
  asm("mov.b64 %0, {%1,%1};" : "=l"(aa) : "f"(a));
  asm("mov.b64 %0, {%1,%1};" : "=l"(cc) : "f"(c));
  asm("fma.rn.f32x2 %0, %0, %1, %2;" : "+l"(xx) : "l"(aa), "l"(cc));
  asm("mov.b64 {%0,%1}, %2;" : "=f"(x0), "=f"(x1) : "l"(xx));
}

struct ItemInfo {
  Slot slot;
  int n0, n_valid, m0;
};

// The partials capture (coli_debug_capture_partials): buffer, and what maps a
// slot row to its capture row token * (K + S) + rank (shared s: rank K + s).
struct DbgArgs {
  int32_t* buf;
  int E, S;
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

// Capture row of token n of the item's tile: token * (K + S) + rank (shared
// expert s: rank K + s), and the capture's words per row.
__device__ __forceinline__ int64_t dbg_row(const ItemInfo& f, const int32_t* perm, int top_k, const DbgArgs& dbg,
                                           int n) {
  if (f.slot.perm_base < 0) return (int64_t)(f.n0 + n) * (top_k + dbg.S) + top_k + (f.slot.table_idx - dbg.E);
  const int pr = perm[f.slot.perm_base + f.n0 + n];
  return (int64_t)(pr / top_k) * (top_k + dbg.S) + pr % top_k;
}
__device__ __forceinline__ int64_t dbg_words(int hidden, int inter) {
  return 2 * (int64_t)inter * (hidden / 32) + (int64_t)hidden * (inter / 32);
}

// Row of token n of the item's tile in the per-token arrays: gate/up: the
// token itself (x's scales and block sums); down: the (slot, token) row.
__device__ __forceinline__ int64_t item_token_row(const ItemInfo& f, bool gu, const int32_t* perm, int top_k, int n) {
  if (!gu) return (int64_t)f.slot.row_base + f.n0 + n;
  return f.slot.perm_base < 0 ? (int64_t)(f.n0 + n) : (int64_t)(perm[f.slot.perm_base + f.n0 + n] / top_k);
}

// GU: gate/up (+ SwiGLU + Q8 of h -> hr int8 rows + hd); !GU: down (-> y).
// ad: the A rows' Q8 scales, [row x nb].
template <bool GU, int BITS, bool DBG, typename Tab>
__global__ void __launch_bounds__(kThreadsP, 1) prefill_kernel(
    const __grid_constant__ Tab tab, const __grid_constant__ CUtensorMap amap,
    const __grid_constant__ CUtensorMap amap32, const Slot* __restrict__ slots,
    const Tile* __restrict__ tiles, const int32_t* __restrict__ n_tiles, const int32_t* __restrict__ perm, int top_k,
    const float* ad, int hidden, int inter, int8_t* hr, float* hd, float* __restrict__ y, int32_t* __restrict__ err,
    DbgArgs dbg) {
  using L = PSmem;
  constexpr int kGroupRows = GU ? kN / 2 : kN;  // output rows of one matrix per item
  __shared__ uint64_t full_bar[kStages], empty_bar[kStages], tfull_bar[kTBufs / kHalf], tempty_bar[kTBufs / kHalf],
      done_bar;
  __shared__ uint32_t tmem_s;
  __shared__ int abort_s;
  __shared__ float s_amax[2][kEpiWarps][32];  // gate/up fold: half-block absmax per (warp, token), by item parity
  // gate/up fold of light items: the up rows' products per (c4, quadrant 2/3, lane, token), by item parity
  __shared__ float s_up[GU ? 2 : 1][kEpiWarps / 4][64][8];
  extern __shared__ unsigned char smem_raw[];

  const int dim_in = GU ? hidden : inter;
  const int dim_out = GU ? inter : hidden;
  const int nb = dim_in / 32;
  const int nst = nb / kBS;  // stages per item
  const int nm = dim_out / kGroupRows;
  const int n_items = *n_tiles * nm;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);  // 1 KB aligned
  unsigned char* op_ring = smem;                                  // [kStages][A | B: kBS x kSubB]
  unsigned char* pk_ring = op_ring + kStages * L::kOpStage;       // [kPkSlots][128 rows][BITS * 16 B]

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 2);  // the stage's producer warp + the TMA warp's expect_tx
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
    // Producer warp pw makes the operand stages gs = pw, pw + kProdWarps, ...
    // of this CTA on its own: it copies the stage's packed weights (4 lanes
    // per 64-byte int4 row, so that each instruction touches few cache lines)
    // kLookW of its stages ahead with cp.async, and expands all 128 weight
    // rows of the stage's 4 blocks into the B operand (lane l: rows l,
    // l + 32, ...).  (The A tiles come from the TMA warp.)
    constexpr int kPkSlots = PkRing<BITS>::kPkSlots, kPk = PkRing<BITS>::kPk;
    constexpr int kLookW = kPkSlots / kProdWarps - 1;  // own stages in flight beyond the one expanded
    const int pw = warp;
    const size_t rb = (size_t)dim_in * BITS / 8;  // bytes per weight row
    constexpr int kChunks = BITS == 4 ? 4 : 8;      // 16-byte chunks per row per stage
    const int n_mine = blockIdx.x < n_items ? (n_items - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
    const int total = n_mine * nst;
    // packed-weight copies of stage gj (the (gj / nst)-th item of this CTA)
    // into pk slot gj % kPkSlots, as one commit group (empty past the end)
    auto issue = [&](int gj) {
      if (gj < total) {
        const int k = gj / nst, ji = gj - k * nst;
        const ItemInfo fi = item_info(slots, tiles, blockIdx.x + k * gridDim.x, nm, kGroupRows);
        const int kb0 = ji * kBS;
        unsigned char* pk = pk_ring + (gj % kPkSlots) * kPk;
#pragma unroll 4
        for (int it = 0; it < kChunks * kN / 32; ++it) {  // row q / kChunks, chunk q % kChunks of the stage's bytes
          const int q = it * 32 + lane;
          const int r = q / kChunks, c = q % kChunks;
          const uint8_t* w;  // weight row r of the item: GU rows 0..63 gate, 64..127 up
          if constexpr (GU)
            w = (r < kGroupRows ? tab.gate_q[fi.slot.table_idx] : tab.up_q[fi.slot.table_idx]) +
                (size_t)(fi.m0 + (r & (kGroupRows - 1))) * rb;
          else
            w = tab.down_q[fi.slot.table_idx] + (size_t)(fi.m0 + r) * rb;
          cp_async16(pk + pk_off<BITS>(r, c), w + (size_t)kb0 * (BITS * 4) + (size_t)c * 16);
        }
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
    };
#pragma unroll
    for (int u = 0; u < kLookW; ++u) issue(pw + u * kProdWarps);
    for (int u = 0;; ++u) {
      const int gs = pw + u * kProdWarps;
      if (gs >= total) break;
      issue(gs + kLookW * kProdWarps);
      asm volatile("cp.async.wait_group %0;" ::"n"(kLookW) : "memory");  // stage gs's copies (this lane's) are in
      __syncwarp();                                                       // ... and the warp's
      const int s = gs % kStages;
      // the MMA is done with the operand stage's previous contents
      if (mbar_wait(&empty_bar[s], ((gs / kStages) & 1) ^ 1, abort, err, 10) && !*abort) {
        const unsigned char* pk = pk_ring + (gs % kPkSlots) * kPk;
        unsigned char* ob = op_ring + s * L::kOpStage + L::kStageA;
#pragma unroll 1
        for (int rr = 0; rr < kN / 32; rr += 2) {
          if constexpr (BITS == 4) {
            // two rows' packed words first, then the expansion and the stores
            uint4 w[2][kBS];
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int c = 0; c < kBS; ++c)
                w[h][c] = *reinterpret_cast<const uint4*>(pk + pk_off<4>(lane + (rr + h) * 32, c));
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int pr = lane + (rr + h) * 32;  // the weight row this lane expands
#pragma unroll
              for (int c = 0; c < kBS; ++c) {
                unsigned char* dst = ob + c * L::kSubB;
                uint4 o0, o1;
                expand_word(w[h][c].x, o0.x, o0.y);
                expand_word(w[h][c].y, o0.z, o0.w);
                expand_word(w[h][c].z, o1.x, o1.y);
                expand_word(w[h][c].w, o1.z, o1.w);
                *reinterpret_cast<uint4*>(dst + op_off(pr, 0)) = o0;
                *reinterpret_cast<uint4*>(dst + op_off(pr, 1)) = o1;
              }
            }
          } else {  // int8 rows are the operand as they are
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int pr = lane + (rr + h) * 32;
#pragma unroll
              for (int c = 0; c < kBS; ++c) {
                unsigned char* dst = ob + c * L::kSubB;
                const uint4 o0 = *reinterpret_cast<const uint4*>(pk + pk_off<8>(pr, 2 * c));
                const uint4 o1 = *reinterpret_cast<const uint4*>(pk + pk_off<8>(pr, 2 * c + 1));
                *reinterpret_cast<uint4*>(dst + op_off(pr, 0)) = o0;
                *reinterpret_cast<uint4*>(dst + op_off(pr, 1)) = o1;
              }
            }
          }
        }
      }
      fence_async_smem();  // this lane's operand writes -> the tensor core
      __syncwarp();
      if (lane == 0) mbar_arrive(&full_bar[s]);
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int gs = 0, gh = 0;
      bool ok = true;
      constexpr uint32_t idesc = idesc_i8_s32(kM, kN);
      constexpr uint32_t idesc_l = idesc_i8_s32(kN, kNL);  // light: weights as M, tokens as N
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        if (item_info(slots, tiles, item, nm, kGroupRows).n_valid <= kNL) {
          // light item: one hand-off per two stages (8 blocks of kNL
          // columns in one 256-column pair of buffers)
          for (int j = 0; j < nst && ok; ++j, ++gs) {
            const int s = gs % kStages;
            if (!mbar_wait(&full_bar[s], (gs / kStages) & 1, abort, err, 11)) {
              ok = false;
              break;
            }
            fence_after_sync();
            const uint32_t opa = smem_u32(op_ring + s * L::kOpStage);
            const uint32_t opb = opa + L::kStageA;
            const int hb = gh % (kTBufs / kHalf);
            if ((j & 1) == 0) {
              if (!mbar_wait(&tempty_bar[hb], (gh / (kTBufs / kHalf)) & 1, abort, err, 12)) {
                ok = false;
                break;
              }
              fence_after_sync();
            }
#pragma unroll
            for (int c = 0; c < kBS; ++c) {
              const uint32_t d = tmem + hb * kHalf * kN + (j & 1) * kBS * kNL + c * kNL;
              const uint64_t da = smem_desc_k_noswizzle(opb + c * L::kSubB, 128, 256);
              const uint64_t db = smem_desc_k_sw128(opa + c * 32);
              mma_i8(d, da, db, idesc_l);
            }
            if ((j & 1) == 1 || j == nst - 1) {
              mma_commit(&tfull_bar[hb]);
              ++gh;
            }
            mma_commit(&empty_bar[s]);
          }
          continue;
        }
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
            // the fold has read the pair's previous values and written their starting values
            if (!mbar_wait(&tempty_bar[hb], (gh / (kTBufs / kHalf)) & 1, abort, err, 12)) {
              ok = false;
              break;
            }
            fence_after_sync();
#pragma unroll
            for (int i = 0; i < kHalf; ++i) {
              const int c = hh * kHalf + i;  // block within the stage: one K=32 step
              const uint32_t d = tmem + (hb * kHalf + i) * kN;
              const uint64_t da = smem_desc_k_sw128(opa + c * 32);
              const uint64_t db = smem_desc_k_noswizzle(opb + c * L::kSubB, 128, 256);
              mma_i8(d, da, db, idesc);
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
    // expect_tx arrival on `full` and one TMA load of 128 rows x 128 bytes
    // (128-byte swizzle) of the row-ordered activations (gate/up) or h
    // (down), rows [row_base + n0, +128) of the item's slot; a light item (at
    // most kNL tokens): rows [row_base + n0, +kNL) only.
    if (lane == 0) {
      int gs = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        const ItemInfo f = item_info(slots, tiles, item, nm, kGroupRows);
        const int row0 = f.slot.row_base + f.n0;
        const bool light = f.n_valid <= kNL;
        for (int j = 0; j < nst; ++j, ++gs) {
          const int s = gs % kStages;
          if (!mbar_wait(&empty_bar[s], ((gs / kStages) & 1) ^ 1, abort, err, 16)) {
            ok = false;
            break;
          }
          unsigned char* oa = op_ring + s * L::kOpStage;
          if (light) {
            mbar_arrive_expect_tx(&full_bar[s], kNL * 128);
            tma_load_2d(oa, &amap32, j * kBS * 32, row0, &full_bar[s]);
          } else {
            mbar_arrive_expect_tx(&full_bar[s], L::kStageA);
            tma_load_2d(oa, &amap, j * kBS * 32, row0, &full_bar[s]);
          }
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ fold
    // warp w: TMEM lanes 32*(w%4).. (tokens); columns c0.. and c1.. (16 each):
    // gate/up: gate rows [16 c4, 16 c4 + 16) of the group and the same up
    // rows (64 columns on); down: columns [32 c4, 32 c4 + 32).
    // A light item (at most kNL tokens) has the weight rows as the TMEM lanes
    // and the tokens as columns (kNL per block): warp w folds weight rows
    // 32 (w%4).. for tokens [8 c4, 8 c4 + 8).
    const int quad = warp & 3, c4 = (warp - kEpi0) >> 2;
    const int c0 = GU ? 16 * c4 : 32 * c4;
    const int c1 = GU ? kGroupRows + 16 * c4 : 32 * c4 + 16;
    int n_done = 0;  // items this warp has folded (parity of the exchange buffers)
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    constexpr int kHandPerStage = kBS / kHalf;
    // isum from an accumulator read as binary32: int4 (B = 16 q): the value
    // is 0x4B400000 + 16 isum, so fma(v, 1/16, -C/16) = isum exactly (the
    // exact result is an integer below 2^22); int8 (B = q): v - C.
    constexpr float kIsumScale = BITS == 4 ? 0.0625f : 1.0f;
    constexpr float kIsumOffset = -kMagicF * kIsumScale;
    // every buffer is free for its first use
    if ((int)blockIdx.x < n_items) {
      __syncwarp();
      if (lane == 0)
        for (int h = 0; h < kTBufs / kHalf; ++h) mbar_arrive(&tempty_bar[h]);
    }
    // (float)isum of two accumulator values (S + 0x4B400000 read as binary32
    // is 1.5 * 2^23 + S, |S| < 2^22)
    auto isum2 = [&](uint32_t a, uint32_t b, float& v0, float& v1) {
      v0 = __uint_as_float(a + kMagic);
      v1 = __uint_as_float(b + kMagic);
      fma2c(v0, v1, kIsumScale, kIsumOffset);
    };
    int gh = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
      const bool light = item_info(slots, tiles, item, nm, kGroupRows).n_valid <= kNL;  // CTA-uniform
      float acc0[16], acc1[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        acc0[j] = 0.0f;
        acc1[j] = 0.0f;
      }
      if (!light) {
        bool active, valid;
        const int n = quad * 32 + lane;  // this thread's token within the tile
        const float* drow;               // the token's Q8 scales, one per block
        // capture: this token's row and the first output row of each column range
        int32_t* dbg0 = nullptr;
        int32_t* dbg1 = nullptr;
        {  // the item's description is read again for the epilogue: fewer live registers in the block loop
          const ItemInfo f = item_info(slots, tiles, item, nm, kGroupRows);
          active = quad * 32 < f.n_valid;  // warp-uniform
          valid = n < f.n_valid;
          drow = ad + (valid ? item_token_row(f, GU, perm, top_k, n) : 0) * nb;
          if constexpr (DBG) {
            if (valid) {
              int32_t* base = dbg.buf + dbg_row(f, perm, top_k, dbg, n) * dbg_words(hidden, inter);
              const int nbh = hidden / 32, nbi = inter / 32;
              if constexpr (GU) {
                dbg0 = base + (int64_t)(f.m0 + c0) * nbh;                         // gate rows
                dbg1 = base + (int64_t)inter * nbh + (int64_t)(f.m0 + c0) * nbh;  // up rows
              } else {
                dbg0 = base + 2 * (int64_t)inter * nbh + (int64_t)(f.m0 + c0) * nbi;
                dbg1 = base + 2 * (int64_t)inter * nbh + (int64_t)(f.m0 + c1) * nbi;
              }
            }
          }
        }
        // the token's Q8 scales of a hand-off (kHalf blocks), one hand-off ahead
        float dnext[kHalf], dcur[kHalf];
#pragma unroll
        for (int i = 0; i < kHalf; ++i) dnext[i] = valid ? __ldg(drow + i) : 0.0f;
        for (int j = 0; j < nst; ++j) {
#pragma unroll
          for (int hs = 0; hs < kHandPerStage; ++hs, ++gh) {
            const int hn = j * kHandPerStage + hs + 1;  // next hand-off of this item
#pragma unroll
            for (int i = 0; i < kHalf; ++i) {
              dcur[i] = dnext[i];
              if (valid && hn < nst * kHandPerStage) dnext[i] = __ldg(drow + hn * kHalf + i);
            }
            const int hb = gh % (kTBufs / kHalf);
            // warp-uniform: tcgen05.ld is a warp-wide instruction
            const bool ok =
                __all_sync(0xffffffffu, mbar_wait(&tfull_bar[hb], (gh / (kTBufs / kHalf)) & 1, abort, err, 13));
            fence_after_sync();
#pragma unroll
            for (int i = 0; i < kHalf; ++i) {
              const int b = j * kBS + hs * kHalf + i;  // block of this item
              const uint32_t col = tmem + lane_base + (hb * kHalf + i) * kN;
              if (active && ok) {
                const float dx = dcur[i];
                // 8 columns of each range at a time (16 TMEM values live)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                  uint32_t r0[8], r1[8];
                  tmem_ld8(col + c0 + 8 * h, r0);
                  tmem_ld8(col + c1 + 8 * h, r1);
                  tmem_ld_wait();
#pragma unroll
                  for (int jj = 0; jj < 8; jj += 2) {
                    float v0, v1, u0, u1;
                    isum2(r0[jj], r0[jj + 1], v0, v1);
                    isum2(r1[jj], r1[jj + 1], u0, u1);
                    const int colw = 8 * h + jj;
                    if constexpr (DBG) {
                      if (valid) {
                        dbg0[(int64_t)colw * nb + b] = (int32_t)v0;
                        dbg0[(int64_t)(colw + 1) * nb + b] = (int32_t)v1;
                        dbg1[(int64_t)colw * nb + b] = (int32_t)u0;
                        dbg1[(int64_t)(colw + 1) * nb + b] = (int32_t)u1;
                      }
                    }
                    fma2(acc0[colw], acc0[colw + 1], dx, dx, v0, v1);
                    fma2(acc1[colw], acc1[colw + 1], dx, dx, u0, u1);
                  }
                }
              }
            }
            fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty_bar[hb]);  // the hand-off's TMEM buffers may be rewritten now
          }
        }
        if (active) {  // warp-uniform, and the same for both warps of a pair (one quadrant)
          const bool go = !*abort;  // this warp's writes only: both warps meet the barrier regardless
          const ItemInfo f = item_info(slots, tiles, item, nm, kGroupRows);
          const int64_t row = (int64_t)f.slot.row_base + f.n0 + n;
          if constexpr (GU) {
            const int o = f.m0 + c0;  // this thread's 16 intermediate rows (half of a Q8 block of h)
            const float* sgp = tab.gate_s[f.slot.table_idx] + o;
            const float* sup = tab.up_s[f.slot.table_idx] + o;
            float amax = 0.0f;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float gv = __fmul_rn(__ldg(sgp + j), acc0[j]);
              const float u = __fmul_rn(__ldg(sup + j), acc1[j]);
              acc0[j] = __fmul_rn(__fmul_rn(gv, sigmoid_cw(gv)), u);
              amax = fmaxf(amax, fabsf(acc0[j]));
            }
            // the block's absmax: this half's and the partner warp's (c4 ^ 1)
            float* xa = &s_amax[n_done & 1][0][0];
            xa[(warp - kEpi0) * 32 + lane] = valid ? amax : 0.0f;
            named_bar(2 + quad * 2 + (c4 >> 1), 64);
            amax = fmaxf(amax, xa[(warp - kEpi0 + 4 * ((c4 ^ 1) - c4)) * 32 + lane]);
            const float d = __fdiv_rn(amax, 127.0f);
            if (go && valid) {
              // q in the operand order (int4 weights: per 8 elements 0,2,4,6,1,3,5,7;
              // int8: the elements' order)
              uint32_t pk[4];
#pragma unroll
              for (int e8 = 0; e8 < 2; ++e8) {
                uint32_t lo = 0, hi = 0;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  const int qe = q8_of(acc0[8 * e8 + 2 * i], d), qo = q8_of(acc0[8 * e8 + 2 * i + 1], d);
                  lo |= ((uint32_t)qe & 0xFFu) << (8 * i);
                  hi |= ((uint32_t)qo & 0xFFu) << (8 * i);
                }
                if constexpr (BITS == 4) {
                  pk[2 * e8] = lo;
                  pk[2 * e8 + 1] = hi;
                } else {  // back to element order: even / odd bytes interleaved
                  pk[2 * e8] = __byte_perm(lo, hi, 0x5140);
                  pk[2 * e8 + 1] = __byte_perm(lo, hi, 0x7362);
                }
              }
              *reinterpret_cast<uint4*>(hr + row * inter + o) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
              if ((c4 & 1) == 0) hd[row * (inter / 32) + (o >> 5)] = d;
            }
          } else if (go && valid) {
            const float* sdp = tab.down_s[f.slot.table_idx] + f.m0;
            float4* dst0 = reinterpret_cast<float4*>(y + row * hidden + f.m0 + c0);
            float4* dst1 = reinterpret_cast<float4*>(y + row * hidden + f.m0 + c1);
#pragma unroll
            for (int j = 0; j < 16; j += 4) {
              const float4 s0 = __ldg(reinterpret_cast<const float4*>(sdp + c0 + j));
              const float4 s1 = __ldg(reinterpret_cast<const float4*>(sdp + c1 + j));
              dst0[j / 4] = make_float4(__fmul_rn(s0.x, acc0[j]), __fmul_rn(s0.y, acc0[j + 1]),
                                        __fmul_rn(s0.z, acc0[j + 2]), __fmul_rn(s0.w, acc0[j + 3]));
              dst1[j / 4] = make_float4(__fmul_rn(s1.x, acc1[j]), __fmul_rn(s1.y, acc1[j + 1]),
                                        __fmul_rn(s1.z, acc1[j + 2]), __fmul_rn(s1.w, acc1[j + 3]));
            }
          }
        }
      } else {
        // light item: this thread's weight row r (0..127 of the item's 128
        // rows) for the warp's tw tokens t0 + t (the item's tokens split over
        // the four warps of a quadrant, tw = 2, 4, 6 or 8); lane 4 t + c holds
        // the Q8 scale of token t0 + t for block c of the current stage
        const int r = quad * 32 + lane;
        int tw, t0;
        bool active;
        const float* dl;  // lane's token's scales
        int32_t* dbgt[8];
        {
          const ItemInfo f = item_info(slots, tiles, item, nm, kGroupRows);
          tw = 2 * ((f.n_valid + 7) / 8);  // tokens per warp
          t0 = tw * c4;
          active = t0 < f.n_valid;  // warp-uniform (the same for the four warps of this c4)
          const int tl = t0 + (lane >> 2);
          dl = (lane >> 2) < tw && tl < f.n_valid ? ad + item_token_row(f, GU, perm, top_k, tl) * nb : nullptr;
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            dbgt[t] = nullptr;
            if constexpr (DBG) {
              if (t < tw && t0 + t < f.n_valid) {
                int32_t* base = dbg.buf + dbg_row(f, perm, top_k, dbg, t0 + t) * dbg_words(hidden, inter);
                const int nbh = hidden / 32, nbi = inter / 32;
                if constexpr (GU)
                  dbgt[t] = r < kGroupRows ? base + (int64_t)(f.m0 + r) * nbh
                                           : base + (int64_t)inter * nbh + (int64_t)(f.m0 + r - kGroupRows) * nbh;
                else
                  dbgt[t] = base + 2 * (int64_t)inter * nbh + (int64_t)(f.m0 + r) * nbi;
              }
            }
          }
        }
        const int nh = (nst + 1) / 2;  // hand-offs: two stages each
        // the lane's Q8 scales for the next two stages, loaded two stages ahead
        float dxn = dl != nullptr ? __ldg(dl + (lane & 3)) : 0.0f;
        float dxn2 = dl != nullptr && nst > 1 ? __ldg(dl + kBS + (lane & 3)) : 0.0f;
        for (int hh = 0; hh < nh; ++hh, ++gh) {
          const int hb = gh % (kTBufs / kHalf);
          const bool ok =
              __all_sync(0xffffffffu, mbar_wait(&tfull_bar[hb], (gh / (kTBufs / kHalf)) & 1, abort, err, 13));
          fence_after_sync();
          if (active && ok) {
            for (int jj = 0; jj < 2 && 2 * hh + jj < nst; ++jj) {
              const int j = 2 * hh + jj;  // stage of this item
              uint32_t rv[kBS][8];
#pragma unroll
              for (int c = 0; c < kBS; ++c)
                tmem_ld8(tmem + lane_base + hb * kHalf * kN + jj * kBS * kNL + c * kNL + t0, rv[c]);
              const float dxl = dxn;
              dxn = dxn2;
              if (dl != nullptr && j + 2 < nst) dxn2 = __ldg(dl + (j + 2) * kBS + (lane & 3));
              tmem_ld_wait();
#pragma unroll
              for (int c = 0; c < kBS; ++c) {
                const int b = j * kBS + c;
#pragma unroll
                for (int t = 0; t < 8; t += 2) {
                  if (t >= tw) break;  // warp-uniform
                  float v0, v1;
                  isum2(rv[c][t], rv[c][t + 1], v0, v1);
                  const float d0 = __shfl_sync(0xffffffffu, dxl, 4 * t + c);
                  const float d1 = __shfl_sync(0xffffffffu, dxl, 4 * (t + 1) + c);
                  if constexpr (DBG) {
                    if (dbgt[t] != nullptr) dbgt[t][b] = (int32_t)v0;
                    if (dbgt[t + 1] != nullptr) dbgt[t + 1][b] = (int32_t)v1;
                  }
                  fma2(acc0[t], acc0[t + 1], d0, d1, v0, v1);
                }
              }
            }
          }
          fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty_bar[hb]);
        }
        if (active) {
          const bool go = !*abort;
          const ItemInfo f = item_info(slots, tiles, item, nm, kGroupRows);
          if constexpr (GU) {
            // up rows (quadrants 2, 3) hand their products to the gate rows'
            // threads (quadrants 0, 1: same lane and c4) through shared memory
            float* xu = &s_up[n_done & 1][c4][0][0];
            const int o = f.m0 + (r & (kGroupRows - 1));  // intermediate row
            if (r >= kGroupRows) {
              const float su = __ldg(tab.up_s[f.slot.table_idx] + o);
#pragma unroll
              for (int t = 0; t < 8; ++t)
                if (t < tw) xu[((quad - 2) * 32 + lane) * 8 + t] = __fmul_rn(su, acc0[t]);
            }
            named_bar(12 + c4, 128);  // the four warps of this c4
            if (r < kGroupRows) {
              const float sg = __ldg(tab.gate_s[f.slot.table_idx] + o);
#pragma unroll
              for (int t = 0; t < 8; ++t) {
                if (t >= tw) break;  // warp-uniform
                const float gv = __fmul_rn(sg, acc0[t]);
                const float u = xu[(quad * 32 + lane) * 8 + t];
                const float h = __fmul_rn(__fmul_rn(gv, sigmoid_cw(gv)), u);
                // Q8_0 block of h: the warp's 32 lanes are its 32 rows
                const float d = __fdiv_rn(warp_max(fabsf(h)), 127.0f);
                if (go && t0 + t < f.n_valid) {
                  const int64_t row = (int64_t)f.slot.row_base + f.n0 + t0 + t;
                  int pos = lane;  // int4 weights: element e of a group of 8 at e / 2 or 4 + e / 2
                  if constexpr (BITS == 4) pos = (lane & ~7) + ((lane & 1) ? 4 + ((lane & 7) >> 1) : ((lane & 7) >> 1));
                  hr[row * inter + (o & ~31) + pos] = (int8_t)q8_of(h, d);
                  if (lane == 0) hd[row * (inter / 32) + (o >> 5)] = d;
                }
              }
            }
          } else if (go) {
            const int o = f.m0 + r;  // output row
            const float sd = __ldg(tab.down_s[f.slot.table_idx] + o);
#pragma unroll
            for (int t = 0; t < 8; ++t)
              if (t < tw && t0 + t < f.n_valid)
                y[((int64_t)f.slot.row_base + f.n0 + t0 + t) * hidden + o] = __fmul_rn(sd, acc0[t]);
          }
        }
      }
      ++n_done;
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

// A 2D tensor map over `rows` int8 rows of `cols` bytes (row-major), box
// 128 bytes x box_rows rows, 128-byte swizzle: the A operand tiles (kM rows,
// or 32 for the quarters of a light item's tile).
cudaError_t make_rows_map(CUtensorMap* m, const void* base, int64_t rows, int cols, int box_rows) {
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
  const cuuint64_t strides[1] = {(cuuint64_t)cols};
  const cuuint32_t box[2] = {128, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

namespace {

// The two GEMMs of one weight width; DBG: the capture instantiation.
template <int BITS, bool DBG>
cudaError_t prefill_pair(const GateUpTable& gu, const DownTable& dn, const CUtensorMap& map_x,
                         const CUtensorMap& map_x32, const CUtensorMap& map_h, const CUtensorMap& map_h32,
                         const Slot* slots, const Tile* t, const int32_t* n_tiles,
                         const int32_t* perm, int K, const float* xd, int hidden, int inter, int8_t* hri, float* hd,
                         float* y, int32_t* err, int grid, DbgArgs dbg, cudaStream_t st, cudaEvent_t ev_mid) {
  static int mask_gu[64] = {}, mask_dn[64] = {};
  const size_t smem = PSmem::bytes();
  cudaError_t e;
  if ((e = smem_opt_in(prefill_kernel<true, BITS, DBG, GateUpTable>, (int)smem, mask_gu)) != cudaSuccess) return e;
  if ((e = smem_opt_in(prefill_kernel<false, BITS, DBG, DownTable>, (int)smem, mask_dn)) != cudaSuccess) return e;
  prefill_kernel<true, BITS, DBG, GateUpTable><<<grid, kThreadsP, smem, st>>>(
      gu, map_x, map_x32, slots, t, n_tiles, perm, K, xd, hidden, inter, hri, hd, y, err, dbg);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (ev_mid && (e = cudaEventRecordWithFlags(ev_mid, st, cudaEventRecordExternal)) != cudaSuccess) return e;
  prefill_kernel<false, BITS, DBG, DownTable><<<grid, kThreadsP, smem, st>>>(
      dn, map_h, map_h32, slots, t, n_tiles, perm, K, hd, hidden, inter, hri, hd, y, err, dbg);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_experts(const GateUpTable& gu, const DownTable& dn, const Slot* slots,
                                   const int32_t* n_slots, void* tiles, int32_t* n_tiles, const int32_t* perm,
                                   int K, int n_shared, int bits, const int8_t* xq, const float* xd, int n_tok,
                                   int hidden, int inter, void* xr, void* hr, float* hd, float* y, int32_t* err,
                                   cudaStream_t st, cudaEvent_t ev_mid, int32_t* dbg_buf, int n_experts) {
  Tile* t = reinterpret_cast<Tile*>(tiles);
  const int64_t rows = (int64_t)n_tok * (K + n_shared);
  const int64_t n16 = rows * hidden / 16;
  if (bits == 8)
    act_rows_i8_kernel<8><<<(unsigned)((n16 + 255) / 256), 256, 0, st>>>(xq, perm, n_tok, K, rows, hidden,
                                                                         reinterpret_cast<uint4*>(xr));
  else
    act_rows_i8_kernel<4><<<(unsigned)((n16 + 255) / 256), 256, 0, st>>>(xq, perm, n_tok, K, rows, hidden,
                                                                         reinterpret_cast<uint4*>(xr));
  build_tiles_kernel<<<1, 32, 0, st>>>(slots, n_slots, t, n_tiles);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap map_x, map_h, map_x32, map_h32;
  if ((e = make_rows_map(&map_x, xr, rows, hidden, kM)) != cudaSuccess) return e;
  if ((e = make_rows_map(&map_h, hr, rows, inter, kM)) != cudaSuccess) return e;
  if ((e = make_rows_map(&map_x32, xr, rows, hidden, 32)) != cudaSuccess) return e;
  if ((e = make_rows_map(&map_h32, hr, rows, inter, 32)) != cudaSuccess) return e;
  static int sms_cache[64] = {};
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (sms_cache[dev] == 0 &&
      (e = cudaDeviceGetAttribute(&sms_cache[dev], cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  const int grid = sms_cache[dev];
  int8_t* hri = reinterpret_cast<int8_t*>(hr);
  const DbgArgs dbg{dbg_buf, n_experts, n_shared};
  if (bits == 8)
    return dbg_buf ? prefill_pair<8, true>(gu, dn, map_x, map_x32, map_h, map_h32, slots, t, n_tiles, perm, K, xd, hidden, inter, hri,
                                           hd, y, err, grid, dbg, st, ev_mid)
                   : prefill_pair<8, false>(gu, dn, map_x, map_x32, map_h, map_h32, slots, t, n_tiles, perm, K, xd, hidden, inter, hri,
                                            hd, y, err, grid, dbg, st, ev_mid);
  return dbg_buf ? prefill_pair<4, true>(gu, dn, map_x, map_x32, map_h, map_h32, slots, t, n_tiles, perm, K, xd, hidden, inter, hri, hd,
                                         y, err, grid, dbg, st, ev_mid)
                 : prefill_pair<4, false>(gu, dn, map_x, map_x32, map_h, map_h32, slots, t, n_tiles, perm, K, xd, hidden, inter, hri, hd,
                                          y, err, grid, dbg, st, ev_mid);
}

}  // namespace coli
