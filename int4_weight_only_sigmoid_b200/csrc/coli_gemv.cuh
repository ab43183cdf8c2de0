// coli_gemv.cuh -- device pieces shared by the expert GEMV kernels
// (coli_gemv.cu: general token counts; coli_decode.cu: decode batches).
// See coli_gemv.cu for the work layout and the sources.
#pragma once

#include "coli_launch.h"

namespace coli {
namespace gemv {

constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;
constexpr int kRows = 16;  // rows per warp
constexpr int kSPad = 33;  // padded row of the isum park: conflict-free fold reads

template <int TT>
struct GemvSmem {
  static size_t bytes(int dim_in) {
    const int nb = dim_in / 32;
    return (size_t)2 * TT * nb * 16        // even / odd activation planes
           + (size_t)TT * nb * 4           // block scales
           + (size_t)kWarps * TT * kRows * kSPad * 4  // isum park
           + (size_t)TT * 32 * 4;          // h tile (gate/up)
  }
};

__device__ __forceinline__ Slot load_slot(const GemvSlots& sl, int y, bool& live) {
  if (sl.slots == nullptr) {
    live = (y == 0);
    return sl.one;
  }
  live = y < *sl.n_slots;
  return live ? sl.slots[y] : Slot{0, 0, 0, -1};
}

__device__ __forceinline__ int token_of(const GemvSlots& sl, const Slot& s, int i) {
  return s.perm_base < 0 ? i : sl.perm[s.perm_base + i] / sl.top_k;
}

// Stage n_valid activation rows (Q8 bytes + block scales) into shared memory
// as even/odd byte planes.  act_row(i) gives the source row of token i.
template <int TT, typename RowFn>
__device__ __forceinline__ void stage_acts(const int8_t* aq, const float* ad, int dim_in,
                                           int n_valid, RowFn act_row, uint4* xe_s, uint4* xo_s, float* xd_s) {
  const int nb = dim_in / 32;
  for (int i = threadIdx.x; i < n_valid * nb; i += kThreads) {
    const int t = i / nb, b = i - t * nb;
    const int64_t row = act_row(t);
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

// The warp's 16 rows against n_valid staged tokens; facc[m] ends with the
// fold of chain (row = lane % 16, token = lane / 16 + 2m).
template <int TT, typename RowPtrFn>
__device__ __forceinline__ void warp_rows_fold(RowPtrFn row_ptr, int nb, int n_valid, const uint4* xe_s,
                                               const uint4* xo_s, const float* xd_s, int32_t* Sw,
                                               float (&facc)[(TT + 1) / 2]) {
  const int lane = threadIdx.x & 31;
  const int cr = lane & 15, ct = lane >> 4;
#pragma unroll
  for (int m = 0; m < (TT + 1) / 2; ++m) facc[m] = 0.0f;
  const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
  for (int s0 = 0; s0 < nb; s0 += 32) {
    const int b = s0 + lane;
    const bool valid = b < nb;
    uint4 wv[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) wv[r] = valid ? ldg_stream(row_ptr(r) + 16 * b) : zero;
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
    const int nsteps = min(32, nb - s0);
#pragma unroll
    for (int m = 0; m < (TT + 1) / 2; ++m) {
      const int t = ct + 2 * m;
      if (t < n_valid && t < TT) {
        const int32_t* srow = Sw + (t * kRows + cr) * kSPad;
        const float* dsrc = xd_s + t * nb + s0;
        float a = facc[m];
        for (int j = 0; j < nsteps; ++j) a = __fmaf_rn(dsrc[j], (float)srow[j], a);
        facc[m] = a;
      }
    }
    __syncwarp();
  }
}


}  // namespace gemv
}  // namespace coli
