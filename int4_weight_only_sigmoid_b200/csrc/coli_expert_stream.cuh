// coli_expert_stream.cuh -- the streaming layout of a layer's expert weights
// (host and device): where every packed 16-byte Q8 block of every expert
// row sits in the private copy that coli_moe_prepare writes and the
// streaming decode kernel reads.
//
// The copy is made of "stages": the exact shared-memory image of one step
// of a warp's work, so that one bulk copy moves a stage from HBM to shared
// memory with no gather.
//  - gate/up unit u of an expert (intermediate outputs 32u .. 32u+31):
//    stages s = 0 .. nbh/G - 1 of 64 stage rows x G blocks; stage row
//    r < 32 is gate row 32u + r, r >= 32 is up row 32u + r - 32; block j of
//    stage s is Q8 block sG + j of the row, stored in 16-byte slot
//    j ^ (r & swz) of the stage row (rows on lanes: lane l reads row l, and
//    the XOR spreads the 8 lanes of each shared-memory phase over 8 bank
//    groups).  G = min(16, nbh).
//  - down unit v (output rows 32v .. 32v+31): stages of 32 rows x G blocks,
//    G = min(32, nbi), the same slot rule.
//  - then the F32 row scales: gate [I], up [I], down [H].
// Per expert: gate/up units | down units | scales, each expert padded to
// 256 bytes; expert j (routed 0..E-1, then shared) at j * expert_bytes.
#pragma once

#include <cstddef>
#include <cstdint>

namespace coli {

constexpr int kStreamStageMax = 16 * 1024;  // bytes of the largest stage (and of a ring slot)

struct StreamGeom {
  int H, I;          // hidden, expert inter
  int nbh, nbi;      // Q8 blocks per gate/up row (H/32) and per down row (I/32)
  int g_gu, g_dn;    // blocks per stage row
  int swz_gu, swz_dn;
  int st_gu, st_dn;  // stages per unit
  int cpu_gu, cpu_dn;  // units per expert (I/32 gate/up, H/32 down)
  uint32_t sb_gu, sb_dn;  // stage bytes
  uint64_t ub_gu, ub_dn;  // unit bytes
  uint64_t dn_off, sc_off, expert_bytes;
};

__host__ __device__ inline bool stream_shape_ok(int H, int I) {
  if (H <= 0 || I <= 0 || H % 128 != 0 || I % 128 != 0) return false;
  const int nbh = H / 32, nbi = I / 32;
  const bool gu = nbh % 16 == 0 || nbh == 4 || nbh == 8;
  const bool dn = nbi % 32 == 0 || nbi == 4 || nbi == 8 || nbi == 16;
  return gu && dn;
}

__host__ __device__ inline StreamGeom stream_geom(int H, int I) {
  StreamGeom g{};
  g.H = H;
  g.I = I;
  g.nbh = H / 32;
  g.nbi = I / 32;
  g.g_gu = g.nbh < 16 ? g.nbh : 16;
  g.g_dn = g.nbi < 32 ? g.nbi : 32;
  g.swz_gu = (g.g_gu < 8 ? g.g_gu : 8) - 1;
  g.swz_dn = (g.g_dn < 8 ? g.g_dn : 8) - 1;
  g.st_gu = g.nbh / g.g_gu;
  g.st_dn = g.nbi / g.g_dn;
  g.cpu_gu = I / 32;
  g.cpu_dn = H / 32;
  g.sb_gu = (uint32_t)(64 * g.g_gu * 16);
  g.sb_dn = (uint32_t)(32 * g.g_dn * 16);
  g.ub_gu = (uint64_t)g.st_gu * g.sb_gu;
  g.ub_dn = (uint64_t)g.st_dn * g.sb_dn;
  g.dn_off = (uint64_t)g.cpu_gu * g.ub_gu;
  g.sc_off = g.dn_off + (uint64_t)g.cpu_dn * g.ub_dn;
  g.expert_bytes = (g.sc_off + (uint64_t)(2 * I + H) * 4 + 255) & ~uint64_t(255);
  return g;
}

// Byte offset, within an expert's streaming copy, of Q8 block b of row r of
// matrix m (0 gate, 1 up, 2 down).
__host__ __device__ inline uint64_t stream_block_offset(const StreamGeom& g, int m, int r, int b) {
  if (m < 2) {
    const int u = r / 32, sr = (m == 0 ? 0 : 32) + (r & 31);
    const int s = b / g.g_gu, j = b - s * g.g_gu;
    return (uint64_t)u * g.ub_gu + (uint64_t)s * g.sb_gu + (uint64_t)sr * g.g_gu * 16 +
           (uint64_t)((j ^ (sr & g.swz_gu)) * 16);
  }
  const int v = r / 32, sr = r & 31;
  const int s = b / g.g_dn, j = b - s * g.g_dn;
  return g.dn_off + (uint64_t)v * g.ub_dn + (uint64_t)s * g.sb_dn + (uint64_t)sr * g.g_dn * 16 +
         (uint64_t)((j ^ (sr & g.swz_dn)) * 16);
}

}  // namespace coli
