// coli_expert_stream.cuh -- the streaming layout of a layer's expert weights
// (host and device): where every Q8 block of every expert row sits in the
// private copy that coli_moe_prepare writes and the streaming decode kernel
// reads.
//
// The copy is made of "stages": the exact shared-memory image of one step
// of a warp's work (32 weight rows x 256 bytes, 8 KB), so that one bulk copy
// moves a stage from HBM to shared memory with no gather.  A weight block
// (32 weights) is 16 bytes of packed int4 or 32 bytes of int8; an int8
// block is stored as its even elements (16 bytes: 0, 2, .., 30) then its odd
// elements, so both widths meet the activations as even / odd byte planes.
// The 16-byte chunks of a stage row are XOR-rotated: chunk c of stage row r
// sits in slot c ^ (r & swz) (rows on lanes: lane l reads row l, and the XOR
// spreads the 8 lanes of each shared-memory phase over 8 bank groups).
//  - gate/up unit u of an expert (intermediate outputs 32u .. 32u+31) is
//    two halves h = 0, 1 (outputs 32u + 16h .. +15); a half's stage row
//    r < 16 is gate row 32u + 16h + r, r >= 16 the up row of the same
//    output; block j of stage s is Q8 block sG + j of the row.
//  - down unit v: 32 rows, or 16 rows on lane pairs when every row spans an
//    even number of whole stages (and so do the gate/up rows).  Single rows:
//    stage row r is down row 32v + r, block j of stage s is block sG + j.
//    Lane pairs (unit rows 16v .. 16v+15): stage row p * 16 + r holds piece
//    p = 0, 1 of down row 16v + r, block j of it is block 2sG + pG + j (the
//    two lanes of a row fold its blocks in order, piece 0 first).
//  - G = 16 blocks per stage row for int4, 8 for int8 (fewer when a row is
//    shorter than one stage).
//  - then the F32 row scales: gate [I], up [I], down [H].
// Per expert: gate/up halves (unit-major) | down units | scales, each expert
// padded to 256 bytes; expert j (routed 0..E-1, then shared) at
// j * expert_bytes.
#pragma once

#include <cstddef>
#include <cstdint>

namespace coli {

constexpr int kStreamStageMax = 8 * 1024;  // bytes of the largest stage (and of a ring slot)

struct StreamGeom {
  int H, I;          // hidden, expert inter
  int bits;          // 4 (packed int4) or 8 (int8)
  int bpb;           // bytes per weight block: 16 or 32
  int nbh, nbi;      // Q8 blocks per gate/up row (H/32) and per down row (I/32)
  int g_gu, g_dn;    // blocks per stage row
  int swz_gu, swz_dn;
  int st_gu, st_dn;  // stages per unit
  int cpu_gu, cpu_dn;  // units per expert (I/32 gate/up, H/rpu_dn down)
  int lpr_dn, rpu_dn;  // lanes per down row (1 or 2), down rows per unit (32 / lpr_dn)
  uint32_t sb_gu, sb_dn;  // stage bytes
  uint64_t ub_gu, ub_dn;  // bytes of a gate/up half unit, of a down unit
  uint64_t dn_off, sc_off, expert_bytes;
};

__host__ __device__ inline bool stream_pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }

// A row of nb blocks splits into stages of gmax blocks, or is one stage of
// a power-of-two number of 16-byte chunks.
__host__ __device__ inline bool stream_row_ok(int nb, int gmax, int bpb) {
  return nb % gmax == 0 || (nb < gmax && stream_pow2(nb * bpb / 16));
}

__host__ __device__ inline bool stream_shape_ok(int H, int I, int bits) {
  if (H <= 0 || I <= 0 || H % 128 != 0 || I % 128 != 0 || (bits != 4 && bits != 8)) return false;
  const int bpb = bits == 8 ? 32 : 16;
  return stream_row_ok(H / 32, 256 / bpb, bpb) && stream_row_ok(I / 32, 256 / bpb, bpb);
}

__host__ __device__ inline StreamGeom stream_geom(int H, int I, int bits) {
  StreamGeom g{};
  g.H = H;
  g.I = I;
  g.bits = bits;
  g.bpb = bits == 8 ? 32 : 16;
  g.nbh = H / 32;
  g.nbi = I / 32;
  const int gmax = 256 / g.bpb;  // blocks in a 256-byte stage row
  g.g_gu = g.nbh < gmax ? g.nbh : gmax;
  g.g_dn = g.nbi < gmax ? g.nbi : gmax;
  const int ch_gu = g.g_gu * g.bpb / 16, ch_dn = g.g_dn * g.bpb / 16;  // 16-byte chunks per stage row
  g.swz_gu = (ch_gu < 8 ? ch_gu : 8) - 1;
  g.swz_dn = (ch_dn < 8 ? ch_dn : 8) - 1;
  g.lpr_dn = (g.nbh % gmax == 0 && g.nbi % (2 * gmax) == 0) ? 2 : 1;
  g.rpu_dn = 32 / g.lpr_dn;
  g.st_gu = g.nbh / g.g_gu;
  g.st_dn = g.nbi / (g.lpr_dn * g.g_dn);
  g.cpu_gu = I / 32;
  g.cpu_dn = H / g.rpu_dn;
  g.sb_gu = (uint32_t)(32 * g.g_gu * g.bpb);
  g.sb_dn = (uint32_t)(32 * g.g_dn * g.bpb);
  g.ub_gu = (uint64_t)g.st_gu * g.sb_gu;  // one half of a gate/up unit
  g.ub_dn = (uint64_t)g.st_dn * g.sb_dn;
  g.dn_off = (uint64_t)g.cpu_gu * 2 * g.ub_gu;
  g.sc_off = g.dn_off + (uint64_t)g.cpu_dn * g.ub_dn;
  g.expert_bytes = (g.sc_off + (uint64_t)(2 * I + H) * 4 + 255) & ~uint64_t(255);
  return g;
}

// Byte offset, within an expert's streaming copy, of 16-byte chunk h of Q8
// block b of row r of matrix m (0 gate, 1 up, 2 down).  int4: h = 0 (the
// whole block); int8: h = 0 the even elements, h = 1 the odd ones.
__host__ __device__ inline uint64_t stream_chunk_offset(const StreamGeom& g, int m, int r, int b, int h) {
  const int cpb = g.bpb / 16;  // chunks per block
  if (m < 2) {
    const int u = r / 32, half = (r / 16) & 1, sr = (m == 0 ? 0 : 16) + (r & 15);
    const int s = b / g.g_gu, j = b - s * g.g_gu;
    const int c = j * cpb + h;
    return (uint64_t)(u * 2 + half) * g.ub_gu + (uint64_t)s * g.sb_gu + (uint64_t)sr * g.g_gu * g.bpb +
           (uint64_t)((c ^ (sr & g.swz_gu)) * 16);
  }
  const int v = r / g.rpu_dn, rr = r - v * g.rpu_dn;
  const int span = g.lpr_dn * g.g_dn;  // blocks of a row in one stage
  const int s = b / span, jj = b - s * span;
  const int piece = jj / g.g_dn, j = jj - piece * g.g_dn;
  const int sr = piece * g.rpu_dn + rr;
  const int c = j * cpb + h;
  return g.dn_off + (uint64_t)v * g.ub_dn + (uint64_t)s * g.sb_dn + (uint64_t)sr * g.g_dn * g.bpb +
         (uint64_t)((c ^ (sr & g.swz_dn)) * 16);
}

}  // namespace coli
