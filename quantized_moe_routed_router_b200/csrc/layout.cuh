// Repacked weight layout and the work partition shared by host and device code.
//
// Repacked expert matrix ("tile-major for the tensor-core fragment"):
//   A tile is 16 MMA rows.  Gate/up tiles interleave 8 gate rows (tile rows
//   0..7) with the same 8 rows of up (tile rows 8..15), so one thread holds
//   gate and up of the same act row and forms the activation in registers.
//   Down tiles are 16 consecutive rows of the [H][I] matrix.
//   K is cut into chunks of KC elements (64 for MXFP4, 32 for Q8_0 and
//   INT4-affine).  One (tile, chunk) unit of Q8_0 or MXFP4 is 544 bytes: 512
//   bytes of quants, lane l of a warp owning bytes [16 l, 16 l + 16) (its
//   whole A fragment for the chunk), followed by 32 bytes of block scales, 4
//   per lane quad.  An INT4-affine unit is 320 bytes: 256 bytes of 4-bit codes
//   (lane l owns bytes [8 l, 8 l + 8)), then per lane quad g the fp16 scales
//   and offsets {d(g), d(g+8), m(g), m(g+8)} (8 bytes).  Every format's unit
//   holds as many bytes as the user blocks it comes from.
//   Tiles are grouped (GS tiles per group, the last group may be short) and a
//   group is stored chunk-major: [chunk][tile in group][544 B], so any run of
//   chunks of one group is one contiguous range -- one bulk copy.
#pragma once
#include <stdint.h>

#ifndef TSM_HD
#define TSM_HD __host__ __device__ __forceinline__
#endif

namespace tsm {

constexpr int UNIT_BYTES = 544;       // one Q8_0 / MXFP4 (tile, chunk): 512 B quants + 32 B scales
constexpr int QUANT_BYTES = 512;
constexpr int UNIT_BYTES_I4 = 320;    // one INT4-affine (tile, chunk): 256 B codes + 64 B scales and offsets
constexpr int QUANT_BYTES_I4 = 256;
enum { FMT_Q8_0 = 0, FMT_MXFP4 = 1, FMT_INT4_AFFINE = 2 };
constexpr int GS_MAX = 30;            // tiles per group (= consumer warps x tiles per warp)
constexpr int MAX_TOK = 16;           // tokens of one routing block (a router item's columns; an entry's routes)
constexpr int MAX_LT = 64;            // tokens of one layer-kernel launch (up to four routing blocks)
constexpr int MAX_K = 8;
constexpr int MAX_E = 256;
// Entries: every touched expert's routes in blocks of at most 16 (so an expert
// with r routes is ceil(r / 16) entries), then the shared expert in blocks of
// 16 tokens.  M <= 64 tokens x K <= 8 routes give at most E + 32 routed entries.
constexpr int MAX_ENTRIES = MAX_E + MAX_LT * MAX_K / MAX_TOK + MAX_LT / MAX_TOK;

TSM_HD int chunk_k(int fmt) { return fmt == FMT_MXFP4 ? 64 : 32; }  // elements of K per chunk
TSM_HD int unit_bytes(int fmt) { return fmt == FMT_INT4_AFFINE ? UNIT_BYTES_I4 : UNIT_BYTES; }
TSM_HD int round_up(int a, int b) { return (a + b - 1) / b * b; }

struct MatGeom {
  int tiles;       // 16-row MMA tiles per expert
  int chunks;      // K chunks
  int gs;          // tiles per group
  int ngroups;     // groups per expert
  int kdim;        // K (unpadded)
  int fmt;         // FMT_*
  int ub;          // bytes per (tile, chunk) unit
  uint64_t bytes;  // bytes per expert matrix = tiles * chunks * ub
};

// Tiles per group: the group is one tile per consumer-warp slot (GS_MAX), so
// the size in [15, 30] that keeps the most slots busy -- tiles over
// ceil(tiles / g) * GS_MAX -- wins, ties going to the larger size (whole
// 30-tile groups take the unguarded MMA path); the last group may be short.
inline int pick_group_size(int tiles) {
  if (tiles <= GS_MAX) return tiles;
  int best = GS_MAX;
  long long best_slots = 0;  // slots of the best so far (fewer = more busy)
  for (int g = GS_MAX; g >= GS_MAX / 2; --g) {
    const long long slots = (long long)((tiles + g - 1) / g) * GS_MAX;
    if (best_slots == 0 || slots < best_slots) {
      best = g;
      best_slots = slots;
    }
  }
  return best;
}

inline MatGeom make_geom(int rows_tiles, int kdim, int fmt) {
  MatGeom m;
  m.tiles = rows_tiles;
  m.kdim = kdim;
  m.fmt = fmt;
  m.chunks = (kdim + chunk_k(fmt) - 1) / chunk_k(fmt);
  m.gs = pick_group_size(rows_tiles);
  m.ngroups = (rows_tiles + m.gs - 1) / m.gs;
  m.ub = unit_bytes(fmt);
  m.bytes = (uint64_t)rows_tiles * m.chunks * m.ub;
  return m;
}

// The router: one tile per group, i.e. tile-major [tile][chunk][544 B], so
// each 16-expert tile is one contiguous range (one bulk copy).
inline MatGeom make_router_geom(int num_experts, int kdim) {
  MatGeom m = make_geom((num_experts + 15) / 16, kdim, 0);
  m.gs = 1;
  m.ngroups = m.tiles;
  return m;
}

TSM_HD uint64_t group_offset(int gs, int chunks, int grp, int ub) { return (uint64_t)grp * gs * chunks * ub; }
TSM_HD int group_tiles(int tiles, int gs, int grp) {
  int t = tiles - grp * gs;
  return t < gs ? t : gs;
}

// ----------------------------------------------------------------------------- stream-K partition
// The units of one launch -- every touched entry's (group, chunk) pairs, in
// entry-major order (entry, group, chunk) for gate/up and group-major order
// (group, entry, chunk) for down -- are split into NB contiguous ranges:
// block b owns [range_start(b), range_start(b + 1)).
// floor(b * U / NB) in 32-bit arithmetic (U < 2^32, b <= NB <= 512): with
// U = q NB + r, b U / NB = b q + b r / NB and b r < 2^18.  (A 64-bit integer
// division is a long software sequence on the GPU.)
TSM_HD uint64_t range_start(uint64_t U, int NB, int b) {
  const unsigned u = (unsigned)U, nb = (unsigned)NB, q = u / nb, r = u - q * nb;
  return (uint64_t)((unsigned)b * q + (unsigned)b * r / nb);
}

// The block whose range contains unit u (0 <= u < U): the largest b with
// range_start(b) <= u, i.e. floor(((u + 1) * NB - 1) / U).
TSM_HD int owner_of(uint64_t U, int NB, uint64_t u) { return (int)(((u + 1) * (uint64_t)NB - 1) / U); }

// Partial-sum slot of block b for the group starting at unit g0: 0 when the
// group is b's first segment (b's range starts inside it), else 1 (its last).
TSM_HD int partial_slot(uint64_t U, int NB, int b, uint64_t g0) { return range_start(U, NB, b) >= g0 ? 0 : 1; }

// Group-aligned partition, for few groups (G <= NB): CTA i works in group
// floor(i * G / NB) only, and the CTAs of one group split its chunks evenly,
// so no CTA carries two partial groups (a CTA that did would finish its second
// group late and, as its last contributor, also pay for its reduction).
// (32-bit arithmetic: the aligned partition is used only with G <= NB <= 512.)
TSM_HD int aligned_group_of(int i, int G, int NB) { return i * G / NB; }
TSM_HD int aligned_first_cta(int g, int G, int NB) { return (g * NB + G - 1) / G; }
// First unit of CTA i inside its group of `chunks` units.
TSM_HD int aligned_offset(int i, int G, int NB, int chunks) {
  const int g = aligned_group_of(i, G, NB);
  const int f = aligned_first_cta(g, G, NB), n = aligned_first_cta(g + 1, G, NB) - f;
  return chunks * (i - f) / n;
}
// Used when the busiest CTA then does at most 10 % more than the mean
// (G <= NB and NB <= 1.1 * G * floor(NB / G)); otherwise plain contiguous ranges.
TSM_HD bool use_aligned(int G, int NB) { return G >= 1 && G <= NB && 10LL * NB <= 11LL * G * (NB / G); }

}  // namespace tsm
