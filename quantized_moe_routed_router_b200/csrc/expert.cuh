// The routed MoE half of one layer as ONE persistent kernel per layer
// (one CTA per SM, all resident):
//
//   1. route   -- every CTA computes the routing itself (router GEMV on the
//                 tensor cores, top-k, route list; see route.cuh), so no CTA
//                 waits for another and no separate launch sits in front;
//   2. gate/up -- grouped GEMV of the touched experts (+ shared expert) and
//                 the activation, written as FP16 acts (gpt-oss state page,
//                 `BatchedRoutedScratch`: phase 1 fills `batch_acts` from the
//                 route list);
//   3. down    -- grouped GEMV of the acts; a CTA whose down work needs an
//                 expert's acts waits (bounded) until every gate/up group of
//                 that expert is done, prefetching its weights meanwhile;
//   4. combine -- after a bounded grid-wide barrier each CTA forms 1/NB of
//                 y[t] = sum_k w[t][k] down_k[t] (+ shared, deepseek2 state
//                 page, `shared_out`: the shared output seeds the sum) and
//                 resid += y.
//
// Work split: the (entry, group, chunk) units of each GEMV phase are cut into
// one equal contiguous range per CTA (stream-K), so every SM streams the same
// number of weight bytes whatever the routing.  A group split between CTAs is
// finished from per-CTA partial slots added in CTA order: results do not
// depend on timing.
//
// Per CTA: one producer warp issues 1-D bulk copies (TMA, no multicast) of
// weight stages (contiguous runs of a group's chunks) into a 4-deep ring, and
// of activation windows (512 K-elements of each column's FP16 row) into a
// 2-deep ring, each completing on an mbarrier.  Fifteen consumer warps own two
// tiles each; per chunk they convert their A fragments in registers (MXFP4:
// cvt e2m1x2 -> f16x2; Q8_0: byte permute into 1024+u and subtract), run
// m16n8k16 tensor-core MMAs against the activation columns (tokens or routes,
// padded to 8 or 16) and fold each 32-block's partial sum into FP32
// accumulators with the block scale.  Every wait is bounded.
#pragma once
#include "common.cuh"
#include "layout.cuh"
#include "route.cuh"

namespace tsm {

constexpr int NWC = 15;                    // consumer warps
constexpr int RW = 2;                      // tiles per consumer warp
constexpr int NTHREADS = (NWC + 1) * 32;   // + one producer warp
constexpr int KS = 2;                      // chunks per weight stage (Q8_0, MXFP4)
constexpr int KS_I4 = 3;                   // chunks per weight stage (INT4-affine: 320-byte units)
template <int FMT> constexpr int stage_chunks() { return FMT == FMT_INT4_AFFINE ? KS_I4 : KS; }
template <int FMT> constexpr int unit_b() { return FMT == FMT_INT4_AFFINE ? UNIT_BYTES_I4 : UNIT_BYTES; }
constexpr int NSW = 4;                     // weight stages in the ring
constexpr int NSX = 2;                     // activation windows in the ring
constexpr int KW = 512;                    // K elements per activation window
constexpr int XROW = KW * 2 + 32;          // bytes per window row; 1056 = 32 mod 128 keeps the B loads conflict-free
constexpr int WSTAGE = GS_MAX * KS * UNIT_BYTES;
constexpr int XWIN = 16 * XROW;
constexpr int SLOT_FLOATS = GS_MAX * 16 * 16;
constexpr int MAX_NB = 512;                // CTAs per launch (one per SM)
static_assert(GS_MAX == NWC * RW, "a group is one tile per consumer-warp slot");
static_assert(GS_MAX * KS_I4 * UNIT_BYTES_I4 <= WSTAGE, "an INT4-affine stage fits the weight ring");
static_assert(ROUTE_WARPS <= NWC + 1, "routing uses the first ROUTE_WARPS warps");

struct LayerParams {
  RouteParams rp;           // routing inputs; its output pointers are written by CTA 0 only
  __half* xh;               // [M][Hp] FP16 x (the gate/up B operand), written by the routing CTAs of tile 0
  unsigned* xh_cnt;         // slices of xh written (reset at the end of each launch)
  float* part_pub;          // [S][M][item_ld(E)] router items (block tb, tile j, slice c by CTA (tb T + j) S + c)
  float* max_pub;           // [S][MAX_LT] |x| max of each slice
  unsigned* route_cnt;      // router items published (reset at the end of each launch)
  const uint8_t* wB;        // gate/up: expert e at wB + e * wB_stride
  uint64_t wB_stride;
  const uint8_t* wBs;       // shared gate/up or null
  const uint8_t* wC;        // down
  uint64_t wC_stride;
  const uint8_t* wCs;       // shared down or null
  MatGeom gB, gBs, gC, gCs;
  __half* acts;             // [M*K][Ip]
  __half* acts_sh;          // [M][Sp]
  int Ip, Sp;
  float* P;                 // [M*K + M][H] down outputs of whole segments
  float* partial0;          // [NB][2][SLOT_FLOATS] gate/up partial slots
  float* partial1;          // [NB][2][SLOT_FLOATS] down partial slots
  unsigned* cnt_group;      // [MAX_ENTRIES * ng_max * NWC] gate/up chunk counters per (entry, group, consumer warp)
  int ng_max;
  unsigned* entry_done;     // [MAX_ENTRIES] gate/up (group, consumer warp) shares finished per entry
  unsigned long long* grid_cnt;  // grid barrier arrivals, never reset: NB per launch (64-bit: never wraps)
  int debug_skip_arrival;   // test hook: CTA 0 does not arrive, so the barrier's bounded wait runs out
  // decode launches: the unit-equal range tables (gate/up then down,
  // part_stride(NB) entries each) for every count nT = 1 .. part_nmax of
  // routed entries, table nT - 1 at part_all + (nT - 1) 2 part_stride(NB),
  // computed at open; null for prefill launches
  const unsigned* part_all;
  int part_nmax;
  float* y;                 // [M][H] or null
  __nv_bfloat16* resid;     // [M][H] in/out or null
  unsigned* err;
  int act;
  float alpha, limit;
};

// Range tables of NB + 1 entries, padded to whole 16-byte rows (a table of
// part_stride entries is one bulk copy).
constexpr int RS_LEN = (MAX_NB + 1 + 3) / 4 * 4;
TSM_HD int part_stride(int NB) { return (NB + 1 + 3) / 4 * 4; }

struct __align__(128) LayerSmem {
  uint8_t w[NSW][WSTAGE];
  uint8_t x[NSX][XWIN];
  uint64_t wfull[NSW], wempty[NSW], xfull[NSX], xempty[NSX];
  RouteState r;
  unsigned cp0[MAX_ENTRIES + 1];     // gate/up: cost of the entries before entry j (units x weight)
  unsigned cq1[MAX_ENTRIES + 1];     // down: cost of the entries before entry j within one group
  __align__(16) unsigned rs0[RS_LEN];  // gate/up: first unit of each CTA's range
  __align__(16) unsigned rs1[RS_LEN];  // down: first unit of each CTA's range
  int dead;
  int tab_nT;               // routed entries whose range tables were fetched after the top-k (0: none)
  uint64_t tbar;            // completion of that fetch
  unsigned long long gen0;  // launches completed before this one
};

struct Seg {
  int j;          // entry
  bool sh;        // shared-expert entry
  int grp, c0, c1;
  int chunks, tiles, gs, ntg;
  int nc, ro;
  long long g0;   // unit index of the (entry, group)'s first chunk
};

// First unit of entry j (the nT routed entries, then the shared expert's
// entries from nT on): gate/up units are entry-major, so entry j starts at
// upre0(j); down units are group-major, and inside a group entry j starts at
// cpre1(j).
TSM_DEV long long upre0(const LayerParams& p, int nT, int j) {
  return (long long)min(j, nT) * p.gB.ngroups * p.gB.chunks +
         (j > nT ? (long long)(j - nT) * p.gBs.ngroups * p.gBs.chunks : 0);
}
TSM_DEV int cpre1(const LayerParams& p, int nT, int j) {
  return min(j, nT) * p.gC.chunks + (j > nT ? (j - nT) * p.gCs.chunks : 0);
}

// Relative cost of a unit of an entry with nc columns: with more than 8
// columns the consumers run two n8 MMA tiles per fragment, and the MXFP4 and
// INT4-affine consumers, bound by their conversion issue, then take about
// 1.4x the time per unit.  (Q8_0 stays within its memory time either way, so
// its ranges stay equal in units.)
TSM_DEV unsigned unit_weight(int nc) { return nc > 8 ? 7u : 5u; }

// Warp 0: the cost prefixes of the entries (gate/up: units x weight, entry
// major; down: chunks x weight within a group), so that CTA ranges are equal
// in cost, not in units.  With equal weights the ranges are the same as by
// units (floor(floor(b U w / NB) / w) = floor(b U / NB)).
TSM_DEV void cost_tables(LayerSmem& s, const LayerParams& p, int lane) {
  const int nE = s.r.nE, nT = s.r.nT;
  const int per = (nE + 31) / 32, j0 = lane * per;
  unsigned c0[MAX_ENTRIES / 32 + 1], c1[MAX_ENTRIES / 32 + 1], t0 = 0, t1 = 0;
#pragma unroll
  for (int i = 0; i < MAX_ENTRIES / 32 + 1; ++i) {
    const int j = j0 + i;
    c0[i] = c1[i] = 0u;
    if (i < per && j < nE) {
      const bool sh = j >= nT;
      const unsigned w = unit_weight(s.r.nc[j]);
      c0[i] = (unsigned)(sh ? p.gBs.ngroups * p.gBs.chunks : p.gB.ngroups * p.gB.chunks) * w;
      c1[i] = (unsigned)(sh ? p.gCs.chunks : p.gC.chunks) * w;
    }
    t0 += c0[i];
    t1 += c1[i];
  }
  unsigned i0 = t0, i1 = t1;
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned a = __shfl_up_sync(0xffffffffu, i0, o), b2 = __shfl_up_sync(0xffffffffu, i1, o);
    if (lane >= o) {
      i0 += a;
      i1 += b2;
    }
  }
  unsigned r0 = i0 - t0, r1 = i1 - t1;
#pragma unroll
  for (int i = 0; i < MAX_ENTRIES / 32 + 1; ++i) {
    const int j = j0 + i;
    if (i < per && j <= nE) {
      s.cp0[j] = r0;
      s.cq1[j] = r1;
    }
    r0 += c0[i];
    r1 += c1[i];
  }
  if (lane == 31) {  // totals (the last lane's inclusive sums)
    s.cp0[nE] = i0;
    s.cq1[nE] = i1;
  }
}

// Largest j in [0, n] with tab[j] <= c (tab non-decreasing, tab[0] = 0 <= c).
TSM_DEV int last_le(const unsigned* tab, int n, unsigned c) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tab[mid] <= c)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

// First unit of CTA b's range in phase PH (b = NB: the total): ranges equal
// in units, or with COST equal in cost (cost_tables), or for gate/up with few
// groups the group-aligned partition (aligned_* in layout.cuh).
template <int PH, bool COST>
TSM_DEV unsigned cta_start(const LayerSmem* sp, const LayerParams& p, int nT, int nE, int NB, bool aligned, int G0,
                           int b) {
  if (PH == 1 && !COST) return (unsigned)range_start((uint64_t)p.gC.ngroups * cpre1(p, nT, nE), NB, b);
  if (PH == 0 && !COST && (!aligned || b >= NB)) return (unsigned)range_start((uint64_t)upre0(p, nT, nE), NB, b);
  if (PH == 1) {  // (COST only from here on: the cost tables in *sp)
    const LayerSmem& s = *sp;
    const unsigned upg = (unsigned)cpre1(p, nT, nE), W1 = s.cq1[nE];
    if (b >= NB) return (unsigned)p.gC.ngroups * upg;
    const unsigned c = (unsigned)range_start((uint64_t)p.gC.ngroups * W1, NB, b);
    const unsigned grp = c / W1, r = c - grp * W1;
    const int j = min(last_le(s.cq1, nE, r), nE - 1);
    return grp * upg + (unsigned)cpre1(p, nT, j) + (r - s.cq1[j]) / unit_weight(s.r.nc[j]);
  }
  if (b >= NB) return (unsigned)upre0(p, nT, nE);
  if (!aligned) {
    const LayerSmem& s = *sp;
    const unsigned c = (unsigned)range_start((uint64_t)s.cp0[nE], NB, b);
    const int j = min(last_le(s.cp0, nE, c), nE - 1);
    return (unsigned)upre0(p, nT, j) + (c - s.cp0[j]) / unit_weight(s.r.nc[j]);
  }
  const int g = aligned_group_of(b, G0, NB);
  const bool shg = g >= nT * p.gB.ngroups;
  const int gs_ = g - nT * p.gB.ngroups;
  const int j = shg ? nT + gs_ / p.gBs.ngroups : g / p.gB.ngroups;
  const int grp = shg ? gs_ % p.gBs.ngroups : g % p.gB.ngroups;
  const int ch = shg ? p.gBs.chunks : p.gB.chunks;
  return (unsigned)(upre0(p, nT, j) + (long long)grp * ch + aligned_offset(b, G0, NB, ch));
}

// The unit-equal range tables of decode launches, computed once at open with
// cta_start: block t for nT = t + 1 routed entries (and nsh shared ones) writes
// out[2 t stride + b] = gate/up start of CTA b, out[(2 t + 1) stride + b] =
// down start (b <= NB).
__global__ void partition_table_kernel(const LayerParams p, int nsh, int NB, int stride, unsigned* out) {
  const int nT = blockIdx.x + 1, nE = nT + nsh;
  const int G0 = nT * p.gB.ngroups + nsh * p.gBs.ngroups;
  const bool aligned = use_aligned(G0, NB);
  unsigned* o = out + (size_t)blockIdx.x * 2 * stride;
  for (int i = threadIdx.x; i <= NB; i += blockDim.x) {
    o[i] = cta_start<0, false>(nullptr, p, nT, nE, NB, aligned, G0, i);
    o[stride + i] = cta_start<1, false>(nullptr, p, nT, nE, NB, aligned, G0, i);
  }
}

// Next segment (one entry's group, a run of its chunks) of [u, u1) of phase PH
// (0: entry-major gate/up units, 1: group-major down units).
template <int PH>
TSM_DEV bool next_seg(const LayerSmem& s, const LayerParams& p, long long& u, long long u1, int& j, Seg& sg) {
  if (u >= u1) return false;
  const MatGeom& gr = PH == 0 ? p.gB : p.gC;
  const MatGeom& gsh = PH == 0 ? p.gBs : p.gCs;
  const int nT = s.r.nT;
  // unit indices fit in 32 bits (at most 257 entries x 546 groups x 512 chunks)
  const unsigned uu = (unsigned)u;
  int grp, c0;
  unsigned base;
  if (PH == 1) {
    const unsigned upg = (unsigned)cpre1(p, nT, s.r.nE);
    grp = (int)(uu / upg);
    const int r = (int)(uu - (unsigned)grp * upg);
    j = r < nT * gr.chunks ? r / gr.chunks : nT + (r - nT * gr.chunks) / gsh.chunks;
    c0 = r - cpre1(p, nT, j);
    base = (unsigned)grp * upg + (unsigned)cpre1(p, nT, j);
  } else {
    const unsigned ub = (unsigned)(gr.ngroups * gr.chunks);
    const unsigned ush = (unsigned)(gsh.ngroups * gsh.chunks);
    j = uu < (unsigned)nT * ub ? (int)(uu / ub) : nT + (int)((uu - (unsigned)nT * ub) / ush);
    const bool sh = p.rp.has_shared && j >= nT;
    const unsigned chunks = (unsigned)(sh ? gsh.chunks : gr.chunks);
    const unsigned e0 = (unsigned)upre0(p, nT, j);
    grp = (int)((uu - e0) / chunks);
    c0 = (int)(uu - e0 - (unsigned)grp * chunks);
    base = e0 + (unsigned)grp * chunks;
  }
  sg.j = j;
  sg.sh = p.rp.has_shared && j >= s.r.nT;
  const MatGeom& g = sg.sh ? gsh : gr;
  sg.chunks = g.chunks;
  sg.tiles = g.tiles;
  sg.gs = g.gs;
  sg.grp = grp;
  sg.c0 = c0;
  const long long rem = u1 - u;
  sg.c1 = (int)((long long)c0 + rem < g.chunks ? c0 + rem : g.chunks);
  sg.ntg = group_tiles(g.tiles, g.gs, grp);
  sg.nc = s.r.nc[j];
  sg.ro = s.r.ro[j];
  sg.g0 = base;
  u += sg.c1 - sg.c0;
  return true;
}

// The CTA whose range holds unit u: the largest b with rs[b] <= u.
TSM_DEV int owner_tab(const unsigned* rs, int NB, unsigned u) {
  int lo = 0, hi = NB - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (rs[mid] <= u)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

TSM_DEV float act_fn(int act, float alpha, float limit, float g, float u) {
  if (act == 0) return g / (1.f + expf(-g)) * u;
  const float gc = fminf(g, limit);
  const float uc = fminf(fmaxf(u, -limit), limit);
  return gc / (1.f + expf(-alpha * gc)) * (uc + 1.f);
}

// One chunk of K for this warp's tiles: A from the weight stage, B from the
// activation window (column c of the n8 tile nt is window row nt*8 + c).
// FULL: the group has all GS_MAX tiles, so no tile of the warp is skipped and
// the compiler may interleave the tiles' work freely.
template <int FMT, int NT, bool FULL = false>
TSM_DEV void mma_chunk(float (&acc)[RW][NT][4], const uint8_t* chunk, int ntg, int warp, const uint8_t* xc,
                       int lane) {
  constexpr int STEPS = FMT == FMT_MXFP4 ? 4 : 2;
  constexpr int UB = unit_b<FMT>();
  const int g = lane >> 2, c = lane & 3;
  uint32_t b[STEPS][NT][2];
#pragma unroll
  for (int s = 0; s < STEPS; ++s)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const uint2 v = *reinterpret_cast<const uint2*>(xc + (nt * 8 + g) * XROW + (16 * s + 4 * c) * 2);
      b[s][nt][0] = v.x;
      b[s][nt][1] = v.y;
    }
  // INT4-affine: the block's column sums of B (an MMA with an all-ones A), for
  // the offset term m * sum(x); lane (g, c) gets columns 2c, 2c + 1 in [0], [1]
  float csum[NT][4];
  if constexpr (FMT == FMT_INT4_AFFINE) {
    const uint32_t ones[4] = {0x3C003C00u, 0x3C003C00u, 0x3C003C00u, 0x3C003C00u};
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      mma_f16_zc(csum[nt], ones, b[0][nt][0], b[0][nt][1]);
      mma_f16_acc(csum[nt], ones, b[1][nt][0], b[1][nt][1]);
    }
  }
#pragma unroll
  for (int r = 0; r < RW; ++r) {
    const int jt = warp * RW + r;
    if (!FULL && jt >= ntg) break;
    const uint8_t* t = chunk + jt * UB;
    if constexpr (FMT == FMT_INT4_AFFINE) {
      // One block.  The MMA gives D = sum((1024 + q) x) = 1024 S + Q for row g
      // and sum((1024 + 16 q) x) = 1024 S + 16 Q for row g + 8 (S = sum(x), Q =
      // sum(q x)), so d Q + m S = d D + (m - 1024 d) S for row g and
      // (d / 16) D + (m - 64 d) S for row g + 8.
      const uint2 qw = *reinterpret_cast<const uint2*>(t + lane * 8);
      const uint2 dm = *reinterpret_cast<const uint2*>(t + QUANT_BYTES_I4 + g * 8);
      float2 d = __half22float2(*reinterpret_cast<const __half2*>(&dm.x));
      float2 m = __half22float2(*reinterpret_cast<const __half2*>(&dm.y));
      m.x = fmaf(-1024.f, d.x, m.x);
      m.y = fmaf(-64.f, d.y, m.y);
      d.y *= 0.0625f;
      uint32_t a0[4], a1[4];
      i4x8_to_f16x8_biased(qw.x, a0);
      i4x8_to_f16x8_biased(qw.y, a1);
      float tmp[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        mma_f16_zc(tmp[nt], a0, b[0][nt][0], b[0][nt][1]);
        mma_f16_acc(tmp[nt], a1, b[1][nt][0], b[1][nt][1]);
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        acc[r][nt][0] = fmaf(d.x, tmp[nt][0], fmaf(m.x, csum[nt][0], acc[r][nt][0]));
        acc[r][nt][1] = fmaf(d.x, tmp[nt][1], fmaf(m.x, csum[nt][1], acc[r][nt][1]));
        acc[r][nt][2] = fmaf(d.y, tmp[nt][2], fmaf(m.y, csum[nt][0], acc[r][nt][2]));
        acc[r][nt][3] = fmaf(d.y, tmp[nt][3], fmaf(m.y, csum[nt][1], acc[r][nt][3]));
      }
      continue;
    }
    const uint4 q = *reinterpret_cast<const uint4*>(t + lane * 16);
    const uint32_t sc = *reinterpret_cast<const uint32_t*>(t + QUANT_BYTES + g * 4);
    if constexpr (FMT == FMT_MXFP4) {
      const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int blk = 0; blk < 2; ++blk) {
        float tmp[NT][4];
        uint32_t a[4];
        e2m1x8_to_f16x8(qw[2 * blk], a);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_f16_zc(tmp[nt], a, b[2 * blk][nt][0], b[2 * blk][nt][1]);
        e2m1x8_to_f16x8(qw[2 * blk + 1], a);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_f16_acc(tmp[nt], a, b[2 * blk + 1][nt][0], b[2 * blk + 1][nt][1]);
        const float sg = blk == 0 ? e8m0_byte_to_f32<0>(sc) : e8m0_byte_to_f32<2>(sc);
        const float sg8 = blk == 0 ? e8m0_byte_to_f32<1>(sc) : e8m0_byte_to_f32<3>(sc);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          acc[r][nt][0] = fmaf(sg, tmp[nt][0], acc[r][nt][0]);
          acc[r][nt][1] = fmaf(sg, tmp[nt][1], acc[r][nt][1]);
          acc[r][nt][2] = fmaf(sg8, tmp[nt][2], acc[r][nt][2]);
          acc[r][nt][3] = fmaf(sg8, tmp[nt][3], acc[r][nt][3]);
        }
      }
    } else {
      const float2 d = __half22float2(*reinterpret_cast<const __half2*>(&sc));
      float tmp[NT][4];
      const uint32_t a0[4] = {u8x2_to_f16x2<0x4140>(q.x), u8x2_to_f16x2<0x4342>(q.x), u8x2_to_f16x2<0x4140>(q.y),
                              u8x2_to_f16x2<0x4342>(q.y)};
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_f16_zc(tmp[nt], a0, b[0][nt][0], b[0][nt][1]);
      const uint32_t a1[4] = {u8x2_to_f16x2<0x4140>(q.z), u8x2_to_f16x2<0x4342>(q.z), u8x2_to_f16x2<0x4140>(q.w),
                              u8x2_to_f16x2<0x4342>(q.w)};
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_f16_acc(tmp[nt], a1, b[1][nt][0], b[1][nt][1]);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        acc[r][nt][0] = fmaf(d.x, tmp[nt][0], acc[r][nt][0]);
        acc[r][nt][1] = fmaf(d.x, tmp[nt][1], acc[r][nt][1]);
        acc[r][nt][2] = fmaf(d.y, tmp[nt][2], acc[r][nt][2]);
        acc[r][nt][3] = fmaf(d.y, tmp[nt][3], acc[r][nt][3]);
      }
    }
  }
}

// First / last CTA that worked on the down segment (entry j, row group grp),
// packed as bf | bl << 16.
TSM_DEV unsigned down_owners(const LayerSmem& s, const LayerParams& p, int NB, int grp, int j) {
  const bool sh = p.rp.has_shared && j >= s.r.nT;
  const unsigned C = (unsigned)(sh ? p.gCs.chunks : p.gC.chunks);
  const unsigned g0 = (unsigned)grp * (unsigned)cpre1(p, s.r.nT, s.r.nE) + (unsigned)cpre1(p, s.r.nT, j);
  return (unsigned)owner_tab(s.rs1, NB, g0) | ((unsigned)owner_tab(s.rs1, NB, g0 + C - 1) << 16);
}

// Loads of the down output of entry j, column n, row h (row group `grp`): the
// value written to P when one CTA covered the whole (group, entry) segment,
// else the contributing CTAs' partial slots, to be added in CTA order.
// down_loads issues the first DV_LOADS of them (predicated, all in flight
// together) into t and returns how many it covered; down_rest adds the rest.
constexpr int DV_LOADS = 8;

struct DownSrc {
  const float* base;  // P row, or the partial-slot base of contributor bf
  int bf, bl;         // contributing CTAs (bf == bl: one owner, value in P)
  unsigned g0;        // first unit of the segment
  int off;            // element offset inside a partial slot
};

TSM_DEV DownSrc down_src(const LayerSmem& s, const LayerParams& p, unsigned owners, int grp, int gs, int j, int n,
                         int h, int route) {
  DownSrc d;
  d.bf = owners & 0xFFFF;
  d.bl = owners >> 16;
  d.g0 = (unsigned)grp * (unsigned)cpre1(p, s.r.nT, s.r.nE) + (unsigned)cpre1(p, s.r.nT, j);
  const int rel = h - grp * gs * 16;
  d.off = ((rel >> 4) * 16 + (rel & 15)) * 16 + n;
  d.base = p.P + (size_t)route * p.rp.H + h;
  return d;
}

TSM_DEV const float* slot_ptr(const LayerSmem& s, const LayerParams& p, const DownSrc& d, int bb) {
  return p.partial1 + ((size_t)bb * 2 + (s.rs1[bb] >= d.g0 ? 0 : 1)) * SLOT_FLOATS + d.off;
}

TSM_DEV void down_loads(const LayerSmem& s, const LayerParams& p, const DownSrc& d, bool use, float (&t)[DV_LOADS]) {
#pragma unroll
  for (int q = 0; q < DV_LOADS; ++q) {
    const int bb = d.bf + q;
    t[q] = 0.f;  // past bl or an empty range: adds nothing
    if (!use) continue;
    if (d.bf == d.bl) {
      if (q == 0) t[q] = ld_cg(d.base);
    } else if (bb <= d.bl && s.rs1[bb] != s.rs1[bb + 1]) {
      t[q] = ld_cg(slot_ptr(s, p, d, bb));
    }
  }
}

TSM_DEV float down_sum(const LayerSmem& s, const LayerParams& p, const DownSrc& d, const float (&t)[DV_LOADS]) {
  if (d.bf == d.bl) return t[0];
  float v = 0.f;
#pragma unroll
  for (int q = 0; q < DV_LOADS; ++q) v += t[q];
  for (int bb = d.bf + DV_LOADS; bb <= d.bl; ++bb)  // more contributors than DV_LOADS (small M)
    if (s.rs1[bb] != s.rs1[bb + 1]) v += ld_cg(slot_ptr(s, p, d, bb));
  return v;
}

// This CTA's 1/NB slice [lo, hi) of the M x H outputs.
// (32-bit: M H <= 64 x 16384 = 2^20 and NB <= 512.)
TSM_DEV void combine_range(const LayerParams& p, int NB, int& lo, int& hi) {
  const unsigned MH = (unsigned)p.rp.M * (unsigned)p.rp.H, nb = (unsigned)NB, b = blockIdx.x;
  lo = (int)(MH * b / nb);
  hi = (int)(MH * (b + 1) / nb);
}

// Before the grid barrier (nothing here depends on other CTAs' down work):
// the (row group, entry) -> contributing CTAs table, in the routing scratch
// when it fits (returns whether it does), and the residual of this thread's
// first output of the combine.
TSM_DEV bool combine_prepare(LayerSmem& s, const LayerParams& p, int NB, int ctid, float& r0) {
  const int nE = s.r.nE;
  unsigned* tab = reinterpret_cast<unsigned*>(&s.r.part[0][0][0]);
  constexpr int TAB_CAP = (int)(sizeof(s.r.part) / sizeof(unsigned));
  const bool use_tab = p.gC.ngroups * nE <= TAB_CAP;
  if (use_tab)
    for (int i = ctid; i < p.gC.ngroups * nE; i += NWC * 32) tab[i] = down_owners(s, p, NB, i / nE, i % nE);
  int lo, hi;
  combine_range(p, NB, lo, hi);
  r0 = (p.resid && lo + ctid < hi) ? __bfloat162float(p.resid[lo + ctid]) : 0.f;
  return use_tab;
}

// floor(a / b) for 0 <= a < 2^21 and b >= 1 by a float reciprocal rb = 1 / b:
// the product's relative error is below 2^-23, so its absolute error is below
// 2^-23 (a + 0.5) / b < 0.25 / b, while (a + 0.5) / b lies at least 0.5 / b
// from every integer; the truncation is exact.
TSM_DEV int fdiv(int a, float rb) { return (int)(((float)a + 0.5f) * rb); }

// After the grid barrier: y[t][h] = sum_k w[t][k] * down_k[t][h] (+ shared)
// in slot order over this CTA's slice; resid += y.  Two passes, so that the
// loads of many (output, slot) pairs are in flight together: (1) each pair's
// down value -- the K slots, then the shared expert -- into the idle weight
// ring, CB pairs per thread with all of their loads issued before any is
// used; (2) each output sums its values in slot order.  The barrier orders the
// owner table written by combine_prepare before its reads here.  CB = 2 for
// a decode launch, where a thread has at most a few pairs; 3 for more tokens.
template <int CB>
TSM_DEV void final_combine(LayerSmem& s, const LayerParams& p, int NB, int ctid, bool use_tab, float r0) {
  constexpr int CT = NWC * 32;
  const int K = p.rp.K, H = p.rp.H, gs = p.gC.gs, MK = p.rp.M * K, nE = s.r.nE;
  const unsigned* tab = reinterpret_cast<const unsigned*>(&s.r.part[0][0][0]);
  int lo, hi;
  combine_range(p, NB, lo, hi);
  const int KP = K + (p.rp.has_shared ? 1 : 0);
  const float rKP = 1.f / (float)KP, rH = 1.f / (float)H, rG = 1.f / (float)(gs * 16);
  float* vbuf = reinterpret_cast<float*>(&s.w[0][0]);
  const int cap = (int)((sizeof(s.w) + sizeof(s.x)) / sizeof(float)) / KP;  // outputs per batch
  for (int base = lo; base < hi; base += cap) {
    const int nb = min(cap, hi - base), npair = nb * KP;
    for (int q0 = ctid; q0 < npair; q0 += CT * CB) {
      DownSrc d[CB];
      float t[CB][DV_LOADS];
#pragma unroll
      for (int u = 0; u < CB; ++u) {
        const int q = q0 + u * CT;
        const bool use = q < npair;
        const int o = use ? fdiv(q, rKP) : 0, k = q - o * KP, i = base + o;
        const int tk = fdiv(i, rH), h = i - tk * H, grp = fdiv(h, rG);
        int j, n, route;
        if (k < K) {
          route = s.r.rpos[tk * K + k];
          j = s.r.rj[route];
          n = route - s.r.ro[j];
        } else {  // the shared expert: its entries take 16 tokens each
          j = s.r.nT + tk / MAX_TOK;
          n = tk % MAX_TOK;
          route = MK + tk;
        }
        const unsigned own = use_tab ? tab[grp * nE + j] : down_owners(s, p, NB, grp, j);
        d[u] = down_src(s, p, own, grp, gs, j, n, h, route);
        down_loads(s, p, d[u], use, t[u]);
      }
#pragma unroll
      for (int u = 0; u < CB; ++u) {
        const int q = q0 + u * CT;
        if (q < npair) vbuf[q] = down_sum(s, p, d[u], t[u]);
      }
    }
    bar_sync(1, CT);
    for (int o = ctid; o < nb; o += CT) {
      const int i = base + o, tk = i / H, h = i - tk * H;
      float y = 0.f;
      for (int k = 0; k < K; ++k) y = fmaf(s.r.w[tk * K + k], vbuf[o * KP + k], y);
      if (p.rp.has_shared) y += vbuf[o * KP + K];
      if (p.y) p.y[(size_t)tk * H + h] = y;
      if (p.resid) {
        __nv_bfloat16* r = p.resid + (size_t)tk * H + h;
        *r = __float2bfloat16_rn((i == lo + ctid ? r0 : __bfloat162float(*r)) + y);
      }
    }
    bar_sync(1, CT);  // vbuf is rewritten by the next batch
  }
}

// Grid-wide barrier among the consumer warps of all CTAs (one CTA per SM, all
// resident).  The 64-bit arrival counter is never reset, so launch number
// gen0 = floor(count / NB) read at the start is right even when other CTAs of
// this launch have already arrived (at most NB - 1 of them can have), and the
// launch is complete when the count reaches (gen0 + 1) * NB.  Each CTA arrives
// with a release reduction (nothing to wait for on the way in) and polls with
// acquire loads.  Bounded: a CTA that waits longer than WAIT_LIMIT_NS records
// ERR_TIMEOUT_GRID and goes on.
TSM_DEV void grid_barrier(const LayerSmem& s, const LayerParams& p, int NB, int ctid) {
  bar_sync(1, NWC * 32);  // orders every consumer's stores before thread 0's release
  if (ctid == 0) {
    if (!(p.debug_skip_arrival && blockIdx.x == 0)) red_release_add_u64(p.grid_cnt, 1ull);
    const unsigned long long target = (s.gen0 + 1ull) * (unsigned long long)NB;
    const unsigned long long t0 = globaltimer();
    while (ld_acquire_u64(p.grid_cnt) < target) {
      if (globaltimer() - t0 > WAIT_LIMIT_NS) {
        atomicOr(p.err, ERR_TIMEOUT_GRID);
        break;
      }
    }
  }
  bar_sync(1, NWC * 32);  // thread 0's acquire, then the CTA barrier, orders the other CTAs' writes before our reads
}

// A warp's share of a finished gate/up group (its tiles' acts written):
// count it for the entry.  __syncwarp orders the warp's stores before lane
// 0's release increment (cumulative, so the whole warp's acts are published
// with it); an entry is complete when its count reaches ngroups * NWC.
TSM_DEV void entry_warp_done(const LayerParams& p, const Seg& sg, int lane) {
  __syncwarp();
  if (lane == 0) red_release_add_u32(p.entry_done + sg.j, 1u);
}

// Group epilogue with complete sums in acc.
template <int PH, int NT>
TSM_DEV void group_epilogue(const LayerSmem& s, const LayerParams& p, const Seg& sg, float (&acc)[RW][NT][4],
                            int warp, int lane, int ctid) {
  const int g = lane >> 2, c = lane & 3;
  if constexpr (PH == 0) {
#pragma unroll
    for (int r = 0; r < RW; ++r) {
      const int jt = warp * RW + r;
      if (jt >= sg.ntg) break;
      const int arow = (sg.grp * sg.gs + jt) * 8 + g;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int n = nt * 8 + 2 * c + h;
          if (n < sg.nc) {
            const int tk = sg.sh ? sg.ro - p.rp.M * p.rp.K + n : s.r.tok[sg.ro + n];
            const float scl = __uint_as_float((uint32_t)(127 - s.r.shift[tk]) << 23);
            const float a = act_fn(p.act, p.alpha, p.limit, acc[r][nt][h] * scl, acc[r][nt][2 + h] * scl);
            __half* dst = sg.sh ? p.acts_sh + (size_t)tk * p.Sp : p.acts + (size_t)(sg.ro + n) * p.Ip;
            dst[arow] = __float2half_rn(a);
          }
        }
    }
    entry_warp_done(p, sg, lane);
  } else {
#pragma unroll
    for (int r = 0; r < RW; ++r) {
      const int jt = warp * RW + r;
      if (jt >= sg.ntg) break;
      const int h0 = (sg.grp * sg.gs + jt) * 16 + g;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int n = nt * 8 + 2 * c + hh;
          if (n < sg.nc) {
            const int route = sg.ro + n;  // (shared entries start at M K + their first token)
            float* dst = p.P + (size_t)route * p.rp.H + h0;
            dst[0] = acc[r][nt][hh];
            dst[8] = acc[r][nt][2 + hh];
          }
        }
    }
  }
}

template <int FMT, int PH, int NT>
TSM_DEV void consume_seg(LayerSmem& s, const LayerParams& p, const Seg& sg, int& wi, int& wph, int& xi, int& xph,
                         int warp, int lane, int ctid, int NB) {
  constexpr int KC = FMT == FMT_MXFP4 ? 64 : 32;
  constexpr int KWC = KW / KC;
  constexpr int KS = stage_chunks<FMT>(), UB = unit_b<FMT>();
  float acc[RW][NT][4];
#pragma unroll
  for (int r = 0; r < RW; ++r)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[r][nt][0] = acc[r][nt][1] = acc[r][nt][2] = acc[r][nt][3] = 0.f;

  for (int ws = sg.c0; ws < sg.c1;) {
    const int we = min(sg.c1, (ws / KWC + 1) * KWC);
    mbar_wait(&s.xfull[xi], xph, &s.dead, p.err, ERR_TIMEOUT_XFULL);
    const uint8_t* xw = s.x[xi];
    for (int k = ws; k < we; k += KS) {
      const int kk = min(KS, we - k);
      mbar_wait(&s.wfull[wi], wph, &s.dead, p.err, ERR_TIMEOUT_WFULL);
      const uint8_t* st = s.w[wi];
      if (kk == KS && sg.ntg == GS_MAX) {  // whole stage of a whole group: no guards
#pragma unroll
        for (int q = 0; q < KS; ++q)
          mma_chunk<FMT, NT, true>(acc, st + q * GS_MAX * UB, GS_MAX, warp, xw + (k + q - ws) * KC * 2, lane);
      } else {
#pragma unroll
        for (int q = 0; q < KS; ++q)
          if (q < kk)
            mma_chunk<FMT, NT>(acc, st + q * sg.ntg * UB, sg.ntg, warp, xw + (k + q - ws) * KC * 2, lane);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.wempty[wi]);
      if (++wi == NSW) {
        wi = 0;
        wph ^= 1;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.xempty[xi]);
    if (++xi == NSX) {
      xi = 0;
      xph ^= 1;
    }
    ws = we;
  }

  if (sg.c0 == 0 && sg.c1 == sg.chunks) {
    group_epilogue<PH, NT>(s, p, sg, acc, warp, lane, ctid);
    return;
  }
  // split group: publish this CTA's partial
  const int b = blockIdx.x;
  const int g = lane >> 2, c = lane & 3;
  const unsigned* rs = PH == 0 ? s.rs0 : s.rs1;
  float* slots = PH == 0 ? p.partial0 : p.partial1;
  {
    const int slot = rs[b] >= (unsigned)sg.g0 ? 0 : 1;
    float* sp = slots + ((size_t)b * 2 + slot) * SLOT_FLOATS;
#pragma unroll
    for (int r = 0; r < RW; ++r) {
      const int jt = warp * RW + r;
      if (jt >= sg.ntg) break;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int col = nt * 8 + 2 * c;
        *reinterpret_cast<float2*>(sp + (jt * 16 + g) * 16 + col) = make_float2(acc[r][nt][0], acc[r][nt][1]);
        *reinterpret_cast<float2*>(sp + (jt * 16 + g + 8) * 16 + col) = make_float2(acc[r][nt][2], acc[r][nt][3]);
      }
    }
  }
  if (PH == 1) return;  // down partials are combined after the grid barrier
  // gate/up: per warp (its own tiles), the last contributing CTA finishes the
  // group.  __syncwarp orders the warp's partial stores before lane 0's
  // acquire-release chunk count, which publishes them and, for the last
  // contributor, makes the others' slots visible; the second __syncwarp
  // orders the other lanes' reads after it.  No other warp of the CTA waits.
  const unsigned key = ((unsigned)sg.j * p.ng_max + sg.grp) * NWC + warp;
  __syncwarp();
  unsigned last = 0;
  if (lane == 0) {
    const unsigned inc = (unsigned)(sg.c1 - sg.c0);
    last = atom_acq_rel_add_u32(p.cnt_group + key, inc) + inc == (unsigned)sg.chunks;
  }
  __syncwarp();
  if (!__shfl_sync(0xffffffffu, last, 0)) return;
#pragma unroll
  for (int r = 0; r < RW; ++r)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[r][nt][0] = acc[r][nt][1] = acc[r][nt][2] = acc[r][nt][3] = 0.f;
  const int bf = owner_tab(rs, NB, (unsigned)sg.g0);
  const int bl = owner_tab(rs, NB, (unsigned)(sg.g0 + sg.chunks - 1));
  // the contributors' slots in CTA order, two CTAs' loads in flight at a time
  for (int b2 = bf; b2 <= bl; b2 += 2) {
    float2 v[2][RW][NT][2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int bb = b2 + q;
      const bool use = bb <= bl && rs[bb] != rs[bb + 1];  // past bl or an empty range: adds nothing
      const float* sp = slots + ((size_t)bb * 2 + (use && rs[bb] < (unsigned)sg.g0 ? 1 : 0)) * SLOT_FLOATS;
#pragma unroll
      for (int r = 0; r < RW; ++r) {
        const int jt = warp * RW + r;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int col = nt * 8 + 2 * c;
          const bool ld = use && jt < sg.ntg;
          v[q][r][nt][0] = ld ? ld_cg2(sp + (jt * 16 + g) * 16 + col) : make_float2(0.f, 0.f);
          v[q][r][nt][1] = ld ? ld_cg2(sp + (jt * 16 + g + 8) * 16 + col) : make_float2(0.f, 0.f);
        }
      }
    }
#pragma unroll
    for (int q = 0; q < 2; ++q)
#pragma unroll
      for (int r = 0; r < RW; ++r)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          acc[r][nt][0] += v[q][r][nt][0].x;
          acc[r][nt][1] += v[q][r][nt][0].y;
          acc[r][nt][2] += v[q][r][nt][1].x;
          acc[r][nt][3] += v[q][r][nt][1].y;
        }
  }
  if (lane == 0) p.cnt_group[key] = 0u;
  group_epilogue<PH, NT>(s, p, sg, acc, warp, lane, ctid);
}

// Producer: weight stages and activation windows of phase PH in consumer order.
// Before the first activation window whose data another CTA writes (down:
// every segment's acts; gate/up: the shared FP16 x when xh_wait) it issues
// weight stages (down: up to NSW, as the acts may take long; gate/up: one, as
// x is soon ready), then waits (bounded) for the data to be published.
template <int FMT, int PH>
TSM_DEV bool produce_phase(LayerSmem& s, const LayerParams& p, long long u0, long long u1, int& wi, int& wph, int& xi,
                           int& xph, int& wcount, int& xcount, uint64_t pol, int lane, const __half* xh_src,
                           bool xh_wait) {
  constexpr int KC = FMT == FMT_MXFP4 ? 64 : 32;
  constexpr int KWC = KW / KC;
  constexpr int KS = stage_chunks<FMT>(), UB = unit_b<FMT>();
  long long u = u0;
  int j = 0;
  Seg sg;
  bool alive = true;
  while (alive && next_seg<PH>(s, p, u, u1, j, sg)) {
    const uint8_t* mat = PH == 0 ? (sg.sh ? p.wBs : p.wB + (uint64_t)s.r.ex[sg.j] * p.wB_stride)
                                 : (sg.sh ? p.wCs : p.wC + (uint64_t)s.r.ex[sg.j] * p.wC_stride);
    const uint8_t* gbase = mat + group_offset(sg.gs, sg.chunks, sg.grp, UB);  // (a shared expert only with Q8_0)
    const __half* brow = nullptr;
    if (lane < sg.nc) {
      const int shtok = sg.ro - p.rp.M * p.rp.K + lane;  // shared entries: the token of column `lane`
      if (PH == 0)
        brow = xh_src + (size_t)(sg.sh ? shtok : s.r.tok[sg.ro + lane]) * p.rp.Hp;
      else
        brow = sg.sh ? p.acts_sh + (size_t)shtok * p.Sp : p.acts + (size_t)(sg.ro + lane) * p.Ip;
    }
    const unsigned ustride = (unsigned)sg.ntg * UB;
    int k_issued = sg.c0;  // first chunk whose weight stage is not yet issued
    for (int ws = sg.c0; alive && ws < sg.c1;) {
      const int we = min(sg.c1, (ws / KWC + 1) * KWC);
      if (PH == 1 ? ws == sg.c0 : xh_wait) {
        // prefetch weight stages of the first window, then wait until the
        // expert's acts (down) or the shared x (gate/up) are published
        for (int pre = 0; pre < (PH == 1 ? NSW : 1) && k_issued < we && alive; ++pre) {
          const int kk = min(KS, we - k_issued);
          if (lane == 0) {
            alive = mbar_wait(&s.wempty[wi], wph ^ 1, &s.dead, p.err, ERR_TIMEOUT_WEMPTY);
            if (alive) {
              mbar_arrive_expect_tx(&s.wfull[wi], (unsigned)kk * ustride);
              bulk_g2s_hint(s.w[wi], gbase + (uint64_t)k_issued * ustride, (unsigned)kk * ustride, &s.wfull[wi], pol);
            }
          }
          alive = __shfl_sync(0xffffffffu, alive, 0);
          ++wcount;
          if (++wi == NSW) {
            wi = 0;
            wph ^= 1;
          }
          k_issued += kk;
        }
        if (lane == 0 && alive) {
          // gate/up: every routing block's tile-0 CTAs wrote their slices of xh
          const unsigned need = PH == 1 ? (unsigned)(sg.sh ? p.gBs.ngroups : p.gB.ngroups) * NWC
                                        : (unsigned)(p.rp.S * ((p.rp.M + MAX_TOK - 1) / MAX_TOK));
          const unsigned* flag = PH == 1 ? p.entry_done + sg.j : p.xh_cnt;
          const unsigned long long t0 = globaltimer();
          while (ld_acquire_u32(flag) < need) {
            if (s.dead) break;
            if (globaltimer() - t0 > WAIT_LIMIT_NS) {
              s.dead = 1;
              atomicOr(p.err, PH == 1 ? ERR_TIMEOUT_ACTS : ERR_TIMEOUT_XH);
              break;
            }
          }
        }
        xh_wait = false;
        alive = __shfl_sync(0xffffffffu, alive && !s.dead, 0);
        if (!alive) break;
        // the data were written through the generic proxy by other CTAs and
        // acquired above; the bulk copies below read them through the async proxy
        fence_proxy_async_global();
      }
      const unsigned xbytes = (unsigned)(we - ws) * KC * 2;
      if (lane == 0) {
        alive = mbar_wait(&s.xempty[xi], xph ^ 1, &s.dead, p.err, ERR_TIMEOUT_XEMPTY);
        if (alive) mbar_arrive_expect_tx(&s.xfull[xi], xbytes * (unsigned)sg.nc);
      }
      alive = __shfl_sync(0xffffffffu, alive, 0);
      if (!alive) break;
      if (lane < sg.nc) bulk_g2s(s.x[xi] + lane * XROW, brow + (size_t)ws * KC, xbytes, &s.xfull[xi]);
      ++xcount;
      if (++xi == NSX) {
        xi = 0;
        xph ^= 1;
      }
      for (int k = max(ws, k_issued); k < we; k += KS) {
        const int kk = min(KS, we - k);
        if (lane == 0) {
          alive = mbar_wait(&s.wempty[wi], wph ^ 1, &s.dead, p.err, ERR_TIMEOUT_WEMPTY);
          if (alive) {
            mbar_arrive_expect_tx(&s.wfull[wi], (unsigned)kk * ustride);
            bulk_g2s_hint(s.w[wi], gbase + (uint64_t)k * ustride, (unsigned)kk * ustride, &s.wfull[wi], pol);
          }
        }
        alive = __shfl_sync(0xffffffffu, alive, 0);
        if (!alive) break;
        ++wcount;
        if (++wi == NSW) {
          wi = 0;
          wph ^= 1;
        }
      }
      k_issued = max(k_issued, we);
      ws = we;
    }
  }
  return alive;
}

// BIG: a launch of more than 16 tokens (several routing blocks, experts cut
// into entries of 16 routes); the other instance is the decode launch.
// RONLY: the routing of such a launch alone (ts_moe_route), then a grid
// barrier so that the item counters can be reset; FMT does not matter there.
// NARROW: decode launches of one kind (1: at most 8 tokens; 2: one token,
// whole router; 3: 9 to 16 tokens, router items).  Such an instance holds
// only the code those launches run -- one n8 MMA tile per entry up to 8
// tokens, one routing form for 2 and 3 -- so the once-per-launch phases
// fetch fewer instructions.
template <int FMT, bool BIG, bool RONLY = false, int NARROW = 0>
__global__ void __maxnreg__(120) layer_kernel(const LayerParams p) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  LayerSmem& s = *reinterpret_cast<LayerSmem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int NB = gridDim.x, b = blockIdx.x;

  // ---- 1. route.  The launch's M <= 64 tokens are cut into routing blocks
  // of 16.  CTA b < T S NTB computes router item (block tb, tile j, slice c)
  // with b = (tb T + j) S + c, exactly as route_kernel computes it for that
  // block, and publishes it with the slice's |x| max; every CTA then adds the
  // items in slice order, forms the top-k and the route list itself.  The
  // CTAs of tile 0 also write their block's slice of the FP16 x that the
  // gate/up phase reads.
  RouteParams rp = p.rp;
  if constexpr (NARROW == 2) {
    rp.M = 1;
    rp.whole = 1;
  }
  if constexpr (NARROW == 3) rp.whole = 0;
  rp.logits = nullptr;  // written below by CTA 0 from the summed items
  if (b != 0) {
    rp.idx_out = nullptr;
    rp.w_out = nullptr;
    rp.logits_out = nullptr;
    rp.idx = nullptr;
    rp.w = nullptr;
    rp.shift = nullptr;
    rp.meta = nullptr;
    rp.routes = nullptr;
    rp.rpos = nullptr;
  }
  const int M = rp.M, NTB = BIG ? (M + MAX_TOK - 1) / MAX_TOK : 1;
  // A token selects K distinct experts: a one-token launch routed with the
  // whole router fetches its range tables (nT = K) with the router.
  const bool tab_pro = !BIG && p.part_all && rp.whole && M == 1;
  const int S = rp.S, TS = rp.rg.tiles * S, nR = rp.whole ? 0 : TS * NTB;
  const bool rcta = b < nR;
  const int rtb = rcta ? b / TS : 0, rrem = rcta ? b % TS : 0;
  const int rj = rrem / S, rcs = rrem % S;
  const int t0 = rtb * MAX_TOK;
  RouteParams bp = rp;  // this CTA's routing block: rows t0 .. t0 + mb - 1 of x
  bp.x = rp.x + (size_t)t0 * rp.H;
  bp.M = min(MAX_TOK, M - t0);
  // the routing buffers sit in the still idle weight and window rings
  const SliceSmem L(min(M, MAX_TOK), rp.CS, rp.xscale != nullptr);
  const WholeSmem WS(M, rp.H, rp.rg.tiles, rp.rg.chunks, S, rp.CS, rp.E, rp.xscale != nullptr);
  uint8_t* ring = &s.w[0][0];
  constexpr size_t ring_bytes = sizeof(s.w) + sizeof(s.x);  // w and x are adjacent
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(ring + L.xs);
  __half* xin = reinterpret_cast<__half*>(ring + L.xin);
  uint8_t* rt = ring + L.rt;
  const RouteConst rc = route_const_load(rp, tid);
  if (tid == 0) {
    for (int i = 0; i < NSW; ++i) {
      mbar_init(&s.wfull[i], 1);
      mbar_init(&s.wempty[i], NWC);
    }
    for (int i = 0; i < NSX; ++i) {
      mbar_init(&s.xfull[i], 1);
      mbar_init(&s.xempty[i], NWC);
    }
    mbar_init(&s.r.xbar, 1);
    mbar_init(&s.r.rbar, 1);
    mbar_init(&s.r.pbar, 1);
    mbar_init(&s.tbar, 1);
    fence_barrier_init();
    s.dead = 0;
    s.tab_nT = 0;
    if (rp.whole) {  // the router is a weight: fetched before the dependency wait
      const unsigned rbytes = (unsigned)rp.rg.tiles * rp.rg.chunks * UNIT_BYTES;
      const unsigned tbytes = tab_pro ? (unsigned)part_stride(NB) * 4u : 0u;  // and the one-token range tables
      mbar_arrive_expect_tx(&s.r.rbar, rbytes + 2 * tbytes);
      bulk_g2s(ring + WS.rt, rp.rw, rbytes, &s.r.rbar);
      if (tab_pro) {
        const unsigned* t = p.part_all + (size_t)(rp.K - 1) * 2 * part_stride(NB);
        bulk_g2s(s.rs0, t, tbytes, &s.r.rbar);
        bulk_g2s(s.rs1, t + part_stride(NB), tbytes, &s.r.rbar);
      }
    } else if (rcta) {
      slice_issue_router(bp, s.r, rj, rcs, rt);
    }
  }
  grid_dep_wait();
  grid_dep_launch();
  if (tid == 0) {
    if (rp.whole) {
      const unsigned xbytes = (unsigned)M * rp.H * 2;
      mbar_arrive_expect_tx(&s.r.xbar, xbytes);
      bulk_g2s(ring + WS.x, rp.x, xbytes, &s.r.xbar);
    } else if (rcta) {
      slice_issue_x(bp, s.r, rcs, xs);
    }
    // floor(count / NB), exact in FP64 for counts below 2^53 (no 64-bit integer division)
    s.gen0 = (unsigned long long)floor((double)ld_acquire_u64(p.grid_cnt) / (double)NB);
  }
  route_init_smem(s.r, rc, tid);
  __syncthreads();
  __half* xh_src = p.xh;
  bool xwriter = false;
  if (rp.whole) {
    // few tokens, small router: every CTA routes by itself (and writes the whole xh)
    route_whole(rp, s.r, ring, WS, xh_src, &s.dead, warp, lane, tid, NTHREADS);
    for (int i = tid; i < M * rp.E; i += NTHREADS)
      if (b == 0 && p.rp.logits) p.rp.logits[i] = s.r.lg[i];
    if (tid < M && rp.shift) rp.shift[tid] = s.r.shift[tid];
  } else {
    if (rcta) {
      mbar_wait(&s.r.xbar, 0, &s.dead, p.err, ERR_TIMEOUT_XSTAGE);
      slice_max(bp, s.r, rcs, xs, warp, lane);
      __syncthreads();
      slice_input(bp, s.r, rcs, xs, xin, tid, NTHREADS);
      __syncthreads();
      mbar_wait(&s.r.rbar, 0, &s.dead, p.err, ERR_TIMEOUT_XSTAGE);
      float* pub = p.part_pub + ((size_t)rcs * M + t0) * item_ld(rp.E);
      if (bp.M > 8)
        slice_gemv<2>(bp, s.r, rj, rcs, xin, rt, warp, lane, tid, NTHREADS, pub);
      else
        slice_gemv<1>(bp, s.r, rj, rcs, xin, rt, warp, lane, tid, NTHREADS, pub);
      if (rj == 0 && tid < bp.M) p.max_pub[rcs * MAX_LT + t0 + tid] = s.r.smax[tid];
      __syncthreads();
      if (tid == 0) red_release_add_u32(p.route_cnt, 1u);  // publishes the item written by the whole CTA
    }
    // every item published (bounded); then the S items and slice maxima are
    // brought in by two bulk copies when they fit past the item buffers (with
    // the logits after them)
    const int ild = item_ld(rp.E);
    const unsigned ibytes = (unsigned)((size_t)S * M * ild * 4), mbytes = (unsigned)S * MAX_LT * 4;
    const size_t pst = align128(L.total), lgbytes = (size_t)M * rp.E * 4;
    const bool bulk_items = pst + ibytes + mbytes + lgbytes <= ring_bytes;
    const float* items = bulk_items ? reinterpret_cast<const float*>(ring + pst) : p.part_pub;
    const float* maxes = bulk_items ? reinterpret_cast<const float*>(ring + pst + ibytes) : p.max_pub;
    s.r.lg = reinterpret_cast<float*>(ring + (bulk_items ? pst + ibytes + mbytes : pst));  // fits: checked at open
    s.r.lgld = rp.E;
    if (tid == 0) {
      const unsigned long long tw = globaltimer();
      while (ld_acquire_u32(p.route_cnt) < (unsigned)nR) {
        if (globaltimer() - tw > WAIT_LIMIT_NS) {
          s.dead = 1;
          atomicOr(p.err, ERR_TIMEOUT_ROUTE);
          break;
        }
      }
      if (bulk_items && !s.dead) {  // (no copy left in flight when the wait gave up)
        fence_proxy_async_global();  // written by other CTAs' generic stores, read by bulk copies
        mbar_arrive_expect_tx(&s.r.pbar, ibytes + mbytes);
        bulk_g2s(ring + pst, p.part_pub, ibytes, &s.r.pbar);
        bulk_g2s(ring + pst + ibytes, p.max_pub, mbytes, &s.r.pbar);
      }
    }
    __syncthreads();
    if (bulk_items) mbar_wait(&s.r.pbar, 0, &s.dead, p.err, ERR_TIMEOUT_ROUTE);
    // logits: the items added in slice order; shift from the max of the slice maxima
    for (int i = tid; i < M * rp.E; i += NTHREADS) {
      const int t = i / rp.E, e = i - t * rp.E;
      float v = 0.f;
  #pragma unroll 8
      for (int c = 0; c < S; ++c) {
        const float* src = items + ((size_t)c * M + t) * ild + e;
        v += bulk_items ? *src : ld_cg(src);
      }
      s.r.lg[i] = v;
      if (b == 0 && p.rp.logits) p.rp.logits[i] = v;
    }
    if (tid < M) {
      float m = 0.f;
      for (int c = 0; c < S; ++c) {
        const float* src = maxes + c * MAX_LT + tid;
        m = fmaxf(m, bulk_items ? *src : ld_cg(src));
      }
      s.r.shift[tid] = shift_of_max(m);
      if (rp.shift) rp.shift[tid] = s.r.shift[tid];
    }
    __syncthreads();
    // gate/up B operand: this CTA's slice of its block's x as FP16, published with the count of slices written
    xwriter = rcta && rj == 0;
    if (xwriter) slice_xh(bp, s.r, rcs, xs, xh_src, t0, tid, NTHREADS);
  }
  route_topk<BIG>(rp, s.r, warp, lane, NTHREADS / 32);
  __syncthreads();
  if (xwriter && tid == 0) red_release_add_u32(p.xh_cnt, 1u);  // after the barrier: the CTA's slice of xh
  if (!BIG && p.part_all && !tab_pro && warp == NWC) {
    // other decode launches: the routed-entry count is known from the token
    // masks now, so the producer fetches its tables while the list is built
    const int nw = (rp.E + 31) / 32;
    int cnt = 0;
    for (int w = 0; w < nw; ++w)
      cnt += __popc(__ballot_sync(0xffffffffu, lane + 32 * w < rp.E && s.r.tmask[lane + 32 * w] != 0ull));
    if (lane == 0 && cnt >= 1 && cnt <= p.part_nmax) {
      const unsigned tbytes = (unsigned)part_stride(NB) * 4u;
      const unsigned* t = p.part_all + (size_t)(cnt - 1) * 2 * part_stride(NB);
      s.tab_nT = cnt;  // published by the route list's first barrier
      mbar_arrive_expect_tx(&s.tbar, 2 * tbytes);
      bulk_g2s(s.rs0, t, tbytes, &s.tbar);
      bulk_g2s(s.rs1, t + part_stride(NB), tbytes, &s.tbar);
    }
  }
  route_list<BIG>(rp, s.r, warp, lane, tid, NTHREADS);
  if constexpr (RONLY) {
    // every CTA has read the router items once all are past the barrier
    if (warp == NWC) return;
    grid_barrier(s, p, NB, tid);
    if (b == 0 && tid == 0) {
      *p.route_cnt = 0u;
      *p.xh_cnt = 0u;
    }
    return;
  }
  fence_proxy_async_smem();  // the rings are rewritten by bulk copies from here on
  // Cost-weighted ranges where units differ in cost: a launch of more than
  // 16 tokens cuts experts into entries of up to 16 columns.
  constexpr bool COST = BIG && FMT != FMT_Q8_0;
  if (COST) {
    if (warp == 0) cost_tables(s, p, lane);
    __syncthreads();
  }

  // ---- this CTA's ranges of both phases, in closed form: the producer's four
  // bounds one per lane, so that it starts at once; the consumer warps
  // tabulate every CTA's range starts (for the owners of split groups and the
  // combine) while the first stages load
  const int nE = s.r.nE, nT = s.r.nT;
  // gate/up: with few groups, each CTA stays inside one group (aligned_* in layout.cuh)
  const int G0 = nT * p.gB.ngroups + (nE - nT) * p.gBs.ngroups;
  const bool aligned = use_aligned(G0, NB);
  // decode launches: the tables fetched with the router (one token, unless
  // NaN logits made it select fewer than K experts) or after the top-k hold
  // every range
  const bool tab_post = s.tab_nT != 0 && s.tab_nT == nT;
  const bool tab = (tab_pro && nT == rp.K) || tab_post;

  if (warp == NWC) {
    // ------------------------------------------------------------ producer warp
    unsigned bound = 0;
    if (tab_post) mbar_wait(&s.tbar, 0, &s.dead, p.err, ERR_TIMEOUT_TABLES);
    if (tab)
      bound = lane < 2 ? s.rs0[b + lane] : s.rs1[b + (lane & 1)];
    else if (lane < 2)
      bound = cta_start<0, COST>(&s, p, nT, nE, NB, aligned, G0, b + lane);
    else if (lane < 4)
      bound = cta_start<1, COST>(&s, p, nT, nE, NB, aligned, G0, b + lane - 2);
    const long long a0 = __shfl_sync(0xffffffffu, bound, 0), a1 = __shfl_sync(0xffffffffu, bound, 1);
    const long long d0 = __shfl_sync(0xffffffffu, bound, 2), d1 = __shfl_sync(0xffffffffu, bound, 3);
    const uint64_t pol = policy_evict_first();
    int wi = 0, wph = 0, xi = 0, xph = 0;
    int wcount = 0, xcount = 0;  // copies issued into the weight / window rings (round robin)
    // gate/up reads x written by the routing CTAs: wait for all their slices;
    // routed with the whole router, this CTA wrote all of x itself, before the
    // barriers above (its generic writes, read by the window bulk copies)
    if (rp.whole) fence_proxy_async_global();
    bool alive = produce_phase<FMT, 0>(s, p, a0, a1, wi, wph, xi, xph, wcount, xcount, pol, lane, xh_src, !rp.whole);
    if (alive) produce_phase<FMT, 1>(s, p, d0, d1, wi, wph, xi, xph, wcount, xcount, pol, lane, xh_src, false);
    // Copies still in flight must land before the CTA can exit (only matters
    // when a wait gave up): wait, bounded, for each slot's last issued phase.
    if (lane == 0 && s.dead) {
      const unsigned long long t0 = globaltimer();
      if (s.tab_nT)
        while (!mbar_try_wait(&s.tbar, 0) && globaltimer() - t0 < WAIT_LIMIT_NS) {
        }
      // slot i of a ring of n was used count / n + (i < count % n) times
      for (int i = 0; i < NSW; ++i) {
        const int uses = wcount / NSW + (i < wcount % NSW ? 1 : 0);
        if (uses)
          while (!mbar_try_wait(&s.wfull[i], (uses - 1) & 1) && globaltimer() - t0 < WAIT_LIMIT_NS) {
          }
      }
      for (int i = 0; i < NSX; ++i) {
        const int uses = xcount / NSX + (i < xcount % NSX ? 1 : 0);
        if (uses)
          while (!mbar_try_wait(&s.xfull[i], (uses - 1) & 1) && globaltimer() - t0 < WAIT_LIMIT_NS) {
          }
      }
    }
    return;
  }

  // ------------------------------------------------------------ consumer warps
  if (tab_post) mbar_wait(&s.tbar, 0, &s.dead, p.err, ERR_TIMEOUT_TABLES);
  if (!tab)
    for (int i = tid; i < 2 * (NB + 1); i += NWC * 32) {
      if (i <= NB)
        s.rs0[i] = cta_start<0, COST>(&s, p, nT, nE, NB, aligned, G0, i);
      else
        s.rs1[i - NB - 1] = cta_start<1, COST>(&s, p, nT, nE, NB, aligned, G0, i - NB - 1);
    }
  bar_sync(1, NWC * 32);
  int wi = 0, wph = 0, xi = 0, xph = 0;
  {
    long long u = s.rs0[b];
    const long long a1 = s.rs0[b + 1];
    int j = 0;
    Seg sg;
    while (next_seg<0>(s, p, u, a1, j, sg)) {
      if ((NARROW == 0 || NARROW == 3) && sg.nc > 8)
        consume_seg<FMT, 0, 2>(s, p, sg, wi, wph, xi, xph, warp, lane, tid, NB);
      else
        consume_seg<FMT, 0, 1>(s, p, sg, wi, wph, xi, xph, warp, lane, tid, NB);
    }
  }
  {
    long long u = s.rs1[b];
    const long long d1 = s.rs1[b + 1];
    int j = 0;
    Seg sg;
    while (next_seg<1>(s, p, u, d1, j, sg)) {
      if ((NARROW == 0 || NARROW == 3) && sg.nc > 8)
        consume_seg<FMT, 1, 2>(s, p, sg, wi, wph, xi, xph, warp, lane, tid, NB);
      else
        consume_seg<FMT, 1, 1>(s, p, sg, wi, wph, xi, xph, warp, lane, tid, NB);
    }
  }
  float r0;
  const bool use_tab = combine_prepare(s, p, NB, tid, r0);
  grid_barrier(s, p, NB, tid);
  final_combine<BIG ? 3 : 2>(s, p, NB, tid, use_tab, r0);
  if (b == 0) {  // every readiness wait of this launch is over
    for (int j = tid; j < nE; j += NWC * 32) p.entry_done[j] = 0u;
    if (tid == 0) {
      *p.route_cnt = 0u;
      *p.xh_cnt = 0u;
    }
  }
}

}  // namespace tsm
