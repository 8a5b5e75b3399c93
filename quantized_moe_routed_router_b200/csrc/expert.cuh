// Grouped expert kernels: phase 1 = gate/up GEMV + activation, phase 2 =
// down GEMV + weighted combine + shared expert + residual add.
//
// Both phases are the same persistent, stream-K kernel over the route list
// the route kernel built (gpt-oss state page, `BatchedRoutedScratch`: phase 1
// writes `batch_acts [M*top_k, moe_inter]` from the route list, the fused
// phase 2 writes the per-token sum that the residual add reads; deepseek2
// state page: phase 2 is seeded with the shared expert, "y = shared +
// sum(w * expert)").
//
// Work: every touched expert (plus the shared expert as one more entry with
// all M tokens) contributes (group, chunk) units -- a group is up to 30
// tiles of 16 MMA rows, a chunk 64 (MXFP4) or 32 (Q8_0) elements of K.  The
// units of the launch are cut into one equal contiguous range per CTA (one
// CTA per SM), so every SM streams the same number of weight bytes whatever
// the routing.  A group split between CTAs is finished by the last CTA to
// add its chunk count to the group's counter: partial sums go to per-CTA
// slots and are added back in CTA order, so results do not depend on timing.
//
// Per CTA: one producer warp issues 1-D bulk copies (TMA, no multicast) of
// weight stages (contiguous runs of a group's chunks) into a 4-deep ring,
// and of activation windows (512 K-elements of each column's FP16 row) into a
// 2-deep ring, each completing on an mbarrier.  Fifteen consumer warps own two
// tiles each; per chunk they convert their A fragments in registers (MXFP4:
// cvt e2m1x2 -> f16x2; Q8_0: byte permute into 1024+u and subtract), run
// m16n8k16 tensor-core MMAs against the activation columns (tokens or
// routes, padded to 8 or 16) and fold each 32-block's partial sum into FP32
// accumulators with the block scale.  Every wait is bounded.
#pragma once
#include "common.cuh"
#include "layout.cuh"
#include "route.cuh"

namespace tsm {

constexpr int NWC = 15;                    // consumer warps
constexpr int RW = 2;                      // tiles per consumer warp
constexpr int NTHREADS = (NWC + 1) * 32;   // + one producer warp
constexpr int KS = 2;                      // chunks per weight stage
constexpr int NSW = 4;                     // weight stages in the ring
constexpr int NSX = 2;                     // activation windows in the ring
constexpr int KW = 512;                    // K elements per activation window
constexpr int XROW = KW * 2 + 32;          // bytes per window row; 1056 = 32 mod 128 keeps the B loads conflict-free
constexpr int WSTAGE = GS_MAX * KS * UNIT_BYTES;
constexpr int XWIN = 16 * XROW;
constexpr int SLOT_FLOATS = GS_MAX * 16 * 16;
constexpr int MAX_NB = 1024;               // CTAs per launch (one per SM)
static_assert(GS_MAX == NWC * RW, "a group is one tile per consumer-warp slot");

struct PhaseParams {
  const uint8_t* w_routed;  // expert e's matrix at w_routed + e * w_stride
  uint64_t w_stride;
  const uint8_t* w_shared;  // shared expert matrix or null
  MatGeom gr, gsh;          // routed / shared geometry
  const __half* b_routed;   // B rows: phase 1 x (FP16, scaled) [M][ld]; phase 2 acts [M*K][ld]
  int b_routed_ld;
  const __half* b_shared;   // phase 1: x; phase 2: shared acts [M][ld]
  int b_shared_ld;
  const int* meta;
  const Route* routes;
  const int* shift;         // [M] x scale exponents (phase 1)
  __half* acts;             // phase 1 out: [M*K][acts_ld]
  int acts_ld;
  __half* acts_sh;          // phase 1 out: shared [M][acts_sh_ld]
  int acts_sh_ld;
  float* P;                 // phase 2: per-route down outputs [M*K + M][H]
  const float* wts;         // [M][K] routing weights
  const int* rpos;          // [M][K] route positions
  float* y;                 // [M][H] or null
  __nv_bfloat16* resid;     // [M][H] in/out or null
  float* partial;           // [NB][2][SLOT_FLOATS]
  unsigned* cnt_group;      // [(E+1) * ng_max]
  int ng_max;
  unsigned* grid_cnt;       // phase 2: grid barrier arrivals
  unsigned* grid_gen;       // phase 2: grid barrier generation
  unsigned* err;
  int H, K, E;
  int act;
  float alpha, limit;
};

struct __align__(128) PhaseSmem {
  uint8_t w[NSW][WSTAGE];
  uint8_t x[NSX][XWIN];
  uint64_t wfull[NSW], wempty[NSW], xfull[NSX], xempty[NSX];
  long long upre[MAX_ENTRIES + 1];  // entry-major: first unit of each entry
  int cpre[MAX_ENTRIES + 1];        // group-major: first unit of each entry inside a group
  int ex[MAX_ENTRIES], ro[MAX_ENTRIES], nc[MAX_ENTRIES];
  int tok[MAX_TOK * MAX_K];
  int rj[MAX_TOK * MAX_K];          // entry index of each route position
  unsigned rs[MAX_NB + 1];          // first unit of each CTA's range
  unsigned gen0;                    // grid barrier generation seen at kernel start
  int nE, nT, M, MK, has_shared;
  int dead;
  int flag;
};

struct Seg {
  int j;          // entry
  bool sh;        // shared-expert entry
  int grp, c0, c1;
  int chunks, tiles, gs, ntg;
  int nc, ro;
  long long g0;   // unit index of the group's first chunk
};

// Next segment (one entry's group, a run of its chunks) of [u, u1).
// GM = group-major order (the down phase: every entry has the same groups).
template <bool GM>
TSM_DEV bool next_seg(const PhaseSmem& s, const PhaseParams& p, long long& u, long long u1, int& j, Seg& sg) {
  if (u >= u1) return false;
  int grp, c0;
  long long base;
  if (GM) {
    const int upg = s.cpre[s.nE];
    grp = (int)(u / upg);
    const int r = (int)(u - (long long)grp * upg);
    j = 0;
    while (r >= s.cpre[j + 1]) ++j;
    c0 = r - s.cpre[j];
    base = (long long)grp * upg + s.cpre[j];
  } else {
    while (u >= s.upre[j + 1]) ++j;
    const bool sh = s.has_shared && j == s.nT;
    const int chunks = sh ? p.gsh.chunks : p.gr.chunks;
    const long long local = u - s.upre[j];
    grp = (int)(local / chunks);
    c0 = (int)(local - (long long)grp * chunks);
    base = s.upre[j] + (long long)grp * chunks;
  }
  sg.j = j;
  sg.sh = s.has_shared && j == s.nT;
  const MatGeom& g = sg.sh ? p.gsh : p.gr;
  sg.chunks = g.chunks;
  sg.tiles = g.tiles;
  sg.gs = g.gs;
  sg.grp = grp;
  sg.c0 = c0;
  const long long rem = u1 - u;
  sg.c1 = (int)((long long)c0 + rem < g.chunks ? c0 + rem : g.chunks);
  sg.ntg = group_tiles(g.tiles, g.gs, grp);
  sg.nc = s.nc[j];
  sg.ro = s.ro[j];
  sg.g0 = base;
  u += sg.c1 - sg.c0;
  return true;
}

// The CTA whose range holds unit u: the largest b with rs[b] <= u.
TSM_DEV int owner_tab(const PhaseSmem& s, int NB, unsigned u) {
  int lo = 0, hi = NB - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s.rs[mid] <= u)
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
template <int FMT, int NT>
TSM_DEV void mma_chunk(float (&acc)[RW][NT][4], const uint8_t* chunk, int ntg, int warp, const uint8_t* xc,
                       int lane) {
  constexpr int STEPS = FMT == 1 ? 4 : 2;
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
#pragma unroll
  for (int r = 0; r < RW; ++r) {
    const int jt = warp * RW + r;
    if (jt >= ntg) break;
    const uint8_t* t = chunk + jt * UNIT_BYTES;
    const uint4 q = *reinterpret_cast<const uint4*>(t + lane * 16);
    const uint32_t sc = *reinterpret_cast<const uint32_t*>(t + QUANT_BYTES + g * 4);
    if constexpr (FMT == 1) {
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

// Value of the down output of entry j, column n, row h (row group `grp`):
// written to P when one CTA covered the whole (group, entry) segment, else
// the sum of the contributing CTAs' partial slots in CTA order.
TSM_DEV float down_value(const PhaseSmem& s, const PhaseParams& p, int NB, int grp, int gs, int j, int n, int h,
                         int route) {
  const bool sh = s.has_shared && j == s.nT;
  const unsigned C = (unsigned)(sh ? p.gsh.chunks : p.gr.chunks);
  const unsigned g0 = (unsigned)grp * (unsigned)s.cpre[s.nE] + (unsigned)s.cpre[j];
  const int bf = owner_tab(s, NB, g0), bl = owner_tab(s, NB, g0 + C - 1);
  if (bf == bl) return ld_cg(p.P + (size_t)route * p.H + h);
  const int rel = h - grp * gs * 16;
  const int off = ((rel >> 4) * 16 + (rel & 15)) * 16 + n;
  float v = 0.f;
  for (int b2 = bf; b2 <= bl; ++b2) {
    if (s.rs[b2] == s.rs[b2 + 1]) continue;  // empty range
    const int slot = s.rs[b2] >= g0 ? 0 : 1;
    v += ld_cg(p.partial + ((size_t)b2 * 2 + slot) * SLOT_FLOATS + off);
  }
  return v;
}

// Phase 2 finish, after the grid barrier: this CTA's 1/NB slice of the M x H
// outputs, y[t][h] = sum_k w[t][k] * down_k[t][h] (+ shared) in slot order;
// resid += y (BF16).
TSM_DEV void final_combine(const PhaseSmem& s, const PhaseParams& p, int NB, int ctid) {
  const int M = s.M, K = p.K, H = p.H, gs = p.gr.gs;
  const long long MH = (long long)M * H;
  const int lo = (int)(MH * blockIdx.x / NB), hi = (int)(MH * (blockIdx.x + 1) / NB);
  for (int i = lo + ctid; i < hi; i += NWC * 32) {
    const int t = i / H, h = i - t * H, grp = h / (gs * 16);
    float y = 0.f;
    for (int k = 0; k < K; ++k) {
      const int pos = p.rpos[t * K + k];
      const int j = s.rj[pos];
      y = fmaf(p.wts[t * K + k], down_value(s, p, NB, grp, gs, j, pos - s.ro[j], h, pos), y);
    }
    if (s.has_shared) y += down_value(s, p, NB, grp, gs, s.nT, t, h, s.MK + t);
    if (p.y) p.y[(size_t)t * H + h] = y;
    if (p.resid) {
      __nv_bfloat16* r = p.resid + (size_t)t * H + h;
      *r = __float2bfloat16_rn(__bfloat162float(*r) + y);
    }
  }
}

// Grid-wide barrier among the consumer warps of all CTAs (one CTA per SM, all
// resident).  Bounded: a CTA that waits longer than WAIT_LIMIT_NS records
// ERR_TIMEOUT_GRID and goes on.
TSM_DEV void grid_barrier(const PhaseSmem& s, const PhaseParams& p, int NB, int ctid) {
  __threadfence();
  bar_sync(1, NWC * 32);
  if (ctid == 0) {
    if (atomicAdd(p.grid_cnt, 1u) == (unsigned)NB - 1) {
      *p.grid_cnt = 0u;
      __threadfence();
      atomicAdd(p.grid_gen, 1u);
    } else {
      const unsigned long long t0 = globaltimer();
      while (ld_acquire_u32(p.grid_gen) == s.gen0) {
        if (globaltimer() - t0 > WAIT_LIMIT_NS) {
          atomicOr(p.err, ERR_TIMEOUT_GRID);
          break;
        }
      }
    }
  }
  bar_sync(1, NWC * 32);
  __threadfence();
}

// Group epilogue with complete sums in acc.
template <int PHASE, int NT>
TSM_DEV void group_epilogue(PhaseSmem& s, const PhaseParams& p, const Seg& sg, float (&acc)[RW][NT][4], int warp,
                            int lane, int ctid) {
  const int g = lane >> 2, c = lane & 3;
  if constexpr (PHASE == 0) {
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
            const int tk = sg.sh ? n : s.tok[sg.ro + n];
            const float scl = __uint_as_float((uint32_t)(127 - p.shift[tk]) << 23);
            const float a = act_fn(p.act, p.alpha, p.limit, acc[r][nt][h] * scl, acc[r][nt][2 + h] * scl);
            __half* dst = sg.sh ? p.acts_sh + (size_t)n * p.acts_sh_ld : p.acts + (size_t)(sg.ro + n) * p.acts_ld;
            dst[arow] = __float2half_rn(a);
          }
        }
    }
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
            const int route = sg.sh ? s.MK + n : sg.ro + n;
            float* dst = p.P + (size_t)route * p.H + h0;
            dst[0] = acc[r][nt][hh];
            dst[8] = acc[r][nt][2 + hh];
          }
        }
    }
  }
}

template <int FMT, int PHASE, int NT>
TSM_DEV void consume_seg(PhaseSmem& s, const PhaseParams& p, const Seg& sg, int& wi, int& wph, int& xi, int& xph,
                         int warp, int lane, int ctid, long long U, int NB) {
  constexpr int KC = FMT == 1 ? 64 : 32;
  constexpr int KWC = KW / KC;
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
#pragma unroll
      for (int q = 0; q < KS; ++q)
        if (q < kk)
          mma_chunk<FMT, NT>(acc, st + q * sg.ntg * UNIT_BYTES, sg.ntg, warp, xw + (k + q - ws) * KC * 2, lane);
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

  const bool whole = sg.c0 == 0 && sg.c1 == sg.chunks;
  if (whole) {
    group_epilogue<PHASE, NT>(s, p, sg, acc, warp, lane, ctid);
    return;
  }
  // split group: publish this CTA's partial
  const int b = blockIdx.x;
  const int g = lane >> 2, c = lane & 3;
  {
    const int slot = s.rs[b] >= (unsigned)sg.g0 ? 0 : 1;
    float* sp = p.partial + ((size_t)b * 2 + slot) * SLOT_FLOATS;
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
  if (PHASE == 1) return;  // phase 2 combines everything after the grid barrier
  // phase 1: the last contributor of the group finishes it
  __threadfence();
  bar_sync(1, NWC * 32);
  const int key = (sg.sh ? p.E : s.ex[sg.j]) * p.ng_max + sg.grp;
  if (ctid == 0) {
    const unsigned inc = (unsigned)(sg.c1 - sg.c0);
    s.flag = (atomicAdd(p.cnt_group + key, inc) + inc == (unsigned)sg.chunks);
  }
  bar_sync(1, NWC * 32);
  if (!s.flag) return;
  __threadfence();
#pragma unroll
  for (int r = 0; r < RW; ++r)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[r][nt][0] = acc[r][nt][1] = acc[r][nt][2] = acc[r][nt][3] = 0.f;
  const int bf = owner_tab(s, NB, (unsigned)sg.g0);
  const int bl = owner_tab(s, NB, (unsigned)(sg.g0 + sg.chunks - 1));
  for (int b2 = bf; b2 <= bl; ++b2) {
    if (s.rs[b2] == s.rs[b2 + 1]) continue;  // empty range
    const int slot = s.rs[b2] >= (unsigned)sg.g0 ? 0 : 1;
    const float* sp = p.partial + ((size_t)b2 * 2 + slot) * SLOT_FLOATS;
#pragma unroll
    for (int r = 0; r < RW; ++r) {
      const int jt = warp * RW + r;
      if (jt >= sg.ntg) break;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int col = nt * 8 + 2 * c;
        const float2 v0 = ld_cg2(sp + (jt * 16 + g) * 16 + col);
        const float2 v1 = ld_cg2(sp + (jt * 16 + g + 8) * 16 + col);
        acc[r][nt][0] += v0.x;
        acc[r][nt][1] += v0.y;
        acc[r][nt][2] += v1.x;
        acc[r][nt][3] += v1.y;
      }
    }
  }
  if (ctid == 0) p.cnt_group[key] = 0u;
  group_epilogue<PHASE, NT>(s, p, sg, acc, warp, lane, ctid);
}

template <int FMT, int PHASE>
__global__ void __launch_bounds__(NTHREADS, 1) expert_kernel(const PhaseParams p) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  PhaseSmem& s = *reinterpret_cast<PhaseSmem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int NB = gridDim.x;
  constexpr int KC = FMT == 1 ? 64 : 32;
  constexpr int KWC = KW / KC;

  if (tid == 0) {
    for (int i = 0; i < NSW; ++i) {
      mbar_init(&s.wfull[i], 1);
      mbar_init(&s.wempty[i], NWC);
    }
    for (int i = 0; i < NSX; ++i) {
      mbar_init(&s.xfull[i], 1);
      mbar_init(&s.xempty[i], NWC);
    }
    fence_barrier_init();
    s.dead = 0;
    if (PHASE == 1) s.gen0 = ld_acquire_u32(p.grid_gen);
  }
  grid_dep_wait();
  grid_dep_launch();
  if (tid == 0) {
    s.M = p.meta[META_M];
    s.nT = p.meta[META_NT];
    s.MK = p.meta[META_MK];
    s.has_shared = p.meta[META_HAS_SHARED];
    s.nE = p.meta[META_NE];
    if (s.nE < 0 || s.nE > MAX_ENTRIES || s.MK > MAX_TOK * MAX_K || s.nT > MAX_E || s.M > MAX_TOK) {
      atomicOr(p.err, ERR_BAD_META);
      s.nE = 0;
      s.nT = 0;
    }
  }
  __syncthreads();
  {
    // entries in parallel; every routed entry has the same geometry, so the
    // unit prefixes have closed forms
    const long long units_r = (long long)p.gr.ngroups * p.gr.chunks;
    for (int j = tid; j < s.nE; j += NTHREADS) {
      int ex = p.meta[META_EX + j], ro = p.meta[META_RO + j], nc = p.meta[META_NC + j];
      const bool sh = s.has_shared && j == s.nT;
      if (nc < 1 || nc > MAX_TOK || ro < 0 || (!sh && (ex < 0 || ex >= p.E || ro + nc > MAX_TOK * MAX_K))) {
        atomicOr(p.err, ERR_BAD_META);
        nc = 1;
        ex = 0;
        ro = 0;
      }
      s.ex[j] = ex;
      s.ro[j] = ro;
      s.nc[j] = nc;
      s.upre[j] = (long long)j * units_r;
      s.cpre[j] = j * p.gr.chunks;
      if (!sh)
        for (int n = 0; n < nc; ++n) s.rj[ro + n] = j;
    }
    if (tid == 0) {
      const bool hs = s.has_shared && s.nE > s.nT;
      s.upre[s.nE] = (long long)s.nT * units_r + (hs ? (long long)p.gsh.ngroups * p.gsh.chunks : 0);
      s.cpre[s.nE] = s.nT * p.gr.chunks + (hs ? p.gsh.chunks : 0);
    }
  }
  for (int i = tid; i < MAX_TOK * MAX_K; i += NTHREADS) {
    int tk = 0;
    if (i < s.MK) {
      tk = p.routes[i].token;
      if (tk < 0 || tk >= MAX_TOK) {
        atomicOr(p.err, ERR_BAD_INDEX);
        tk = 0;
      }
    }
    s.tok[i] = tk;
  }
  __syncthreads();

  const long long U = s.upre[s.nE];
  if (U == 0) return;
  for (int b = tid; b <= NB; b += NTHREADS) s.rs[b] = (unsigned)range_start((uint64_t)U, NB, b);
  __syncthreads();
  const long long u0 = (long long)range_start((uint64_t)U, NB, blockIdx.x);
  const long long u1 = (long long)range_start((uint64_t)U, NB, blockIdx.x + 1);
  if (u0 >= u1 && PHASE == 0) return;

  if (warp == NWC) {
    // ---------------------------------------------------------------- producer warp
    const uint64_t pol = policy_evict_first();
    int wi = 0, wph = 0, xi = 0, xph = 0;
    int wuse[NSW], xuse[NSX];
    for (int i = 0; i < NSW; ++i) wuse[i] = 0;
    for (int i = 0; i < NSX; ++i) xuse[i] = 0;
    long long u = u0;
    int j = 0;
    Seg sg;
    bool alive = true;
    while (alive && next_seg<PHASE == 1>(s, p, u, u1, j, sg)) {
      const uint8_t* mat = sg.sh ? p.w_shared : p.w_routed + (uint64_t)s.ex[sg.j] * p.w_stride;
      const uint8_t* gbase = mat + group_offset(sg.gs, sg.chunks, sg.grp);
      const __half* brow = nullptr;
      if (lane < sg.nc) {
        if (PHASE == 0)
          brow = sg.sh ? p.b_shared + (size_t)lane * p.b_shared_ld
                       : p.b_routed + (size_t)s.tok[sg.ro + lane] * p.b_routed_ld;
        else
          brow = sg.sh ? p.b_shared + (size_t)lane * p.b_shared_ld : p.b_routed + (size_t)(sg.ro + lane) * p.b_routed_ld;
      }
      const unsigned ustride = (unsigned)sg.ntg * UNIT_BYTES;
      for (int ws = sg.c0; alive && ws < sg.c1;) {
        const int we = min(sg.c1, (ws / KWC + 1) * KWC);
        const unsigned xbytes = (unsigned)(we - ws) * KC * 2;
        if (lane == 0) {
          alive = mbar_wait(&s.xempty[xi], xph ^ 1, &s.dead, p.err, ERR_TIMEOUT_XEMPTY);
          if (alive) mbar_arrive_expect_tx(&s.xfull[xi], xbytes * (unsigned)sg.nc);
        }
        alive = __shfl_sync(0xffffffffu, alive, 0);
        if (!alive) break;
        if (lane < sg.nc) bulk_g2s(s.x[xi] + lane * XROW, brow + (size_t)ws * KC, xbytes, &s.xfull[xi]);
        ++xuse[xi];
        if (++xi == NSX) {
          xi = 0;
          xph ^= 1;
        }
        for (int k = ws; k < we; k += KS) {
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
          ++wuse[wi];
          if (++wi == NSW) {
            wi = 0;
            wph ^= 1;
          }
        }
        ws = we;
      }
    }
    // Copies still in flight must land before the CTA can exit (only matters
    // when a wait gave up): wait, bounded, for each slot's last issued phase.
    if (lane == 0 && s.dead) {
      unsigned long long t0 = globaltimer();
      for (int i = 0; i < NSW; ++i)
        if (wuse[i])
          while (!mbar_try_wait(&s.wfull[i], (wuse[i] - 1) & 1) && globaltimer() - t0 < WAIT_LIMIT_NS) {
          }
      for (int i = 0; i < NSX; ++i)
        if (xuse[i])
          while (!mbar_try_wait(&s.xfull[i], (xuse[i] - 1) & 1) && globaltimer() - t0 < WAIT_LIMIT_NS) {
          }
    }
    return;
  }

  // ------------------------------------------------------------------ consumer warps
  int wi = 0, wph = 0, xi = 0, xph = 0;
  long long u = u0;
  int j = 0;
  Seg sg;
  while (next_seg<PHASE == 1>(s, p, u, u1, j, sg)) {
    if (sg.nc > 8)
      consume_seg<FMT, PHASE, 2>(s, p, sg, wi, wph, xi, xph, warp, lane, tid, U, NB);
    else
      consume_seg<FMT, PHASE, 1>(s, p, sg, wi, wph, xi, xph, warp, lane, tid, U, NB);
  }
  if (PHASE == 1) {
    grid_barrier(s, p, NB, tid);
    final_combine(s, p, NB, tid);
  }
}

}  // namespace tsm
