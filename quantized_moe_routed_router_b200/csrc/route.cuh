// Route kernel: router GEMV -> (bias) -> top-k + weights -> route list.
//
// One CTA does the whole micro-batch.  The router GEMV runs on the tensor
// cores: the Q8_0 router is repacked at open into the same 16-row MMA
// fragment layout as the experts (rows past E are zero), x * router_xscale is
// staged in shared memory as FP16 scaled by a per-token power of two (|x| max
// lands in [2^13, 2^14); with a non-trivial xscale the product is split into
// an FP16 hi + lo pair so it stays exact), and the FP32 logits come out of
// m16n8k16 MMAs with the block scale folded in per 32-block (llama state page,
// `router_ones`: the INT8 router kernel scales x[n] per element;
// `router_logits_f32`: one FP32 row of logits per token).  One warp per token
// then selects the top K by (selection logit desc, index asc), where the
// selection logit is l + b when a router bias is present (gpt-oss state page,
// `router_bias`: added BEFORE the top-k), and forms the weights:
//   softmax over the selected ("selection reduces to softmax over the
//   selected", `per_expert_ones`), or the full softmax over all experts taken
//   at the selected indices without renormalisation (deepseek2 layer sketch),
// times the per-expert scale.  The reference does this part on the host after
// reading the logits back; here it never leaves the device.
//
// The same CTA then groups the M*K (token, slot) pairs by expert into the
// route list the expert kernels walk: per touched expert its first route and
// count, routes sorted by (expert, token) -- each expert's weights are then
// streamed once per micro-batch.  The pages' route list is a host-written
// 16-byte record per route (gpt-oss state page, `batch_routes`); ours is
// built on the device.
//
// It also writes x as FP16 with the same per-token scale (no xscale), the B
// operand of the gate/up MMA; that kernel undoes the shift exactly.
#pragma once
#include "common.cuh"
#include "layout.cuh"

namespace tsm {

struct Route {
  int token;
  int slot;
  int expert;
  float w;
};

// meta[] layout (int32), written by the route kernel.
enum { META_M = 0, META_NT = 1, META_MK = 2, META_HAS_SHARED = 3, META_NE = 4, META_EX = 8,
       META_RO = META_EX + MAX_ENTRIES, META_NC = META_RO + MAX_ENTRIES, META_INTS = META_NC + MAX_ENTRIES };

struct RouteParams {
  const __nv_bfloat16* x;  // [M][H]
  int M, H, Hp, E, K;
  const uint8_t* rw;       // router, repacked Q8_0 fragment tiles (rows padded to 16)
  MatGeom rg;              // its geometry
  const float* xscale;     // [H] or null (null = ones)
  const float* bias;       // [E] or null
  const float* pes;        // [E] or null
  int bias_mode, score, has_shared;
  float* logits;           // [M][E] (optional)
  int* idx;                // [M][K] (optional)
  float* w;                // [M][K] (optional)
  int* shift;              // [M] (optional)
  __half* xh;              // [M][Hp] x as FP16 * 2^shift
  __half* rin;             // [2][M][Hp] router input hi/lo (used only with an x-scale)
  int* meta;               // optional global copies of the route list
  Route* routes;           // [M*K]
  int* rpos;               // [M][K] -> position in routes
  unsigned* err;
  int* idx_out;            // optional user outputs
  float* w_out;
  float* logits_out;
};

TSM_DEV bool topk_better(float v1, int i1, float v2, int i2) { return v1 > v2 || (v1 == v2 && i1 < i2); }

constexpr int ROUTE_WARPS = 16;           // warps that do the router GEMV (tiles are split over them)
constexpr int ROUTE_PRE = 4;              // router units per warp fetched before x is ready

// Routing results, in the shared memory of the kernel that routes.
struct RouteState {
  float part[ROUTE_WARPS][16][16];        // per-warp partial logits [row][token]
  float lg[MAX_TOK][MAX_E];               // logits (before bias)
  int shift[MAX_TOK];                     // per-token power-of-two scale of x
  int idx[MAX_TOK * MAX_K];               // selected experts, slot order
  float w[MAX_TOK * MAX_K];               // their weights
  int cnt[MAX_E], off[MAX_E];
  unsigned tmask[MAX_E];                  // tokens that selected each expert (bit t)
  int ex[MAX_ENTRIES], ro[MAX_ENTRIES], nc[MAX_ENTRIES];  // touched experts (+ shared entry)
  int tok[MAX_TOK * MAX_K];               // token of each route position
  int rpos[MAX_TOK * MAX_K];              // route position of each (token, slot)
  int rj[MAX_TOK * MAX_K];                // entry index of each route position
  int nT, nE;
};

// Router work split: warp w (< ROUTE_WARPS) owns tile w / wpt and every wpt-th chunk of it.
struct RouterSplit {
  int T, C, wpt, tile, wsub, nunits;
  TSM_DEV RouterSplit(const MatGeom& g, int warp) {
    T = g.tiles;
    C = g.chunks;
    wpt = ROUTE_WARPS / T;  // warps per tile (T <= 16)
    tile = warp / wpt;
    wsub = warp % wpt;
    nunits = (warp < ROUTE_WARPS && tile < T) ? (C - wsub + wpt - 1) / wpt : 0;
  }
  TSM_DEV const uint8_t* unit(const RouteParams& p, int k) const {
    const int ck = wsub + k * wpt;
    const int grp = tile / p.rg.gs, jt = tile % p.rg.gs, ntg = group_tiles(T, p.rg.gs, grp);
    return p.rw + group_offset(p.rg.gs, C, grp) + ((uint64_t)ck * ntg + jt) * UNIT_BYTES;
  }
};

struct RoutePrefetch {
  uint4 q[ROUTE_PRE];
  uint32_t sc[ROUTE_PRE];
};

// The router does not depend on the previous kernel: its first units can be
// fetched before griddepcontrol.wait.
TSM_DEV void route_prefetch(const RouteParams& p, const RouterSplit& rs, int lane, RoutePrefetch& pf) {
#pragma unroll
  for (int k = 0; k < ROUTE_PRE; ++k)
    if (k < rs.nunits) {
      const uint8_t* u = rs.unit(p, k);
      pf.q[k] = *reinterpret_cast<const uint4*>(u + lane * 16);
      pf.sc[k] = *reinterpret_cast<const uint32_t*>(u + QUANT_BYTES + (lane >> 2) * 4);
    }
}

// Per-token |x| (and |x * xscale|) max -> power-of-two shift (warp t: token t).
TSM_DEV void route_shift(const RouteParams& p, RouteState& s, int warp, int lane) {
  if (warp >= p.M) return;
  const int t = warp;
  float m = 0.f;
  constexpr int U = 4;
  for (int kb = lane * 8; kb < p.H; kb += 32 * 8 * U) {
    uint4 raw[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int k = kb + u * 256;
      raw[u] = k < p.H ? *reinterpret_cast<const uint4*>(p.x + (size_t)t * p.H + k) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int k = kb + u * 256;
      const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&raw[u]);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = __bfloat1622float2(b2[q]);
        m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
        if (p.xscale && k < p.H) {
          m = fmaxf(m, fabsf(f.x * p.xscale[k + 2 * q]));
          m = fmaxf(m, fabsf(f.y * p.xscale[k + 2 * q + 1]));
        }
      }
    }
  }
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  int sh = 0;
  if (m > 0.f && m <= 3.4e38f) {
    int e2;
    frexpf(m, &e2);  // m in [2^(e2-1), 2^e2)
    sh = min(126, max(-126, 14 - e2));
  }
  if (lane == 0) {
    s.shift[t] = sh;
    if (p.shift) p.shift[t] = sh;
  }
}

// Row stride (halves) of the router input staged in shared memory: 32 bytes
// past a multiple of 128 keeps the B-fragment loads conflict-free.
TSM_DEV int route_bs_ld(int Hp) { return Hp + 16; }

// x -> FP16 * 2^shift into xh [M][Hp] (zero padded).  The router input (the
// same values, or with an x-scale x * xscale * 2^shift as an FP16 hi + lo
// pair) also goes to `bs` (rows route_bs_ld(Hp) halves apart; hi rows 0..M-1,
// lo rows M..2M-1) when bs is not null, else to `rin` [2][M][Hp].
TSM_DEV void route_convert(const RouteParams& p, const RouteState& s, __half* xh, __half* rin, __half* bs, int tid,
                           int nthr) {
  constexpr int U = 4;
  const int per_row = p.Hp / 8, total = p.M * per_row, bld = route_bs_ld(p.Hp);
  const bool split = p.xscale != nullptr;
  for (int base = tid; base < total; base += nthr * U) {
    uint4 raw[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = base + u * nthr;
      raw[u] = make_uint4(0, 0, 0, 0);
      if (i < total) {
        const int t = i / per_row, k = (i - t * per_row) * 8;
        if (k < p.H) raw[u] = *reinterpret_cast<const uint4*>(p.x + (size_t)t * p.H + k);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = base + u * nthr;
      if (i >= total) break;
      const int t = i / per_row, k = (i - t * per_row) * 8;
      const float sc = __uint_as_float((uint32_t)(s.shift[t] + 127) << 23);
      const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&raw[u]);
      __half hx[8], hh[8], hl[8];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = __bfloat1622float2(b2[q]);
        hx[2 * q] = __float2half_rn(f.x * sc);
        hx[2 * q + 1] = __float2half_rn(f.y * sc);
        if (split) {
          const bool in = k + 2 * q < p.H;
          const float xa = f.x * (in ? p.xscale[k + 2 * q] : 1.f) * sc;
          const float xb = f.y * (in ? p.xscale[k + 2 * q + 1] : 1.f) * sc;
          hh[2 * q] = __float2half_rn(xa);
          hh[2 * q + 1] = __float2half_rn(xb);
          hl[2 * q] = __float2half_rn(xa - __half2float(hh[2 * q]));
          hl[2 * q + 1] = __float2half_rn(xb - __half2float(hh[2 * q + 1]));
        }
      }
      *reinterpret_cast<uint4*>(xh + (size_t)t * p.Hp + k) = *reinterpret_cast<uint4*>(hx);
      if (bs) {
        *reinterpret_cast<uint4*>(bs + (size_t)t * bld + k) = *reinterpret_cast<uint4*>(split ? hh : hx);
        if (split) *reinterpret_cast<uint4*>(bs + (size_t)(p.M + t) * bld + k) = *reinterpret_cast<uint4*>(hl);
      } else if (split) {
        *reinterpret_cast<uint4*>(rin + (size_t)t * p.Hp + k) = *reinterpret_cast<uint4*>(hh);
        *reinterpret_cast<uint4*>(rin + (size_t)(p.M + t) * p.Hp + k) = *reinterpret_cast<uint4*>(hl);
      }
    }
  }
}

// One Q8_0 (tile, chunk) unit of the router against x rows in global memory
// (b points at column 32 * chunk of row 0, rows `ld` halves apart): acc += W x.
template <int NT>
TSM_DEV void router_unit(float (&acc)[NT][4], uint4 q, uint32_t sc, const __half* b, int ld, int M, int lane) {
  const int g = lane >> 2, c = lane & 3;
  const float2 d = __half22float2(*reinterpret_cast<const __half2*>(&sc));
  float tmp[NT][4];
  const uint32_t a0[4] = {u8x2_to_f16x2<0x4140>(q.x), u8x2_to_f16x2<0x4342>(q.x), u8x2_to_f16x2<0x4140>(q.y),
                          u8x2_to_f16x2<0x4342>(q.y)};
  const uint32_t a1[4] = {u8x2_to_f16x2<0x4140>(q.z), u8x2_to_f16x2<0x4342>(q.z), u8x2_to_f16x2<0x4140>(q.w),
                          u8x2_to_f16x2<0x4342>(q.w)};
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int row = min(nt * 8 + g, M - 1);  // columns past M repeat the last token; their outputs are unused
    const __half* br = b + (size_t)row * ld;
    const uint2 b0 = *reinterpret_cast<const uint2*>(br + 4 * c);
    const uint2 b1 = *reinterpret_cast<const uint2*>(br + 16 + 4 * c);
    mma_f16_zc(tmp[nt], a0, b0.x, b0.y);
    mma_f16_acc(tmp[nt], a1, b1.x, b1.y);
    acc[nt][0] = fmaf(d.x, tmp[nt][0], acc[nt][0]);
    acc[nt][1] = fmaf(d.x, tmp[nt][1], acc[nt][1]);
    acc[nt][2] = fmaf(d.y, tmp[nt][2], acc[nt][2]);
    acc[nt][3] = fmaf(d.y, tmp[nt][3], acc[nt][3]);
  }
}

// Router GEMV of all tokens -> s.lg (bias not applied).  bsrc: router input
// rows `ld` halves apart (lo rows follow the M hi rows with an x-scale), in
// shared or global memory.  Needs a barrier of the whole CTA after
// route_convert; ends with one.
template <int NT>
TSM_DEV void route_gemv(const RouteParams& p, RouteState& s, const RouterSplit& rs, const RoutePrefetch& pf,
                        const __half* bsrc, int ld, int warp, int lane, int tid, int nthr) {
  float acc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
  const bool split = p.xscale != nullptr;
  // units past the prefetched ones: ROUTE_PRE at a time, the next batch in flight while one is used
  RoutePrefetch nb;
  auto fetch = [&](RoutePrefetch& f, int k0) {
#pragma unroll
    for (int k = 0; k < ROUTE_PRE; ++k)
      if (k0 + k < rs.nunits) {
        const uint8_t* u = rs.unit(p, k0 + k);
        f.q[k] = *reinterpret_cast<const uint4*>(u + lane * 16);
        f.sc[k] = *reinterpret_cast<const uint32_t*>(u + QUANT_BYTES + (lane >> 2) * 4);
      }
  };
  for (int half = 0; half < (split ? 2 : 1); ++half) {
    const __half* b = bsrc + (size_t)half * p.M * ld;
    if (ROUTE_PRE < rs.nunits) fetch(nb, ROUTE_PRE);
#pragma unroll
    for (int k = 0; k < ROUTE_PRE; ++k)
      if (k < rs.nunits) router_unit<NT>(acc, pf.q[k], pf.sc[k], b + (rs.wsub + k * rs.wpt) * 32, ld, p.M, lane);
    for (int kb = ROUTE_PRE; kb < rs.nunits; kb += ROUTE_PRE) {
      RoutePrefetch cur = nb;
      if (kb + ROUTE_PRE < rs.nunits) fetch(nb, kb + ROUTE_PRE);
#pragma unroll
      for (int k = 0; k < ROUTE_PRE; ++k)
        if (kb + k < rs.nunits)
          router_unit<NT>(acc, cur.q[k], cur.sc[k], b + (rs.wsub + (kb + k) * rs.wpt) * 32, ld, p.M, lane);
    }
  }
  if (warp < ROUTE_WARPS) {
    const int gq = lane >> 2, c = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      s.part[warp][gq][nt * 8 + 2 * c] = acc[nt][0];
      s.part[warp][gq][nt * 8 + 2 * c + 1] = acc[nt][1];
      s.part[warp][gq + 8][nt * 8 + 2 * c] = acc[nt][2];
      s.part[warp][gq + 8][nt * 8 + 2 * c + 1] = acc[nt][3];
    }
  }
  __syncthreads();
  // logits[t][e] = sum over the tile's warps in order, times 2^-shift[t]
  for (int i = tid; i < p.M * p.E; i += nthr) {
    const int t = i / p.E, e = i - t * p.E;
    const int tl = e >> 4, r = e & 15;
    float v = 0.f;
    for (int w = 0; w < rs.wpt; ++w) v += s.part[tl * rs.wpt + w][r][t];
    s.lg[t][e] = v * __uint_as_float((uint32_t)(127 - s.shift[t]) << 23);
  }
  __syncthreads();
}

// Top-k and weights: warp t handles token t (lane holds experts lane, lane+32, ...).
TSM_DEV void route_topk(const RouteParams& p, RouteState& s, int warp, int lane) {
  if (warp >= p.M) return;
  const int t = warp;
  constexpr int PER = MAX_E / 32;
  float vsel[PER], vsc[PER];
  unsigned taken = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = lane + 32 * i;
    const float l = e < p.E ? s.lg[t][e] : -INFINITY;
    const float ls = (e < p.E && p.bias && p.bias_mode != 0) ? l + p.bias[e] : l;
    vsel[i] = ls;
    vsc[i] = (p.bias_mode == 1 && p.bias) ? ls : l;
    if (e < p.E) {
      if (p.logits) p.logits[(size_t)t * p.E + e] = l;
      if (p.logits_out) p.logits_out[(size_t)t * p.E + e] = l;
    }
  }
  int selk = 0;  // lane k holds the k-th selected expert and its score logit
  float sck = -INFINITY;
  for (int k = 0; k < p.K; ++k) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int e = lane + 32 * i;
      if (e < p.E && !((taken >> i) & 1u) && topk_better(vsel[i], e, bv, bi)) {
        bv = vsel[i];
        bi = e;
      }
    }
    for (int o = 16; o; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (topk_better(ov, oi, bv, bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if (bi < 0 || bi >= p.E) {  // only with NaN logits
      if (lane == 0) atomicOr(p.err, ERR_BAD_INDEX);
      bi = 0;
    }
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    float mine = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i)
      if (i == (bi >> 5)) mine = vsc[i];
    const float sc = __shfl_sync(0xffffffffu, mine, bi & 31);
    if (lane == k) {
      selk = bi;
      sck = sc;
    }
  }
  const bool act = lane < p.K;
  float m = act ? sck : -INFINITY;
  if (p.score != 0) {
#pragma unroll
    for (int i = 0; i < PER; ++i)
      if (lane + 32 * i < p.E) m = fmaxf(m, vsc[i]);
  }
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float den = 0.f;
  if (p.score == 0) {
    den = act ? expf(sck - m) : 0.f;
  } else {
#pragma unroll
    for (int i = 0; i < PER; ++i)
      if (lane + 32 * i < p.E) den += expf(vsc[i] - m);
  }
  for (int o = 16; o; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
  if (act) {
    const float wv = expf(sck - m) / den * (p.pes ? p.pes[selk] : 1.f);
    s.idx[t * p.K + lane] = selk;
    s.w[t * p.K + lane] = wv;
    if (p.idx) p.idx[t * p.K + lane] = selk;
    if (p.w) p.w[t * p.K + lane] = wv;
    if (p.idx_out) p.idx_out[t * p.K + lane] = selk;
    if (p.w_out) p.w_out[t * p.K + lane] = wv;
  }
}

// Route list: the (token, slot) pairs grouped by expert (touched experts in
// ascending order, tokens ascending), plus the shared expert as the last
// entry with all M tokens.  Needs a CTA barrier after route_topk; ends with one.
TSM_DEV void route_list(const RouteParams& p, RouteState& s, int warp, int lane, int tid, int nthr) {
  for (int e = tid; e < p.E; e += nthr) {
    s.cnt[e] = 0;
    s.tmask[e] = 0u;
  }
  __syncthreads();
  const int MK = p.M * p.K;
  for (int i = tid; i < MK; i += nthr) {
    atomicAdd(&s.cnt[s.idx[i]], 1);
    atomicOr(&s.tmask[s.idx[i]], 1u << (i / p.K));
  }
  __syncthreads();
  if (warp == 0) {
    constexpr int PER = MAX_E / 32;
    int cl[PER], tot = 0, nz = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int e = lane * PER + i;
      cl[i] = e < p.E ? s.cnt[e] : 0;
      tot += cl[i];
      nz += cl[i] > 0;
    }
    int incl = tot, nzincl = nz;
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o), w = __shfl_up_sync(0xffffffffu, nzincl, o);
      if (lane >= o) {
        incl += v;
        nzincl += w;
      }
    }
    int run = incl - tot, slot = nzincl - nz;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int e = lane * PER + i;
      if (e < p.E) {
        s.off[e] = run;
        if (cl[i]) {
          s.ex[slot] = e;
          s.ro[slot] = run;
          s.nc[slot] = cl[i];
          if (p.meta) {
            p.meta[META_EX + slot] = e;
            p.meta[META_RO + slot] = run;
            p.meta[META_NC + slot] = cl[i];
          }
          ++slot;
        }
        run += cl[i];
      }
    }
    const int nT = __shfl_sync(0xffffffffu, nzincl, 31);
    if (lane == 0) {
      s.nT = nT;
      s.nE = nT + (p.has_shared ? 1 : 0);
      if (p.has_shared) {
        s.ex[nT] = p.E;
        s.ro[nT] = MK;
        s.nc[nT] = p.M;
      }
      if (p.meta) {
        if (p.has_shared) {
          p.meta[META_EX + nT] = p.E;
          p.meta[META_RO + nT] = MK;
          p.meta[META_NC + nT] = p.M;
        }
        p.meta[META_M] = p.M;
        p.meta[META_NT] = nT;
        p.meta[META_MK] = MK;
        p.meta[META_HAS_SHARED] = p.has_shared;
        p.meta[META_NE] = s.nE;
      }
    }
  }
  __syncthreads();
  for (int i = tid; i < MK; i += nthr) {
    const int e = s.idx[i], tk = i / p.K;
    const int pos = s.off[e] + __popc(s.tmask[e] & ((1u << tk) - 1u));  // tokens before tk that chose e
    s.tok[pos] = tk;
    s.rpos[i] = pos;
    if (p.routes) {
      Route r;
      r.token = tk;
      r.slot = i % p.K;
      r.expert = e;
      r.w = s.w[i];
      p.routes[pos] = r;
    }
    if (p.rpos) p.rpos[i] = pos;
  }
  __syncthreads();
  // entry index of each route position
  for (int j = tid; j < s.nT; j += nthr)
    for (int n = 0; n < s.nc[j]; ++n) s.rj[s.ro[j] + n] = j;
  __syncthreads();
}

// ---------------------------------------------------------------------------- standalone route kernel
constexpr int ROUTE_THREADS = ROUTE_WARPS * 32;

// Shared memory of route_kernel: RouteState, then the staged router input
// (2 * M rows of route_bs_ld(Hp) halves) when it fits.
TSM_HD size_t route_stage_bytes(int M, int Hp, bool split) { return (size_t)(split ? 2 : 1) * M * (Hp + 16) * 2; }

__global__ void __launch_bounds__(ROUTE_THREADS, 1) route_kernel(const RouteParams p, int stage_in_smem) {
  extern __shared__ __align__(128) uint8_t route_smem_raw[];
  RouteState& s = *reinterpret_cast<RouteState*>(route_smem_raw);
  __half* bs = stage_in_smem ? reinterpret_cast<__half*>(route_smem_raw + ((sizeof(RouteState) + 127) & ~(size_t)127))
                             : nullptr;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const RouterSplit rs(p.rg, warp);
  RoutePrefetch pf;
  route_prefetch(p, rs, lane, pf);
  grid_dep_wait();
  grid_dep_launch();
  route_shift(p, s, warp, lane);
  __syncthreads();
  route_convert(p, s, p.xh, p.rin, bs, tid, ROUTE_THREADS);
  __syncthreads();
  const __half* bsrc = bs ? bs : (p.xscale ? p.rin : p.xh);
  const int ld = bs ? route_bs_ld(p.Hp) : p.Hp;
  if (p.M > 8)
    route_gemv<2>(p, s, rs, pf, bsrc, ld, warp, lane, tid, ROUTE_THREADS);
  else
    route_gemv<1>(p, s, rs, pf, bsrc, ld, warp, lane, tid, ROUTE_THREADS);
  route_topk(p, s, warp, lane);
  __syncthreads();
  route_list(p, s, warp, lane, tid, ROUTE_THREADS);
}

}  // namespace tsm
