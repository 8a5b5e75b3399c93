// Routing: router GEMV -> (bias) -> top-k + weights -> route list.
//
// The router GEMV runs on the tensor cores: the Q8_0 router is repacked at
// open into the 16-row MMA fragment layout of the experts, one 16-expert tile
// after another (rows past E are zero), and the FP32 logits come out of
// m16n8k16 MMAs with the block scale folded in per 32-block (llama state page,
// `router_ones`: the int8 router GEMV scales x[n] per element;
// `router_logits_f32`: one FP32 row of logits per token).
//
// The GEMV is cut into items (tile j, slice c): slice c is the K range of
// chunks [c CS, (c + 1) CS) (32 K per chunk).  An item needs only its slice of
// x and CS units of the router, so in the fused layer kernel the T * S items
// go to T * S CTAs, each loading a few KB (one SM takes in roughly 50 GB/s, so
// the whole x and router in one CTA would cost several microseconds).  Within
// an item, x * router_xscale is staged in shared memory as FP16 scaled by a
// power of two per (token, slice) -- the slice's |x| max lands in
// [2^13, 2^14); with a non-trivial xscale the product is an FP16 hi + lo pair
// so it stays exact -- and the item's 16 warps' partial sums are added in
// warp order and unscaled exactly.  A logit is the sum of its S item values
// in slice order.  route_kernel runs the same items one after another in one
// CTA, so both kernels produce the same bits.
//
// One warp per token then selects the top K by (selection logit desc, index
// asc), where the selection logit is l + b when a router bias is present
// (gpt-oss state page, `router_bias`: the bias enters ahead of the top-k), and forms the
// weights: softmax over the selected (`per_expert_ones`: with unit per-expert
// scales the weights are exactly that softmax), or the full softmax over all experts taken at
// the selected indices without renormalisation (deepseek2 layer sketch), or --
// with sigmoid scoring (llama state page, MiniMax flow) -- the sigmoid scores
// s of the selected experts renormalised to sum 1, the selection then being by
// s + b with the bias as a selection-only correction; times the per-expert
// scale.  The reference does this part on the host after
// reading the logits back; here it never leaves the device.
//
// The (token, slot) pairs are then grouped by expert into the route list the
// expert phases walk: routes sorted by (expert, token), cut into entries of at
// most 16 routes (an expert's weights are streamed once per entry: once per
// micro-batch for up to 16 routes, once per 16 routes beyond).  The pages' route list is a host-written 16-byte record
// per route (gpt-oss state page, `batch_routes`); ours is built on the device.
//
// The gate/up B operand is x as FP16 scaled by a per-token power of two taken
// from the |x| max over the whole row (the max of the slice maxima); the
// gate/up epilogue undoes it exactly.
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

constexpr int ROUTE_WARPS = 16;  // warps of a routing CTA; an item's chunks are split over them
constexpr int MAX_SLICES = 64;   // router slices along K

struct RouteParams {
  const __nv_bfloat16* x;  // [M][H]
  int M, H, Hp, E, K;      // M: tokens of the launch (layer kernel <= 64, route kernel <= 16)
  int S, CS;               // router slices: S slices of CS chunks (32 K each), the last may be shorter
  const uint8_t* rw;       // router, repacked Q8_0 fragment tiles, tile-major (rows padded to 16)
  MatGeom rg;              // its geometry
  const float* xscale;     // [H] or null (null = ones)
  const float* bias;       // [E] or null
  const float* pes;        // [E] or null
  int bias_mode, score, has_shared;
  float* logits;           // [M][E] (optional)
  int* idx;                // [M][K] (optional)
  float* w;                // [M][K] (optional)
  int* shift;              // [M] (optional)
  int* meta;               // optional global copies of the route list
  Route* routes;           // [M*K]
  int* rpos;               // [M][K] -> position in routes
  unsigned* err;
  int* idx_out;            // optional user outputs
  float* w_out;
  float* logits_out;
  const unsigned* pre_err; // route_kernel only: a word an earlier kernel of the same call set on bad input, or null
  int sentinel;            // route_kernel only: on any error, overwrite idx_out / w_out with -1 / 0
  int whole;               // 1: every routing CTA holds the whole router and x (route_whole), 0: router items
};

// Routing results, in the shared memory of the kernel that routes.
struct RouteState {
  float part[ROUTE_WARPS][16][16];        // per-warp partial logits [row][token] of one router item
  float* lg;                              // logits (before bias) [M][lgld], in the caller's scratch
  int lgld;
  int shift[MAX_LT];                      // per-token power-of-two scale of x (whole row)
  float smax[MAX_TOK];                    // |x| max of the current slice (one routing block)
  int sshift[MAX_TOK];                    // its power-of-two scale
  float gmax[MAX_TOK];                    // running |x| max over the slices (route_kernel)
  int idx[MAX_LT * MAX_K];                // selected experts, slot order
  float w[MAX_LT * MAX_K];                // their weights
  int off[MAX_E];                         // first route position of each expert
  int eslot[MAX_E];                       // first entry index of each touched expert
  unsigned long long tmask[MAX_E];        // tokens that selected each expert (bit t)
  float bias[MAX_E], pes[MAX_E];          // router bias and per-expert scale (read before the dependency wait)
  int ex[MAX_ENTRIES], ro[MAX_ENTRIES], nc[MAX_ENTRIES];  // entries: expert, first route, routes (<= 16)
  int tok[MAX_LT * MAX_K];                // token of each route position
  int rpos[MAX_LT * MAX_K];               // route position of each (token, slot)
  int rj[MAX_LT * MAX_K];                 // entry index of each route position
  int nT, nE;                             // routed entries; routed + shared entries
  uint64_t xbar;                          // completion of the bulk copy of an x slice
  uint64_t rbar;                          // completion of the bulk copy of an item's router units
  uint64_t pbar;                          // completion of the bulk copy of the published items
  int xdead;                              // set when a wait of the routing gave up
};

// ---------------------------------------------------------------------------- slices
TSM_HD int slice_lo(int CS, int c) { return c * CS; }
TSM_HD int slice_hi(int CS, int C, int c) { return (c + 1) * CS < C ? (c + 1) * CS : C; }
// Row stride (halves) of the FP16 router input: 32 bytes past a multiple of
// 128 keeps the B-fragment loads conflict-free.
TSM_HD int slice_ld(int CS) { return round_up(CS * 32, 64) + 16; }
TSM_HD size_t align128(size_t n) { return (n + 127) & ~(size_t)127; }
// Row stride (floats) of a published item [M][.]: a multiple of 4, so an
// item block is whole 16-byte units (one bulk copy).
TSM_HD int item_ld(int E) { return (E + 3) & ~3; }

// Shared-memory buffers of one item: x slice (BF16, [M][CS*32]), router input
// (FP16, hi rows then lo rows with an x-scale, slice_ld apart) and the item's
// CS router units.
struct SliceSmem {
  size_t xs, xin, rt, total;
  TSM_HD SliceSmem(int M, int CS, bool split) {
    xs = 0;
    xin = align128((size_t)M * CS * 64);
    rt = xin + align128((size_t)(split ? 2 : 1) * M * slice_ld(CS) * 2);
    total = rt + align128((size_t)CS * UNIT_BYTES);
  }
};

// Shared memory of route_whole: the whole repacked router [T][C] units, x
// [M][H] BF16, the router input of every slice [S][halves][M][slice_ld(CS)]
// FP16, the slice maxima and shifts [M][S], the items [T][S][16][M] FP32 and
// the logits [M][E] FP32.
struct WholeSmem {
  size_t rt, x, xin, smx, ssh, item, lg, total;
  TSM_HD WholeSmem(int M, int H, int T, int C, int S, int CS, int E, bool split) {
    rt = 0;
    x = align128((size_t)T * C * UNIT_BYTES);
    xin = x + align128((size_t)M * H * 2);
    smx = xin + align128((size_t)S * (split ? 2 : 1) * M * slice_ld(CS) * 2);
    ssh = smx + align128((size_t)M * S * 4);
    item = ssh + align128((size_t)M * S * 4);
    lg = item + align128((size_t)T * S * 16 * M * 4);
    total = lg + align128((size_t)M * E * 4);
  }
};

// Router bias and per-expert scale of expert `tid` (0 and 1 where absent).
// They are weights, so they are read before the dependency wait.
struct RouteConst {
  float b, s;
};
TSM_DEV RouteConst route_const_load(const RouteParams& p, int tid) {
  RouteConst c{0.f, 1.f};
  if (tid < p.E) {
    if (p.bias) c.b = p.bias[tid];
    if (p.pes) c.s = p.pes[tid];
  }
  return c;
}

// Shared-memory state that must be set before the first CTA barrier: the
// prefetched constants and the cleared per-expert token masks.
TSM_DEV void route_init_smem(RouteState& s, const RouteConst& c, int tid) {
  if (tid < MAX_E) {
    s.bias[tid] = c.b;
    s.pes[tid] = c.s;
    s.tmask[tid] = 0ull;
  }
}

// Running max of |x| (and |x * xscale|) over the 8 BF16 values of `raw` at column k.
TSM_DEV float absmax8(const RouteParams& p, const uint4& raw, int k, float m) {
  const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float2 f = __bfloat1622float2(b2[q]);
    m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
    if (p.xscale && k < p.H) {
      m = fmaxf(m, fabsf(f.x * p.xscale[k + 2 * q]));
      m = fmaxf(m, fabsf(f.y * p.xscale[k + 2 * q + 1]));
    }
  }
  return m;
}

// 8 BF16 values of x at column k (zero past H) -> FP16 * 2^shift (hx) and,
// with an x-scale, x * xscale * 2^shift as an FP16 hi + lo pair (hh, hl).
TSM_DEV void convert8(const RouteParams& p, const uint4& raw, int k, float sc, bool split, uint4& hx, uint4& hh,
                      uint4& hl) {
  const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
  __half2* ox = reinterpret_cast<__half2*>(&hx);
  __half* oh = reinterpret_cast<__half*>(&hh);
  __half* ol = reinterpret_cast<__half*>(&hl);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float2 f = __bfloat1622float2(b2[q]);
    ox[q] = __floats2half2_rn(f.x * sc, f.y * sc);  // each half rounded to nearest, as one conversion each
    if (split) {
      const bool in = k + 2 * q < p.H;
      const float xa = f.x * (in ? p.xscale[k + 2 * q] : 1.f) * sc;
      const float xb = f.y * (in ? p.xscale[k + 2 * q + 1] : 1.f) * sc;
      oh[2 * q] = __float2half_rn(xa);
      oh[2 * q + 1] = __float2half_rn(xb);
      ol[2 * q] = __float2half_rn(xa - __half2float(oh[2 * q]));
      ol[2 * q + 1] = __float2half_rn(xb - __half2float(oh[2 * q + 1]));
    }
  }
}

// One thread: bulk copies of the M rows of x slice c into xs ([M][CS*32]
// BF16), completing on s.xbar.  x is 16-byte aligned and H a multiple of 32,
// so every source starts on a 64-byte boundary.
TSM_DEV void slice_issue_x(const RouteParams& p, RouteState& s, int c, __nv_bfloat16* xs) {
  const int lo = slice_lo(p.CS, c), hi = slice_hi(p.CS, p.rg.chunks, c);
  const unsigned row = (unsigned)(hi - lo) * 64u;
  mbar_arrive_expect_tx(&s.xbar, row * (unsigned)p.M);
  for (int t = 0; t < p.M; ++t)
    bulk_g2s(xs + (size_t)t * p.CS * 32, p.x + (size_t)t * p.H + lo * 32, row, &s.xbar);
}

// One thread: bulk copy of item (j, c)'s router units (contiguous: the router
// is tile-major) into rt, completing on s.rbar.  The router is constant, so
// this may be issued before the dependency wait.
TSM_DEV void slice_issue_router(const RouteParams& p, RouteState& s, int j, int c, uint8_t* rt) {
  const int lo = slice_lo(p.CS, c), hi = slice_hi(p.CS, p.rg.chunks, c);
  const unsigned bytes = (unsigned)(hi - lo) * UNIT_BYTES;
  mbar_arrive_expect_tx(&s.rbar, bytes);
  bulk_g2s(rt, p.rw + ((size_t)j * p.rg.chunks + lo) * UNIT_BYTES, bytes, &s.rbar);
}

// Power-of-two scale that puts |x| max m in [2^13, 2^14) (0 for m = 0 or not finite).
TSM_DEV int shift_of_max(float m) {
  int sh = 0;
  if (m > 0.f && m <= 3.4e38f) {
    int e2;
    frexpf(m, &e2);  // m in [2^(e2-1), 2^e2)
    sh = min(126, max(-126, 14 - e2));
  }
  return sh;
}

TSM_DEV float pow2f(int e) { return __uint_as_float((uint32_t)(e + 127) << 23); }

// Per-token |x| max of slice c (warp t: token t) -> s.smax, s.sshift.
TSM_DEV void slice_max(const RouteParams& p, RouteState& s, int c, const __nv_bfloat16* xs, int warp, int lane) {
  if (warp >= p.M) return;
  const int t = warp, lo = slice_lo(p.CS, c), n = (slice_hi(p.CS, p.rg.chunks, c) - lo) * 32;
  const __nv_bfloat16* row = xs + (size_t)t * p.CS * 32;
  float m = 0.f;
  for (int k = lane * 8; k < n; k += 256) m = absmax8(p, *reinterpret_cast<const uint4*>(row + k), lo * 32 + k, m);
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) {
    s.smax[t] = m;
    s.sshift[t] = shift_of_max(m);
  }
}

// Router input of slice c: x (* xscale) * 2^sshift[t] as FP16 (hi, and lo in
// rows M..2M-1 with an x-scale), rows slice_ld(CS) halves apart.
TSM_DEV void slice_input(const RouteParams& p, const RouteState& s, int c, const __nv_bfloat16* xs, __half* xin,
                         int tid, int nthr) {
  const int lo = slice_lo(p.CS, c), per_row = (slice_hi(p.CS, p.rg.chunks, c) - lo) * 4, ld = slice_ld(p.CS);
  const bool split = p.xscale != nullptr;
  for (int i = tid; i < p.M * per_row; i += nthr) {
    const int t = i / per_row, k = (i - t * per_row) * 8;
    const uint4 raw = *reinterpret_cast<const uint4*>(xs + (size_t)t * p.CS * 32 + k);
    uint4 hx, hh, hl;
    convert8(p, raw, lo * 32 + k, pow2f(s.sshift[t]), split, hx, hh, hl);
    *reinterpret_cast<uint4*>(xin + (size_t)t * ld + k) = split ? hh : hx;
    if (split) *reinterpret_cast<uint4*>(xin + (size_t)(p.M + t) * ld + k) = hl;
  }
}

// x slice c of a routing block (p.M <= 16 rows, the launch's tokens t0 ..)
// -> FP16 * 2^shift[t0 + t] (whole-row scale) into rows t0 + t of xh [.][Hp].
TSM_DEV void slice_xh(const RouteParams& p, const RouteState& s, int c, const __nv_bfloat16* xs, __half* xh, int t0,
                      int tid, int nthr) {
  const int lo = slice_lo(p.CS, c), per_row = (slice_hi(p.CS, p.rg.chunks, c) - lo) * 4;
  for (int i = tid; i < p.M * per_row; i += nthr) {
    const int t = i / per_row, k = (i - t * per_row) * 8;
    const uint4 raw = *reinterpret_cast<const uint4*>(xs + (size_t)t * p.CS * 32 + k);
    uint4 hx, hh, hl;
    convert8(p, raw, lo * 32 + k, pow2f(s.shift[t0 + t]), false, hx, hh, hl);
    *reinterpret_cast<uint4*>(xh + (size_t)(t0 + t) * p.Hp + lo * 32 + k) = hx;
  }
}

// One Q8_0 (tile, chunk) unit of the router against the FP16 router input
// (b points at the chunk's column 0 of row 0, rows `ld` halves apart): acc += W x.
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

// Item (tile j, slice c): the slice's router units (at `units`, shared or
// global memory: unit of local chunk q at units + q * UNIT_BYTES) against the
// router input xin.  Warp w takes local chunks w, w + ROUTE_WARPS, ...; the
// warps' partial sums are added in warp order and multiplied by
// 2^-sshift[t].  The value of (token t, expert e = 16 j + r) goes to
// pub[t * item_ld(E) + e] when pub is not null, else is added to s.lg[t][e].
// Needs a CTA barrier after slice_input; ends with one.
template <int NT>
TSM_DEV void slice_gemv(const RouteParams& p, RouteState& s, int j, int c, const __half* xin, const uint8_t* units,
                        int warp, int lane, int tid, int nthr, float* pub) {
  float acc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
  const int nck = slice_hi(p.CS, p.rg.chunks, c) - slice_lo(p.CS, c), ld = slice_ld(p.CS);
  const int halves = p.xscale ? 2 : 1;
  if (warp < ROUTE_WARPS) {
#pragma unroll 2
    for (int q = warp; q < nck; q += ROUTE_WARPS) {
      const uint8_t* u = units + (size_t)q * UNIT_BYTES;
      const uint4 qw = *reinterpret_cast<const uint4*>(u + lane * 16);
      const uint32_t sc = *reinterpret_cast<const uint32_t*>(u + QUANT_BYTES + (lane >> 2) * 4);
      for (int h = 0; h < halves; ++h)
        router_unit<NT>(acc, qw, sc, xin + (size_t)h * p.M * ld + q * 32, ld, p.M, lane);
    }
    const int gq = lane >> 2, cq = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      s.part[warp][gq][nt * 8 + 2 * cq] = acc[nt][0];
      s.part[warp][gq][nt * 8 + 2 * cq + 1] = acc[nt][1];
      s.part[warp][gq + 8][nt * 8 + 2 * cq] = acc[nt][2];
      s.part[warp][gq + 8][nt * 8 + 2 * cq + 1] = acc[nt][3];
    }
  }
  __syncthreads();
  for (int i = tid; i < p.M * 16; i += nthr) {
    const int t = i >> 4, r = i & 15, e = j * 16 + r;
    if (e >= p.E) continue;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < ROUTE_WARPS; ++w) v += s.part[w][r][t];
    v *= pow2f(-s.sshift[t]);
    if (pub)
      pub[(size_t)t * item_ld(p.E) + e] = v;
    else
      s.lg[t * s.lgld + e] += v;
  }
  __syncthreads();
}

// Order-preserving map of an FP32 value to an unsigned key (larger value,
// larger key; -0 and +0 share a key); NaN maps to 0, below every number.
TSM_DEV unsigned order_key(float f) {
  if (f != f) return 0u;
  const unsigned u = __float_as_uint(f + 0.f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
TSM_DEV float key_value(unsigned k) { return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k); }

// Top-k and weights: warp w handles tokens w, w + nwarps, ... (MULTI; else
// the launch has at most 16 tokens and warp w handles token w; lane holds
// experts lane, lane + 32, ...; PER = ceil(E / 32)).  The selection order is
// (selection logit desc, expert index asc): each step takes the largest key
// over the warp, then the smallest index holding it.  Each selected (token,
// expert) also sets the token's bit in the expert's token mask.
template <int PER, bool MULTI>
TSM_DEV void route_topk_t(const RouteParams& p, RouteState& s, int warp, int lane, int nwarps) {
  const bool biased = p.bias && p.bias_mode != 0;
  const bool score_biased = p.bias && p.bias_mode == 1;
  const bool sig = p.score == 2;  // sigmoid scores; the bias is a selection-only correction
  for (int t = warp; t < p.M; t += MULTI ? nwarps : p.M) {
    const float* lgt = s.lg + (size_t)t * s.lgld;
    unsigned key[PER];
    float vsc[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int e = lane + 32 * i;
      const float l = e < p.E ? lgt[e] : -INFINITY;
      const float base = sig ? 1.f / (1.f + expf(-l)) : l;
      const float ls = (e < p.E && biased) ? base + s.bias[e] : base;
      key[i] = e < p.E ? order_key(ls) : 0u;
      vsc[i] = score_biased ? ls : l;
      if (e < p.E) {
        if (p.logits) p.logits[(size_t)t * p.E + e] = l;
        if (p.logits_out) p.logits_out[(size_t)t * p.E + e] = l;
      }
    }
    int selk = 0;  // lane k: the k-th selected expert
    for (int k = 0; k < p.K; ++k) {
      unsigned bk = 0u;
      int be = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < PER; ++i)
        if (key[i] > bk) {  // strict: the lowest index wins among this lane's equal keys
          bk = key[i];
          be = lane + 32 * i;
        }
      const unsigned kmax = __reduce_max_sync(0xffffffffu, bk);
      int bi = (int)__reduce_min_sync(0xffffffffu, bk == kmax && kmax != 0u ? (unsigned)be : 0x7fffffffu);
      if (kmax == 0u || bi >= p.E) {  // no candidate left: only with NaN logits
        if (lane == 0) atomicOr(p.err, ERR_BAD_INDEX);
        bi = 0;
      }
#pragma unroll
      for (int i = 0; i < PER; ++i)
        if (lane + 32 * i == bi) key[i] = 0u;
      if (lane == k) selk = bi;
    }
    const bool act = lane < p.K;
    float wv = 0.f;
    if (sig) {  // weights: the selected sigmoid scores renormalised to sum 1
      const float sk = act ? 1.f / (1.f + expf(-lgt[selk])) : 0.f;
      float den = sk;
      for (int o = 16; o; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
      wv = act ? sk / den * s.pes[selk] : 0.f;
    } else {
      // score logit of the selected expert, recomputed exactly as above
      float sck = -INFINITY;
      if (act) {
        const float l = lgt[selk];
        sck = score_biased ? l + s.bias[selk] : l;
      }
      unsigned mk = act ? order_key(sck) : 0u;
      if (p.score != 0) {
#pragma unroll
        for (int i = 0; i < PER; ++i)
          if (lane + 32 * i < p.E) mk = max(mk, order_key(vsc[i]));
      }
      const float m = key_value(__reduce_max_sync(0xffffffffu, mk));
      float den = 0.f;
      if (p.score == 0) {
        den = act ? expf(sck - m) : 0.f;
      } else {
#pragma unroll
        for (int i = 0; i < PER; ++i)
          if (lane + 32 * i < p.E) den += expf(vsc[i] - m);
      }
      for (int o = 16; o; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
      if (act) wv = expf(sck - m) / den * s.pes[selk];
    }
    if (act) {
      s.idx[t * p.K + lane] = selk;
      s.w[t * p.K + lane] = wv;
      atomicOr(&s.tmask[selk], 1ull << t);
      if (p.idx) p.idx[t * p.K + lane] = selk;
      if (p.w) p.w[t * p.K + lane] = wv;
      if (p.idx_out) p.idx_out[t * p.K + lane] = selk;
      if (p.w_out) p.w_out[t * p.K + lane] = wv;
    }
  }
}

template <bool MULTI>
TSM_DEV void route_topk(const RouteParams& p, RouteState& s, int warp, int lane, int nwarps) {
  if (p.E <= 32)
    route_topk_t<1, MULTI>(p, s, warp, lane, nwarps);
  else if (p.E <= 64)
    route_topk_t<2, MULTI>(p, s, warp, lane, nwarps);
  else if (p.E <= 128)
    route_topk_t<4, MULTI>(p, s, warp, lane, nwarps);
  else
    route_topk_t<8, MULTI>(p, s, warp, lane, nwarps);
}

// Route list: the (token, slot) pairs grouped by expert (touched experts in
// ascending order, tokens ascending), cut into entries of at most 16 routes,
// then the shared expert's entries (all M tokens, 16 per entry).  A token
// selects an expert at most once, so the expert's route count is the
// popcount of its token mask (set by route_topk) and a token's rank among
// them the popcount of the mask's lower bits.  A shared entry's routes are
// M K + its tokens, so every entry's route r of column n is ro + n.  Without
// MULTI the launch has at most 16 tokens: one entry per touched expert.
// Warp 0 counts the routes, lane l holding experts l PER .. l PER + PER - 1
// (PER: the power of two at or above E / 32).  Needs s.tmask cleared
// (route_init_smem) and a CTA barrier after route_topk; ends with one.
template <int PER, bool MULTI>
TSM_DEV void route_list_t(const RouteParams& p, RouteState& s, int warp, int lane, int tid, int nthr) {
  const int MK = p.M * p.K;
  if (warp == 0) {
    int cl[PER], tot = 0, ne = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int e = lane * PER + i;
      cl[i] = e < p.E ? __popcll(s.tmask[e]) : 0;
      tot += cl[i];
      ne += MULTI ? (cl[i] + MAX_TOK - 1) / MAX_TOK : (cl[i] > 0);
    }
    int incl = tot, neincl = ne;
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o), w = __shfl_up_sync(0xffffffffu, neincl, o);
      if (lane >= o) {
        incl += v;
        neincl += w;
      }
    }
    int run = incl - tot, slot = neincl - ne;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int e = lane * PER + i;
      if (e < p.E) {
        s.off[e] = run;
        s.eslot[e] = slot;
        for (int q = 0; q < cl[i]; q += MAX_TOK, ++slot) {
          s.ex[slot] = e;
          s.ro[slot] = run + q;
          s.nc[slot] = min(MAX_TOK, cl[i] - q);
          if (p.meta) {
            p.meta[META_EX + slot] = e;
            p.meta[META_RO + slot] = run + q;
            p.meta[META_NC + slot] = min(MAX_TOK, cl[i] - q);
          }
          if (!MULTI) {
            ++slot;
            break;
          }
        }
        run += cl[i];
      }
    }
    const int nT = __shfl_sync(0xffffffffu, neincl, 31);
    const int nsh = p.has_shared ? (MULTI ? (p.M + MAX_TOK - 1) / MAX_TOK : 1) : 0;
    if (lane < nsh) {
      const int j = nT + lane, n = min(MAX_TOK, p.M - MAX_TOK * lane);
      s.ex[j] = p.E;
      s.ro[j] = MK + MAX_TOK * lane;
      s.nc[j] = n;
      if (p.meta) {
        p.meta[META_EX + j] = p.E;
        p.meta[META_RO + j] = MK + MAX_TOK * lane;
        p.meta[META_NC + j] = n;
      }
    }
    if (lane == 0) {
      s.nT = nT;
      s.nE = nT + nsh;
      if (p.meta) {
        p.meta[META_M] = p.M;
        p.meta[META_NT] = nT;
        p.meta[META_MK] = MK;
        p.meta[META_HAS_SHARED] = p.has_shared;
        p.meta[META_NE] = nT + nsh;
      }
    }
  }
  __syncthreads();
  for (int i = tid; i < MK; i += nthr) {
    const int e = s.idx[i], tk = i / p.K;
    const int rank = __popcll(s.tmask[e] & ((1ull << tk) - 1ull));  // tokens before tk that chose e
    const int pos = s.off[e] + rank;
    s.tok[pos] = tk;
    s.rpos[i] = pos;
    s.rj[pos] = s.eslot[e] + (MULTI ? rank / MAX_TOK : 0);
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
}

template <bool MULTI>
TSM_DEV void route_list(const RouteParams& p, RouteState& s, int warp, int lane, int tid, int nthr) {
  if (p.E <= 32)
    route_list_t<1, MULTI>(p, s, warp, lane, tid, nthr);
  else if (p.E <= 64)
    route_list_t<2, MULTI>(p, s, warp, lane, tid, nthr);
  else if (p.E <= 128)
    route_list_t<4, MULTI>(p, s, warp, lane, tid, nthr);
  else
    route_list_t<8, MULTI>(p, s, warp, lane, tid, nthr);
}

// ---------------------------------------------------------------------------- routing with the whole router
// For a few tokens and a router that fits in shared memory, a CTA can compute
// all logits by itself with four CTA barriers: (1) the |x| max of every
// (token, slice), (2) x (* xscale) as FP16 scaled per (token, slice) as in
// slice_input, and the gate/up operand xh (scaled per token) to global
// memory, (3) warp w computes the items (tile j, slice c) = w, w + nwarps, ...
// -- the slice's units in order, one accumulator -- unscaled into `item`, (4)
// the logits, each the sum of its S items in slice order.  The router must be
// in smem at w.rt and x at w.x (bulk copies issued by the caller, completing
// on s.rbar and s.xbar).  Every CTA that runs it, and route_kernel for the
// same call, gets the same bits.  Leaves the logits in s.lg (= smem + w.lg)
// and the per-token shifts in s.shift; ends with a CTA barrier.
TSM_DEV void route_whole(const RouteParams& p, RouteState& s, uint8_t* smem, const WholeSmem& ws, __half* xh,
                         volatile int* dead, int warp, int lane, int tid, int nthr) {
  const int M = p.M, H = p.H, S = p.S, CS = p.CS, C = p.rg.chunks, T = p.rg.tiles, E = p.E;
  const bool split = p.xscale != nullptr;
  const int ld = slice_ld(CS), halves = split ? 2 : 1, nwarps = nthr / 32;
  const __nv_bfloat16* xr = reinterpret_cast<const __nv_bfloat16*>(smem + ws.x);
  __half* xin = reinterpret_cast<__half*>(smem + ws.xin);
  float* smx = reinterpret_cast<float*>(smem + ws.smx);
  int* ssh = reinterpret_cast<int*>(smem + ws.ssh);
  float* item = reinterpret_cast<float*>(smem + ws.item);
  const uint8_t* rt = smem + ws.rt;
  s.lg = reinterpret_cast<float*>(smem + ws.lg);
  s.lgld = E;
  mbar_wait(&s.xbar, 0, dead, p.err, ERR_TIMEOUT_XSTAGE);
  mbar_wait(&s.rbar, 0, dead, p.err, ERR_TIMEOUT_XSTAGE);
  // (1) slice maxima, one warp per (token, slice)
  for (int q = warp; q < M * S; q += nwarps) {
    const int t = q / S, c = q - t * S, lo = slice_lo(CS, c), n = (slice_hi(CS, C, c) - lo) * 32;
    const __nv_bfloat16* row = xr + (size_t)t * H + lo * 32;
    float m = 0.f;
    for (int k = lane * 8; k < n; k += 256) m = absmax8(p, *reinterpret_cast<const uint4*>(row + k), lo * 32 + k, m);
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) {
      smx[t * S + c] = m;
      ssh[t * S + c] = shift_of_max(m);
    }
  }
  __syncthreads();
  if (tid < M) {
    float m = 0.f;
    for (int c = 0; c < S; ++c) m = fmaxf(m, smx[tid * S + c]);
    s.shift[tid] = shift_of_max(m);
  }
  // (2) router input per (slice, token) and the gate/up operand xh
  for (int i = tid; i < M * (H / 8); i += nthr) {
    const int t = i / (H / 8), k = (i - t * (H / 8)) * 8, c = k / (CS * 32), kk = k - c * CS * 32;
    const uint4 raw = *reinterpret_cast<const uint4*>(xr + (size_t)t * H + k);
    uint4 hx, hh, hl;
    convert8(p, raw, k, pow2f(ssh[t * S + c]), split, hx, hh, hl);
    __half* dst = xin + ((size_t)c * halves * M + t) * ld + kk;
    *reinterpret_cast<uint4*>(dst) = split ? hh : hx;
    if (split) *reinterpret_cast<uint4*>(dst + (size_t)M * ld) = hl;
  }
  if (xh) {
    __syncthreads();  // s.shift
    for (int i = tid; i < M * (H / 8); i += nthr) {
      const int t = i / (H / 8), k = (i - t * (H / 8)) * 8;
      const uint4 raw = *reinterpret_cast<const uint4*>(xr + (size_t)t * H + k);
      uint4 hx, hh, hl;
      convert8(p, raw, k, pow2f(s.shift[t]), false, hx, hh, hl);
      *reinterpret_cast<uint4*>(xh + (size_t)t * p.Hp + k) = hx;
    }
  }
  __syncthreads();
  // (3) items: warp w takes (tile j, slice c) pairs w, w + nwarps, ...; the
  // slice's units in order into one accumulator, unscaled per token
  for (int q = warp; q < T * S; q += nwarps) {
    const int j = q / S, c = q - j * S, lo = slice_lo(CS, c), nck = slice_hi(CS, C, c) - lo;
    const __half* xc = xin + (size_t)c * halves * M * ld;
    float acc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
    for (int u = 0; u < nck; ++u) {
      const uint8_t* un = rt + ((size_t)j * C + lo + u) * UNIT_BYTES;
      const uint4 qw = *reinterpret_cast<const uint4*>(un + lane * 16);
      const uint32_t sc = *reinterpret_cast<const uint32_t*>(un + QUANT_BYTES + (lane >> 2) * 4);
      for (int h = 0; h < halves; ++h) {
        if (M > 8)
          router_unit<2>(acc, qw, sc, xc + (size_t)h * M * ld + u * 32, ld, M, lane);
        else
          router_unit<1>(reinterpret_cast<float(&)[1][4]>(acc[0]), qw, sc, xc + (size_t)h * M * ld + u * 32, ld, M,
                         lane);
      }
    }
    const int gq = lane >> 2, cq = lane & 3;
    float* it = item + (size_t)q * 16 * M;  // [row][token]
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int t = nt * 8 + 2 * cq + hh;
        if (t < M) {
          const float sc = pow2f(-ssh[t * S + c]);
          it[gq * M + t] = acc[nt][hh] * sc;
          it[(gq + 8) * M + t] = acc[nt][2 + hh] * sc;
        }
      }
  }
  __syncthreads();
  // (4) logits: each the sum of its items in slice order
  for (int i = tid; i < M * E; i += nthr) {
    const int t = i / E, e = i - t * E, j = e >> 4, r = e & 15;
    float v = 0.f;
    for (int c = 0; c < S; ++c) v += item[((size_t)(j * S + c) * 16 + r) * M + t];
    s.lg[i] = v;
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------- standalone route kernel
constexpr int ROUTE_THREADS = ROUTE_WARPS * 32;

// End of a route_kernel run with p.sentinel set: if this call's error word or
// the earlier kernel's word (p.pre_err) holds any bit, every (token, slot) of
// idx_out / w_out becomes -1 / 0, so a failed call cannot pass for a routing.
// Needs a CTA barrier after every write of idx_out / w_out and every error bit.
TSM_DEV void route_sentinel(const RouteParams& p, int tid) {
  __shared__ unsigned bad;
  if (tid == 0) bad = *reinterpret_cast<volatile unsigned*>(p.err) | (p.pre_err ? *p.pre_err : 0u);
  __syncthreads();
  if (!bad) return;
  for (int i = tid; i < p.M * p.K; i += ROUTE_THREADS) {
    if (p.idx_out) p.idx_out[i] = -1;
    if (p.w_out) p.w_out[i] = 0.f;
  }
}

// One CTA: the items (j, c) in slice order, each slice's x staged by bulk copy,
// router units read from global memory; logits accumulated in slice order.
// Dynamic shared memory: RouteState, then the slice buffers (SliceSmem).
__global__ void __launch_bounds__(ROUTE_THREADS, 1) route_kernel(const RouteParams p) {
  extern __shared__ __align__(128) uint8_t route_smem_raw[];
  RouteState& s = *reinterpret_cast<RouteState*>(route_smem_raw);
  uint8_t* sbuf = route_smem_raw + align128(sizeof(RouteState));
  if (p.whole) {
    // the whole-router algorithm, exactly as the layer kernel runs it
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const WholeSmem ws(p.M, p.H, p.rg.tiles, p.rg.chunks, p.S, p.CS, p.E, p.xscale != nullptr);
    const RouteConst rc = route_const_load(p, tid);
    if (tid == 0) {
      mbar_init(&s.xbar, 1);
      mbar_init(&s.rbar, 1);
      fence_barrier_init();
      s.xdead = 0;
      const unsigned rbytes = (unsigned)p.rg.tiles * p.rg.chunks * UNIT_BYTES;
      mbar_arrive_expect_tx(&s.rbar, rbytes);
      bulk_g2s(sbuf + ws.rt, p.rw, rbytes, &s.rbar);
    }
    grid_dep_wait();
    grid_dep_launch();
    if (tid == 0) {
      const unsigned xbytes = (unsigned)p.M * p.H * 2;
      mbar_arrive_expect_tx(&s.xbar, xbytes);
      bulk_g2s(sbuf + ws.x, p.x, xbytes, &s.xbar);
    }
    if (tid < p.E && !(isfinite(rc.b) && isfinite(rc.s))) atomicOr(p.err, ERR_BAD_ROUTER_INPUT);
    route_init_smem(s, rc, tid);
    __syncthreads();
    route_whole(p, s, sbuf, ws, nullptr, &s.xdead, warp, lane, tid, ROUTE_THREADS);
    if (tid < p.M && p.shift) p.shift[tid] = s.shift[tid];
    route_topk<false>(p, s, warp, lane, ROUTE_WARPS);
    __syncthreads();
    route_list<false>(p, s, warp, lane, tid, ROUTE_THREADS);
    if (p.sentinel) route_sentinel(p, tid);
    return;
  }
  const SliceSmem L(p.M, p.CS, p.xscale != nullptr);
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(sbuf + L.xs);
  __half* xin = reinterpret_cast<__half*>(sbuf + L.xin);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const RouteConst rc = route_const_load(p, tid);
  s.lg = reinterpret_cast<float*>(sbuf + align128(L.total));  // [M][E]
  s.lgld = p.E;
  if (tid == 0) {
    mbar_init(&s.xbar, 1);
    fence_barrier_init();
    s.xdead = 0;
  }
  grid_dep_wait();
  grid_dep_launch();
  if (tid == 0) slice_issue_x(p, s, 0, xs);
  // the bias and per-expert scale are device inputs here: a non-finite one is an error of the call
  if (tid < p.E && !(isfinite(rc.b) && isfinite(rc.s))) atomicOr(p.err, ERR_BAD_ROUTER_INPUT);
  route_init_smem(s, rc, tid);
  for (int i = tid; i < p.M * p.E; i += ROUTE_THREADS) s.lg[i] = 0.f;
  if (tid < MAX_TOK) s.gmax[tid] = 0.f;
  __syncthreads();
  for (int c = 0; c < p.S; ++c) {
    mbar_wait(&s.xbar, c & 1, &s.xdead, p.err, ERR_TIMEOUT_XSTAGE);
    slice_max(p, s, c, xs, warp, lane);
    __syncthreads();
    slice_input(p, s, c, xs, xin, tid, ROUTE_THREADS);
    if (tid < p.M) s.gmax[tid] = fmaxf(s.gmax[tid], s.smax[tid]);
    fence_proxy_async_smem();  // xs is rewritten by the next slice's bulk copies
    __syncthreads();
    if (tid == 0 && c + 1 < p.S) slice_issue_x(p, s, c + 1, xs);
    for (int j = 0; j < p.rg.tiles; ++j) {
      const uint8_t* units = p.rw + ((size_t)j * p.rg.chunks + slice_lo(p.CS, c)) * UNIT_BYTES;
      if (p.M > 8)
        slice_gemv<2>(p, s, j, c, xin, units, warp, lane, tid, ROUTE_THREADS, nullptr);
      else
        slice_gemv<1>(p, s, j, c, xin, units, warp, lane, tid, ROUTE_THREADS, nullptr);
    }
  }
  if (tid < p.M) {
    s.shift[tid] = shift_of_max(s.gmax[tid]);
    if (p.shift) p.shift[tid] = s.shift[tid];
  }
  __syncthreads();
  route_topk<false>(p, s, warp, lane, ROUTE_WARPS);
  __syncthreads();
  route_list<false>(p, s, warp, lane, tid, ROUTE_THREADS);
  if (p.sentinel) route_sentinel(p, tid);
}

}  // namespace tsm
