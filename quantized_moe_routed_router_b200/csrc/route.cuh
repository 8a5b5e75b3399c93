// Route kernel: router GEMV -> (bias) -> top-k + weights -> route list.
//
// One CTA per token.  The router GEMV reads the Q8_0 router rows (int8 plane
// + FP32 block scales, repacked at open) against x * router_xscale in FP32
// (llama state page, `router_ones`: the INT8 router kernel scales x[n] per
// element; `router_logits_f32`: one FP32 row of logits per token).  One warp
// then selects the top K by (selection logit desc, index asc), where the
// selection logit is l + b when a router bias is present (gpt-oss state page,
// `router_bias`: added BEFORE the top-k), and forms the weights:
//   softmax over the selected ("selection reduces to softmax over the
//   selected", `per_expert_ones`), or the full softmax over all experts taken
//   at the selected indices without renormalisation (deepseek2 layer sketch),
// times the per-expert scale.  The reference does this part on the host after
// reading the logits back; here it never leaves the device.
//
// The last CTA to finish (one atomic counter, no waiting) groups the M*K
// (token, slot) pairs by expert into the route list the expert kernels walk:
// per touched expert its first route and count, routes sorted by (expert,
// token) -- each expert's weights are then streamed once per micro-batch.
// The pages' route list is a host-written 16-byte record per route
// (gpt-oss state page, `batch_routes`); ours is built on the device.
//
// Each CTA also writes its token's x as FP16 scaled by a power of two
// 2^shift (|x| max lands in [2^13, 2^14)), the B operand of the gate/up
// tensor-core MMA; the shift is undone exactly in that kernel's epilogue.
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

// meta[] layout (int32), written by the route kernel's last CTA.
enum { META_M = 0, META_NT = 1, META_MK = 2, META_HAS_SHARED = 3, META_NE = 4, META_EX = 8,
       META_RO = META_EX + MAX_ENTRIES, META_NC = META_RO + MAX_ENTRIES, META_INTS = META_NC + MAX_ENTRIES };

struct RouteParams {
  const __nv_bfloat16* x;  // [M][H]
  int M, H, Hp, E, K;
  const int8_t* rq;        // [E][H] router quants
  const float* rd;         // [E][H/32] router block scales
  const float* xscale;     // [H] or null
  const float* bias;       // [E] or null
  const float* pes;        // [E] or null
  int bias_mode, score, has_shared;
  float* logits;           // [M][E] workspace
  int* idx;                // [M][K] workspace
  float* w;                // [M][K] workspace
  int* shift;              // [M]
  __half* xh;              // [M][Hp]
  int* meta;
  Route* routes;           // [M*K]
  int* rpos;               // [M][K] -> position in routes
  unsigned* cnt;
  unsigned* err;
  int* idx_out;            // optional user outputs
  float* w_out;
  float* logits_out;
};

TSM_DEV bool topk_better(float v1, int i1, float v2, int i2) { return v1 > v2 || (v1 == v2 && i1 < i2); }

constexpr int ROUTE_THREADS = 256;

__global__ void __launch_bounds__(ROUTE_THREADS) route_kernel(const RouteParams p) {
  extern __shared__ float rsm[];
  float* xs = rsm;          // [H] router input x * xscale
  float* lg = rsm + p.H;    // [E] logits
  __shared__ float red[ROUTE_THREADS / 32];
  __shared__ int s_last;
  __shared__ int s_cnt[MAX_E], s_off[MAX_E], s_idx[MAX_TOK * MAX_K];

  grid_dep_wait();
  grid_dep_launch();

  const int t = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const __nv_bfloat16* xr = p.x + (size_t)t * p.H;

  // ---- x: router input, |x| max
  float amax = 0.f;
  for (int n = tid; n < p.H; n += ROUTE_THREADS) {
    float v = __bfloat162float(xr[n]);
    amax = fmaxf(amax, fabsf(v));
    xs[n] = p.xscale ? v * p.xscale[n] : v;
  }
  for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (lane == 0) red[warp] = amax;
  __syncthreads();
  amax = red[0];
  for (int i = 1; i < ROUTE_THREADS / 32; ++i) amax = fmaxf(amax, red[i]);
  int sh = 0;
  if (amax > 0.f && amax <= 3.4e38f) {
    int e2;
    frexpf(amax, &e2);  // amax in [2^(e2-1), 2^e2)
    sh = min(126, max(-126, 14 - e2));
  }
  const float xsc = __uint_as_float((uint32_t)(sh + 127) << 23);
  __half* xhr = p.xh + (size_t)t * p.Hp;
  for (int n = tid; n < p.Hp; n += ROUTE_THREADS)
    xhr[n] = n < p.H ? __float2half_rn(__bfloat162float(xr[n]) * xsc) : __ushort_as_half(0);
  if (tid == 0) p.shift[t] = sh;
  __syncthreads();

  // ---- router GEMV: warp per expert, lane per 32-block
  const int nb = p.H / 32;
  for (int e = warp; e < p.E; e += ROUTE_THREADS / 32) {
    const int8_t* q = p.rq + (size_t)e * p.H;
    const float* d = p.rd + (size_t)e * nb;
    float acc = 0.f;
    for (int b = lane; b < nb; b += 32) {
      const int4* qv = reinterpret_cast<const int4*>(q + (size_t)b * 32);
      int4 qa = qv[0], qb = qv[1];
      int qw[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
      const float* xb = xs + b * 32;
      float s = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
#pragma unroll
        for (int k = 0; k < 4; ++k) s = fmaf((float)(int8_t)(qw[i] >> (8 * k)), xb[4 * i + k], s);
      }
      acc = fmaf(d[b], s, acc);
    }
    for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) lg[e] = acc;
  }
  __syncthreads();

  // ---- top-k and weights (warp 0; lane holds experts lane, lane+32, ...)
  if (warp == 0) {
    constexpr int PER = MAX_E / 32;
    float vsel[PER], vsc[PER];
    unsigned taken = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int e = lane + 32 * i;
      float l = e < p.E ? lg[e] : -INFINITY;
      float ls = (e < p.E && p.bias && p.bias_mode != 0) ? l + p.bias[e] : l;
      vsel[i] = ls;
      vsc[i] = (p.bias_mode == 1 && p.bias) ? ls : l;
      if (e < p.E && p.logits_out) p.logits_out[(size_t)t * p.E + e] = l;
      if (e < p.E) p.logits[(size_t)t * p.E + e] = l;
    }
    int sel[MAX_K];
    float ssc[MAX_K];
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
        float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (topk_better(ov, oi, bv, bi)) {
          bv = ov;
          bi = oi;
        }
      }
      if (bi < 0 || bi >= p.E) {  // only with NaN logits
        if (lane == 0) atomicOr(p.err, ERR_BAD_INDEX);
        bi = 0;
      }
      sel[k] = bi;
      if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
      // score logit of the chosen expert, from its owner lane
      float mine = 0.f;
#pragma unroll
      for (int i = 0; i < PER; ++i)
        if (i == (bi >> 5)) mine = vsc[i];
      ssc[k] = __shfl_sync(0xffffffffu, mine, bi & 31);
    }
    float wk[MAX_K];
    if (p.score == 0) {
      float m = -INFINITY;
      for (int k = 0; k < p.K; ++k) m = fmaxf(m, ssc[k]);
      float den = 0.f;
      for (int k = 0; k < p.K; ++k) {
        wk[k] = expf(ssc[k] - m);
        den += wk[k];
      }
      for (int k = 0; k < p.K; ++k) wk[k] /= den;
    } else {
      float m = -INFINITY;
#pragma unroll
      for (int i = 0; i < PER; ++i)
        if (lane + 32 * i < p.E) m = fmaxf(m, vsc[i]);
      for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      float den = 0.f;
#pragma unroll
      for (int i = 0; i < PER; ++i)
        if (lane + 32 * i < p.E) den += expf(vsc[i] - m);
      for (int o = 16; o; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
      for (int k = 0; k < p.K; ++k) wk[k] = expf(ssc[k] - m) / den;
    }
    if (lane == 0) {
      for (int k = 0; k < p.K; ++k) {
        const float wv = wk[k] * (p.pes ? p.pes[sel[k]] : 1.f);
        p.idx[t * p.K + k] = sel[k];
        p.w[t * p.K + k] = wv;
        if (p.idx_out) p.idx_out[t * p.K + k] = sel[k];
        if (p.w_out) p.w_out[t * p.K + k] = wv;
      }
    }
  }

  // ---- last CTA builds the route list (no waiting: the other CTAs are done)
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(p.cnt, 1u) == (unsigned)(p.M - 1));
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const int MK = p.M * p.K;
  for (int i = tid; i < MK; i += ROUTE_THREADS) s_idx[i] = ld_cg_i(p.idx + i);
  for (int e = tid; e < p.E; e += ROUTE_THREADS) s_cnt[e] = 0;
  __syncthreads();
  for (int i = tid; i < MK; i += ROUTE_THREADS) {
    int e = s_idx[i];
    if (e < 0 || e >= p.E) {
      atomicOr(p.err, ERR_BAD_INDEX);
      e = s_idx[i] = 0;
    }
    atomicAdd(&s_cnt[e], 1);
  }
  __syncthreads();
  if (tid == 0) {
    int run = 0, nT = 0;
    for (int e = 0; e < p.E; ++e) {
      s_off[e] = run;
      if (s_cnt[e]) {
        p.meta[META_EX + nT] = e;
        p.meta[META_RO + nT] = run;
        p.meta[META_NC + nT] = s_cnt[e];
        ++nT;
      }
      run += s_cnt[e];
    }
    if (p.has_shared) {
      p.meta[META_EX + nT] = p.E;
      p.meta[META_RO + nT] = MK;
      p.meta[META_NC + nT] = p.M;
    }
    p.meta[META_M] = p.M;
    p.meta[META_NT] = nT;
    p.meta[META_MK] = MK;
    p.meta[META_HAS_SHARED] = p.has_shared;
    p.meta[META_NE] = nT + (p.has_shared ? 1 : 0);
    *p.cnt = 0u;
  }
  __syncthreads();
  for (int i = tid; i < MK; i += ROUTE_THREADS) {
    const int e = s_idx[i], tk = i / p.K;
    int rank = 0;
    for (int i2 = 0; i2 < MK; ++i2)
      if (s_idx[i2] == e && i2 / p.K < tk) ++rank;
    const int pos = s_off[e] + rank;
    Route r;
    r.token = tk;
    r.slot = i % p.K;
    r.expert = e;
    r.w = ld_cg(p.w + i);
    p.routes[pos] = r;
    p.rpos[i] = pos;
  }
}

}  // namespace tsm
