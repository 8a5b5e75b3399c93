// C-ABI library: open-time validation, device allocation and repack; per-call
// launch of the route kernel and the two expert kernels on the caller's
// stream with programmatic dependent launch (each kernel's prologue overlaps
// the previous kernel's tail; griddepcontrol.wait orders the data).
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/ts_moe.h"
#include "../../include/ts_moe_debug.h"
#include "common.cuh"
#include "expert.cuh"
#include "layout.cuh"
#include "repack.cuh"
#include "route.cuh"

using namespace tsm;

namespace {

thread_local std::string g_open_error;

struct LayerDev {
  uint8_t* rw = nullptr;   // router, repacked Q8_0 fragment tiles
  float* bias = nullptr;
  float* pes = nullptr;
  float* xscale = nullptr;
  bool has_xscale = false; // some router x-scale differs from 1
  uint8_t* wB = nullptr;   // routed gate/up, E matrices
  uint8_t* wC = nullptr;   // routed down
  uint8_t* wBs = nullptr;  // shared gate/up
  uint8_t* wCs = nullptr;  // shared down
};

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Bytes of one user row of `cols` weights: 32-element blocks of 34 (Q8_0), 17 (MXFP4) or 20 (INT4-affine) bytes.
size_t blob_row_bytes(int fmt, int cols) {
  return (size_t)(cols / 32) * (fmt == TS_FMT_Q8_0 ? 34 : fmt == TS_FMT_MXFP4 ? 17 : 20);
}

}  // namespace

struct ts_moe {
  ts_moe_config cfg{};
  int sm_count = 0, nb = 0;
  int slices[MAX_TOK + 1] = {};  // router slices per token count (calls of at most 16 tokens)
  int lt = 0;                    // tokens per layer-kernel launch: 64, or 16 when no slicing fits four blocks
  int s_chunk = 0;               // router slices of every launch of a call with more than 16 tokens
  int Hp = 0, Ip = 0, Sp = 0;
  MatGeom gR{}, gB{}, gC{}, gBs{}, gCs{};
  int ng_max_B = 0;
  bool any_xscale = false;
  uint8_t* arena = nullptr;
  size_t arena_bytes = 0;
  uint8_t* ws = nullptr;
  size_t ws_bytes = 0;
  std::vector<LayerDev> layers;
  // workspace views
  float* logits = nullptr;
  int* idx = nullptr;
  float* w = nullptr;
  int* rpos = nullptr;
  int* shift = nullptr;
  int* meta = nullptr;
  Route* routes = nullptr;
  __half* xh = nullptr;         // layer kernel: FP16 x, the gate/up B operand
  float* part_pub = nullptr;    // layer kernel: router items [MAX_SLICES][Mmax][item_ld(E)]
  float* max_pub = nullptr;     // layer kernel: slice |x| maxima [MAX_SLICES][MAX_TOK]
  __half* acts = nullptr;
  __half* acts_sh = nullptr;
  float* P = nullptr;
  float* partial0 = nullptr;
  float* partial1 = nullptr;
  unsigned* entry_done = nullptr;
  unsigned* cnt_gB = nullptr;   // gate/up: per (expert, group, consumer warp) chunk counters
  unsigned long long* arrivals = nullptr;  // grid barrier arrivals (64-bit, never reset while the handle lives)
  unsigned* grid = nullptr;     // {x slices written, router items published}
  unsigned* part_all = nullptr;  // decode launches' range tables for 1 .. part_nmax routed entries, computed at open
  int part_nmax = 0;
  bool debug_skip_arrival = false;
  unsigned* err = nullptr;
  size_t counters_bytes = 0;
  uint8_t* counters = nullptr;
  cudaEvent_t ev[4] = {nullptr, nullptr, nullptr, nullptr};
  bool timing = false;
  std::string error;
  uint64_t expert_bytes = 0, router_bytes = 0, shared_bytes = 0;
};

namespace {

ts_moe_status fail(ts_moe* h, ts_moe_status st, const std::string& msg) {
  if (h)
    h->error = msg;
  else
    g_open_error = msg;
  return st;
}

ts_moe_status cuda_fail(ts_moe* h, cudaError_t e, const char* what) {
  return fail(h, TS_MOE_ECUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

#define TSM_CUDA(h, call)                                     \
  do {                                                        \
    cudaError_t e_ = (call);                                  \
    if (e_ != cudaSuccess) return cuda_fail((h), e_, #call);  \
  } while (0)

// Host-side validation: everything that can be refused before device memory exists.
ts_moe_status validate(const ts_moe_config* c, const ts_moe_layer_weights* L) {
  if (!c) return fail(nullptr, TS_MOE_EINVAL, "config is NULL");
  if (c->abi_version != TS_MOE_ABI_VERSION) return fail(nullptr, TS_MOE_EINVAL, "abi_version mismatch");
  auto bad = [&](const std::string& m) { return fail(nullptr, TS_MOE_EINVAL, m); };
  auto uns = [&](const std::string& m) { return fail(nullptr, TS_MOE_EUNSUPPORTED, m); };
  if (c->hidden <= 0 || c->hidden % 32) return bad("hidden must be a positive multiple of 32 (whole Q8_0/MXFP4 blocks)");
  if (c->hidden > 16384) return uns("hidden > 16384 is not supported");
  if (c->moe_inter <= 0 || c->moe_inter % 32) return bad("moe_inter must be a positive multiple of 32");
  if (c->moe_inter > 65536) return uns("moe_inter > 65536 is not supported");
  if (c->num_experts < 1 || c->num_experts > TS_MOE_MAX_EXPERTS) return bad("num_experts must be in [1, 256]");
  if (c->top_k < 1 || c->top_k > TS_MOE_MAX_TOPK || c->top_k > c->num_experts)
    return bad("top_k must be in [1, min(8, num_experts)] (the 8-slot phase-2 reduce)");
  if (c->num_layers < 1 || c->num_layers > 1024) return bad("num_layers must be in [1, 1024]");
  if (c->max_tokens < 1 || c->max_tokens > TS_MOE_MAX_PREFILL) return bad("max_tokens must be in [1, 65536]");
  if (c->expert_fmt != TS_FMT_Q8_0 && c->expert_fmt != TS_FMT_MXFP4 && c->expert_fmt != TS_FMT_INT4_AFFINE)
    return bad("unknown expert_fmt");
  if (c->score != TS_SCORE_SOFTMAX_SELECTED && c->score != TS_SCORE_SOFTMAX_ALL_NORENORM &&
      c->score != TS_SCORE_SIGMOID_RENORM)
    return bad("unknown score");
  if (c->score == TS_SCORE_SIGMOID_RENORM && c->bias_mode == TS_BIAS_LOGITS)
    return bad("sigmoid scoring takes its correction bias as TS_BIAS_SELECT_ONLY");
  if (c->bias_mode < TS_BIAS_NONE || c->bias_mode > TS_BIAS_SELECT_ONLY) return bad("unknown bias_mode");
  if (c->act != TS_ACT_SWIGLU && c->act != TS_ACT_SWIGLU_CLAMPED) return bad("unknown act");
  if (c->act == TS_ACT_SWIGLU_CLAMPED &&
      (!std::isfinite(c->act_alpha) || !std::isfinite(c->act_limit) || c->act_limit <= 0.f))
    return bad("clamped SwiGLU needs a finite alpha and a finite limit > 0");
  if (c->shared_inter < 0 || c->shared_inter % 32) return bad("shared_inter must be 0 or a multiple of 32");
  if (c->shared_inter > 65536) return uns("shared_inter > 65536 is not supported");
  if (c->shared_inter > 0 && c->expert_fmt != TS_FMT_Q8_0)
    return uns("a shared expert is only supported with Q8_0 routed experts (no family on the pages mixes them)");
  if (c->weights_mem != TS_MEM_HOST && c->weights_mem != TS_MEM_DEVICE) return bad("unknown weights_mem");
  if (c->device < 0) return bad("device must be >= 0");
  if (!L) return bad("layers is NULL");
  for (int l = 0; l < c->num_layers; ++l) {
    const ts_moe_layer_weights& w = L[l];
    const std::string at = " (layer " + std::to_string(l) + ")";
    if (!w.router || !w.gate || !w.up || !w.down) return bad("router/gate/up/down must be non-NULL" + at);
    if ((c->bias_mode != TS_BIAS_NONE) != (w.router_bias != nullptr))
      return bad("router_bias must be given iff bias_mode != NONE" + at);
    if (w.router_bias)
      for (int e = 0; e < c->num_experts; ++e)
        if (!std::isfinite(w.router_bias[e])) return bad("non-finite router bias" + at);
    if (w.per_expert_scale)
      for (int e = 0; e < c->num_experts; ++e)
        if (!std::isfinite(w.per_expert_scale[e])) return bad("non-finite per_expert_scale" + at);
    if (w.router_xscale)
      for (int n = 0; n < c->hidden; ++n)
        if ((w.router_xscale[n] & 0x7F80u) == 0x7F80u) return bad("non-finite router_xscale" + at);
    const bool sh = w.sh_gate || w.sh_up || w.sh_down;
    if (c->shared_inter > 0 && !(w.sh_gate && w.sh_up && w.sh_down))
      return bad("shared_inter > 0 needs sh_gate, sh_up and sh_down" + at);
    if (c->shared_inter == 0 && sh) return bad("shared expert blobs given with shared_inter == 0" + at);
  }
  return TS_MOE_OK;
}

// Dynamic shared memory of route_kernel: RouteState, one item's slice buffers, the logits.
constexpr int ROUTE_SMEM_MAX = 220 * 1024;
size_t route_smem(const RouteParams& rp) {
  if (rp.whole)
    return align128(sizeof(RouteState)) +
           WholeSmem(rp.M, rp.H, rp.rg.tiles, rp.rg.chunks, rp.S, rp.CS, rp.E, rp.xscale != nullptr).total;
  return align128(sizeof(RouteState)) + align128(SliceSmem(rp.M, rp.CS, rp.xscale != nullptr).total) +
         (size_t)rp.M * rp.E * 4;
}

// Router slices for a launch of `ml` tokens cut into `ntb` routing blocks of
// at most M tokens: the count S (CS = ceil(C / S) chunks each) that balances
// the bytes a routing CTA loads (its block's x slice and CS router units)
// against the bytes every CTA reads back (S items of ml x E logits), with the
// T * S * ntb routing CTAs within the grid and one item's buffers plus the
// launch's logits within the layer kernel's weight and window rings.
// Returns 0 when no S fits.
constexpr size_t RING_BYTES = sizeof(LayerSmem::w) + sizeof(LayerSmem::x);
int choose_slices(int M, int C, int T, int E, int nb, bool split, int ntb, int ml) {
  int best = 0;
  double best_cost = 0.0;
  const int smax = std::min({C, MAX_SLICES, nb / std::max(T * ntb, 1)});
  for (int S = 1; S <= smax; ++S) {
    const int CS = (C + S - 1) / S;
    if ((C + CS - 1) / CS != S) continue;  // S must be the slice count CS gives
    if (align128(SliceSmem(M, CS, split).total) + (size_t)ml * E * 4 > RING_BYTES) continue;
    const double load = (double)M * CS * 64 + (double)CS * UNIT_BYTES;
    const double read = (double)S * (ml * item_ld(E) + MAX_LT) * 4;
    const double cost = std::max(load, read);
    if (best == 0 || cost < best_cost) {
      best = S;
      best_cost = cost;
    }
  }
  return best;
}

// Calls of at most WHOLE_MAX_M tokens whose router and routing buffers fit in
// the rings route with the whole router in every CTA (route_whole): S and CS
// give every warp of a CTA about one (tile, slice) item.  Both the handle path
// and the allocation-free entry point decide here.
#ifndef TSM_WHOLE_MAX_M
#define TSM_WHOLE_MAX_M 1
#endif
constexpr int WHOLE_MAX_M = TSM_WHOLE_MAX_M;
bool whole_slicing(int M, const MatGeom& gR, int E, int H, bool split, int& S, int& CS) {
  if (M > WHOLE_MAX_M) return false;
  const int C = gR.chunks, T = gR.tiles;
  int s = std::max(1, std::min(C, (ROUTE_WARPS + T - 1) / T));
  CS = (C + s - 1) / s;
  S = (C + CS - 1) / CS;
  const size_t need = WholeSmem(M, H, T, C, S, CS, E, split).total;
  return need <= RING_BYTES && align128(sizeof(RouteState)) + need <= (size_t)ROUTE_SMEM_MAX;
}

// CTAs of one layer-kernel launch on a device with `sm_count` SMs: one per SM.
int layer_ctas(int sm_count) { return std::min(sm_count, MAX_NB); }

// Router slicing (count S and chunks per slice CS) for M tokens.  The handle
// path and the allocation-free entry point both take it from here, so that for
// the same router and SM count both sum a logit's partial products in the same
// order (the allocation-free path matches a handle opened without an x-scale).
bool router_slicing(int M, const MatGeom& gR, int E, int nb, bool split, int& S, int& CS) {
  const int s = choose_slices(M, gR.chunks, gR.tiles, E, nb, split, 1, M);
  if (s == 0) return false;
  CS = (gR.chunks + s - 1) / s;
  S = (gR.chunks + CS - 1) / CS;
  return true;
}

// The layer kernel's grid barrier and readiness waits need all `nb` CTAs
// resident at once.  With `per_sm` CTAs of it fitting on one SM (from the
// occupancy calculator) and `sm_count` SMs, that holds on an otherwise idle
// device iff per_sm >= 1 and nb <= per_sm * sm_count.
bool coresident(int per_sm, int sm_count, int nb) { return per_sm >= 1 && (long long)nb <= (long long)per_sm * sm_count; }

// The layer-kernel instance of a forward launch: prefill (more than 16
// tokens); decode of one token routed with the whole router; decode of at
// most 8 tokens (every entry one n8 tile); decode of 9 to 16 tokens routed
// with router items; or any other decode launch.
template <int FMT>
void (*layer_instance(const RouteParams& rp))(LayerParams) {
  if (rp.M > MAX_TOK) return layer_kernel<FMT, true>;
  if (rp.whole && rp.M == 1) return layer_kernel<FMT, false, false, 2>;
  if (rp.M <= 8) return layer_kernel<FMT, false, false, 1>;
  if (!rp.whole && rp.M > 8) return layer_kernel<FMT, false, false, 3>;
  return layer_kernel<FMT, false>;
}

template <int FMT>
cudaError_t set_narrow_smem(int bytes) {
  const auto a = cudaFuncAttributeMaxDynamicSharedMemorySize;
  cudaError_t e = cudaFuncSetAttribute(layer_kernel<FMT, false, false, 1>, a, bytes);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(layer_kernel<FMT, false, false, 2>, a, bytes);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(layer_kernel<FMT, false, false, 3>, a, bytes);
  return e;
}

template <typename... Args>
cudaError_t launch_pdl(void (*k)(Args...), int grid, int block, size_t smem, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(grid);
  lc.blockDim = dim3(block);
  lc.dynamicSmemBytes = smem;
  lc.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  return cudaLaunchKernelEx(&lc, k, args...);
}

ts_moe_status set_smem_attrs(ts_moe* h) {
  const int bytes = (int)sizeof(LayerSmem);
  TSM_CUDA(h, cudaFuncSetAttribute(layer_kernel<0, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  TSM_CUDA(h, cudaFuncSetAttribute(layer_kernel<1, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  TSM_CUDA(h, cudaFuncSetAttribute(layer_kernel<2, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  TSM_CUDA(h, cudaFuncSetAttribute(layer_kernel<0, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  TSM_CUDA(h, cudaFuncSetAttribute(layer_kernel<1, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  TSM_CUDA(h, cudaFuncSetAttribute(layer_kernel<2, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  TSM_CUDA(h, set_narrow_smem<0>(bytes));
  TSM_CUDA(h, set_narrow_smem<1>(bytes));
  TSM_CUDA(h, set_narrow_smem<2>(bytes));
  TSM_CUDA(h, cudaFuncSetAttribute(layer_kernel<0, false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  TSM_CUDA(h, cudaFuncSetAttribute(layer_kernel<0, true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  return TS_MOE_OK;
}

template <int PHASE>
void launch_repack(int fmt, const uint8_t* a, const uint8_t* b, int row_bytes, int nblocks, const MatGeom& g,
                   uint8_t* dst, unsigned* bad, cudaStream_t st, int nrows) {
  const long long units = (long long)g.tiles * g.chunks;
  const int threads = 256;
  const long long blocks = std::min<long long>((units + 7) / 8, 65535LL * 8);
  if (fmt == TS_FMT_MXFP4)
    repack_kernel<1, PHASE><<<(int)std::max<long long>(1, blocks), threads, 0, st>>>(a, b, row_bytes, nblocks, g.tiles,
                                                                                      g.chunks, g.gs, dst, bad, nrows);
  else if (fmt == TS_FMT_INT4_AFFINE)
    repack_kernel<2, PHASE><<<(int)std::max<long long>(1, blocks), threads, 0, st>>>(a, b, row_bytes, nblocks, g.tiles,
                                                                                      g.chunks, g.gs, dst, bad, nrows);
  else
    repack_kernel<0, PHASE><<<(int)std::max<long long>(1, blocks), threads, 0, st>>>(a, b, row_bytes, nblocks, g.tiles,
                                                                                      g.chunks, g.gs, dst, bad, nrows);
}

}  // namespace

extern "C" {

ts_moe_status ts_moe_open(const ts_moe_config* cfg, const ts_moe_layer_weights* layers, ts_moe** out) {
  if (!out) return fail(nullptr, TS_MOE_EINVAL, "out is NULL");
  *out = nullptr;
  ts_moe_status st = validate(cfg, layers);
  if (st != TS_MOE_OK) return st;

  int ndev = 0;
  cudaError_t ce = cudaGetDeviceCount(&ndev);
  if (ce != cudaSuccess || ndev == 0)
    return fail(nullptr, TS_MOE_ECUDA, std::string("no CUDA device: ") + cudaGetErrorString(ce));
  if (cfg->device >= ndev) return fail(nullptr, TS_MOE_EINVAL, "device ordinal out of range");
  ce = cudaSetDevice(cfg->device);
  if (ce != cudaSuccess) return fail(nullptr, TS_MOE_ECUDA, std::string("cudaSetDevice: ") + cudaGetErrorString(ce));
  cudaDeviceProp prop;
  ce = cudaGetDeviceProperties(&prop, cfg->device);
  if (ce != cudaSuccess) return fail(nullptr, TS_MOE_ECUDA, cudaGetErrorString(ce));
  if (prop.major != 10)
    return fail(nullptr, TS_MOE_EUNSUPPORTED, "the kernels are built for sm_100a (B200); this device is sm_" +
                                                  std::to_string(prop.major) + std::to_string(prop.minor));

  ts_moe* h = new ts_moe();
  h->cfg = *cfg;
  const ts_moe_config& c = h->cfg;
  const int H = c.hidden, I = c.moe_inter, E = c.num_experts, K = c.top_k, S = c.shared_inter;
  // Calls above 16 tokens run in launches of up to 64 tokens (four routing
  // blocks) when a router slicing fits that, else of 16; the workspace holds
  // one launch's tokens.
  h->nb = layer_ctas(prop.multiProcessorCount);
  h->gR = make_router_geom(E, H);
  for (int l = 0; l < c.num_layers && !h->any_xscale; ++l)
    if (layers[l].router_xscale)
      for (int n = 0; n < H; ++n)
        if (layers[l].router_xscale[n] != 0x3F80u) {
          h->any_xscale = true;
          break;
        }
  h->s_chunk = choose_slices(MAX_TOK, h->gR.chunks, h->gR.tiles, E, h->nb, h->any_xscale, MAX_LT / MAX_TOK, MAX_LT);
  h->lt = h->s_chunk ? MAX_LT : MAX_TOK;
  if (!h->s_chunk) h->s_chunk = choose_slices(MAX_TOK, h->gR.chunks, h->gR.tiles, E, h->nb, h->any_xscale, 1, MAX_TOK);
  const int Mx = std::min(c.max_tokens, h->lt);
  const int fmt = c.expert_fmt;
  h->sm_count = prop.multiProcessorCount;
  h->Hp = round_up(H, 64);
  h->Ip = round_up(I, 64);
  h->Sp = S ? round_up(S, 64) : 0;
  h->gB = make_geom(I / 8, H, fmt);
  h->gC = make_geom(H / 16, I, fmt);
  if (S) {
    h->gBs = make_geom(S / 8, H, TS_FMT_Q8_0);
    h->gCs = make_geom(H / 16, S, TS_FMT_Q8_0);
  }
  h->ng_max_B = std::max(h->gB.ngroups, S ? h->gBs.ngroups : 0);
  if (c.max_tokens > MAX_TOK && h->s_chunk == 0) {
    g_open_error = "no router slicing fits these sizes (too many experts for the SM count, or hidden too large)";
    ts_moe_close(h);
    return TS_MOE_EUNSUPPORTED;
  }
  for (int m = 1; m <= std::min(Mx, MAX_TOK); ++m) {
    int S_m = 0, CS_m = 0;
    h->slices[m] = router_slicing(m, h->gR, E, h->nb, h->any_xscale, S_m, CS_m) ? S_m : 0;
    if (h->slices[m] == 0) {
      g_open_error = "no router slicing fits these sizes (too many experts for the SM count, or hidden too large)";
      ts_moe_close(h);
      return TS_MOE_EUNSUPPORTED;
    }
  }
  h->expert_bytes = 2ull * I * blob_row_bytes(fmt, H) + (uint64_t)H * blob_row_bytes(fmt, I);
  h->router_bytes = (uint64_t)E * blob_row_bytes(TS_FMT_Q8_0, H);
  h->shared_bytes = S ? 2ull * S * blob_row_bytes(TS_FMT_Q8_0, H) + (uint64_t)H * blob_row_bytes(TS_FMT_Q8_0, S) : 0;

  auto cleanup = [&](ts_moe_status s2) {
    ts_moe_close(h);
    return s2;
  };

  // ---- arena
  size_t per_layer = 0;
  per_layer += align256(h->gR.bytes);             // router
  per_layer += align256((size_t)E * 4) * 2;        // bias, pes
  per_layer += align256((size_t)H * 4);            // xscale
  per_layer += align256(h->gB.bytes * E);
  per_layer += align256(h->gC.bytes * E);
  if (S) per_layer += align256(h->gBs.bytes) + align256(h->gCs.bytes);
  h->arena_bytes = per_layer * c.num_layers;
  ce = cudaMalloc(&h->arena, h->arena_bytes);
  if (ce != cudaSuccess) {
    g_open_error = "arena allocation of " + std::to_string(h->arena_bytes) + " bytes failed";
    ts_moe_close(h);
    return TS_MOE_ENOMEM;
  }
  h->layers.resize(c.num_layers);
  {
    uint8_t* p = h->arena;
    auto take = [&](size_t n) {
      uint8_t* r = p;
      p += align256(n);
      return r;
    };
    for (int l = 0; l < c.num_layers; ++l) {
      LayerDev& d = h->layers[l];
      d.rw = take(h->gR.bytes);
      d.bias = (float*)take((size_t)E * 4);
      d.pes = (float*)take((size_t)E * 4);
      d.xscale = (float*)take((size_t)H * 4);
      d.wB = take(h->gB.bytes * E);
      d.wC = take(h->gC.bytes * E);
      if (S) {
        d.wBs = take(h->gBs.bytes);
        d.wCs = take(h->gCs.bytes);
      }
    }
  }

  // ---- workspace (sized once for max_tokens; the calls allocate nothing)
  {
    size_t off = 0;
    auto slot = [&](size_t n) {
      size_t r = off;
      off += align256(n);
      return r;
    };
    const size_t o_logits = slot((size_t)Mx * E * 4);
    const size_t o_idx = slot((size_t)Mx * K * 4);
    const size_t o_w = slot((size_t)Mx * K * 4);
    const size_t o_rpos = slot((size_t)Mx * K * 4);
    const size_t o_shift = slot((size_t)Mx * 4);
    const size_t o_meta = slot((size_t)META_INTS * 4);
    const size_t o_routes = slot((size_t)Mx * K * sizeof(Route));
    const size_t o_xh = slot((size_t)Mx * h->Hp * 2);
    const size_t o_part = slot((size_t)MAX_SLICES * Mx * item_ld(E) * 4);
    const size_t o_max = slot((size_t)MAX_SLICES * MAX_LT * 4);
    const size_t o_acts = slot((size_t)Mx * K * h->Ip * 2);
    const size_t o_acts_sh = slot((size_t)Mx * std::max(h->Sp, 64) * 2);
    const size_t o_P = slot((size_t)(Mx * K + Mx) * H * 4);
    const size_t o_part0 = slot((size_t)h->nb * 2 * SLOT_FLOATS * 4);
    const size_t o_part1 = slot((size_t)h->nb * 2 * SLOT_FLOATS * 4);
    h->part_nmax = std::min(E, MAX_TOK * K);  // routed entries of a decode launch
    const size_t o_tab = slot((size_t)h->part_nmax * 2 * part_stride(h->nb) * 4);
    const size_t o_cnt = off;
    const size_t n_cnt = 2 + (size_t)MAX_ENTRIES * h->ng_max_B * NWC + MAX_ENTRIES + 2 + 1;  // arrivals (u64) + ... + grid[2] + error word
    slot(n_cnt * 4);
    h->ws_bytes = off;
    ce = cudaMalloc(&h->ws, h->ws_bytes);
    if (ce != cudaSuccess) {
      g_open_error = "workspace allocation failed";
      ts_moe_close(h);
      return TS_MOE_ENOMEM;
    }
    h->logits = (float*)(h->ws + o_logits);
    h->idx = (int*)(h->ws + o_idx);
    h->w = (float*)(h->ws + o_w);
    h->rpos = (int*)(h->ws + o_rpos);
    h->shift = (int*)(h->ws + o_shift);
    h->meta = (int*)(h->ws + o_meta);
    h->routes = (Route*)(h->ws + o_routes);
    h->xh = (__half*)(h->ws + o_xh);
    h->part_pub = (float*)(h->ws + o_part);
    h->max_pub = (float*)(h->ws + o_max);
    h->acts = (__half*)(h->ws + o_acts);
    h->acts_sh = (__half*)(h->ws + o_acts_sh);
    h->P = (float*)(h->ws + o_P);
    h->partial0 = (float*)(h->ws + o_part0);
    h->partial1 = (float*)(h->ws + o_part1);
    h->part_all = (unsigned*)(h->ws + o_tab);
    unsigned* cn = (unsigned*)(h->ws + o_cnt);
    h->counters = (uint8_t*)cn;
    h->counters_bytes = n_cnt * 4;
    h->arrivals = (unsigned long long*)cn;  // 256-byte aligned: first in the counter block
    h->cnt_gB = cn + 2;
    h->entry_done = h->cnt_gB + (size_t)MAX_ENTRIES * h->ng_max_B * NWC;
    h->grid = h->entry_done + MAX_ENTRIES;  // x slices written, router items published
    h->err = h->grid + 2;
    // zeros: counters, error word, and the padding columns of x / acts
    ce = cudaMemset(h->ws, 0, h->ws_bytes);
    if (ce != cudaSuccess) {
      g_open_error = std::string("workspace memset: ") + cudaGetErrorString(ce);
      return cleanup(TS_MOE_ECUDA);
    }
  }
  if ((st = set_smem_attrs(h)) != TS_MOE_OK) {
    g_open_error = h->error;
    return cleanup(st);
  }
  {
    // a decode launch's unit-equal range tables depend only on the geometry and
    // its count of routed entries: computed once here for every count
    LayerParams lp;
    std::memset(&lp, 0, sizeof(lp));
    lp.gB = h->gB;
    lp.gBs = h->gBs;
    lp.gC = h->gC;
    lp.gCs = h->gCs;
    lp.rp.has_shared = c.shared_inter > 0;
    partition_table_kernel<<<h->part_nmax, 256>>>(lp, lp.rp.has_shared ? 1 : 0, h->nb, part_stride(h->nb), h->part_all);
    ce = cudaGetLastError();
    if (ce == cudaSuccess) ce = cudaStreamSynchronize(nullptr);
    if (ce != cudaSuccess) {
      g_open_error = std::string("partition tables: ") + cudaGetErrorString(ce);
      return cleanup(TS_MOE_ECUDA);
    }
  }
  {
    // every CTA of a layer launch must be resident at once (grid barrier)
    int per_sm = 0;
    ce = fmt == TS_FMT_MXFP4
             ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, layer_kernel<1, false>, NTHREADS, sizeof(LayerSmem))
         : fmt == TS_FMT_INT4_AFFINE
             ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, layer_kernel<2, false>, NTHREADS, sizeof(LayerSmem))
             : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, layer_kernel<0, false>, NTHREADS, sizeof(LayerSmem));
    if (ce != cudaSuccess) {
      g_open_error = std::string("occupancy query: ") + cudaGetErrorString(ce);
      return cleanup(TS_MOE_ECUDA);
    }
    if (!coresident(per_sm, h->sm_count, h->nb)) {
      g_open_error = "the layer kernel's " + std::to_string(h->nb) + " CTAs cannot all be resident at once (" +
                     std::to_string(per_sm) + " per SM on " + std::to_string(h->sm_count) + " SMs)";
      return cleanup(TS_MOE_EUNSUPPORTED);
    }
  }

  // ---- upload + repack every layer
  unsigned* d_bad = nullptr;
  uint8_t* stage = nullptr;
  size_t stage_bytes = 0;
  const size_t gate_bytes = (size_t)E * I * blob_row_bytes(fmt, H);
  const size_t down_bytes = (size_t)E * H * blob_row_bytes(fmt, I);
  const size_t router_b = (size_t)E * blob_row_bytes(TS_FMT_Q8_0, H);
  const size_t shg = S ? (size_t)S * blob_row_bytes(TS_FMT_Q8_0, H) : 0;
  const size_t shd = S ? (size_t)H * blob_row_bytes(TS_FMT_Q8_0, S) : 0;
  ce = cudaMalloc(&d_bad, 4);
  if (ce == cudaSuccess) ce = cudaMemset(d_bad, 0, 4);
  if (ce == cudaSuccess && c.weights_mem == TS_MEM_HOST) {
    stage_bytes = std::max({2 * gate_bytes, down_bytes, router_b, 2 * shg, shd});
    ce = cudaMalloc(&stage, stage_bytes);
  }
  if (ce != cudaSuccess) {
    g_open_error = std::string("repack staging: ") + cudaGetErrorString(ce);
    cudaFree(d_bad);
    cudaFree(stage);
    ts_moe_close(h);
    return TS_MOE_ENOMEM;
  }
  cudaStream_t st0 = 0;
  std::vector<float> ones((size_t)std::max(H, E), 1.0f);
  std::vector<float> tmp((size_t)std::max(H, E));
  for (int l = 0; l < c.num_layers && ce == cudaSuccess; ++l) {
    const ts_moe_layer_weights& w = layers[l];
    LayerDev& d = h->layers[l];
    auto src = [&](const void* p, size_t bytes, size_t at) -> const uint8_t* {
      if (c.weights_mem == TS_MEM_DEVICE) return (const uint8_t*)p;
      if (ce == cudaSuccess) ce = cudaMemcpy(stage + at, p, bytes, cudaMemcpyHostToDevice);
      return stage + at;
    };
    // router + small vectors
    const uint8_t* r = src(w.router, router_b, 0);
    if (ce != cudaSuccess) break;
    launch_repack<1>(TS_FMT_Q8_0, r, nullptr, (int)blob_row_bytes(TS_FMT_Q8_0, H), H / 32, h->gR, d.rw, d_bad, st0, E);
    if (ce == cudaSuccess) ce = cudaStreamSynchronize(nullptr);  // the staging buffer is reused next
    if (w.router_bias && ce == cudaSuccess) ce = cudaMemcpy(d.bias, w.router_bias, E * 4, cudaMemcpyHostToDevice);
    if (ce == cudaSuccess)
      ce = cudaMemcpy(d.pes, w.per_expert_scale ? w.per_expert_scale : ones.data(), E * 4, cudaMemcpyHostToDevice);
    if (w.router_xscale) {
      for (int n = 0; n < H; ++n) {
        uint32_t u = (uint32_t)w.router_xscale[n] << 16;
        std::memcpy(&tmp[n], &u, 4);
        if (tmp[n] != 1.0f) d.has_xscale = true;
      }
    } else {
      std::fill(tmp.begin(), tmp.begin() + H, 1.0f);
    }
    if (ce == cudaSuccess) ce = cudaMemcpy(d.xscale, tmp.data(), (size_t)H * 4, cudaMemcpyHostToDevice);
    // gate/up -> phase-1 layout, per expert
    const uint8_t* gsrc = src(w.gate, gate_bytes, 0);
    const uint8_t* usrc = src(w.up, gate_bytes, gate_bytes);
    if (ce != cudaSuccess) break;
    const int rbH = (int)blob_row_bytes(fmt, H), rbI = (int)blob_row_bytes(fmt, I);
    for (int e = 0; e < E; ++e)
      launch_repack<0>(fmt, gsrc + (size_t)e * I * rbH, usrc + (size_t)e * I * rbH, rbH, H / 32, h->gB,
                       d.wB + (size_t)e * h->gB.bytes, d_bad, st0, I);
    ce = cudaDeviceSynchronize();
    if (ce != cudaSuccess) break;
    const uint8_t* dsrc = src(w.down, down_bytes, 0);
    if (ce != cudaSuccess) break;
    for (int e = 0; e < E; ++e)
      launch_repack<1>(fmt, dsrc + (size_t)e * H * rbI, nullptr, rbI, I / 32, h->gC, d.wC + (size_t)e * h->gC.bytes,
                       d_bad, st0, H);
    ce = cudaDeviceSynchronize();
    if (ce != cudaSuccess) break;
    if (S) {
      const int rbHq = (int)blob_row_bytes(TS_FMT_Q8_0, H), rbS = (int)blob_row_bytes(TS_FMT_Q8_0, S);
      const uint8_t* sg = src(w.sh_gate, shg, 0);
      const uint8_t* su = src(w.sh_up, shg, shg);
      if (ce != cudaSuccess) break;
      launch_repack<0>(TS_FMT_Q8_0, sg, su, rbHq, H / 32, h->gBs, d.wBs, d_bad, st0, S);
      ce = cudaDeviceSynchronize();
      if (ce != cudaSuccess) break;
      const uint8_t* sd = src(w.sh_down, shd, 0);
      if (ce != cudaSuccess) break;
      launch_repack<1>(TS_FMT_Q8_0, sd, nullptr, rbS, S / 32, h->gCs, d.wCs, d_bad, st0, H);
      ce = cudaDeviceSynchronize();
    }
  }
  unsigned bad = 0;
  if (ce == cudaSuccess) ce = cudaMemcpy(&bad, d_bad, 4, cudaMemcpyDeviceToHost);
  cudaFree(d_bad);
  cudaFree(stage);
  if (ce != cudaSuccess) {
    g_open_error = std::string("repack: ") + cudaGetErrorString(ce);
    ts_moe_close(h);
    return TS_MOE_ECUDA;
  }
  if (bad) {
    g_open_error = std::string("refused at open: ") + ((bad & BAD_E8M0_NAN) ? "MXFP4 block scale e8m0 = 255 (NaN); " : "") +
                   ((bad & BAD_Q8_SCALE) ? "non-finite Q8_0 block scale; " : "") +
                   ((bad & BAD_I4_SCALE) ? "non-finite INT4-affine block scale or offset; " : "") +
                   ((bad & BAD_ROUTER_SCALE) ? "non-finite router block scale; " : "");
    ts_moe_close(h);
    return TS_MOE_EINVAL;
  }
  *out = h;
  return TS_MOE_OK;
}

// A launch of M tokens within a call of call_m tokens: calls of at most 16
// tokens take the slicing chosen for their M, every launch of a longer call
// the one chosen for chunks, so that ts_moe_route and ts_moe_forward on the
// same call sum each logit's partial products in the same order.
static RouteParams route_params(ts_moe* h, int layer, const void* x, int M, int call_m) {
  const ts_moe_config& c = h->cfg;
  const LayerDev& d = h->layers[layer];
  RouteParams rp;
  std::memset(&rp, 0, sizeof(rp));
  rp.x = (const __nv_bfloat16*)x;
  rp.M = M;
  rp.H = c.hidden;
  rp.Hp = h->Hp;
  rp.E = c.num_experts;
  rp.K = c.top_k;
  rp.rw = d.rw;
  rp.rg = h->gR;
  rp.xscale = d.has_xscale ? d.xscale : nullptr;
  rp.bias = c.bias_mode != TS_BIAS_NONE ? d.bias : nullptr;
  rp.pes = d.pes;
  rp.bias_mode = c.bias_mode;
  rp.score = c.score;
  rp.has_shared = c.shared_inter > 0;
  rp.logits = h->logits;
  rp.idx = h->idx;
  rp.w = h->w;
  rp.shift = h->shift;
  if (call_m > MAX_TOK) {
    rp.CS = (h->gR.chunks + h->s_chunk - 1) / h->s_chunk;
    rp.S = (h->gR.chunks + rp.CS - 1) / rp.CS;
  } else if (whole_slicing(M, h->gR, rp.E, rp.H, h->any_xscale, rp.S, rp.CS)) {
    rp.whole = 1;
  } else {
    router_slicing(M, h->gR, rp.E, h->nb, h->any_xscale, rp.S, rp.CS);  // fits: checked at open
  }
  rp.meta = h->meta;
  rp.routes = h->routes;
  rp.rpos = h->rpos;
  rp.err = h->err;
  return rp;
}

static ts_moe_status check_call(ts_moe* h, int layer, const void* x, int M) {
  if (!h) return TS_MOE_EINVAL;
  if (layer < 0 || layer >= h->cfg.num_layers) return fail(h, TS_MOE_EINVAL, "layer out of range");
  if (M < 0 || M > h->cfg.max_tokens) return fail(h, TS_MOE_EINVAL, "M out of range [0, max_tokens]");
  if (M > 0 && !x) return fail(h, TS_MOE_EINVAL, "x is NULL");
  if (((uintptr_t)x & 15) != 0) return fail(h, TS_MOE_EINVAL, "x must be 16-byte aligned");
  return TS_MOE_OK;
}

// A call of M tokens runs as launches over consecutive row blocks, full ones
// first: ts_moe_forward and ts_moe_route in launches of h->lt (64) tokens,
// each forward launch reading every touched expert's weights once per 16
// routes.  Tokens are independent in the routed half, so the chunking changes
// no token's route (the chunked-prefill driver of the gpt-oss state page,
// `BatchedRoutedScratch`, feeds the routed half MAX_PREFILL_BATCH = 16 rows
// at a time; here a launch takes up to four such blocks).
static inline int chunk_rows(int M, int m0, int n) { return std::min(n, M - m0); }

// The launch parameters of a layer, without the per-launch routing and outputs.
static LayerParams layer_params(ts_moe* h, int layer) {
  const ts_moe_config& c = h->cfg;
  const LayerDev& d = h->layers[layer];
  LayerParams lp;
  std::memset(&lp, 0, sizeof(lp));
  lp.xh = h->xh;
  lp.part_pub = h->part_pub;
  lp.max_pub = h->max_pub;
  lp.wB = d.wB;
  lp.wB_stride = h->gB.bytes;
  lp.wBs = d.wBs;
  lp.wC = d.wC;
  lp.wC_stride = h->gC.bytes;
  lp.wCs = d.wCs;
  lp.gB = h->gB;
  lp.gBs = h->gBs;
  lp.gC = h->gC;
  lp.gCs = h->gCs;
  lp.acts = h->acts;
  lp.acts_sh = h->acts_sh;
  lp.Ip = h->Ip;
  lp.Sp = h->Sp;
  lp.P = h->P;
  lp.partial0 = h->partial0;
  lp.partial1 = h->partial1;
  lp.cnt_group = h->cnt_gB;
  lp.ng_max = h->ng_max_B;
  lp.entry_done = h->entry_done;
  lp.grid_cnt = h->arrivals;
  lp.xh_cnt = h->grid;
  lp.route_cnt = h->grid + 1;
  lp.err = h->err;
  lp.act = c.act;
  lp.alpha = c.act_alpha;
  lp.limit = c.act_limit;
  return lp;
}

// ts_moe_route runs the routing of ts_moe_forward's launches alone (the same
// launches, so every token's logits, experts and weights are the forward's).
ts_moe_status ts_moe_route(ts_moe* h, int layer, const void* x, int M, int32_t* idx, float* w, float* logits,
                           void* stream) {
  ts_moe_status s = check_call(h, layer, x, M);
  if (s != TS_MOE_OK) return s;
  if (M == 0) return TS_MOE_OK;
  if (!idx || !w) return fail(h, TS_MOE_EINVAL, "idx and w must be non-NULL");
  const int H = h->cfg.hidden, E = h->cfg.num_experts, K = h->cfg.top_k;
  LayerParams lp = layer_params(h, layer);
  for (int m0 = 0; m0 < M; m0 += h->lt) {
    lp.rp = route_params(h, layer, (const __nv_bfloat16*)x + (size_t)m0 * H, chunk_rows(M, m0, h->lt), M);
    lp.rp.idx_out = idx + (size_t)m0 * K;
    lp.rp.w_out = w + (size_t)m0 * K;
    lp.rp.logits_out = logits ? logits + (size_t)m0 * E : nullptr;
    const cudaError_t e = launch_pdl(lp.rp.M > MAX_TOK ? layer_kernel<0, true, true> : layer_kernel<0, false, true>,
                                     h->nb, NTHREADS, sizeof(LayerSmem), (cudaStream_t)stream, lp);
    if (e != cudaSuccess) return cuda_fail(h, e, "routing launch");
  }
  return TS_MOE_OK;
}

ts_moe_status ts_moe_forward(ts_moe* h, int layer, const void* x, int M, void* resid, float* y, void* stream) {
  ts_moe_status s = check_call(h, layer, x, M);
  if (s != TS_MOE_OK) return s;
  if (!resid && !y) return fail(h, TS_MOE_EINVAL, "resid and y are both NULL");
  if (M == 0) return TS_MOE_OK;
  cudaStream_t st = (cudaStream_t)stream;
  const ts_moe_config& c = h->cfg;
  LayerParams lp = layer_params(h, layer);
  lp.debug_skip_arrival = h->debug_skip_arrival ? 1 : 0;
  h->debug_skip_arrival = false;  // the next forward launch only
  const size_t smem = sizeof(LayerSmem);
  const int H = c.hidden;
  if (h->timing) cudaEventRecord(h->ev[0], st);
  for (int m0 = 0; m0 < M; m0 += h->lt) {
    lp.rp = route_params(h, layer, (const __nv_bfloat16*)x + (size_t)m0 * H, chunk_rows(M, m0, h->lt), M);
    lp.y = y ? y + (size_t)m0 * H : nullptr;
    lp.resid = resid ? (__nv_bfloat16*)resid + (size_t)m0 * H : nullptr;
    lp.part_all = lp.rp.M <= MAX_TOK ? h->part_all : nullptr;  // decode launches
    lp.part_nmax = h->part_nmax;
    cudaError_t e;
    if (c.expert_fmt == TS_FMT_MXFP4)
      e = launch_pdl(layer_instance<1>(lp.rp), h->nb, NTHREADS, smem, st, lp);
    else if (c.expert_fmt == TS_FMT_INT4_AFFINE)
      e = launch_pdl(layer_instance<2>(lp.rp), h->nb, NTHREADS, smem, st, lp);
    else
      e = launch_pdl(layer_instance<0>(lp.rp), h->nb, NTHREADS, smem, st, lp);
    if (e != cudaSuccess) return cuda_fail(h, e, "layer kernel launch");
  }
  if (h->timing) cudaEventRecord(h->ev[1], st);
  return TS_MOE_OK;
}

ts_moe_status ts_moe_device_status(ts_moe* h, void* stream) {
  if (!h) return TS_MOE_EINVAL;
  TSM_CUDA(h, cudaSetDevice(h->cfg.device));
  TSM_CUDA(h, cudaStreamSynchronize((cudaStream_t)stream));
  unsigned err = 0;
  TSM_CUDA(h, cudaMemcpy(&err, h->err, 4, cudaMemcpyDeviceToHost));
  if (!err) return TS_MOE_OK;
  TSM_CUDA(h, cudaMemset(h->counters, 0, h->counters_bytes));
  char buf[768];
  std::snprintf(buf, sizeof buf, "device error word 0x%x (bit0/1: weight-stage wait gave up, bit2/3: activation-window "
                "wait gave up, bit4: bad index, bit5: bad route metadata, bit6: grid barrier wait gave up, bit7: "
                "wait for an expert's activations gave up, bit8: wait for the staged x gave up, bit9: wait for the "
                "shared FP16 x gave up, bit10: wait for the router logits gave up, bit11: non-finite router bias or per-expert scale, bit12: wait for the precomputed range tables gave up)", err);
  return fail(h, TS_MOE_EDEVICE, buf);
}

ts_moe_status ts_moe_get_info(const ts_moe* h, ts_moe_info* info) {
  if (!h || !info) return TS_MOE_EINVAL;
  info->arena_bytes = h->arena_bytes;
  info->workspace_bytes = h->ws_bytes;
  info->expert_bytes = h->expert_bytes;
  info->router_bytes = h->router_bytes;
  info->shared_bytes = h->shared_bytes;
  info->num_ctas = h->nb;
  info->sm_count = h->sm_count;
  info->launch_tokens = h->lt;
  return TS_MOE_OK;
}

ts_moe_status ts_moe_set_timing_events(ts_moe* h, void* const* events4) {
  if (!h) return TS_MOE_EINVAL;
  if (!events4) {
    h->timing = false;
    return TS_MOE_OK;
  }
  for (int i = 0; i < 4; ++i) {
    if (!events4[i]) return fail(h, TS_MOE_EINVAL, "timing events must be non-NULL");
    h->ev[i] = (cudaEvent_t)events4[i];
  }
  h->timing = true;
  return TS_MOE_OK;
}

const char* ts_moe_last_error(const ts_moe* h) { return h ? h->error.c_str() : g_open_error.c_str(); }

ts_moe_status ts_moe_close(ts_moe* h) {
  if (!h) return TS_MOE_OK;
  cudaSetDevice(h->cfg.device);
  if (h->arena) cudaFree(h->arena);
  if (h->ws) cudaFree(h->ws);
  delete h;
  return TS_MOE_OK;
}

// ----------------------------------------------------------------------------- routing without allocation
// Scratch for ts_moe_route_noalloc: a file-scope device array.  Host code must
// not use the symbol itself as a device pointer (on the host it names a
// host-side stand-in); the device address is looked up once per device.
static __device__ __align__(256) uint8_t g_noalloc_scratch[TS_MOE_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int NOALLOC_MAX_DEVICES = 64;
std::mutex g_noalloc_mu;
uint8_t* g_noalloc_ptr[NOALLOC_MAX_DEVICES] = {};

// Once per device, with that device current: the array's device address and
// the route kernel's shared-memory attribute.
ts_moe_status noalloc_setup(int dev, uint8_t** out) {
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* ptr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return fail(nullptr, TS_MOE_ECUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
    e = cudaFuncSetAttribute(route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, ROUTE_SMEM_MAX);
    if (e != cudaSuccess) return fail(nullptr, TS_MOE_ECUDA, std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e));
    g_noalloc_ptr[dev] = (uint8_t*)ptr;
  }
  *out = g_noalloc_ptr[dev];
  return TS_MOE_OK;
}
}  // namespace

ts_moe_status ts_moe_route_noalloc(const void* router, const float* router_bias, const float* per_expert_scale, int E,
                                   int H, int K, int score, int bias_mode, const void* x, int M, int32_t* idx,
                                   float* w, float* logits, void* stream) {
  if (E < 1 || E > TS_MOE_MAX_EXPERTS) return fail(nullptr, TS_MOE_EINVAL, "num_experts must be in [1, 256]");
  if (K < 1 || K > TS_MOE_MAX_TOPK || K > E) return fail(nullptr, TS_MOE_EINVAL, "top_k must be in [1, min(8, E)]");
  if (H <= 0 || H % 32 || H > 16384) return fail(nullptr, TS_MOE_EINVAL, "hidden must be a positive multiple of 32, <= 16384");
  if (M < 0 || M > TS_MOE_MAX_TOKENS) return fail(nullptr, TS_MOE_EINVAL, "M must be in [0, 16]");
  if (score != TS_SCORE_SOFTMAX_SELECTED && score != TS_SCORE_SOFTMAX_ALL_NORENORM && score != TS_SCORE_SIGMOID_RENORM)
    return fail(nullptr, TS_MOE_EINVAL, "unknown score");
  if (score == TS_SCORE_SIGMOID_RENORM && bias_mode == TS_BIAS_LOGITS)
    return fail(nullptr, TS_MOE_EINVAL, "sigmoid scoring takes its correction bias as TS_BIAS_SELECT_ONLY");
  if (bias_mode < TS_BIAS_NONE || bias_mode > TS_BIAS_SELECT_ONLY) return fail(nullptr, TS_MOE_EINVAL, "unknown bias_mode");
  if ((bias_mode != TS_BIAS_NONE) != (router_bias != nullptr))
    return fail(nullptr, TS_MOE_EINVAL, "router_bias must be given iff bias_mode != NONE");
  if (M == 0) return TS_MOE_OK;
  if (!router || !x || !idx || !w) return fail(nullptr, TS_MOE_EINVAL, "router, x, idx and w must be non-NULL");
  if (((uintptr_t)x & 15) != 0) return fail(nullptr, TS_MOE_EINVAL, "x must be 16-byte aligned");

  // scratch layout: repacked router | logits | idx | w | shift | meta | routes | rpos | error word
  const MatGeom gR = make_router_geom(E, H);
  const int Hp = round_up(H, 64);
  size_t off = 0;
  auto take = [&](size_t n) {
    const size_t r = off;
    off += align256(n);
    return r;
  };
  const size_t o_rw = take(gR.bytes), o_lg = take((size_t)M * E * 4),
               o_idx = take((size_t)M * K * 4), o_w = take((size_t)M * K * 4), o_sh = take((size_t)M * 4),
               o_meta = take((size_t)META_INTS * 4), o_rt = take((size_t)M * K * sizeof(Route)),
               o_rpos = take((size_t)M * K * 4), o_err = take(8);
  if (off > TS_MOE_NOALLOC_SCRATCH_BYTES)
    return fail(nullptr, TS_MOE_EINVAL, "routing needs " + std::to_string(off) + " bytes of scratch, more than the " +
                                            std::to_string(TS_MOE_NOALLOC_SCRATCH_BYTES) + " this entry point has");
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(nullptr, TS_MOE_ECUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= NOALLOC_MAX_DEVICES) return fail(nullptr, TS_MOE_EUNSUPPORTED, "device ordinal >= 64");
  uint8_t* sc = nullptr;
  ts_moe_status st = noalloc_setup(dev, &sc);
  if (st != TS_MOE_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;

  unsigned* errw = (unsigned*)(sc + o_err);  // the error and repack words must start at zero
  e = cudaMemsetAsync(errw, 0, 8, s);
  if (e != cudaSuccess) return fail(nullptr, TS_MOE_ECUDA, std::string("cudaMemsetAsync: ") + cudaGetErrorString(e));
  launch_repack<1>(TS_FMT_Q8_0, (const uint8_t*)router, nullptr, (int)blob_row_bytes(TS_FMT_Q8_0, H), H / 32, gR,
                   sc + o_rw, errw + 1, s, E);
  e = cudaGetLastError();
  if (e != cudaSuccess) return fail(nullptr, TS_MOE_ECUDA, std::string("router repack launch: ") + cudaGetErrorString(e));

  RouteParams rp;
  std::memset(&rp, 0, sizeof(rp));
  rp.x = (const __nv_bfloat16*)x;
  rp.M = M;
  rp.H = H;
  rp.Hp = Hp;
  rp.E = E;
  rp.K = K;
  rp.rw = sc + o_rw;
  rp.rg = gR;
  rp.xscale = nullptr;
  rp.bias = bias_mode != TS_BIAS_NONE ? router_bias : nullptr;
  rp.pes = per_expert_scale;
  rp.bias_mode = bias_mode;
  rp.score = score;
  rp.has_shared = 0;
  rp.logits = (float*)(sc + o_lg);
  rp.idx = (int*)(sc + o_idx);
  rp.w = (float*)(sc + o_w);
  rp.shift = (int*)(sc + o_sh);
  rp.meta = (int*)(sc + o_meta);
  rp.routes = (Route*)(sc + o_rt);
  rp.rpos = (int*)(sc + o_rpos);
  rp.err = errw;
  rp.idx_out = idx;
  rp.w_out = w;
  rp.logits_out = logits;
  rp.pre_err = errw + 1;  // the repack's bad-scale word
  rp.sentinel = 1;
  int nsm = 0;
  e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return fail(nullptr, TS_MOE_ECUDA, std::string("cudaDeviceGetAttribute: ") + cudaGetErrorString(e));
  if (whole_slicing(M, gR, E, H, false, rp.S, rp.CS))
    rp.whole = 1;
  else if (!router_slicing(M, gR, E, layer_ctas(nsm), false, rp.S, rp.CS))
    return fail(nullptr, TS_MOE_EUNSUPPORTED, "no router slicing fits these sizes");
  e = launch_pdl(route_kernel, 1, ROUTE_THREADS, route_smem(rp), s, rp);
  if (e != cudaSuccess) return fail(nullptr, TS_MOE_ECUDA, std::string("route_kernel launch: ") + cudaGetErrorString(e));
  return TS_MOE_OK;
}

// ----------------------------------------------------------------------------- debug helpers (host-only arithmetic; one failure-path test hook)
uint64_t ts_moe_debug_range_start(uint64_t U, int NB, int b) { return range_start(U, NB, b); }
int ts_moe_debug_owner_of(uint64_t U, int NB, uint64_t u) { return owner_of(U, NB, u); }
int ts_moe_debug_partial_slot(uint64_t U, int NB, int b, uint64_t g0) { return partial_slot(U, NB, b, g0); }
int ts_moe_debug_group_size(int tiles) { return pick_group_size(tiles); }
uint64_t ts_moe_debug_aligned_start(int G, int NB, int chunks, int b) {
  if (b >= NB) return (uint64_t)G * chunks;
  return (uint64_t)aligned_group_of(b, G, NB) * chunks + aligned_offset(b, G, NB, chunks);
}
int ts_moe_debug_use_aligned(int G, int NB) { return use_aligned(G, NB) ? 1 : 0; }
int ts_moe_debug_coresident(int per_sm, int sm_count, int nb) { return coresident(per_sm, sm_count, nb) ? 1 : 0; }
int ts_moe_debug_layer_ctas(int sm_count) { return layer_ctas(sm_count); }
ts_moe_status ts_moe_debug_skew_barrier(ts_moe* h, void* stream) {
  if (!h) return TS_MOE_EINVAL;
  TSM_CUDA(h, cudaSetDevice(h->cfg.device));
  TSM_CUDA(h, cudaStreamSynchronize((cudaStream_t)stream));
  h->debug_skip_arrival = true;  // the next launch's CTA 0 does not arrive: only NB - 1 of NB arrivals come
  return TS_MOE_OK;
}

ts_moe_status ts_moe_debug_validate(const ts_moe_config* cfg, const ts_moe_layer_weights* layers) {
  return validate(cfg, layers);
}

}  // extern "C"
