// FP64 CPU oracle of the routed (MoE) half of one decoder layer.
//
// TEST INFRASTRUCTURE ONLY.  Nothing in the product (the CUDA library, its
// binding, its kernels) links, includes or calls this file; only the test
// suite, the smoke check and the benchmark's CPU-baseline leg load it.  It
// shares no code, header, table or helper with the CUDA path.
//
// What it computes, step by step, for each token m of a micro-batch (the
// order of the pages; citations are page title + section):
//   1. dequantise a weight row from its block format (Q8_0: fp16 scale times
//      int8; MXFP4: E2M1 code times 2^(e-127); INT4-affine: fp16 scale times
//      a 4-bit code plus an fp16 offset)                       [format defs]
//      INT4-affine is only named by the pages (gpt-oss state page,
//      `BatchedRoutedScratch`: the batched-GEMV seam takes only INT4-affine
//      tensors); its block -- 32
//      weights, fp16 d and m, w = d * q + m with q in [0, 15] -- is this
//      library's reading, matched to the 32-element blocks of the other formats
//   2. router logits  l[e] = sum_n Wr[e,n] * s[n] * x[n]  with s the per-element
//      router x-scale (all ones when absent), stored as FP32 as the pages'
//      `router_logits_f32` buffer is                 [llama state: router_ones,
//                                                     router_logits_f32]
//   3. selection logits l'[e] = l[e] + b[e] (FP32 add) when a router bias is
//      present; the bias joins the logits ahead of top-k  [gpt-oss state:
//                                                        router_bias]
//   4. S = top-K of l' by (value desc, index asc) (sigmoid scoring: of s + b, below)
//   5. weights: softmax over the selected experts (SOFTMAX_WEIGHT, norm_w
//      false: with all per-expert scales 1 the weights are exactly the
//      softmax of the selected logits)                  [llama / gpt-oss state:
//                                                        per_expert_ones]
//      or, for the deepseek2 rule, the full softmax over all experts taken at
//      the selected indices, with no renormalisation  [deepseek2 state, layer
//                                                      sketch: "softmax(f @
//                                                      router) top-6, NO renorm"]
//      or, for sigmoid scoring (the MiniMax flow of the llama state page:
//      `router_scoring_func` "sigmoid" with an FP32 `e_score_correction_bias`
//      per expert), scores s[e] = sigmoid(l[e]); the correction bias moves
//      only the selection, S = top-K of s[e] + b[e]; and the weights are the
//      selected scores renormalised, w_j = s[S_j] / sum_{i in S} s[i]
//      (reading: the pages name the rule and the bias but not the weight
//      formula; this is the plainest one consistent with "the bias only
//      moves the selection")
//      then w_j *= per-expert scale (ones when absent)
//   6. per selected expert j: g = Wg x, u = Wu x, a = act(g, u), y += w_j Wd a
//      act = SwiGLU silu(g)*u, or the clamped SwiGLU of the gpt-oss family
//      (gate <= L, |up| <= L, g*sigmoid(alpha g)*(u+1))    [gpt-oss state
//                                                           header]
//   7. shared expert (deepseek2): y += Wd_s act(Wg_s x, Wu_s x), weight 1
//                                 [deepseek2 state, layer sketch: the
//                                  shared SwiGLU joins the routed sum]
//   8. out = resid + y, also rounded to BF16          [llama state: h2 "added
//                                                     back to the stream"]
// All arithmetic after the FP32 logits buffer is FP64.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

// IEEE binary16 -> double, from the format definition (1 sign, 5 exponent
// bits with bias 15, 10 fraction bits; exponent 0 = subnormal; 31 = inf/nan).
double half_to_double(uint16_t h) {
  int sign = (h >> 15) & 1;
  int ex = (h >> 10) & 31;
  int fr = h & 1023;
  double v;
  if (ex == 0) {
    v = std::ldexp((double)fr, -24);
  } else if (ex == 31) {
    v = fr ? NAN : INFINITY;
  } else {
    v = std::ldexp(1024.0 + fr, ex - 25);
  }
  return sign ? -v : v;
}

// bfloat16 -> double: the upper 16 bits of an IEEE binary32.
double bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return (double)f;
}

// E2M1 (OCP MX): bit 3 sign, bits 2..1 exponent (bias 1), bit 0 mantissa;
// exponent 0 is subnormal (0 or 0.5).
double e2m1_to_double(int code) {
  int sign = (code >> 3) & 1;
  int ex = (code >> 1) & 3;
  int m = code & 1;
  double v = (ex == 0) ? 0.5 * m : std::ldexp(1.0 + 0.5 * m, ex - 1);
  return sign ? -v : v;
}

// E8M0 (OCP MX): 2^(e-127); 255 is NaN.
double e8m0_to_double(int e) { return e == 255 ? NAN : std::ldexp(1.0, e - 127); }

const int FMT_Q8_0 = 0;
const int FMT_MXFP4 = 1;
const int FMT_INT4_AFFINE = 2;

// Bytes of one 32-weight block: Q8_0 {fp16 d; int8 q[32]}, MXFP4 {e8m0 e;
// u8 qs[16]}, INT4-affine {fp16 d; fp16 m; u8 qs[16]}.
size_t block_bytes(int fmt) { return fmt == FMT_Q8_0 ? 34 : fmt == FMT_MXFP4 ? 17 : 20; }

size_t row_bytes(int fmt, int cols) { return (size_t)(cols / 32) * block_bytes(fmt); }

// Dequantise one row of `cols` weights.
void dequant_row(int fmt, const uint8_t* row, int cols, double* out) {
  int nb = cols / 32;
  for (int b = 0; b < nb; ++b) {
    if (fmt == FMT_Q8_0) {
      const uint8_t* blk = row + (size_t)b * 34;
      uint16_t dbits = (uint16_t)(blk[0] | (blk[1] << 8));
      double d = half_to_double(dbits);
      for (int i = 0; i < 32; ++i) out[b * 32 + i] = d * (double)(int8_t)blk[2 + i];
    } else if (fmt == FMT_MXFP4) {
      const uint8_t* blk = row + (size_t)b * 17;
      double s = e8m0_to_double(blk[0]);
      for (int j = 0; j < 16; ++j) {
        out[b * 32 + 2 * j] = s * e2m1_to_double(blk[1 + j] & 15);
        out[b * 32 + 2 * j + 1] = s * e2m1_to_double(blk[1 + j] >> 4);
      }
    } else {
      // INT4-affine: element 2j is the low nibble of qs[j], 2j+1 the high one
      const uint8_t* blk = row + (size_t)b * 20;
      double d = half_to_double((uint16_t)(blk[0] | (blk[1] << 8)));
      double m = half_to_double((uint16_t)(blk[2] | (blk[3] << 8)));
      for (int j = 0; j < 16; ++j) {
        out[b * 32 + 2 * j] = d * (double)(blk[4 + j] & 15) + m;
        out[b * 32 + 2 * j + 1] = d * (double)(blk[4 + j] >> 4) + m;
      }
    }
  }
}

double dot(const double* a, const double* b, int n) {
  double s = 0.0;
  for (int i = 0; i < n; ++i) s += a[i] * b[i];
  return s;
}

double sigmoid(double z) { return 1.0 / (1.0 + std::exp(-z)); }

// double -> bfloat16 bits, one correctly rounded step (nearest, ties to even).
uint16_t double_to_bf16(double v) {
  if (std::isnan(v)) return 0x7FC0;
  float f;
  if (std::isinf(v)) {
    f = (float)v;
  } else if (v == 0.0) {
    f = (float)v;
  } else {
    int e;
    std::frexp(v, &e);                 // |v| in [2^(e-1), 2^e)
    int q = std::max(e, -125) - 8;     // bf16 keeps 8 significant bits; subnormal quantum 2^-133
    double r = std::nearbyint(std::ldexp(v, -q));
    double rv = std::ldexp(r, q);
    if (std::fabs(rv) >= std::ldexp(1.0, 128)) rv = v > 0 ? INFINITY : -INFINITY;
    f = (float)rv;                     // exactly representable
  }
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return (uint16_t)(u >> 16);
}

}  // namespace

extern "C" {

struct oracle_cfg {
  int32_t hidden, moe_inter, num_experts, top_k;
  int32_t expert_fmt, score, bias_mode, act;
  double act_alpha, act_limit;
  int32_t shared_inter;
};

struct oracle_layer {
  const uint8_t* router;          // [E][H] Q8_0
  const uint16_t* router_xscale;  // [H] bf16 bits or NULL (ones)
  const float* router_bias;       // [E] or NULL
  const float* per_expert_scale;  // [E] or NULL (ones)
  const uint8_t* gate;            // [E][I][H] expert_fmt
  const uint8_t* up;              // [E][I][H]
  const uint8_t* down;            // [E][H][I]
  const uint8_t* sh_gate;         // [S][H] Q8_0 or NULL
  const uint8_t* sh_up;           // [S][H]
  const uint8_t* sh_down;         // [H][S]
};

double oracle_half_to_double(uint16_t h) { return half_to_double(h); }
double oracle_bf16_to_double(uint16_t b) { return bf16_to_double(b); }
double oracle_e2m1_to_double(int code) { return e2m1_to_double(code); }
double oracle_e8m0_to_double(int e) { return e8m0_to_double(e); }
uint16_t oracle_double_to_bf16(double v) { return double_to_bf16(v); }

void oracle_dequant(int fmt, const uint8_t* blob, int rows, int cols, double* out) {
  for (int r = 0; r < rows; ++r) dequant_row(fmt, blob + (size_t)r * row_bytes(fmt, cols), cols, out + (size_t)r * cols);
}

// Activation: 0 = SwiGLU silu(g)*u, 1 = clamped SwiGLU of the gpt-oss family.
double oracle_act(int act, double alpha, double limit, double g, double u) {
  if (act == 0) return g * sigmoid(g) * u;
  double gc = std::min(g, limit);
  double uc = std::min(std::max(u, -limit), limit);
  return gc * sigmoid(alpha * gc) * (uc + 1.0);
}

// Step 2: FP32 router logits [M][E].
void oracle_router_logits(const oracle_cfg* c, const oracle_layer* L, const uint16_t* x, int M, float* logits32) {
  const int H = c->hidden, E = c->num_experts;
  std::vector<double> wr(H), xs(H);
  for (int m = 0; m < M; ++m) {
    for (int n = 0; n < H; ++n) {
      double s = L->router_xscale ? bf16_to_double(L->router_xscale[n]) : 1.0;
      xs[n] = s * bf16_to_double(x[(size_t)m * H + n]);
    }
    for (int e = 0; e < E; ++e) {
      dequant_row(FMT_Q8_0, L->router + (size_t)e * row_bytes(FMT_Q8_0, H), H, wr.data());
      logits32[(size_t)m * E + e] = (float)dot(wr.data(), xs.data(), H);
    }
  }
}

// Steps 3-5 for M tokens.  idx/w are [M][K] in slot order (descending
// selection logit, lower index first on ties); lsel [M][E] receives the FP32
// selection logits.  forced (optional [M][K]) replaces step 4's choice.
void oracle_select(const oracle_cfg* c, const float* bias, const float* pes, const float* logits32, int M,
                   const int32_t* forced, int32_t* idx, double* w, float* lsel) {
  const int E = c->num_experts, K = c->top_k;
  std::vector<float> ls(E);
  std::vector<double> sc(E);
  std::vector<int> order(E);
  for (int m = 0; m < M; ++m) {
    const float* l = logits32 + (size_t)m * E;
    for (int e = 0; e < E; ++e) {
      if (c->score == 2) {  // sigmoid scores; the bias only moves the selection
        const double sg = 1.0 / (1.0 + std::exp(-(double)l[e]));
        ls[e] = (bias && c->bias_mode != 0) ? (float)(sg + (double)bias[e]) : (float)sg;
        sc[e] = sg;
      } else {
        ls[e] = (bias && c->bias_mode != 0) ? (float)((double)l[e] + (double)bias[e]) : l[e];
        sc[e] = (c->bias_mode == 1 && bias) ? (double)ls[e] : (double)l[e];
      }
      if (lsel) lsel[(size_t)m * E + e] = ls[e];
    }
    int* sel = idx + (size_t)m * K;
    if (forced) {
      for (int j = 0; j < K; ++j) sel[j] = forced[(size_t)m * K + j];
    } else {
      for (int e = 0; e < E; ++e) order[e] = e;
      std::stable_sort(order.begin(), order.end(), [&](int a, int b) {
        if (ls[a] != ls[b]) return ls[a] > ls[b];
        return a < b;
      });
      for (int j = 0; j < K; ++j) sel[j] = order[j];
    }
    double* wm = w + (size_t)m * K;
    if (c->score == 2) {
      double den = 0.0;
      for (int j = 0; j < K; ++j) den += sc[sel[j]];
      for (int j = 0; j < K; ++j) wm[j] = sc[sel[j]] / den;
    } else if (c->score == 0) {
      double mx = -INFINITY;
      for (int j = 0; j < K; ++j) mx = std::max(mx, sc[sel[j]]);
      double den = 0.0;
      for (int j = 0; j < K; ++j) den += std::exp(sc[sel[j]] - mx);
      for (int j = 0; j < K; ++j) wm[j] = std::exp(sc[sel[j]] - mx) / den;
    } else {
      double mx = -INFINITY;
      for (int e = 0; e < E; ++e) mx = std::max(mx, sc[e]);
      double den = 0.0;
      for (int e = 0; e < E; ++e) den += std::exp(sc[e] - mx);
      for (int j = 0; j < K; ++j) wm[j] = std::exp(sc[sel[j]] - mx) / den;
    }
    for (int j = 0; j < K; ++j) wm[j] *= pes ? (double)pes[sel[j]] : 1.0;
  }
}

// One expert's FFN on one token: returns Wd act(Wg x, Wu x) in `out` [H].
static void expert_ffn(int fmt, int act, double alpha, double limit, const uint8_t* gate, const uint8_t* up,
                       const uint8_t* down, int H, int I, const double* x, double* out) {
  std::vector<double> row(std::max(H, I)), a(I);
  for (int i = 0; i < I; ++i) {
    dequant_row(fmt, gate + (size_t)i * row_bytes(fmt, H), H, row.data());
    double g = dot(row.data(), x, H);
    dequant_row(fmt, up + (size_t)i * row_bytes(fmt, H), H, row.data());
    double u = dot(row.data(), x, H);
    a[i] = oracle_act(act, alpha, limit, g, u);
  }
  for (int h = 0; h < H; ++h) {
    dequant_row(fmt, down + (size_t)h * row_bytes(fmt, I), I, row.data());
    out[h] = dot(row.data(), a.data(), I);
  }
}

static void forward_tokens(const oracle_cfg* c, const oracle_layer* L, const uint16_t* x, const uint16_t* resid,
                           const int32_t* idx, const double* w, int m0, int m1, double* y, double* out,
                           uint16_t* out_bf16) {
  const int H = c->hidden, I = c->moe_inter, K = c->top_k, S = c->shared_inter, fmt = c->expert_fmt;
  const size_t gsz = (size_t)I * row_bytes(fmt, H);
  const size_t dsz = (size_t)H * row_bytes(fmt, I);
  std::vector<double> xv(H), p(H);
  for (int m = m0; m < m1; ++m) {
    for (int n = 0; n < H; ++n) xv[n] = bf16_to_double(x[(size_t)m * H + n]);
    double* ym = y + (size_t)m * H;
    for (int h = 0; h < H; ++h) ym[h] = 0.0;
    for (int j = 0; j < K; ++j) {
      int e = idx[(size_t)m * K + j];
      expert_ffn(fmt, c->act, c->act_alpha, c->act_limit, L->gate + e * gsz, L->up + e * gsz, L->down + e * dsz, H, I,
                 xv.data(), p.data());
      double wj = w[(size_t)m * K + j];
      for (int h = 0; h < H; ++h) ym[h] += wj * p[h];
    }
    if (S > 0 && L->sh_gate) {
      expert_ffn(FMT_Q8_0, c->act, c->act_alpha, c->act_limit, L->sh_gate, L->sh_up, L->sh_down, H, S, xv.data(),
                 p.data());
      for (int h = 0; h < H; ++h) ym[h] += p[h];
    }
    for (int h = 0; h < H; ++h) {
      double r = resid ? bf16_to_double(resid[(size_t)m * H + h]) : 0.0;
      double o = r + ym[h];
      if (out) out[(size_t)m * H + h] = o;
      if (out_bf16) out_bf16[(size_t)m * H + h] = double_to_bf16(o);
    }
  }
}

// The whole routed half for M tokens.  Outputs (each optional except idx/w/y):
//   logits32 [M][E] FP32 router logits; lsel [M][E] FP32 selection logits;
//   idx [M][K]; w [M][K]; y [M][H] routed(+shared) sum; out [M][H] = resid + y;
//   out_bf16 [M][H].  forced [M][K] (optional) fixes the selected experts.
// nthreads > 1 splits the tokens over std::threads (tokens are independent).
int oracle_forward(const oracle_cfg* c, const oracle_layer* L, const uint16_t* x, int M, const uint16_t* resid,
                   const int32_t* forced, int nthreads, float* logits32, float* lsel, int32_t* idx, double* w,
                   double* y, double* out, uint16_t* out_bf16) {
  if (M <= 0) return 0;
  const int E = c->num_experts;
  std::vector<float> lg((size_t)M * E);
  oracle_router_logits(c, L, x, M, lg.data());
  if (logits32) std::memcpy(logits32, lg.data(), lg.size() * sizeof(float));
  oracle_select(c, L->router_bias, L->per_expert_scale, lg.data(), M, forced, idx, w, lsel);
  int nt = std::max(1, std::min(nthreads, M));
  if (nt == 1) {
    forward_tokens(c, L, x, resid, idx, w, 0, M, y, out, out_bf16);
  } else {
    std::vector<std::thread> th;
    for (int t = 0; t < nt; ++t) {
      int m0 = (int)((long)M * t / nt), m1 = (int)((long)M * (t + 1) / nt);
      th.emplace_back(forward_tokens, c, L, x, resid, idx, w, m0, m1, y, out, out_bf16);
    }
    for (auto& t : th) t.join();
  }
  return 0;
}

}  // extern "C"
