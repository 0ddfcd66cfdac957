// CPU oracle for the routed Mixture-of-Experts layer (sigmoid top-k routing,
// expert-major block plan, SwiGLU experts, top-k finalize + residual + RMSNorm).
//
// TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously-correct
// statement of what the GPU library computes.  Only the test suite, the
// smoke check in __graft_entry__ and the CPU-baseline leg of bench.py may
// load it.  It shares no code, header, table or constant with the CUDA
// library under prefill_sigmoid_top_b200/, and it includes nothing from it.
//
// Arithmetic is fp64 except where the layer fixes fp32 (the router logit and
// the NVFP4 quantisation recipe).  Build flags: -O2 -ffp-contract=off, no
// fast-math, so every fp32 operation below is one IEEE-rounded operation.
//
// Sources (web pages on the method; cited by page title and section):
//  * "[sglang] [NPU] GLM-4.7-Flash 성능 최적화" (sglang PR #29509 analysis),
//    §2 "MoE TopK Scoring Function": expert scores use sigmoid (norm_type=1)
//    instead of softmax.
//  * "[flashinfer] ... AlphaMoE NVFP4 커널 최적화" (flashinfer PR #6511
//    analysis), §5 "moe_align_block_size_kernel 동기화 개선": the align step
//    is a per-expert histogram, a prefix scan into prefix[], and a search
//    that gives each padded block its expert; §6: the route chain is
//    up -> down -> finalize with the plan built before the up kernel;
//    intro: NVFP4 weights (e2m1 values, e4m3 block scales).
//  * "[flashinfer] Kimi K3를 위한 초고속 통신 최적화" (flashinfer PR #5701
//    analysis), intro and §3: MoE finalize fused with RMSNorm for H=7168,
//    top_k=16, RMS_EPS=1e-5 and WEIGHT_BIAS=0 (gamma used as is).
// Where the pages leave a step open the plainest reading is taken; each such
// reading is named at the function that takes it.
//
// Parity pins live in tests/test_oracle_*.py (brute force, closed forms,
// library special cases, a hand-computed case).

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

// ---------------------------------------------------------------- bf16 ----
// bfloat16 = the top 16 bits of an IEEE binary32.
double bf16_value(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return static_cast<double>(f);
}

float bf16_value_f(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

// Round a double straight to bf16, round-to-nearest-even, in one step (no
// intermediate float, so no double rounding).  bf16 has 8 significant bits;
// in the binade [2^ex, 2^(ex+1)) its spacing is 2^(ex-7); below 2^-126 the
// spacing stays 2^-133 (subnormals).  Values at or beyond the largest finite
// bf16 plus half a spacing round to infinity.
uint16_t bf16_round(double v) {
  if (std::isnan(v)) return 0x7FC0;
  const bool neg = std::signbit(v);
  const double a = std::fabs(v);
  uint16_t mag;
  if (std::isinf(a)) {
    mag = 0x7F80;
  } else if (a == 0.0) {
    mag = 0;
  } else {
    int e2;
    std::frexp(a, &e2);          // a = f * 2^e2 with f in [0.5, 1)
    int ex = e2 - 1;             // a in [2^ex, 2^(ex+1))
    if (ex < -126) ex = -126;    // subnormal spacing is fixed
    const double q = std::ldexp(1.0, ex - 7);
    const double r = std::nearbyint(a / q);  // exact scaling; RNE rounding
    const double res = r * q;
    if (res >= std::ldexp(1.0, 128)) {
      mag = 0x7F80;
    } else {
      const float f = static_cast<float>(res);  // exact: res is a bf16 value
      uint32_t u;
      std::memcpy(&u, &f, 4);
      mag = static_cast<uint16_t>(u >> 16);
    }
  }
  return static_cast<uint16_t>(mag | (neg ? 0x8000 : 0));
}

double sigmoid(double z) { return 1.0 / (1.0 + std::exp(-z)); }

// ---------------------------------------------------------------- NVFP4 ---
// e2m1: 1 sign, 2 exponent (bias 1), 1 mantissa bit.  Exponent field 0 is
// subnormal: value = m * 2^(1-1) * 0.5.  No inf/NaN.
double e2m1_value(uint8_t code) {
  const int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
  double mag = (e == 0) ? std::ldexp(m * 0.5, 0)            // 0 or 0.5
                        : std::ldexp(1.0 + m * 0.5, e - 1);  // 1 .. 6
  return s ? -mag : mag;
}

// e4m3 (the "fn" variant): 1 sign, 4 exponent (bias 7), 3 mantissa bits;
// exponent field 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN; no inf.
// The largest finite value is S.1111.110 = 448.
double e4m3_value(uint8_t code) {
  const int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
  double mag;
  if (e == 15 && m == 7) return std::nan("");
  if (e == 0)
    mag = std::ldexp(m / 8.0, -6);
  else
    mag = std::ldexp(1.0 + m / 8.0, e - 7);
  return s ? -mag : mag;
}

// Round |v| onto a finite grid given as the sorted list of representable
// magnitudes (with their codes), round-to-nearest, ties to the even code
// (even mantissa bit), saturating at the largest magnitude ("satfinite").
template <int N>
uint8_t round_to_grid(double a, const double (&vals)[N], const uint8_t (&codes)[N]) {
  if (a >= vals[N - 1]) return codes[N - 1];
  for (int i = 0; i + 1 < N; ++i) {
    const double lo = vals[i], hi = vals[i + 1];
    if (a == lo) return codes[i];
    if (a < hi) {
      const double mid = 0.5 * (lo + hi);  // exact: both are short binary fractions
      if (a < mid) return codes[i];
      if (a > mid) return codes[i + 1];
      return (codes[i] & 1) ? codes[i + 1] : codes[i];  // tie -> even mantissa
    }
  }
  return codes[N - 1];
}

struct E2m1Grid {
  double vals[8];
  uint8_t codes[8];
  E2m1Grid() {
    for (int c = 0; c < 8; ++c) { vals[c] = e2m1_value(static_cast<uint8_t>(c)); codes[c] = static_cast<uint8_t>(c); }
  }
};

struct E4m3Grid {
  double vals[127];
  uint8_t codes[127];
  E4m3Grid() {
    for (int c = 0; c < 127; ++c) { vals[c] = e4m3_value(static_cast<uint8_t>(c)); codes[c] = static_cast<uint8_t>(c); }
  }
};

uint8_t e2m1_encode(float v) {
  static const E2m1Grid grid;  // thread-safe one-time construction
  if (std::isnan(v)) return 0;  // outside the contract; never produced by the recipe
  const uint8_t mag = round_to_grid(std::fabs(static_cast<double>(v)), grid.vals, grid.codes);
  return static_cast<uint8_t>(mag | (std::signbit(v) ? 8 : 0));
}

uint8_t e4m3_encode(float v) {
  static const E4m3Grid grid;
  if (std::isnan(v)) return 0x7F;
  const uint8_t mag = round_to_grid(std::fabs(static_cast<double>(v)), grid.vals, grid.codes);
  return static_cast<uint8_t>(mag | (std::signbit(v) ? 0x80 : 0));
}

}  // namespace

extern "C" {

// ------------------------------------------------------------ scalar codecs
double oracle_bf16_value(uint16_t b) { return bf16_value(b); }
uint16_t oracle_bf16_round(double v) { return bf16_round(v); }
double oracle_e2m1_value(uint8_t c) { return e2m1_value(c); }
double oracle_e4m3_value(uint8_t c) { return e4m3_value(c); }
uint8_t oracle_e2m1_encode(float v) { return e2m1_encode(v); }
uint8_t oracle_e4m3_encode(float v) { return e4m3_encode(v); }

// ------------------------------------------------------------ router -------
// Router logit for one (token, expert) pair in the canonical fp32 order.
//
// The pages do not state a reduction order; bit-exact routing needs one, so
// the order is fixed here (reading): 32 partial sums p[l]; p[l] accumulates,
// with one fused multiply-add per element and in increasing h, every h whose
// 8-element chunk index floor(h/8) is congruent to l mod 32; then the
// partials are combined pairwise, p[l] += p[l+16] for l < 16, then +8, +4,
// +2, +1; finally the fp32 bias is added.  Requires H % 256 == 0.
float canonical_logit(const uint16_t* x, const uint16_t* w, int H, float bias) {
  float p[32];
  for (int l = 0; l < 32; ++l) {
    float acc = 0.0f;
    for (int j = 0; j * 256 < H; ++j)
      for (int i = 0; i < 8; ++i) {
        const int h = 256 * j + 8 * l + i;
        acc = std::fma(bf16_value_f(x[h]), bf16_value_f(w[h]), acc);
      }
    p[l] = acc;
  }
  for (int s = 16; s >= 1; s /= 2)
    for (int l = 0; l < s; ++l) p[l] = p[l] + p[l + s];
  return p[0] + bias;
}

// z32[M,E] canonical fp32 logits; z64[M,E] (nullable) the exact fp64 dot
// product plus bias, for error-bound checks.
void oracle_router_logits(const uint16_t* x, const uint16_t* w_router, const float* bias,
                          int M, int H, int E, float* z32, double* z64) {
#pragma omp parallel for schedule(dynamic)
  for (int t = 0; t < M; ++t)
    for (int e = 0; e < E; ++e) {
      const float b = bias ? bias[e] : 0.0f;
      z32[static_cast<size_t>(t) * E + e] =
          canonical_logit(x + static_cast<size_t>(t) * H, w_router + static_cast<size_t>(e) * H, H, b);
      if (z64) {
        double acc = 0.0;
        for (int h = 0; h < H; ++h)
          acc += bf16_value(x[static_cast<size_t>(t) * H + h]) * bf16_value(w_router[static_cast<size_t>(e) * H + h]);
        z64[static_cast<size_t>(t) * E + e] = acc + static_cast<double>(b);
      }
    }
}

// Non-finite logits are outside the pages' workloads; a NaN logit is read as
// -inf, so it ranks below every other logit (its expert is picked only when
// nothing else is left) and its sigmoid score is 0.
static float key_of(float z) { return std::isnan(z) ? -INFINITY : z; }

// Sigmoid top-k selection and renormalisation for each token.
// Selection key: the fp32 logit z (sigmoid is monotone, so this is the
// order of the sigmoid scores; keeping z avoids depending on how exp is
// evaluated).  Slots hold the K largest keys in descending order; equal keys
// (compared as floats, so +0 == -0) go to the lower expert id.
// Weights: s_k = sigmoid(z_k), w_k = s_k / sum_j s_j (fp64), no extra
// scaling factor (sglang PR #29509 analysis, §2: scoring fixed to sigmoid).
void oracle_topk(const float* z32, int M, int E, int K, int32_t* topk_ids, double* topk_w) {
#pragma omp parallel for schedule(static)
  for (int t = 0; t < M; ++t) {
    std::vector<float> z(E);
    for (int e = 0; e < E; ++e) z[e] = key_of(z32[static_cast<size_t>(t) * E + e]);
    std::vector<int> order(E);
    for (int e = 0; e < E; ++e) order[e] = e;
    std::sort(order.begin(), order.end(), [&z](int a, int b) {
      if (z[a] > z[b]) return true;
      if (z[a] < z[b]) return false;
      return a < b;
    });
    double total = 0.0;
    for (int k = 0; k < K; ++k) total += sigmoid(static_cast<double>(z[order[k]]));
    for (int k = 0; k < K; ++k) {
      topk_ids[static_cast<size_t>(t) * K + k] = order[k];
      topk_w[static_cast<size_t>(t) * K + k] = sigmoid(static_cast<double>(z[order[k]])) / total;
    }
  }
}

// Routing variants (sglang PR #29509 analysis, §2: the fused top-k takes a
// norm_type, 0 = softmax scoring and 1 = sigmoid scoring).  z32 is the
// canonical logit; sel_bias (nullable) is a per-expert bias that enters only
// the selection key, key = fp32(z + sel_bias[e]), and not the score.  The K
// experts are those oracle_topk picks on the key.  Scores and weights in fp64:
//   scoring 1 (sigmoid): p_k = sigmoid(z_k)
//   scoring 0 (softmax): p_k = exp(z_k - zmax) / sum_e exp(z_e - zmax), over all E
//   w_k = p_k / sum_j p_j if renormalize, else p_k; then w_k *= scale
void oracle_topk_ex(const float* z32, const float* sel_bias, int M, int E, int K, int scoring, int renormalize,
                    double scale, int32_t* topk_ids, double* topk_w) {
  std::vector<float> key(z32, z32 + static_cast<size_t>(M) * E);
  if (sel_bias != nullptr)
    for (int t = 0; t < M; ++t)
      for (int e = 0; e < E; ++e) {
        volatile float sum = key[static_cast<size_t>(t) * E + e] + sel_bias[e];  // one fp32 add
        key[static_cast<size_t>(t) * E + e] = sum;
      }
  std::vector<double> unused(static_cast<size_t>(M) * K);
  oracle_topk(key.data(), M, E, K, topk_ids, unused.data());
  for (int t = 0; t < M; ++t) {
    std::vector<float> z(E);
    for (int e = 0; e < E; ++e) z[e] = key_of(z32[static_cast<size_t>(t) * E + e]);
    double p[64];
    double denom_all = 0.0, zmax = -INFINITY;
    if (scoring == 0) {
      for (int e = 0; e < E; ++e) zmax = std::max(zmax, static_cast<double>(z[e]));
      for (int e = 0; e < E; ++e) denom_all += std::exp(static_cast<double>(z[e]) - zmax);
    }
    double total = 0.0;
    for (int k = 0; k < K; ++k) {
      const double zk = static_cast<double>(z[topk_ids[static_cast<size_t>(t) * K + k]]);
      p[k] = scoring == 0 ? std::exp(zk - zmax) / denom_all : sigmoid(zk);
      total += p[k];
    }
    for (int k = 0; k < K; ++k)
      topk_w[static_cast<size_t>(t) * K + k] = (renormalize ? p[k] / total : p[k]) * scale;
  }
}

// ------------------------------------------------------------ align --------
// Expert-major block plan (flashinfer PR #6511 analysis, §5): histogram of
// the flat slots f = t*K + k by expert; padded exclusive prefix where each
// expert's count is rounded up to a multiple of the block size B (an empty
// expert gets 0 rows); the slots of expert e, in ascending f, are placed at
// the start of its segment and the rest of the segment holds the sentinel
// M*K; every block of B rows belongs to exactly one expert, found by a
// search over the prefix.  Returns 0, or 4 if an id lies outside [0, E).
int oracle_align(const int32_t* topk_ids, int M, int K, int E, int B,
                 int32_t* sorted_ids, int32_t* block_expert, int32_t* expert_counts,
                 int32_t* expert_offsets, int32_t* num_tokens_post_padded) {
  const int64_t n = static_cast<int64_t>(M) * K;
  for (int64_t f = 0; f < n; ++f)
    if (topk_ids[f] < 0 || topk_ids[f] >= E) return 4;
  std::vector<int64_t> count(E, 0);
  for (int64_t f = 0; f < n; ++f) count[topk_ids[f]]++;
  expert_offsets[0] = 0;
  for (int e = 0; e < E; ++e) {
    expert_counts[e] = static_cast<int32_t>(count[e]);
    const int64_t padded = (count[e] + B - 1) / B * B;
    expert_offsets[e + 1] = static_cast<int32_t>(expert_offsets[e] + padded);
  }
  const int32_t total = expert_offsets[E];
  *num_tokens_post_padded = total;
  for (int e = 0; e < E; ++e) {
    int32_t pos = expert_offsets[e];
    for (int64_t f = 0; f < n; ++f)
      if (topk_ids[f] == e) sorted_ids[pos++] = static_cast<int32_t>(f);
    while (pos < expert_offsets[e + 1]) sorted_ids[pos++] = static_cast<int32_t>(n);
  }
  for (int32_t b = 0; b * B < total; ++b) {
    // the expert whose half-open segment [offsets[e], offsets[e+1]) holds row b*B
    int lo = 0, hi = E - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) / 2;
      if (expert_offsets[mid] <= b * B) lo = mid; else hi = mid - 1;
    }
    block_expert[b] = lo;
  }
  return 0;
}

// ------------------------------------------------------------ experts ------
// One routed slot: the SwiGLU expert e applied to token row x (length H).
//   g = x . W_gate[e]^T, u = x . W_up[e]^T  (fp64 over the exact bf16 inputs)
//   h = bf16(silu(g) * u),  silu(g) = g * sigmoid(g)
//   y = bf16(h . W_down[e]^T)
// h and y are rounded to bf16 because they are the layer's stored
// intermediates (reading: the GPU path rounds at the same two points).
// w_gate/w_up: [I,H] row-major, w_down: [H,I] row-major, all bf16.
void oracle_expert(const uint16_t* x, const uint16_t* w_gate, const uint16_t* w_up,
                   const uint16_t* w_down, int H, int I, uint16_t* h_out, uint16_t* y_out) {
  std::vector<double> xd(H), hd(I);
  for (int c = 0; c < H; ++c) xd[c] = bf16_value(x[c]);
  for (int i = 0; i < I; ++i) {
    double g = 0.0, u = 0.0;
    const uint16_t* wg = w_gate + static_cast<size_t>(i) * H;
    const uint16_t* wu = w_up + static_cast<size_t>(i) * H;
    for (int c = 0; c < H; ++c) {
      g += xd[c] * bf16_value(wg[c]);
      u += xd[c] * bf16_value(wu[c]);
    }
    const uint16_t hb = bf16_round(g * sigmoid(g) * u);
    if (h_out) h_out[i] = hb;
    hd[i] = bf16_value(hb);
  }
  for (int r = 0; r < H; ++r) {
    double acc = 0.0;
    const uint16_t* wd = w_down + static_cast<size_t>(r) * I;
    for (int i = 0; i < I; ++i) acc += hd[i] * bf16_value(wd[i]);
    y_out[r] = bf16_round(acc);
  }
}

// Finalize for one token (flashinfer PR #5701 analysis: MoE finalize fused
// with RMSNorm; WEIGHT_BIAS = 0 so gamma multiplies as is):
//   s = x + sum_k w_k * y_k             (fp64)
//   out = bf16( s / sqrt(mean_h(s^2) + eps) * gamma )
//   residual_out = bf16(s)              (nullable)
// out64 / s64 (nullable) receive the same two values before their final bf16
// rounding: the reference for tolerance comparisons of the layer output
// (reading: the bf16 quantisation the reference applies is that of the stored
// intermediates h and y; the output's own rounding is part of the error
// measured, since two correct bf16 roundings of values that straddle a
// rounding boundary differ by a whole bf16 step).
void oracle_finalize_token(const uint16_t* x, const uint16_t* y, const double* w, const uint16_t* gamma,
                           double eps, int K, int H, uint16_t* out, uint16_t* residual_out, double* out64,
                           double* s64) {
  std::vector<double> s(H);
  for (int c = 0; c < H; ++c) {
    double acc = bf16_value(x[c]);
    for (int k = 0; k < K; ++k) acc += w[k] * bf16_value(y[static_cast<size_t>(k) * H + c]);
    s[c] = acc;
  }
  double ss = 0.0;
  for (int c = 0; c < H; ++c) ss += s[c] * s[c];
  const double inv = 1.0 / std::sqrt(ss / H + eps);
  for (int c = 0; c < H; ++c) {
    const double o = s[c] * inv * bf16_value(gamma[c]);
    out[c] = bf16_round(o);
    if (residual_out) residual_out[c] = bf16_round(s[c]);
    if (out64) out64[c] = o;
    if (s64) s64[c] = s[c];
  }
}

// Finalize over M tokens: y is [M,K,H] bf16, w is [M,K] fp64.
void oracle_finalize(const uint16_t* x, const uint16_t* y, const double* w, const uint16_t* gamma,
                     double eps, int M, int K, int H, uint16_t* out, uint16_t* residual_out, double* out64,
                     double* s64) {
#pragma omp parallel for schedule(static)
  for (int t = 0; t < M; ++t)
    oracle_finalize_token(x + static_cast<size_t>(t) * H, y + static_cast<size_t>(t) * K * H,
                          w + static_cast<size_t>(t) * K, gamma, eps, K, H,
                          out + static_cast<size_t>(t) * H,
                          residual_out ? residual_out + static_cast<size_t>(t) * H : nullptr,
                          out64 ? out64 + static_cast<size_t>(t) * H : nullptr,
                          s64 ? s64 + static_cast<size_t>(t) * H : nullptr);
}

// The whole layer for a chosen subset of tokens.  Expert weights are passed
// as per-expert pointer tables so that a caller may provide only the experts
// the chosen tokens route to; a needed expert given as null makes the call
// return 3.  Returns 4 if routing produced an out-of-range id (cannot happen
// for finite inputs).  Per chosen token i (token index tokens[i]):
//   ids/w   -> topk_ids[i*K..], topk_w[i*K..]
//   y       -> y_out[(i*K + k)*H ..]   (nullable)
//   h       -> h_out[(i*K + k)*I ..]   (nullable)
//   out     -> out[i*H ..], residual_out[i*H ..] (nullable)
int oracle_layer(const uint16_t* x, const uint16_t* w_router, const float* bias,
                 const uint16_t* const* w_gate, const uint16_t* const* w_up,
                 const uint16_t* const* w_down, const uint16_t* gamma, float eps,
                 int M, int H, int I, int E, int K, const int32_t* tokens, int n_tokens,
                 int32_t* topk_ids, double* topk_w, uint16_t* h_out, uint16_t* y_out,
                 uint16_t* out, uint16_t* residual_out, double* out64, double* s64) {
  (void)M;
  std::vector<float> z(static_cast<size_t>(E));
  for (int i = 0; i < n_tokens; ++i) {
    const uint16_t* xt = x + static_cast<size_t>(tokens[i]) * H;
    for (int e = 0; e < E; ++e) z[e] = canonical_logit(xt, w_router + static_cast<size_t>(e) * H, H, bias ? bias[e] : 0.0f);
    oracle_topk(z.data(), 1, E, K, topk_ids + static_cast<size_t>(i) * K, topk_w + static_cast<size_t>(i) * K);
    for (int k = 0; k < K; ++k) {
      const int e = topk_ids[static_cast<size_t>(i) * K + k];
      if (e < 0 || e >= E) return 4;
      if (!w_gate[e] || !w_up[e] || !w_down[e]) return 3;
    }
  }
  std::vector<uint16_t> y_local;
  uint16_t* y = y_out;
  if (!y) {
    y_local.resize(static_cast<size_t>(n_tokens) * K * H);
    y = y_local.data();
  }
  const int n_slots = n_tokens * K;
#pragma omp parallel for schedule(dynamic)
  for (int s = 0; s < n_slots; ++s) {
    const int i = s / K;
    const int e = topk_ids[s];
    oracle_expert(x + static_cast<size_t>(tokens[i]) * H, w_gate[e], w_up[e], w_down[e], H, I,
                  h_out ? h_out + static_cast<size_t>(s) * I : nullptr, y + static_cast<size_t>(s) * H);
  }
  if (out) {
    for (int i = 0; i < n_tokens; ++i)
      oracle_finalize_token(x + static_cast<size_t>(tokens[i]) * H, y + static_cast<size_t>(i) * K * H,
                            topk_w + static_cast<size_t>(i) * K, gamma, static_cast<double>(eps), K, H,
                            out + static_cast<size_t>(i) * H,
                            residual_out ? residual_out + static_cast<size_t>(i) * H : nullptr,
                            out64 ? out64 + static_cast<size_t>(i) * H : nullptr,
                            s64 ? s64 + static_cast<size_t>(i) * H : nullptr);
  }
  return 0;
}

// Dense form of the expert sum, for the sparse-vs-dense pin: every expert is
// evaluated for every token and mixed with weight w (zero for experts not
// selected).  mix[t*H + c] = sum_e wdense[t*E + e] * bf16 y_e[c], in fp64.
void oracle_dense_mixture(const uint16_t* x, const uint16_t* const* w_gate, const uint16_t* const* w_up,
                          const uint16_t* const* w_down, const double* wdense, int M, int H, int I, int E,
                          double* mix) {
#pragma omp parallel for schedule(dynamic)
  for (int t = 0; t < M; ++t) {
    std::vector<uint16_t> y(H);
    for (int c = 0; c < H; ++c) mix[static_cast<size_t>(t) * H + c] = 0.0;
    for (int e = 0; e < E; ++e) {
      oracle_expert(x + static_cast<size_t>(t) * H, w_gate[e], w_up[e], w_down[e], H, I, nullptr, y.data());
      const double we = wdense[static_cast<size_t>(t) * E + e];
      for (int c = 0; c < H; ++c) mix[static_cast<size_t>(t) * H + c] += we * bf16_value(y[c]);
    }
  }
}

// ------------------------------------------------------------ NVFP4 --------
// NVFP4 quantisation (flashinfer PR #6511 analysis, intro: e2m1 values with
// e4m3 block scales).  The pages do not print the recipe; the reading taken:
// per matrix a global scale gs = amax / (6*448) (1 if amax is 0); per block
// of 16 consecutive elements along the contraction dimension a scale
// sb = e4m3(blockamax / 6 / gs); each element q = e2m1(v / (sb*gs)) (0 when
// sb is 0); the dequantised value is q * sb * gs.  All recipe arithmetic is
// IEEE fp32, one rounding per operation, in exactly this order; e4m3 and
// e2m1 conversions round to nearest even and saturate to 448 and 6.

float oracle_nvfp4_global_scale(float amax) {
  if (amax == 0.0f) return 1.0f;
  return amax / 2688.0f;  // 6 * 448
}

// rows x cols fp32 values (cols % 16 == 0), row-major; blocks run along cols.
// codes: [rows, cols] one e2m1 code per byte (low nibble); scales: [rows, cols/16].
void oracle_nvfp4_quantize(const float* v, int64_t rows, int64_t cols, float gs, uint8_t* codes, uint8_t* scales) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t b = 0; b < cols / 16; ++b) {
      const float* blk = v + r * cols + b * 16;
      float bamax = 0.0f;
      for (int i = 0; i < 16; ++i) bamax = std::max(bamax, std::fabs(blk[i]));
      float t = bamax / 6.0f;
      t = t / gs;
      const uint8_t sc = e4m3_encode(t);
      scales[r * (cols / 16) + b] = sc;
      const float sbf = static_cast<float>(e4m3_value(sc));
      const float d = sbf * gs;
      for (int i = 0; i < 16; ++i)
        codes[r * cols + b * 16 + i] = (sc == 0) ? static_cast<uint8_t>(0) : e2m1_encode(blk[i] / d);
    }
}

// Dequantised value of element (r, c).
double oracle_nvfp4_value(const uint8_t* codes, const uint8_t* scales, int64_t cols, float gs, int64_t r, int64_t c) {
  return e2m1_value(codes[r * cols + c]) * e4m3_value(scales[r * (cols / 16) + c / 16]) * static_cast<double>(gs);
}

// Quantise a bf16 matrix (per-matrix amax -> gs); returns gs.
float oracle_nvfp4_quantize_bf16(const uint16_t* w, int64_t rows, int64_t cols, uint8_t* codes, uint8_t* scales) {
  std::vector<float> v(static_cast<size_t>(rows * cols));
  float amax = 0.0f;
  for (int64_t i = 0; i < rows * cols; ++i) {
    v[i] = bf16_value_f(w[i]);
    amax = std::max(amax, std::fabs(v[i]));
  }
  const float gs = oracle_nvfp4_global_scale(amax);
  oracle_nvfp4_quantize(v.data(), rows, cols, gs, codes, scales);
  return gs;
}

// Dequantise a whole matrix to fp64.
void oracle_nvfp4_dequantize(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols, float gs,
                             double* out) {
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c) out[r * cols + c] = oracle_nvfp4_value(codes, scales, cols, gs, r, c);
}

// The NVFP4 layer.  Every GEMM operand is replaced by its dequantised NVFP4
// value; the fp64 math and the bf16 rounding points are those of
// oracle_layer.  Weights: per expert per projection a quantised matrix with
// its own gs (codes one per byte, scales e4m3), given as pointer tables.
// Activations: x is quantised from bf16 with gs from amax over all of x;
// h (after bf16 rounding) is quantised with gs from amax over all M*K slot
// rows of the call, so this computes h for every token, then y and out for
// the chosen tokens.  Work is grouped by expert so that each expert matrix is
// dequantised once.  Returns 3 if a needed expert is missing.
namespace {
struct Fp4Tables {
  double e2m1[16];
  double e4m3[256];
  Fp4Tables() {
    for (int c = 0; c < 16; ++c) e2m1[c] = e2m1_value(static_cast<uint8_t>(c));
    for (int c = 0; c < 256; ++c) e4m3[c] = e4m3_value(static_cast<uint8_t>(c));
  }
};

void dequantize_matrix(const Fp4Tables& T, const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols,
                       float gs, double* out) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c)
      out[r * cols + c] = T.e2m1[codes[r * cols + c]] * T.e4m3[scales[r * (cols / 16) + c / 16]] * static_cast<double>(gs);
}
}  // namespace

int oracle_layer_nvfp4(const uint16_t* x, const uint16_t* w_router, const float* bias,
                       const uint8_t* const* gate_codes, const uint8_t* const* gate_scales, const float* gate_gs,
                       const uint8_t* const* up_codes, const uint8_t* const* up_scales, const float* up_gs,
                       const uint8_t* const* down_codes, const uint8_t* const* down_scales, const float* down_gs,
                       const uint16_t* gamma, float eps, int M, int H, int I, int E, int K,
                       const int32_t* tokens, int n_tokens, int32_t* topk_ids_all, double* topk_w_all,
                       uint16_t* h_all, uint16_t* y_out, uint16_t* out, uint16_t* residual_out,
                       double* out64, double* s64) {
  static const Fp4Tables T;
  // routing for every token (h needs all of them)
  std::vector<float> z(static_cast<size_t>(M) * E);
  oracle_router_logits(x, w_router, bias, M, H, E, z.data(), nullptr);
  oracle_topk(z.data(), M, E, K, topk_ids_all, topk_w_all);
  const int64_t n_slots = static_cast<int64_t>(M) * K;
  for (int64_t s = 0; s < n_slots; ++s) {
    const int e = topk_ids_all[s];
    if (!gate_codes[e] || !up_codes[e] || !gate_scales[e] || !up_scales[e]) return 3;
  }
  for (int i = 0; i < n_tokens; ++i)
    for (int k = 0; k < K; ++k) {
      const int e = topk_ids_all[static_cast<size_t>(tokens[i]) * K + k];
      if (!down_codes[e] || !down_scales[e]) return 3;
    }
  // x -> NVFP4 (gs over all of x), dequantised
  std::vector<float> xf(static_cast<size_t>(M) * H);
  float xamax = 0.0f;
  for (size_t i = 0; i < xf.size(); ++i) {
    xf[i] = bf16_value_f(x[i]);
    xamax = std::max(xamax, std::fabs(xf[i]));
  }
  const float xgs = oracle_nvfp4_global_scale(xamax);
  std::vector<uint8_t> xc(xf.size()), xs(xf.size() / 16);
  oracle_nvfp4_quantize(xf.data(), M, H, xgs, xc.data(), xs.data());
  std::vector<double> xd(xf.size());
  dequantize_matrix(T, xc.data(), xs.data(), M, H, xgs, xd.data());
  // h for every slot, expert by expert
  std::vector<std::vector<int64_t>> by_expert(E);
  for (int64_t s = 0; s < n_slots; ++s) by_expert[topk_ids_all[s]].push_back(s);
  std::vector<double> wg(static_cast<size_t>(I) * H), wu(static_cast<size_t>(I) * H);
  for (int e = 0; e < E; ++e) {
    if (by_expert[e].empty()) continue;
    dequantize_matrix(T, gate_codes[e], gate_scales[e], I, H, gate_gs[e], wg.data());
    dequantize_matrix(T, up_codes[e], up_scales[e], I, H, up_gs[e], wu.data());
    const int64_t ns = static_cast<int64_t>(by_expert[e].size());
#pragma omp parallel for schedule(dynamic)
    for (int64_t j = 0; j < ns * I; ++j) {
      const int64_t s = by_expert[e][j / I];
      const int i = static_cast<int>(j % I);
      const double* xr = xd.data() + (s / K) * H;
      double g = 0.0, u = 0.0;
      for (int c = 0; c < H; ++c) {
        g += xr[c] * wg[static_cast<size_t>(i) * H + c];
        u += xr[c] * wu[static_cast<size_t>(i) * H + c];
      }
      h_all[s * I + i] = bf16_round(g * sigmoid(g) * u);
    }
  }
  // h -> NVFP4 (gs over all slot rows)
  float hamax = 0.0f;
  for (int64_t i = 0; i < n_slots * I; ++i) hamax = std::max(hamax, std::fabs(bf16_value_f(h_all[i])));
  const float hgs = oracle_nvfp4_global_scale(hamax);
  // y for the chosen tokens, expert by expert
  std::vector<uint16_t> y_local;
  uint16_t* y = y_out;
  if (!y) {
    y_local.resize(static_cast<size_t>(n_tokens) * K * H);
    y = y_local.data();
  }
  std::vector<std::vector<int>> chosen_by_expert(E);  // local slot index i*K + k
  for (int i = 0; i < n_tokens; ++i)
    for (int k = 0; k < K; ++k)
      chosen_by_expert[topk_ids_all[static_cast<size_t>(tokens[i]) * K + k]].push_back(i * K + k);
  std::vector<double> wd(static_cast<size_t>(H) * I);
  for (int e = 0; e < E; ++e) {
    if (chosen_by_expert[e].empty()) continue;
    dequantize_matrix(T, down_codes[e], down_scales[e], H, I, down_gs[e], wd.data());
    for (int ls : chosen_by_expert[e]) {
      const int i = ls / K, k = ls % K;
      const int64_t slot = static_cast<int64_t>(tokens[i]) * K + k;
      std::vector<float> hf(I);
      for (int c = 0; c < I; ++c) hf[c] = bf16_value_f(h_all[slot * I + c]);
      std::vector<uint8_t> hc(I), hs(I / 16);
      oracle_nvfp4_quantize(hf.data(), 1, I, hgs, hc.data(), hs.data());
      std::vector<double> hd(I);
      dequantize_matrix(T, hc.data(), hs.data(), 1, I, hgs, hd.data());
#pragma omp parallel for schedule(static)
      for (int r = 0; r < H; ++r) {
        double acc = 0.0;
        for (int c = 0; c < I; ++c) acc += hd[c] * wd[static_cast<size_t>(r) * I + c];
        y[static_cast<size_t>(ls) * H + r] = bf16_round(acc);
      }
    }
  }
  if (out) {
    for (int i = 0; i < n_tokens; ++i)
      oracle_finalize_token(x + static_cast<size_t>(tokens[i]) * H, y + static_cast<size_t>(i) * K * H,
                            topk_w_all + static_cast<size_t>(tokens[i]) * K, gamma, static_cast<double>(eps), K, H,
                            out + static_cast<size_t>(i) * H,
                            residual_out ? residual_out + static_cast<size_t>(i) * H : nullptr,
                            out64 ? out64 + static_cast<size_t>(i) * H : nullptr,
                            s64 ? s64 + static_cast<size_t>(i) * H : nullptr);
  }
  return 0;
}

// ------------------------------------------------------------ tensor parallel
// The layer with the expert intermediate dimension I split over G ranks, and
// the finalize fused with the reduction across the ranks and the RMSNorm
// (flashinfer PR #5701 analysis, intro: "MoE finalize + All-Reduce +
// RMSNorm").  Reading: rank r holds rows [r*I/G, (r+1)*I/G) of W_gate[e] and
// W_up[e] and the same columns of W_down[e]; its h is that slice of the
// unsharded h (each h column depends on its own rows only), and its partial
// down projection is rounded once to bf16, the rank's stored intermediate:
//   y_r[t,k,c] = bf16( sum_{i in slice r} h[t,k,i] * W_down[e][c,i] )   (fp64 sum)
//   p_r[t,c]   = (r == 0 ? x[t,c] : 0) + sum_k w[t,k] * y_r[t,k,c]      (fp64, k in order)
// The residual enters once (on rank 0), so for G = 1 p_0 is exactly the
// finalize's s.  Per chosen token i: p_out[i*H..] (fp64), y_out[(i*K+k)*H..]
// (bf16, nullable), ids/w as oracle_layer.  Returns oracle_layer's codes.
int oracle_tp_partial(const uint16_t* x, const uint16_t* w_router, const float* bias,
                      const uint16_t* const* w_gate, const uint16_t* const* w_up, const uint16_t* const* w_down,
                      int H, int I, int E, int K, int G, int rank, const int32_t* tokens, int n_tokens,
                      int32_t* topk_ids, double* topk_w, double* p_out, uint16_t* y_out) {
  if (G < 1 || rank < 0 || rank >= G || I % G != 0) return 2;
  const int Ir = I / G, i0 = rank * Ir;
  std::vector<float> z(static_cast<size_t>(E));
  for (int i = 0; i < n_tokens; ++i) {
    const uint16_t* xt = x + static_cast<size_t>(tokens[i]) * H;
    for (int e = 0; e < E; ++e) z[e] = canonical_logit(xt, w_router + static_cast<size_t>(e) * H, H, bias ? bias[e] : 0.0f);
    oracle_topk(z.data(), 1, E, K, topk_ids + static_cast<size_t>(i) * K, topk_w + static_cast<size_t>(i) * K);
    for (int k = 0; k < K; ++k) {
      const int e = topk_ids[static_cast<size_t>(i) * K + k];
      if (e < 0 || e >= E) return 4;
      if (!w_gate[e] || !w_up[e] || !w_down[e]) return 3;
    }
  }
  std::vector<uint16_t> y(static_cast<size_t>(n_tokens) * K * H);
  const int n_slots = n_tokens * K;
#pragma omp parallel for schedule(dynamic)
  for (int sl = 0; sl < n_slots; ++sl) {
    const int i = sl / K;
    const int e = topk_ids[sl];
    const uint16_t* xt = x + static_cast<size_t>(tokens[i]) * H;
    std::vector<double> hd(Ir);
    for (int j = 0; j < Ir; ++j) {  // this rank's columns of h, as oracle_expert computes them
      double g = 0.0, u = 0.0;
      const uint16_t* wg = w_gate[e] + static_cast<size_t>(i0 + j) * H;
      const uint16_t* wu = w_up[e] + static_cast<size_t>(i0 + j) * H;
      for (int c = 0; c < H; ++c) {
        g += bf16_value(xt[c]) * bf16_value(wg[c]);
        u += bf16_value(xt[c]) * bf16_value(wu[c]);
      }
      hd[j] = bf16_value(bf16_round(g * sigmoid(g) * u));
    }
    for (int c = 0; c < H; ++c) {
      double acc = 0.0;
      const uint16_t* wd = w_down[e] + static_cast<size_t>(c) * I + i0;
      for (int j = 0; j < Ir; ++j) acc += hd[j] * bf16_value(wd[j]);
      y[static_cast<size_t>(sl) * H + c] = bf16_round(acc);
    }
  }
  for (int i = 0; i < n_tokens; ++i)
    for (int c = 0; c < H; ++c) {
      double acc = rank == 0 ? bf16_value(x[static_cast<size_t>(tokens[i]) * H + c]) : 0.0;
      for (int k = 0; k < K; ++k)
        acc += topk_w[static_cast<size_t>(i) * K + k] * bf16_value(y[(static_cast<size_t>(i) * K + k) * H + c]);
      p_out[static_cast<size_t>(i) * H + c] = acc;
    }
  if (y_out) std::memcpy(y_out, y.data(), y.size() * sizeof(uint16_t));
  return 0;
}

// RMSNorm of rows s [n,H] (fp64): out = bf16(s / sqrt(mean_h(s^2) + eps) * gamma),
// residual_out = bf16(s) (nullable), out64 = out before its rounding (nullable).
void oracle_rmsnorm_rows(const double* s, const uint16_t* gamma, double eps, int n, int H, uint16_t* out,
                         uint16_t* residual_out, double* out64) {
  for (int i = 0; i < n; ++i) {
    const double* st = s + static_cast<size_t>(i) * H;
    double ss = 0.0;
    for (int c = 0; c < H; ++c) ss += st[c] * st[c];
    const double inv = 1.0 / std::sqrt(ss / H + eps);
    for (int c = 0; c < H; ++c) {
      const double o = st[c] * inv * bf16_value(gamma[c]);
      out[static_cast<size_t>(i) * H + c] = bf16_round(o);
      if (residual_out) residual_out[static_cast<size_t>(i) * H + c] = bf16_round(st[c]);
      if (out64) out64[static_cast<size_t>(i) * H + c] = o;
    }
  }
}

// The tensor-parallel layer on G ranks, every rank's part computed here:
// s = p_0 + p_1 + ... + p_{G-1} (fp64, rank order), then oracle_rmsnorm_rows.
// y_parts (nullable) receives each rank's partial rows, [G][n][K][H] bf16.
int oracle_layer_tp(const uint16_t* x, const uint16_t* w_router, const float* bias,
                    const uint16_t* const* w_gate, const uint16_t* const* w_up, const uint16_t* const* w_down,
                    const uint16_t* gamma, float eps, int H, int I, int E, int K, int G, const int32_t* tokens,
                    int n_tokens, int32_t* topk_ids, double* topk_w, uint16_t* y_parts, uint16_t* out,
                    uint16_t* residual_out, double* out64, double* s64) {
  std::vector<double> s(static_cast<size_t>(n_tokens) * H, 0.0), p(static_cast<size_t>(n_tokens) * H);
  for (int r = 0; r < G; ++r) {
    const int st = oracle_tp_partial(x, w_router, bias, w_gate, w_up, w_down, H, I, E, K, G, r, tokens, n_tokens,
                                     topk_ids, topk_w, p.data(),
                                     y_parts ? y_parts + static_cast<size_t>(r) * n_tokens * K * H : nullptr);
    if (st != 0) return st;
    for (size_t j = 0; j < s.size(); ++j) s[j] = r == 0 ? p[j] : s[j] + p[j];
  }
  oracle_rmsnorm_rows(s.data(), gamma, static_cast<double>(eps), n_tokens, H, out, residual_out, out64);
  if (s64) std::memcpy(s64, s.data(), s.size() * sizeof(double));
  return 0;
}

int oracle_num_threads() {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

}  // extern "C"
