// ORACLE -- test infrastructure only.
//
// A plain, slow, fp64 CPU implementation of one decode step of a very
// sparse mixture-of-experts layer with MXFP4 expert weights, used to check
// the CUDA library.  Only tests/, the package's smoke check and the CPU
// baseline leg of bench.py load it; the library never does, and the two
// share no code, table or header.
//
// What the layer computes.  The decode-path pages (aitest123 "how NVIDIA
// optimised Kimi K3 with a 12k-line CuTe DSL megakernel", intro; tmtpost
// article, section on the phenomenon) fix: 896 routed experts of which 16
// are active per token, native MXFP4 4-bit expert weights, and one shared
// expert run beside the routed ones (yeyulingfeng article, section 02; smzdm
// post, section on the four-step rework).  They give no formulas.  The
// shapes, SwiGLU experts, E2M1 + E8M0 per-32 scaling and the softmax
// renormalised over the selected logits come from the workload definition.
// Each function below writes the plain definition out, step by step:
//
//   logits[b][e] = sum_h x[b][h] * Wr[h][e] (+ bias[e])          (router)
//   S_b          = the k largest logits, ties to the lower expert id,
//                  listed in ascending expert id                  (top-k)
//   w[b][j]      = exp(l_j - m) / sum_{i in S_b} exp(l_i - m)     (softmax
//                  over the selected logits, m = their maximum; the
//                  sigmoid variant: s = sigmoid(l), selection by s + bias,
//                  w = s_j / sum of the selected s)
//   buckets      = counting sort of the pairs (b, j) by expert    (bucketing)
//   g = Wg x, u = Wu x, h = silu(g) * u, y = Wd h                 (SwiGLU
//                  expert; MXFP4 weights dequantised exactly)
//   y_s          = the same FFN with the shared bf16 weights
//   out[b]       = residual[b] + y_s[b] + sum_{j, ascending e} w[b][j] y[b][j]
//
// Readings where the definition leaves a choice (also listed with the
// design notes): E2M1 code map per OCP Microscaling v1.0 (codes 0..7 are
// 0, .5, 1, 1.5, 2, 3, 4, 6; bit 3 is the sign); E8M0 byte s is 2^(s-127),
// s = 255 is NaN; the even-K element sits in the low nibble; gate rows come
// before up rows; silu(g) = g / (1 + e^-g); the shared expert is added with
// weight 1; the bias takes part in selection and in the softmax.
//
// All arithmetic is IEEE double; the only rounding to a narrow type is the
// final bf16 (round to nearest even, straight from double).
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

double bf16_value(uint16_t b) {
  const uint32_t u = (uint32_t)b << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return (double)f;
}

// E2M1 element values (OCP Microscaling v1.0, FP4 E2M1): magnitude index 0..7.
const double kE2M1Magnitude[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double e2m1_value(unsigned code) {
  const double m = kE2M1Magnitude[code & 7u];
  return (code & 8u) ? -m : m;
}

double e8m0_value(unsigned s) {
  if (s == 255u) return std::nan("");
  return std::ldexp(1.0, (int)s - 127);
}

// Dequantise K elements of one MXFP4 row (codes K/2 bytes, scales K/32 bytes).
void dequant_row(const uint8_t* codes, const uint8_t* scales, int K, double* out) {
  for (int k = 0; k < K; ++k) {
    const uint8_t byte = codes[k / 2];
    const unsigned code = (k % 2 == 0) ? (byte & 0x0Fu) : (byte >> 4);
    out[k] = e2m1_value(code) * e8m0_value(scales[k / 32]);
  }
}

double silu(double g) { return g / (1.0 + std::exp(-g)); }

// Round a double to bf16 (round to nearest even), straight from double.
uint16_t round_bf16(double v) {
  if (std::isnan(v)) return 0x7FC0;
  const bool neg = std::signbit(v);
  const double a = std::fabs(v);
  uint32_t bits;
  if (a == 0.0) {
    bits = 0;
  } else {
    int e;
    std::frexp(a, &e);            // a = f * 2^e, f in [0.5, 1) -> floor(log2 a) = e - 1
    int el = e - 1;
    if (el < -126) el = -126;     // subnormal range: fixed quantum 2^-133
    const double q = std::ldexp(1.0, el - 7);
    const double n = std::nearbyint(a / q);   // default rounding mode: to nearest even
    const double r = n * q;
    if (r >= std::ldexp(1.0, 128)) {
      bits = 0x7F80u;             // overflow to infinity
    } else {
      float f = (float)r;         // exact: r has at most 8 significant bits
      uint32_t u;
      std::memcpy(&u, &f, 4);
      bits = u >> 16;
    }
  }
  return (uint16_t)(bits | (neg ? 0x8000u : 0u));
}

struct Pair { double logit; int expert; };

}  // namespace

extern "C" {

// ---- single steps, exported for the pins in tests/ -----------------------
double oracle_e2m1_value(int code) { return e2m1_value((unsigned)code & 15u); }
double oracle_e8m0_value(int s) { return e8m0_value((unsigned)s & 255u); }
uint16_t oracle_round_bf16(double v) { return round_bf16(v); }
double oracle_silu(double g) { return silu(g); }

void oracle_dequant_row(const uint8_t* codes, const uint8_t* scales, int K, double* out) {
  dequant_row(codes, scales, K, out);
}

// logits [B][E] in fp64 from bf16 x [B][H] and bf16 Wr [H][E] (+ fp32 bias [E] or NULL)
void oracle_router_logits(const uint16_t* x, const uint16_t* wr, const float* bias, int B, int H,
                          int E, double* logits) {
  for (int b = 0; b < B; ++b)
    for (int e = 0; e < E; ++e) {
      double s = 0.0;
      for (int h = 0; h < H; ++h) s += bf16_value(x[(size_t)b * H + h]) * bf16_value(wr[(size_t)h * E + e]);
      if (bias) s += (double)bias[e];
      logits[(size_t)b * E + e] = s;
    }
}

// Top-k by a full sort of (-logit, expert id); output ascending expert id and
// the softmax over the selected logits.
void oracle_topk_softmax(const double* logits, int B, int E, int k, int32_t* idx, double* w) {
  std::vector<Pair> p(E);
  for (int b = 0; b < B; ++b) {
    for (int e = 0; e < E; ++e) p[e] = Pair{logits[(size_t)b * E + e], e};
    std::sort(p.begin(), p.end(), [](const Pair& a, const Pair& c) {
      if (a.logit != c.logit) return a.logit > c.logit;
      return a.expert < c.expert;
    });
    std::vector<Pair> sel(p.begin(), p.begin() + k);
    std::sort(sel.begin(), sel.end(), [](const Pair& a, const Pair& c) { return a.expert < c.expert; });
    double m = -INFINITY;
    for (int j = 0; j < k; ++j) m = std::max(m, sel[j].logit);
    double z = 0.0;
    for (int j = 0; j < k; ++j) z += std::exp(sel[j].logit - m);
    for (int j = 0; j < k; ++j) {
      idx[(size_t)b * k + j] = sel[j].expert;
      w[(size_t)b * k + j] = std::exp(sel[j].logit - m) / z;
    }
  }
}

// Sigmoid scoring with a selection bias (the bias-corrected router variant):
// s_e = 1 / (1 + e^-l_e) from the raw logits; the k experts with the largest
// s_e + bias_e are selected (equal values to the lower id; bias NULL = 0),
// listed in ascending id, with weights s_j / sum of the selected s -- the
// bias steers the choice only.
void oracle_topk_sigmoid(const double* logits, const float* bias, int B, int E, int k, int32_t* idx, double* w) {
  std::vector<Pair> p(E);
  std::vector<double> sc(E);
  for (int b = 0; b < B; ++b) {
    for (int e = 0; e < E; ++e) {
      sc[e] = 1.0 / (1.0 + std::exp(-logits[(size_t)b * E + e]));
      p[e] = Pair{sc[e] + (bias ? (double)bias[e] : 0.0), e};
    }
    std::sort(p.begin(), p.end(), [](const Pair& a, const Pair& c) {
      if (a.logit != c.logit) return a.logit > c.logit;
      return a.expert < c.expert;
    });
    std::vector<int> sel(k);
    for (int j = 0; j < k; ++j) sel[j] = p[j].expert;
    std::sort(sel.begin(), sel.end());
    double z = 0.0;
    for (int j = 0; j < k; ++j) z += sc[sel[j]];
    for (int j = 0; j < k; ++j) {
      idx[(size_t)b * k + j] = sel[j];
      w[(size_t)b * k + j] = sc[sel[j]] / z;
    }
  }
}

// Counting sort of pairs p = b*k + j by expert: counts[E], offsets[E+1]
// (exclusive scan), pair_ids[B*k] ordered by (expert, b, j), the ascending
// list of experts with a nonzero count and its length.
void oracle_bucket(const int32_t* idx, int B, int k, int E, int32_t* counts, int32_t* offsets,
                   int32_t* pair_ids, int32_t* active, int32_t* n_active) {
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (int p = 0; p < B * k; ++p) counts[idx[p]] += 1;
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  std::vector<int32_t> fill(offsets, offsets + E);
  for (int p = 0; p < B * k; ++p) pair_ids[fill[idx[p]]++] = p;   // p ascending = (b, j) order
  int na = 0;
  for (int e = 0; e < E; ++e)
    if (counts[e] > 0) active[na++] = e;
  *n_active = na;
}

// One SwiGLU expert with MXFP4 weights, fp64: h[I] (may be NULL) and y[H].
void oracle_expert_ffn(const double* x, const uint8_t* gu_codes, const uint8_t* gu_scales,
                       const uint8_t* d_codes, const uint8_t* d_scales, int H, int I, double* h_out,
                       double* y) {
  std::vector<double> row(std::max(H, I)), h(I);
  for (int i = 0; i < I; ++i) {
    dequant_row(gu_codes + (size_t)i * (H / 2), gu_scales + (size_t)i * (H / 32), H, row.data());
    double g = 0.0;
    for (int c = 0; c < H; ++c) g += row[c] * x[c];
    dequant_row(gu_codes + (size_t)(I + i) * (H / 2), gu_scales + (size_t)(I + i) * (H / 32), H, row.data());
    double u = 0.0;
    for (int c = 0; c < H; ++c) u += row[c] * x[c];
    h[i] = silu(g) * u;
  }
  if (h_out) std::memcpy(h_out, h.data(), sizeof(double) * I);
  for (int r = 0; r < H; ++r) {
    dequant_row(d_codes + (size_t)r * (I / 2), d_scales + (size_t)r * (I / 32), I, row.data());
    double s = 0.0;
    for (int i = 0; i < I; ++i) s += row[i] * h[i];
    y[r] = s;
  }
}

// The shared expert with bf16 weights gate/up [2Is][H] (gate rows first) and down [H][Is].
void oracle_shared_ffn(const double* x, const uint16_t* gu, const uint16_t* d, int H, int Is,
                       double* h_out, double* y) {
  std::vector<double> h(Is);
  for (int i = 0; i < Is; ++i) {
    double g = 0.0, u = 0.0;
    for (int c = 0; c < H; ++c) {
      g += bf16_value(gu[(size_t)i * H + c]) * x[c];
      u += bf16_value(gu[(size_t)(Is + i) * H + c]) * x[c];
    }
    h[i] = silu(g) * u;
  }
  if (h_out) std::memcpy(h_out, h.data(), sizeof(double) * Is);
  for (int r = 0; r < H; ++r) {
    double s = 0.0;
    for (int i = 0; i < Is; ++i) s += bf16_value(d[(size_t)r * Is + i]) * h[i];
    y[r] = s;
  }
}

// The whole layer.  Expert tensors are given by slot: expert e lives in slot
// expert_slot[e] of gu_codes [slots][2I][H/2], gu_scales [slots][2I][H/32],
// d_codes [slots][H][I/2], d_scales [slots][H][I/32]; expert_slot NULL means
// slot = e.  Every output pointer may be NULL.  Returns 0, or -1 when a
// selected expert has no slot, -2 on bad sizes.
//
// Variants (scoring, shared expert format): scoring 0 = softmax over the
// selected logits, the bias added to the logits first (as above); scoring 1
// = oracle_topk_sigmoid on the raw logits, the bias steering selection only
// (logits_out then holds the raw logits).  The shared expert is either bf16
// (shared_gu / shared_d) or, when shared_mx_gu_codes is non-NULL, MXFP4
// tensors of the routed experts' layout: gate/up codes [2Is][H/2], scales
// [2Is][H/32], down codes [H][Is/2], scales [H][Is/32], dequantised exactly.
int oracle_layer_v(int B, int H, int E, int k, int I, int Is, const uint16_t* x, const uint16_t* residual,
                   const uint16_t* router_w, const float* router_bias, const uint8_t* gu_codes,
                   const uint8_t* gu_scales, const uint8_t* d_codes, const uint8_t* d_scales,
                   const int32_t* expert_slot, const uint16_t* shared_gu, const uint16_t* shared_d,
                   int n_threads, double* logits_out, int32_t* topk_idx_out, double* topk_w_out,
                   int32_t* counts, int32_t* offsets, int32_t* pair_ids, int32_t* active,
                   int32_t* n_active, double* h_routed, double* y_routed, double* y_shared,
                   double* out, uint16_t* out_bf16, int scoring, const uint8_t* shared_mx_gu_codes,
                   const uint8_t* shared_mx_gu_scales, const uint8_t* shared_mx_d_codes,
                   const uint8_t* shared_mx_d_scales) {
  if (B <= 0 || H <= 0 || E <= 0 || k <= 0 || k > E || I <= 0 || H % 32 || I % 32 || Is < 0) return -2;
  if (scoring != 0 && scoring != 1) return -2;
  if (shared_mx_gu_codes && Is % 32) return -2;
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#else
  (void)n_threads;
#endif
  std::vector<double> logits((size_t)B * E), w((size_t)B * k);
  std::vector<int32_t> idx((size_t)B * k);
  if (scoring == 0) {
    oracle_router_logits(x, router_w, router_bias, B, H, E, logits.data());
    oracle_topk_softmax(logits.data(), B, E, k, idx.data(), w.data());
  } else {
    oracle_router_logits(x, router_w, nullptr, B, H, E, logits.data());
    oracle_topk_sigmoid(logits.data(), router_bias, B, E, k, idx.data(), w.data());
  }
  for (int p = 0; p < B * k; ++p) {
    const int e = idx[p];
    const int slot = expert_slot ? expert_slot[e] : e;
    if (slot < 0) return -1;
  }
  if (logits_out) std::memcpy(logits_out, logits.data(), sizeof(double) * B * E);
  if (topk_idx_out) std::memcpy(topk_idx_out, idx.data(), sizeof(int32_t) * B * k);
  if (topk_w_out) std::memcpy(topk_w_out, w.data(), sizeof(double) * B * k);
  if (counts && offsets && pair_ids && active && n_active)
    oracle_bucket(idx.data(), B, k, E, counts, offsets, pair_ids, active, n_active);

  std::vector<double> xd((size_t)B * H);
  for (size_t i = 0; i < (size_t)B * H; ++i) xd[i] = bf16_value(x[i]);

  // Routed experts: first every h[p][i], then every y[p][r]; each element is
  // the same sequential sum as in oracle_expert_ffn, the loops over
  // independent elements are spread over threads.
  std::vector<double> yr((size_t)B * k * H), hr((size_t)B * k * I);
  auto slot_of = [&](int p) { return (size_t)(expert_slot ? expert_slot[idx[p]] : idx[p]); };
#pragma omp parallel for schedule(dynamic, 16)
  for (long long pi = 0; pi < (long long)B * k * I; ++pi) {
    const int p = (int)(pi / I), i = (int)(pi % I);
    const double* xb = xd.data() + (size_t)(p / k) * H;
    const size_t sl = slot_of(p);
    const uint8_t* gc = gu_codes + sl * (2 * (size_t)I) * (H / 2);
    const uint8_t* gs = gu_scales + sl * (2 * (size_t)I) * (H / 32);
    std::vector<double> row(H);
    dequant_row(gc + (size_t)i * (H / 2), gs + (size_t)i * (H / 32), H, row.data());
    double g = 0.0;
    for (int c = 0; c < H; ++c) g += row[c] * xb[c];
    dequant_row(gc + (size_t)(I + i) * (H / 2), gs + (size_t)(I + i) * (H / 32), H, row.data());
    double u = 0.0;
    for (int c = 0; c < H; ++c) u += row[c] * xb[c];
    hr[pi] = silu(g) * u;
  }
#pragma omp parallel for schedule(dynamic, 64)
  for (long long pr = 0; pr < (long long)B * k * H; ++pr) {
    const int p = (int)(pr / H), r = (int)(pr % H);
    const size_t sl = slot_of(p);
    std::vector<double> row(I);
    dequant_row(d_codes + sl * (size_t)H * (I / 2) + (size_t)r * (I / 2),
                d_scales + sl * (size_t)H * (I / 32) + (size_t)r * (I / 32), I, row.data());
    const double* h = hr.data() + (size_t)p * I;
    double acc = 0.0;
    for (int i = 0; i < I; ++i) acc += row[i] * h[i];
    yr[pr] = acc;
  }
  // Shared expert, same structure.
  std::vector<double> ys((size_t)B * H, 0.0);
  if (Is > 0 && shared_mx_gu_codes) {
    // MXFP4 shared expert: every token, weight 1, exact dequantisation
    std::vector<double> hs((size_t)B * Is);
#pragma omp parallel for schedule(dynamic, 16)
    for (long long bi = 0; bi < (long long)B * Is; ++bi) {
      const int b = (int)(bi / Is), i = (int)(bi % Is);
      const double* xb = xd.data() + (size_t)b * H;
      std::vector<double> row(H);
      dequant_row(shared_mx_gu_codes + (size_t)i * (H / 2), shared_mx_gu_scales + (size_t)i * (H / 32), H,
                  row.data());
      double g = 0.0;
      for (int c = 0; c < H; ++c) g += row[c] * xb[c];
      dequant_row(shared_mx_gu_codes + (size_t)(Is + i) * (H / 2), shared_mx_gu_scales + (size_t)(Is + i) * (H / 32),
                  H, row.data());
      double u = 0.0;
      for (int c = 0; c < H; ++c) u += row[c] * xb[c];
      hs[bi] = silu(g) * u;
    }
#pragma omp parallel for schedule(dynamic, 64)
    for (long long br = 0; br < (long long)B * H; ++br) {
      const int b = (int)(br / H), r = (int)(br % H);
      std::vector<double> row(Is);
      dequant_row(shared_mx_d_codes + (size_t)r * (Is / 2), shared_mx_d_scales + (size_t)r * (Is / 32), Is,
                  row.data());
      double acc = 0.0;
      for (int i = 0; i < Is; ++i) acc += row[i] * hs[(size_t)b * Is + i];
      ys[br] = acc;
    }
  } else if (Is > 0 && shared_gu && shared_d) {
    std::vector<double> hs((size_t)B * Is);
#pragma omp parallel for schedule(dynamic, 16)
    for (long long bi = 0; bi < (long long)B * Is; ++bi) {
      const int b = (int)(bi / Is), i = (int)(bi % Is);
      const double* xb = xd.data() + (size_t)b * H;
      double g = 0.0, u = 0.0;
      for (int c = 0; c < H; ++c) {
        g += bf16_value(shared_gu[(size_t)i * H + c]) * xb[c];
        u += bf16_value(shared_gu[(size_t)(Is + i) * H + c]) * xb[c];
      }
      hs[bi] = silu(g) * u;
    }
#pragma omp parallel for schedule(dynamic, 64)
    for (long long br = 0; br < (long long)B * H; ++br) {
      const int b = (int)(br / H), r = (int)(br % H);
      double acc = 0.0;
      for (int i = 0; i < Is; ++i) acc += bf16_value(shared_d[(size_t)r * Is + i]) * hs[(size_t)b * Is + i];
      ys[br] = acc;
    }
  }
  if (h_routed) std::memcpy(h_routed, hr.data(), sizeof(double) * B * k * I);
  if (y_routed) std::memcpy(y_routed, yr.data(), sizeof(double) * B * k * H);
  if (y_shared) std::memcpy(y_shared, ys.data(), sizeof(double) * B * H);

  for (int b = 0; b < B; ++b)
    for (int r = 0; r < H; ++r) {
      double o = bf16_value(residual[(size_t)b * H + r]) + ys[(size_t)b * H + r];
      for (int j = 0; j < k; ++j)   // idx is ascending in expert id within a token
        o += w[(size_t)b * k + j] * yr[((size_t)b * k + j) * H + r];
      if (out) out[(size_t)b * H + r] = o;
      if (out_bf16) out_bf16[(size_t)b * H + r] = round_bf16(o);
    }
  return 0;
}

// The layer with the default variants: softmax scoring, bf16 shared expert.
int oracle_layer(int B, int H, int E, int k, int I, int Is, const uint16_t* x, const uint16_t* residual,
                 const uint16_t* router_w, const float* router_bias, const uint8_t* gu_codes,
                 const uint8_t* gu_scales, const uint8_t* d_codes, const uint8_t* d_scales,
                 const int32_t* expert_slot, const uint16_t* shared_gu, const uint16_t* shared_d,
                 int n_threads, double* logits_out, int32_t* topk_idx_out, double* topk_w_out,
                 int32_t* counts, int32_t* offsets, int32_t* pair_ids, int32_t* active,
                 int32_t* n_active, double* h_routed, double* y_routed, double* y_shared,
                 double* out, uint16_t* out_bf16) {
  return oracle_layer_v(B, H, E, k, I, Is, x, residual, router_w, router_bias, gu_codes, gu_scales, d_codes,
                        d_scales, expert_slot, shared_gu, shared_d, n_threads, logits_out, topk_idx_out, topk_w_out,
                        counts, offsets, pair_ids, active, n_active, h_routed, y_routed, y_shared, out, out_bf16, 0,
                        nullptr, nullptr, nullptr, nullptr);
}

}  // extern "C"
