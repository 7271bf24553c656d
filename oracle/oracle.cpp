// CPU oracle for the Nemotron-H MoE FFN layer forward pass, in float64.
//
// TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct
// statement of what the layer computes.  Only the tests, the smoke check and
// the benchmark's CPU-baseline leg may load it.  It shares no code, header,
// table or helper with the CUDA library, and the library never calls it.
//
// What it follows (page = "NemotronMoeLayer" rustdoc and its source
// nemotron_moe.rs; "MoeLayer" = the generic MoE component page):
//   * forward order: nemotron_moe.rs, module documentation.  The tokens are
//     normalised, gated and routed (sigmoid top-k); the routed experts run
//     up, relu^2 and down (inside fc1 / fc2 when latent) and are combined
//     with the routing weights; the shared expert (up, relu^2, down) is added,
//     and so is the layer input;
//   * direct vs LatentMoE shapes: same module documentation;
//   * norm -> gate -> shared up -> fc1 order and the scaling factor:
//     nemotron_moe.rs, `prefill`;
//   * sort / grouped GEMM / unpermute + weighted reduce pipeline: MoeLayer,
//     `forward_prefill`;
//   * top_k validation: nemotron_moe.rs, `new` and the module invariants.
// Readings where the pages are silent (each one stated here):
//   R1 the residual buffer receives the pre-layer hidden; output =
//      hidden + routed + shared (its input value is not read);
//   R2 gate logits from the un-rounded normed vector;
//   R3 the gate bias is added to the sigmoid scores for selection only;
//   R4 selected scores are renormalised to sum 1, then multiplied by
//      routed_scaling_factor;
//   R5 ties go to the lower expert index; slots are ordered by key
//      descending, then index ascending;
//   R6 relu^2(x) = max(x, 0)^2; experts are non-gated (up, relu^2, down);
//   R7 the shared expert is unweighted and works on the normed vector in H;
//   R8 LatentMoE: gate on the normed vector, fc1 on the normed vector, the
//      weighted sum in latent space, then fc2;
//   R9 the norm weight multiplies directly (x * r * w);
//   R10 FP8 weights (routed experts, and optionally the shared expert and
//      fc1 / fc2, which the pages also keep as FP8 copies: nemotron_moe.rs
//      `new`) are E4M3 bytes times one float32 scale per output row, taken
//      exactly; activations are never quantised here.
// Parity pins: tests/test_oracle_pins.py (closed forms, brute-force subset
// enumeration, hand-computed cases, invariants).
#include <cmath>
#include <cstdint>
#include <cstring>
#include <algorithm>
#include <thread>
#include <vector>

extern "C" {

typedef struct {
  int32_t H, E, k, I, S, L;  // L = moe_latent_size, 0 = direct
  double eps;                // rms_norm_eps
  double rsf;                // routed_scaling_factor
  int32_t expert_fp8;        // 0: routed weights BF16; 1: FP8 E4M3 + FP32 row scale
  int32_t shared_fp8;        // shared expert weights: 0 BF16, 1 FP8 E4M3 + FP32 row scale
  int32_t latent_fp8;        // fc1 / fc2 weights: 0 BF16, 1 FP8 E4M3 + FP32 row scale
} oracle_cfg;

typedef struct {
  const uint16_t* norm_w;         // [H]    bf16
  const uint16_t* gate_w;         // [E,H]  bf16
  const float* gate_bias;         // [E]    or NULL
  const void* up_w;               // [E,I,D] bf16 or e4m3
  const void* down_w;             // [E,D,I] bf16 or e4m3
  const float* up_scale;          // [E,I]  (fp8 only)
  const float* down_scale;        // [E,D]  (fp8 only)
  const void* shared_up_w;        // [S,H]  bf16 or e4m3
  const void* shared_down_w;      // [H,S]  bf16 or e4m3
  const void* fc1_w;              // [L,H]  bf16 or e4m3 (latent only)
  const void* fc2_w;              // [H,L]  bf16 or e4m3 (latent only)
  const float* shared_up_scale;   // [S]    (shared_fp8 only)
  const float* shared_down_scale; // [H]    (shared_fp8 only)
  const float* fc1_scale;         // [L]    (latent_fp8 only)
  const float* fc2_scale;         // [H]    (latent_fp8 only)
} oracle_weights;

}  // extern "C"

namespace {

// BF16 is the upper half of an IEEE binary32.
double bf16(uint16_t b) {
  uint32_t u = uint32_t(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return double(f);
}

// OCP FP8 E4M3 ("fn" variant: no infinities, S.1111.111 is NaN), bias 7.
double e4m3(uint8_t b) {
  int sign = (b >> 7) & 1;
  int ex = (b >> 3) & 0xF;
  int man = b & 7;
  double v;
  if (ex == 0xF && man == 7) return NAN;
  if (ex == 0)
    v = std::ldexp(double(man) / 8.0, -6);
  else
    v = std::ldexp(1.0 + double(man) / 8.0, ex - 7);
  return sign ? -v : v;
}

// The 256 E4M3 values, each computed once (when the library loads) by
// e4m3() above: looking a byte up here gives exactly e4m3(byte), without its
// per-call ldexp.
struct E4M3Table {
  double v[256];
  E4M3Table() {
    for (int b = 0; b < 256; ++b) v[b] = e4m3(uint8_t(b));
  }
};
const E4M3Table kE4M3;

// Element (e, r, c) of a routed expert stack [E, rows, cols], dequantised.
double expert_w(const oracle_cfg& c, const void* w, const float* scale,
                int e, int r, int rows, int col, int cols) {
  size_t i = (size_t(e) * rows + r) * size_t(cols) + col;
  if (c.expert_fp8)
    return kE4M3.v[static_cast<const uint8_t*>(w)[i]] * double(scale[size_t(e) * rows + r]);
  return bf16(static_cast<const uint16_t*>(w)[i]);
}

// Element (r, col) of a dense [rows, cols] weight (shared expert, fc1,
// fc2), dequantised the same way as the routed experts when fp8 is set:
// e4m3 value times the row's scale.
double dense_w(const void* w, const float* scale, int fp8, int r, int col, int cols) {
  size_t i = size_t(r) * size_t(cols) + col;
  if (fp8) return kE4M3.v[static_cast<const uint8_t*>(w)[i]] * double(scale[r]);
  return bf16(static_cast<const uint16_t*>(w)[i]);
}

double relu2(double x) { return x > 0.0 ? x * x : 0.0; }

double sigmoid(double x) { return 1.0 / (1.0 + std::exp(-x)); }

// RMSNorm of one token: n_i = x_i * w_i / sqrt(mean_j x_j^2 + eps).
void rmsnorm(const oracle_cfg& c, const oracle_weights& w, const uint16_t* x, double* n) {
  double ss = 0.0;
  for (int i = 0; i < c.H; ++i) ss += bf16(x[i]) * bf16(x[i]);
  double r = 1.0 / std::sqrt(ss / c.H + c.eps);
  for (int i = 0; i < c.H; ++i) n[i] = bf16(x[i]) * r * bf16(w.norm_w[i]);
}

// logit_e = sum_i n_i * G[e, i]
void gate(const oracle_cfg& c, const oracle_weights& w, const double* n, double* logit) {
  for (int e = 0; e < c.E; ++e) {
    double a = 0.0;
    for (int i = 0; i < c.H; ++i) a += n[i] * bf16(w.gate_w[size_t(e) * c.H + i]);
    logit[e] = a;
  }
}

// Sigmoid top-k of one token.  key_e = sigmoid(logit_e) + bias_e picks the
// experts; the weights come from the unbiased scores of the picked set.
// If `forced` is given the set (and slot order) is taken from it instead.
void route(const oracle_cfg& c, const double* logit, const float* bias,
           const int32_t* forced, int32_t* idx, double* wts, double* keys) {
  std::vector<double> s(c.E), key(c.E);
  for (int e = 0; e < c.E; ++e) {
    s[e] = sigmoid(logit[e]);
    key[e] = s[e] + (bias ? double(bias[e]) : 0.0);
    if (keys) keys[e] = key[e];
  }
  if (forced) {
    for (int j = 0; j < c.k; ++j) idx[j] = forced[j];
  } else {
    std::vector<int32_t> order(c.E);
    for (int e = 0; e < c.E; ++e) order[e] = e;
    std::stable_sort(order.begin(), order.end(),
                     [&](int32_t a, int32_t b) { return key[a] > key[b]; });
    for (int j = 0; j < c.k; ++j) idx[j] = order[j];
  }
  double sum = 0.0;
  for (int j = 0; j < c.k; ++j) sum += s[idx[j]];
  for (int j = 0; j < c.k; ++j) wts[j] = c.rsf * s[idx[j]] / sum;
}

// y = relu^2(z . Wup_e^T) . Wdown_e^T for one routed expert, z of width D.
void routed_expert(const oracle_cfg& c, const oracle_weights& w, int e, const double* z,
                   double* y, std::vector<double>& u) {
  const int D = c.L > 0 ? c.L : c.H;
  u.assign(c.I, 0.0);
  for (int i = 0; i < c.I; ++i) {
    double a = 0.0;
    for (int d = 0; d < D; ++d) a += z[d] * expert_w(c, w.up_w, w.up_scale, e, i, c.I, d, D);
    u[i] = relu2(a);
  }
  for (int d = 0; d < D; ++d) {
    double a = 0.0;
    for (int i = 0; i < c.I; ++i) a += u[i] * expert_w(c, w.down_w, w.down_scale, e, d, D, i, c.I);
    y[d] = a;
  }
}

// out = x + [fc2](sum_j w_j * expert_j([fc1](n))) + shared(n) for one token.
void token_forward(const oracle_cfg& c, const oracle_weights& w, const uint16_t* x,
                   const int32_t* forced, double* out, int32_t* idx, double* wts) {
  const int H = c.H, D = c.L > 0 ? c.L : c.H;
  std::vector<double> n(H), logit(c.E), z(D), y(D), m(D, 0.0), u, v(c.S);
  rmsnorm(c, w, x, n.data());
  gate(c, w, n.data(), logit.data());
  route(c, logit.data(), w.gate_bias, forced, idx, wts, nullptr);
  if (c.L > 0) {
    for (int l = 0; l < c.L; ++l) {
      double a = 0.0;
      for (int i = 0; i < H; ++i) a += n[i] * dense_w(w.fc1_w, w.fc1_scale, c.latent_fp8, l, i, H);
      z[l] = a;
    }
  } else {
    for (int i = 0; i < H; ++i) z[i] = n[i];
  }
  for (int j = 0; j < c.k; ++j) {
    routed_expert(c, w, idx[j], z.data(), y.data(), u);
    for (int d = 0; d < D; ++d) m[d] += wts[j] * y[d];
  }
  std::vector<double> routed(H);
  if (c.L > 0) {
    for (int h = 0; h < H; ++h) {
      double a = 0.0;
      for (int l = 0; l < c.L; ++l) a += m[l] * dense_w(w.fc2_w, w.fc2_scale, c.latent_fp8, h, l, c.L);
      routed[h] = a;
    }
  } else {
    for (int h = 0; h < H; ++h) routed[h] = m[h];
  }
  for (int s = 0; s < c.S; ++s) {
    double a = 0.0;
    for (int i = 0; i < H; ++i) a += n[i] * dense_w(w.shared_up_w, w.shared_up_scale, c.shared_fp8, s, i, H);
    v[s] = relu2(a);
  }
  for (int h = 0; h < H; ++h) {
    double a = 0.0;
    for (int s = 0; s < c.S; ++s) a += v[s] * dense_w(w.shared_down_w, w.shared_down_scale, c.shared_fp8, h, s, c.S);
    out[h] = bf16(x[h]) + routed[h] + a;
  }
}

template <class F>
void parallel_tokens(int T, int nthreads, F f) {
  if (nthreads <= 0) nthreads = int(std::thread::hardware_concurrency());
  if (nthreads < 1) nthreads = 1;
  if (nthreads > T) nthreads = T;
  if (nthreads <= 1) {
    for (int t = 0; t < T; ++t) f(t);
    return;
  }
  std::vector<std::thread> pool;
  for (int p = 0; p < nthreads; ++p)
    pool.emplace_back([=, &f]() {
      for (int t = p; t < T; t += nthreads) f(t);
    });
  for (auto& th : pool) th.join();
}

int check_cfg(const oracle_cfg* c) {
  if (!c) return 1;
  if (c->H <= 0 || c->E <= 0 || c->I <= 0 || c->S <= 0 || c->L < 0) return 1;
  if (c->k < 1 || c->k > c->E) return 1;
  return 0;
}

}  // namespace

extern "C" {

// Number of threads the forward pass uses for nthreads <= 0.
int oracle_default_threads(void) {
  int n = int(std::thread::hardware_concurrency());
  return n > 0 ? n : 1;
}

// normed [T,H] (float64)
int oracle_rmsnorm(const oracle_cfg* c, const oracle_weights* w, const uint16_t* hidden,
                   int32_t T, double* normed) {
  if (check_cfg(c) || T < 0) return 1;
  for (int t = 0; t < T; ++t) rmsnorm(*c, *w, hidden + size_t(t) * c->H, normed + size_t(t) * c->H);
  return 0;
}

// logits [T,E] from hidden (norm then gate)
int oracle_gate_logits(const oracle_cfg* c, const oracle_weights* w, const uint16_t* hidden,
                       int32_t T, double* logits, int32_t nthreads) {
  if (check_cfg(c) || T < 0) return 1;
  parallel_tokens(T, nthreads, [&](int t) {
    std::vector<double> n(c->H);
    rmsnorm(*c, *w, hidden + size_t(t) * c->H, n.data());
    gate(*c, *w, n.data(), logits + size_t(t) * c->E);
  });
  return 0;
}

// Routing of T tokens from their logits: idx [T,k], wts [T,k], keys [T,E] (nullable).
int oracle_route(const oracle_cfg* c, const double* logits, const float* bias, int32_t T,
                 int32_t* idx, double* wts, double* keys) {
  if (check_cfg(c) || T < 0) return 1;
  for (int t = 0; t < T; ++t)
    route(*c, logits + size_t(t) * c->E, bias, nullptr, idx + size_t(t) * c->k,
          wts + size_t(t) * c->k, keys ? keys + size_t(t) * c->E : nullptr);
  return 0;
}

// Weights of given expert sets: forced [T,k] takes the place of the top-k
// choice (slot order kept), wts [T,k] = rsf * s_e / sum of the set's s_e.
int oracle_route_forced(const oracle_cfg* c, const double* logits, const int32_t* forced,
                        int32_t T, double* wts) {
  if (check_cfg(c) || T < 0 || !forced) return 1;
  std::vector<int32_t> idx(c->k);
  for (int t = 0; t < T; ++t) {
    for (int j = 0; j < c->k; ++j)
      if (forced[size_t(t) * c->k + j] < 0 || forced[size_t(t) * c->k + j] >= c->E) return 1;
    route(*c, logits + size_t(t) * c->E, nullptr, forced + size_t(t) * c->k, idx.data(),
          wts + size_t(t) * c->k, nullptr);
  }
  return 0;
}

// Sort the R = T*k routed rows by expert (counting sort, stable in row
// order f = t*k + j): perm[pos] = f, inv[f] = pos, off[E+1] exclusive prefix
// of the per-expert counts.  Returns 1 on an expert id outside [0, E).
int oracle_sort(const int32_t* idx, int32_t T, int32_t k, int32_t E, int32_t* perm,
                int32_t* inv, int32_t* off) {
  const int R = T * k;
  std::vector<int32_t> cnt(E, 0), fill(E, 0);
  for (int f = 0; f < R; ++f) {
    if (idx[f] < 0 || idx[f] >= E) return 1;
    cnt[idx[f]]++;
  }
  off[0] = 0;
  for (int e = 0; e < E; ++e) off[e + 1] = off[e] + cnt[e];
  for (int f = 0; f < R; ++f) {
    int e = idx[f];
    int pos = off[e] + fill[e]++;
    perm[pos] = f;
    inv[f] = pos;
  }
  return 0;
}

// Full layer: out [T,H] float64 (not rounded), idx [T,k], wts [T,k].
// forced_idx [T,k] (nullable) replaces the top-k choice for every token.
int oracle_forward(const oracle_cfg* c, const oracle_weights* w, const uint16_t* hidden,
                   int32_t T, const int32_t* forced_idx, double* out, int32_t* idx,
                   double* wts, int32_t nthreads) {
  if (check_cfg(c) || T < 0) return 1;
  if (c->L > 0 && (!w->fc1_w || !w->fc2_w)) return 1;
  if (c->expert_fp8 && (!w->up_scale || !w->down_scale)) return 1;
  if (c->shared_fp8 && (!w->shared_up_scale || !w->shared_down_scale)) return 1;
  if (c->L > 0 && c->latent_fp8 && (!w->fc1_scale || !w->fc2_scale)) return 1;
  parallel_tokens(T, nthreads, [&](int t) {
    token_forward(*c, *w, hidden + size_t(t) * c->H,
                  forced_idx ? forced_idx + size_t(t) * c->k : nullptr,
                  out + size_t(t) * c->H, idx + size_t(t) * c->k, wts + size_t(t) * c->k);
  });
  return 0;
}

// Decoders of the storage formats (for the pins).
double oracle_bf16_value(uint16_t b) { return bf16(b); }
double oracle_e4m3_value(uint8_t b) { return e4m3(b); }

}  // extern "C"
