// ORACLE — test infrastructure only.
//
// A plain, slow, obviously correct CPU statement of the sparse MoE layer
// forward and of the SparseClip norm.  Only the test suite, the smoke check
// and the benchmark's CPU-baseline leg may load this library; the product
// path (the CUDA library) never does, and the two share no code.
//
// Sources (page title, then section / equation):
//   * "Switch Transformers: Scaling to Trillion Parameter Models with Simple
//     and Efficient Sparsity" (study notes), sec. 2.1 eq. (1) softmax gate,
//     eq. (2) gate-weighted combine, top-k set T; sec. 2.2 eq. (3) expert
//     capacity and the drop rule (overflowing tokens skip the expert and
//     reach the next layer through the residual, so the layer adds 0 for
//     them); sec. 2.4 "selective precision": the router works in float32.
//   * "[Paper review] TorchScale: Transformers at Scale", proposed method:
//     X-MoE top-1 / top-2 routing; SparseClip ||g||_2 = ||(g_d, kappa g_s)||_2
//     with kappa = 1/sqrt(E); key results: the routing entropy it tracks.
//   * Switch notes sec. 2.2, the differentiable load-balancing loss, eqs.
//     (4)-(6).
//   * "[Paper review] PanGu-Sigma", proposed method: Random Routed Experts —
//     experts grouped by domain, each token sent uniformly at random to an
//     expert of its domain's group through an unweighted gate.
//
// Readings taken where the pages are silent:
//   * capacity: C = floor(T * capacity_factor / E), passed on as an integer;
//   * top-k is taken on the fp32 logits (softmax is monotone), ties go to
//     the lowest expert index; the k gates are the raw softmax values of
//     eq. (1) (no renormalisation over T);
//   * slots are granted in token order, token t's k choices before token
//     t+1's; a choice whose slot is >= C is dropped;
//   * expert FFN: d_model -> d_ff -> d_model, ReLU, no biases; H and the
//     expert output are rounded to the activation type; the combine sums in
//     double and rounds once;
//   * RRE: group g owns experts [g*E/G, (g+1)*E/G); the in-group index is
//     splitmix64(seed, t) mod (E/G), gate 1.
//   * GLU experts ("MosaicBERT" page: GLU in the feed-forward layer, no
//     formula): the GEGLU form, GELU(x W_gate) * (x W_linear), erf GELU, no
//     biases, W1 rows interleaved (gate of unit i in row 2i, linear in 2i+1).
//
// Arithmetic: every product and sum is in double; values are rounded to the
// activation type only at the points named above.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

enum { DT_BF16 = 0, DT_F32 = 1 };

// ---- number formats -------------------------------------------------------

double bf16_bits_to_double(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return static_cast<double>(f);
}

// Round a double to the nearest bfloat16 (8 significant bits, fp32 exponent
// range), ties to even, directly from the double (no intermediate float).
uint16_t double_to_bf16_bits(double v) {
  if (v == 0.0) return std::signbit(v) ? 0x8000 : 0x0000;
  if (std::isnan(v)) return 0x7FC0;
  double a = std::fabs(v);
  int e;
  std::frexp(a, &e);  // a = m * 2^e with m in [0.5, 1)
  // spacing of bf16 numbers around a: 2^(e-8) for normals, 2^-133 below 2^-126
  int q = e - 8;
  if (q < -133) q = -133;
  double scaled = std::ldexp(a, -q);    // exact (power-of-two scaling)
  double r = std::nearbyint(scaled);    // default mode: to nearest, ties to even
  double rounded = std::ldexp(r, q);
  if (rounded > 3.3895313892515355e38) rounded = INFINITY;  // above bf16 max
  float f = static_cast<float>(rounded);                    // exact
  uint32_t u;
  std::memcpy(&u, &f, 4);
  uint16_t bits = static_cast<uint16_t>(u >> 16);
  return std::signbit(v) ? static_cast<uint16_t>(bits | 0x8000) : bits;
}

double load(const void* p, int64_t i, int dtype) {
  if (dtype == DT_BF16) return bf16_bits_to_double(static_cast<const uint16_t*>(p)[i]);
  return static_cast<double>(static_cast<const float*>(p)[i]);
}

// Store a double rounded once to the activation type; returns the stored value.
double store(void* p, int64_t i, int dtype, double v) {
  if (dtype == DT_BF16) {
    uint16_t b = double_to_bf16_bits(v);
    static_cast<uint16_t*>(p)[i] = b;
    return bf16_bits_to_double(b);
  }
  float f = static_cast<float>(v);
  static_cast<float*>(p)[i] = f;
  return static_cast<double>(f);
}

// ---- splitmix64 (Steele, Lea & Flood, OOPSLA 2014) --------------------------
// Output #t (0-based) of the generator seeded with `seed`: the state is
// seed + (t+1) * golden-gamma, passed through the published finaliser.
uint64_t splitmix64_at(uint64_t seed, uint64_t t) {
  uint64_t z = seed + (t + 1) * 0x9E3779B97F4A7C15ULL;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

template <class F>
void parallel_for(int64_t n, int threads, F fn) {
  if (threads <= 1 || n < 2) {
    for (int64_t i = 0; i < n; ++i) fn(i);
    return;
  }
  std::vector<std::thread> pool;
  int64_t chunk = (n + threads - 1) / threads;
  for (int w = 0; w < threads; ++w) {
    int64_t b = w * chunk, e = std::min<int64_t>(n, b + chunk);
    if (b >= e) break;
    pool.emplace_back([=] {
      for (int64_t i = b; i < e; ++i) fn(i);
    });
  }
  for (auto& th : pool) th.join();
}

}  // namespace

extern "C" {

uint64_t oracle_splitmix64(uint64_t seed, uint64_t t) { return splitmix64_at(seed, t); }

uint16_t oracle_round_bf16(double v) { return double_to_bf16_bits(v); }

// Switch notes sec. 2.2, eq. (3): capacity = (tokens per batch / experts) x
// capacity factor, taken as the floor.
int32_t oracle_capacity(int64_t T, int32_t E, double capacity_factor) {
  return static_cast<int32_t>(std::floor(static_cast<double>(T) / E * capacity_factor));
}

// Switch notes sec. 2.1: logits h(x) = W_r . x.  Sec. 2.4: the router runs in
// float32 — here every product and the sum are exact-ish in double and the
// logit is rounded once to fp32.  bias (nullable) is added per expert.
void oracle_router(int64_t T, int32_t d, int32_t E, int32_t dtype, const void* x,
                   const void* Wr, const float* bias, float* logits, int32_t threads) {
  parallel_for(T, threads, [&](int64_t t) {
    for (int32_t e = 0; e < E; ++e) {
      double s = 0.0;
      for (int32_t c = 0; c < d; ++c)
        s += load(x, t * d + c, dtype) * load(Wr, static_cast<int64_t>(e) * d + c, dtype);
      if (bias) s += static_cast<double>(bias[e]);
      logits[t * E + e] = static_cast<float>(s);
    }
  });
}

// Switch notes sec. 2.1, eq. (1) gate p_i = exp(h_i) / sum_j exp(h_j) over all
// E experts (evaluated as exp(h_i - max) / sum exp(h_j - max), the same
// number), and the top-k set T.  Selection order: larger fp32 logit first,
// equal logits -> lower index first.  gate[t*k+j] = p of the j-th choice,
// rounded to fp32.  prob_sum (nullable) receives sum_i p_i per token.
void oracle_gate_topk(int64_t T, int32_t E, int32_t k, const float* logits,
                      int32_t* expert_idx, float* gate, double* prob_sum) {
  std::vector<int32_t> order(E);
  for (int64_t t = 0; t < T; ++t) {
    const float* h = logits + t * E;
    double m = -INFINITY;
    for (int32_t e = 0; e < E; ++e) m = std::max(m, static_cast<double>(h[e]));
    double z = 0.0;
    for (int32_t e = 0; e < E; ++e) z += std::exp(static_cast<double>(h[e]) - m);
    for (int32_t e = 0; e < E; ++e) order[e] = e;
    std::stable_sort(order.begin(), order.end(),
                     [&](int32_t a, int32_t b) { return h[a] > h[b]; });
    for (int32_t j = 0; j < k; ++j) {
      int32_t e = order[j];
      expert_idx[t * k + j] = e;
      gate[t * k + j] = static_cast<float>(std::exp(static_cast<double>(h[e]) - m) / z);
    }
    if (prob_sum) {
      double s = 0.0;
      for (int32_t e = 0; e < E; ++e) s += std::exp(static_cast<double>(h[e]) - m) / z;
      prob_sum[t] = s;
    }
  }
}

// PanGu-Sigma review, Random Routed Experts: token t of domain g goes to an
// expert of group g chosen uniformly at random, with an unweighted gate (1).
// k = 1.  Group g holds experts [g*E/G, (g+1)*E/G).
void oracle_route_rre(int64_t T, int32_t E, int32_t G, uint64_t seed, const int32_t* domain,
                      int32_t* expert_idx, float* gate) {
  const int32_t per = E / G;
  for (int64_t t = 0; t < T; ++t) {
    uint64_t r = splitmix64_at(seed, static_cast<uint64_t>(t));
    expert_idx[t] = domain[t] * per + static_cast<int32_t>(r % static_cast<uint64_t>(per));
    gate[t] = 1.0f;
  }
}

// Switch notes sec. 2.2: each expert takes at most C tokens; the rest are
// dropped.  Walk the assignments in token order; the slot of an assignment is
// the number of earlier assignments to the same expert.  tok_of_row[e*C+s] is
// the token in slot s of expert e (-1 where no token).  Returns nothing;
// arrivals/kept_cnt are per expert, n_dropped the total overflow.
void oracle_assign(int64_t T, int32_t E, int32_t k, int32_t C, const int32_t* expert_idx,
                   int32_t* slot, uint8_t* kept, int32_t* tok_of_row, int32_t* arrivals,
                   int32_t* kept_cnt, int64_t* n_dropped) {
  for (int32_t e = 0; e < E; ++e) arrivals[e] = 0;
  for (int64_t r = 0; r < static_cast<int64_t>(E) * C; ++r) tok_of_row[r] = -1;
  for (int64_t t = 0; t < T; ++t) {
    for (int32_t j = 0; j < k; ++j) {
      int32_t e = expert_idx[t * k + j];
      int32_t s = arrivals[e]++;
      slot[t * k + j] = s;
      kept[t * k + j] = s < C ? 1 : 0;
      if (s < C) tok_of_row[static_cast<int64_t>(e) * C + s] = static_cast<int32_t>(t);
    }
  }
  int64_t dropped = 0;
  for (int32_t e = 0; e < E; ++e) {
    kept_cnt[e] = std::min(arrivals[e], C);
    dropped += std::max(0, arrivals[e] - C);
  }
  *n_dropped = dropped;
}

// Dispatch (the permutation behind the Switch router's dispatch tensor, sec.
// 2.4): xe[e, r, :] = x[tok_of_row[e*C+r], :] for r < kept_cnt[e]; other rows
// are left untouched.
void oracle_dispatch(int64_t T, int32_t d, int32_t E, int32_t C, int32_t dtype, const void* x,
                     const int32_t* tok_of_row, const int32_t* kept_cnt, void* xe) {
  (void)T;
  const size_t es = dtype == DT_BF16 ? 2 : 4;
  for (int32_t e = 0; e < E; ++e)
    for (int32_t r = 0; r < kept_cnt[e]; ++r) {
      int64_t t = tok_of_row[static_cast<int64_t>(e) * C + r];
      std::memcpy(static_cast<char*>(xe) + ((static_cast<int64_t>(e) * C + r) * d) * es,
                  static_cast<const char*>(x) + t * d * es, d * es);
    }
}

// One expert applied to one token row (Switch notes sec. 2.1: E_i(x) is a
// feed-forward network): H = round(ReLU(x . W1^T)), out = round(H . W2^T).
// W1 is [f, d], W2 is [d, f], both row-major.  H_out (nullable) receives H.
void oracle_expert_row(int32_t d, int32_t f, int32_t dtype, const void* x_row, const void* W1,
                       const void* W2, void* out_row, void* H_out) {
  std::vector<double> H(f);
  std::vector<uint32_t> hbuf(f);  // scratch for rounding when H_out is null
  void* hdst = H_out ? H_out : static_cast<void*>(hbuf.data());
  for (int32_t n = 0; n < f; ++n) {
    double a = 0.0;
    for (int32_t c = 0; c < d; ++c)
      a += load(x_row, c, dtype) * load(W1, static_cast<int64_t>(n) * d + c, dtype);
    H[n] = store(hdst, n, dtype, a > 0.0 ? a : 0.0);
  }
  for (int32_t c = 0; c < d; ++c) {
    double o = 0.0;
    for (int32_t n = 0; n < f; ++n) o += H[n] * load(W2, static_cast<int64_t>(c) * f + n, dtype);
    store(out_row, c, dtype, o);
  }
}

// All experts over their kept rows: ye[e, r] = E_e(xe[e, r]) for r < kept_cnt[e].
// W1 is [E, f, d], W2 is [E, d, f].  H (nullable) is [E, C, f].
// Gated linear unit in the feed-forward layer ("MosaicBERT" page: the FFN
// uses GLU), GEGLU form: W1 [2f, d] holds, for hidden unit i, the gate
// projection in row 2i and the linear projection in row 2i+1;
//   H_i = GELU(x . W1[2i]) * (x . W1[2i+1]),  GELU(a) = a * Phi(a) = a (1 + erf(a / sqrt 2)) / 2,
// in double, rounded once to the activation type; out = H . W2^T as for ReLU.
void oracle_expert_row_geglu(int32_t d, int32_t f, int32_t dtype, const void* x_row,
                             const void* W1, const void* W2, void* out_row, void* H_out) {
  std::vector<double> H(f);
  std::vector<uint32_t> hbuf(f);
  void* hdst = H_out ? H_out : static_cast<void*>(hbuf.data());
  for (int32_t i = 0; i < f; ++i) {
    double g = 0.0, l = 0.0;
    for (int32_t c = 0; c < d; ++c) {
      const double xv = load(x_row, c, dtype);
      g += xv * load(W1, static_cast<int64_t>(2 * i) * d + c, dtype);
      l += xv * load(W1, static_cast<int64_t>(2 * i + 1) * d + c, dtype);
    }
    const double gelu = 0.5 * g * (1.0 + std::erf(g / std::sqrt(2.0)));
    H[i] = store(hdst, i, dtype, gelu * l);
  }
  for (int32_t c = 0; c < d; ++c) {
    double o = 0.0;
    for (int32_t n = 0; n < f; ++n) o += H[n] * load(W2, static_cast<int64_t>(c) * f + n, dtype);
    store(out_row, c, dtype, o);
  }
}

// expert network by kind: 0 = ReLU FFN (W1 [f, d]), 1 = GEGLU (W1 [2f, d])
static void expert_row_kind(int32_t kind, int32_t d, int32_t f, int32_t dtype, const void* x_row,
                            const void* W1, const void* W2, void* out_row, void* H_out) {
  if (kind == 1) oracle_expert_row_geglu(d, f, dtype, x_row, W1, W2, out_row, H_out);
  else oracle_expert_row(d, f, dtype, x_row, W1, W2, out_row, H_out);
}

void oracle_expert_ffn(int32_t d, int32_t f, int32_t E, int32_t C, int32_t dtype, const void* xe,
                       const void* W1, const void* W2, const int32_t* kept_cnt, void* H, void* ye,
                       int32_t threads, int32_t kind) {
  const size_t es = dtype == DT_BF16 ? 2 : 4;
  std::vector<int64_t> rows;
  for (int32_t e = 0; e < E; ++e)
    for (int32_t r = 0; r < kept_cnt[e]; ++r) rows.push_back(static_cast<int64_t>(e) * C + r);
  parallel_for(static_cast<int64_t>(rows.size()), threads, [&](int64_t i) {
    int64_t row = rows[i];
    int64_t e = row / C;
    expert_row_kind(kind, d, f, dtype, static_cast<const char*>(xe) + row * d * es,
                      static_cast<const char*>(W1) + e * (kind == 1 ? 2 : 1) * f * d * es,
                      static_cast<const char*>(W2) + e * d * f * es,
                      static_cast<char*>(ye) + row * d * es,
                      H ? static_cast<char*>(H) + row * f * es : nullptr);
  });
}

// Switch notes sec. 2.1 eq. (2): y = sum over kept choices of p_i(x) E_i(x);
// a token with no kept choice gets 0 (sec. 2.2: it reaches the next layer
// through the residual only).  Sum in double, one rounding.
void oracle_combine(int64_t T, int32_t d, int32_t k, int32_t C, int32_t dtype, const void* ye,
                    const int32_t* expert_idx, const float* gate, const int32_t* slot,
                    const uint8_t* kept, void* y) {
  for (int64_t t = 0; t < T; ++t)
    for (int32_t c = 0; c < d; ++c) {
      double s = 0.0;
      for (int32_t j = 0; j < k; ++j) {
        if (!kept[t * k + j]) continue;
        int64_t row = static_cast<int64_t>(expert_idx[t * k + j]) * C + slot[t * k + j];
        s += static_cast<double>(gate[t * k + j]) * load(ye, row * d + c, dtype);
      }
      store(y, t * d + c, dtype, s);
    }
}

// One token's layer output (eq. (2) for a single x): y = sum over its kept
// choices j of gate_j * E_{e_j}(x), each expert output rounded as in
// oracle_expert_row, the sum in double and rounded once.  W1 [E, f, d] and
// W2 [E, d, f] are the full weight tensors.
void oracle_token_forward(int32_t d, int32_t f, int32_t k, int32_t dtype, const void* x_row,
                          const void* W1, const void* W2, const int32_t* expert_idx_row,
                          const float* gate_row, const uint8_t* kept_row, void* y_row,
                          int32_t kind) {
  const size_t es = dtype == DT_BF16 ? 2 : 4;
  std::vector<double> acc(d, 0.0);
  std::vector<uint32_t> out(d);  // room for d fp32 or bf16 values
  for (int32_t j = 0; j < k; ++j) {
    if (!kept_row[j]) continue;
    const int64_t e = expert_idx_row[j];
    expert_row_kind(kind, d, f, dtype, x_row,
                    static_cast<const char*>(W1) + e * (kind == 1 ? 2 : 1) * f * d * es,
                    static_cast<const char*>(W2) + e * d * f * es, out.data(), nullptr);
    for (int32_t c = 0; c < d; ++c)
      acc[c] += static_cast<double>(gate_row[j]) * load(out.data(), c, dtype);
  }
  for (int32_t c = 0; c < d; ++c) store(y_row, c, dtype, acc[c]);
}

// The whole layer, step by step, in the pages' order.  mode 0: softmax
// gate + top-k (Wr, bias used); mode 1: RRE (domain, seed, G used; k = 1).
// Buffers the caller may inspect: logits [T,E] (mode 0), expert_idx/gate/
// slot/kept [T,k], tok_of_row [E*C], arrivals/kept_cnt [E], xe/ye [E*C*d],
// H [E*C*f] (nullable), y [T,d].
void oracle_layer_forward(int64_t T, int32_t d, int32_t f, int32_t E, int32_t k, int32_t C,
                          int32_t dtype, int32_t mode, int32_t G, uint64_t seed, const void* x,
                          const void* Wr, const float* bias, const int32_t* domain,
                          const void* W1, const void* W2, float* logits, int32_t* expert_idx,
                          float* gate, int32_t* slot, uint8_t* kept, int32_t* tok_of_row,
                          int32_t* arrivals, int32_t* kept_cnt, int64_t* n_dropped, void* xe,
                          void* H, void* ye, void* y, int32_t threads, int32_t kind) {
  if (mode == 0) {
    oracle_router(T, d, E, dtype, x, Wr, bias, logits, threads);
    oracle_gate_topk(T, E, k, logits, expert_idx, gate, nullptr);
  } else {
    oracle_route_rre(T, E, G, seed, domain, expert_idx, gate);
  }
  oracle_assign(T, E, k, C, expert_idx, slot, kept, tok_of_row, arrivals, kept_cnt, n_dropped);
  oracle_dispatch(T, d, E, C, dtype, x, tok_of_row, kept_cnt, xe);
  oracle_expert_ffn(d, f, E, C, dtype, xe, W1, W2, kept_cnt, H, ye, threads, kind);
  oracle_combine(T, d, k, C, dtype, ye, expert_idx, gate, slot, kept, y);
}

// TorchScale review, SparseClip: ||g||_2 = ||(g_d, kappa * g_s)||_2 with
// kappa = 1/sqrt(E): sqrt(sum g_d^2 + sum (kappa g_s)^2) = sqrt(Sd + Ss / E).
// Sums of squares in double, segment by segment, in order.
double oracle_sparseclip_norm(const float* const* dense, const int64_t* dense_len,
                              int32_t n_dense, const float* const* sparse,
                              const int64_t* sparse_len, int32_t n_sparse, int32_t E) {
  double sd = 0.0, ss = 0.0;
  for (int32_t s = 0; s < n_dense; ++s)
    for (int64_t i = 0; i < dense_len[s]; ++i) sd += static_cast<double>(dense[s][i]) * dense[s][i];
  for (int32_t s = 0; s < n_sparse; ++s)
    for (int64_t i = 0; i < sparse_len[s]; ++i) ss += static_cast<double>(sparse[s][i]) * sparse[s][i];
  const double kappa = 1.0 / std::sqrt(static_cast<double>(E));
  return std::sqrt(sd + kappa * kappa * ss);
}

// TorchScale review, SparseClip as gradient clipping: every gradient (dense
// and expert) is multiplied by coef = min(1, max_norm / ||g||_2), with the
// reweighted norm of oracle_sparseclip_norm; each product is taken in double
// and rounded once to fp32.  Tensors are updated in place.  Returns coef.
double oracle_sparseclip_clip(float* const* dense, const int64_t* dense_len, int32_t n_dense,
                              float* const* sparse, const int64_t* sparse_len, int32_t n_sparse,
                              int32_t E, double max_norm, double* norm_out) {
  const double norm = oracle_sparseclip_norm(dense, dense_len, n_dense, sparse, sparse_len,
                                             n_sparse, E);
  const double coef = norm > max_norm ? max_norm / norm : 1.0;
  if (norm_out) *norm_out = norm;
  for (int32_t s = 0; s < n_dense; ++s)
    for (int64_t i = 0; i < dense_len[s]; ++i)
      dense[s][i] = static_cast<float>(static_cast<double>(dense[s][i]) * coef);
  for (int32_t s = 0; s < n_sparse; ++s)
    for (int64_t i = 0; i < sparse_len[s]; ++i)
      sparse[s][i] = static_cast<float>(static_cast<double>(sparse[s][i]) * coef);
  return coef;
}

// Switch notes sec. 2.2, "A Differentiable Load Balancing Loss", eqs. (4)-(6):
//   f_i = (1/T) #{tokens x : argmax p(x) = i}          (eq. 5)
//   P_i = (1/T) sum_x p_i(x)                            (eq. 6, p from eq. 1)
//   loss = alpha * N * sum_i f_i P_i   (N = E experts)  (eq. 4)
// The argmax is taken on the fp32 logits with ties to the lower index (the
// top-1 choice of oracle_gate_topk).  Also the routing entropy the TorchScale
// review tracks, read as the mean over tokens of -sum_i p_i(x) ln p_i(x)
// (terms with p_i = 0 contribute 0).  out[0] = loss, out[1] = entropy;
// f, P (nullable) receive the two vectors.  All in double.
void oracle_aux_loss(int64_t T, int32_t E, const float* logits, double alpha, double* out,
                     double* f, double* P) {
  std::vector<double> fs(E, 0.0), Ps(E, 0.0), p(E);
  double ent = 0.0;
  for (int64_t t = 0; t < T; ++t) {
    const float* h = logits + t * E;
    int32_t best = 0;
    for (int32_t e = 1; e < E; ++e)
      if (h[e] > h[best]) best = e;  // strict: the lower index wins a tie
    const double m = h[best];
    double z = 0.0;
    for (int32_t e = 0; e < E; ++e) z += std::exp(static_cast<double>(h[e]) - m);
    double ht = 0.0;
    for (int32_t e = 0; e < E; ++e) {
      p[e] = std::exp(static_cast<double>(h[e]) - m) / z;
      Ps[e] += p[e];
      if (p[e] > 0.0) ht -= p[e] * std::log(p[e]);
    }
    fs[best] += 1.0;
    ent += ht;
  }
  double dot = 0.0;
  for (int32_t e = 0; e < E; ++e) {
    fs[e] /= static_cast<double>(T);
    Ps[e] /= static_cast<double>(T);
    dot += fs[e] * Ps[e];
    if (f) f[e] = fs[e];
    if (P) P[e] = Ps[e];
  }
  out[0] = alpha * E * dot;
  out[1] = ent / static_cast<double>(T);
}

}  // extern "C"
