/*
 * moe_oracle.cpp - CPU oracle of the sparse Mixture-of-Experts layer forward
 * pass, as plain, slow C++ loops in double precision.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * CPU-baseline / reference legs of bench.py load or run this library (through
 * oracle/cpp.py).  It shares no code, header or table with the CUDA library:
 * it includes nothing but the C++ standard library.
 *
 * The layer is the one defined on the page "Mixture of experts"
 * (rayaq.ca/ml-models/mixture-of-experts):
 *   - "Replacing the feed-forward block": h = W_r x, p = softmax(h),
 *     y = sum over the chosen experts of g_i(x) E_i(x);
 *   - "Top-k gating": the k largest logits, largest first; the Switch gate
 *     (k = 1) is the chosen expert's full-softmax probability; the
 *     renormalised gate is the softmax over the k chosen logits;
 *   - "The load-balancing loss": aux = E sum_i f_i P_i with f_i the share of
 *     tokens whose top choice is i and P_i the mean router probability of i;
 *     the router z-loss is the mean over tokens of (log sum_j exp h_j)^2;
 *   - "Capacity and dropped tokens": each expert has capacity slots, filled
 *     in position order; assignments past the capacity are dropped and
 *     contribute nothing (the caller's residual carries the token);
 *   - "Implementation": the SwiGLU expert w2(silu(w1 x) * w3 x), the router
 *     computed in float32, the gated expert outputs summed per token;
 *   - "Total versus active parameters": shared experts that every token
 *     visits.
 * Other pages supply the alternative balance statistics: the coefficient of
 * variation of the expert assignment counts ("Mixture of Experts (MoE)",
 * inferensys.com, training bullets) and cv^2 of the router probabilities
 * ("Mixture of Experts (MoE) Language Models", chipfoundryservices.com,
 * "Load Balancing and Training").
 *
 * Readings where the pages are silent (each with its reason in the design
 * notes of this repository): ties in top-k go to the lower expert index (+0
 * and -0 are equal); capacity C = ceil(capacity_factor * T * k / E), equal to
 * the page's tokens/experts x factor at k = 1, and capacity_factor <= 0 means
 * no limit; slot priority is token order alone; f_i counts first choices of
 * all T tokens before any dropping, P_i is the full softmax over all E
 * experts; gates are not renormalised after drops; the ReLU expert is
 * w2(relu(w1 x)) without biases; router logits are rounded once to float32
 * and every routing decision is taken on those values; a shared expert has
 * the routed experts' shape and activation, weight 1, no part in routing,
 * capacity or losses, and is added after the routed sum.
 *
 * Every sum is a plain loop in index order, accumulated in double.  The only
 * parallelism is over independent tokens (std::thread), which changes no
 * result.
 *
 * Parity pins: tests/test_oracle_pins.py runs every pin against this library
 * and against the NumPy restatement in oracle/moe_oracle.py, and
 * tests/test_oracle_mutants.py plants mistakes in this source and checks that
 * a pin fails for each.
 */
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

// A read-only float tensor held as float64, float32 or bfloat16 bit patterns
// (a bfloat16 number is the upper half of a float32; widening it is exact).
enum { T_F64 = 0, T_F32 = 1, T_BF16 = 2 };

struct View {
  const void* data;
  int type;
  double at(int64_t i) const {
    if (type == T_F64) return static_cast<const double*>(data)[i];
    if (type == T_F32) return static_cast<const float*>(data)[i];
    const uint32_t bits = static_cast<uint32_t>(static_cast<const uint16_t*>(data)[i]) << 16;
    float f;
    std::memcpy(&f, &bits, sizeof f);
    return f;
  }
  bool null() const { return data == nullptr; }
};

// Run body(i) for i in [0, n) on `threads` threads (0: one per hardware thread).
template <class Body>
void for_each_index(int64_t n, int threads, Body body) {
  int nt = threads > 0 ? threads : static_cast<int>(std::thread::hardware_concurrency());
  if (nt < 1) nt = 1;
  if (nt > n) nt = static_cast<int>(std::max<int64_t>(n, 1));
  if (nt == 1) {
    for (int64_t i = 0; i < n; ++i) body(i);
    return;
  }
  std::vector<std::thread> pool;
  for (int w = 0; w < nt; ++w) {
    pool.emplace_back([=, &body]() {
      for (int64_t i = w; i < n; i += nt) body(i);
    });
  }
  for (auto& th : pool) th.join();
}

// "Replacing the feed-forward block": the router is one linear layer with E
// rows, h_e = sum_c W_r[e][c] x[c] (+ b_e); "Implementation": computed in
// float32, so the double sum is rounded once to float32 (unless round_f32 is 0,
// which finite-difference checks use).
void router_logits_row(const View& x, int64_t t, int64_t d, int64_t E, const View& W_r, const View& b_r,
                       int round_f32, double* h) {
  for (int64_t e = 0; e < E; ++e) {
    double s = 0.0;
    for (int64_t c = 0; c < d; ++c) s += W_r.at(e * d + c) * x.at(t * d + c);
    if (!b_r.null()) s += b_r.at(e);
    h[e] = round_f32 ? static_cast<double>(static_cast<float>(s)) : s;
  }
}

// p = softmax(h) over the E experts and lse = log sum_e exp h_e.
void softmax_lse_row(const double* h, int64_t E, double* p, double* lse) {
  double m = h[0];
  for (int64_t e = 1; e < E; ++e) m = std::max(m, h[e]);
  double Z = 0.0;
  for (int64_t e = 0; e < E; ++e) Z += std::exp(h[e] - m);
  for (int64_t e = 0; e < E; ++e) p[e] = std::exp(h[e] - m) / Z;
  *lse = m + std::log(Z);
}

// "Top-k gating": k times, take the largest logit not taken yet; a strictly
// larger value is needed to replace the current best, so among equal logits
// the lower expert index wins.
void top_k_row(const double* h, int64_t E, int64_t k, int64_t* idx) {
  std::vector<char> taken(E, 0);
  for (int64_t j = 0; j < k; ++j) {
    int64_t best = -1;
    for (int64_t e = 0; e < E; ++e) {
      if (taken[e]) continue;
      if (best < 0 || h[e] > h[best]) best = e;
    }
    idx[j] = best;
    taken[best] = 1;
  }
}

// "Top-k gating": Switch gate g_j = p[idx_j]; renormalised gate
// g_j = exp(h[idx_j]) / sum_i exp(h[idx_i]) over the chosen experts, computed
// relative to the largest chosen logit h[idx_0].
void gates_row(const double* h, const double* p, const int64_t* idx, int64_t k, int gate_mode, double* g) {
  if (gate_mode == 0) {
    for (int64_t j = 0; j < k; ++j) g[j] = p[idx[j]];
    return;
  }
  double sum = 0.0;
  for (int64_t j = 0; j < k; ++j) sum += std::exp(h[idx[j]] - h[idx[0]]);
  for (int64_t j = 0; j < k; ++j) g[j] = std::exp(h[idx[j]] - h[idx[0]]) / sum;
}

// One expert on one row xr[d]: SwiGLU w2(silu(w1 x) * w3 x), silu(u) = u/(1+e^-u);
// ReLU w2(relu(w1 x)).  W1e, W3e: [d_ff][d]; W2e: [d][d_ff] (nn.Linear layout),
// given as views with the expert's element offset.
void expert_row(const double* xr, int64_t d, int64_t d_ff, int act, const View& W1, const View& W3,
                const View& W2, int64_t off1, int64_t off2, double* out) {
  std::vector<double> hid(d_ff);
  for (int64_t f = 0; f < d_ff; ++f) {
    double a = 0.0;
    for (int64_t c = 0; c < d; ++c) a += W1.at(off1 + f * d + c) * xr[c];
    if (act == 0) {
      hid[f] = a > 0.0 ? a : 0.0;
    } else {
      double b = 0.0;
      for (int64_t c = 0; c < d; ++c) b += W3.at(off1 + f * d + c) * xr[c];
      hid[f] = a / (1.0 + std::exp(-a)) * b;
    }
  }
  for (int64_t c = 0; c < d; ++c) {
    double s = 0.0;
    for (int64_t f = 0; f < d_ff; ++f) s += W2.at(off2 + c * d_ff + f) * hid[f];
    out[c] = s;
  }
}

// "Capacity and dropped tokens": the rank of assignment (t, j) is the number of
// earlier assignments to the same expert in token order (t outer, j inner);
// kept iff rank < C (C < 0: no limit).  Kept assignments of expert e take rows
// offsets[e] .. offsets[e+1]-1 of the expert-sorted buffer in that order.
void assign_slots_impl(int64_t T, int64_t k, int64_t E, const int64_t* idx, int64_t C, int64_t* counts,
                       int64_t* kept_counts, int64_t* offsets, int64_t* rank, uint8_t* kept, int64_t* dest,
                       int64_t* dropped) {
  for (int64_t e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t j = 0; j < k; ++j) {
      const int64_t a = t * k + j;
      rank[a] = counts[idx[a]]++;
    }
  }
  int64_t n_dropped = 0;
  for (int64_t a = 0; a < T * k; ++a) {
    kept[a] = (C < 0 || rank[a] < C) ? 1 : 0;
    if (!kept[a]) ++n_dropped;
  }
  offsets[0] = 0;
  for (int64_t e = 0; e < E; ++e) {
    kept_counts[e] = C < 0 ? counts[e] : std::min(counts[e], C);
    offsets[e + 1] = offsets[e] + kept_counts[e];
  }
  for (int64_t a = 0; a < T * k; ++a) dest[a] = kept[a] ? offsets[idx[a]] + rank[a] : -1;
  *dropped = n_dropped;
}

// "The load-balancing loss": aux = E sum_i f_i P_i, f_i = share of the T tokens
// whose first choice is i (before capacity), P_i = mean of p_i over the tokens;
// z = mean over tokens of lse^2.  T = 0 gives 0 and 0.
void aux_and_z_impl(int64_t T, int64_t E, int64_t k, const double* p, const double* lse, const int64_t* idx,
                    double* aux, double* z) {
  *aux = 0.0;
  *z = 0.0;
  if (T == 0) return;
  std::vector<double> f(E, 0.0), P(E, 0.0);
  for (int64_t t = 0; t < T; ++t) f[idx[t * k]] += 1.0;
  for (int64_t t = 0; t < T; ++t)
    for (int64_t e = 0; e < E; ++e) P[e] += p[t * E + e];
  double s = 0.0;
  for (int64_t e = 0; e < E; ++e) s += (f[e] / T) * (P[e] / T);
  *aux = E * s;
  double zs = 0.0;
  for (int64_t t = 0; t < T; ++t) zs += lse[t] * lse[t];
  *z = zs / T;
}

// Alternative balance statistics, unscaled:
//   out[0] the Switch loss with f_i over all T k assignments;
//   out[1] coefficient of variation std/mean of the assignment counts c_i;
//   out[2] squared coefficient of variation var/mean^2 of P_i.
// Moments over the E values, divided by E.  T = 0 gives zeros.
void balance_impl(int64_t T, int64_t E, int64_t k, const double* p, const int64_t* idx, double* out) {
  out[0] = out[1] = out[2] = 0.0;
  if (T == 0) return;
  std::vector<double> c(E, 0.0), P(E, 0.0);
  for (int64_t a = 0; a < T * k; ++a) c[idx[a]] += 1.0;
  for (int64_t t = 0; t < T; ++t)
    for (int64_t e = 0; e < E; ++e) P[e] += p[t * E + e];
  for (int64_t e = 0; e < E; ++e) P[e] /= T;
  double mean_c = 0.0, mean_p = 0.0;
  for (int64_t e = 0; e < E; ++e) {
    mean_c += c[e];
    mean_p += P[e];
  }
  mean_c /= E;
  mean_p /= E;
  double var_c = 0.0, var_p = 0.0, aux_all = 0.0;
  for (int64_t e = 0; e < E; ++e) {
    var_c += (c[e] - mean_c) * (c[e] - mean_c);
    var_p += (P[e] - mean_p) * (P[e] - mean_p);
    aux_all += c[e] / static_cast<double>(T * k) * P[e];
  }
  var_c /= E;
  var_p /= E;
  out[0] = E * aux_all;
  out[1] = std::sqrt(var_c) / mean_c;
  out[2] = var_p / (mean_p * mean_p);
}

}  // namespace

extern "C" {

// Results of orc_moe_forward; every array is caller-allocated host memory.
struct orc_result {
  double* logits;        // [T][E] the routing logits (float32 values unless not rounded)
  double* p;             // [T][E] full softmax
  double* lse;           // [T]
  int64_t* idx;          // [T][k] chosen experts, largest logit first
  double* gate;          // [T][k]
  int64_t* counts;       // [E] assignments per expert before capacity
  int64_t* kept_counts;  // [E]
  int64_t* offsets;      // [E + 1]
  int64_t* rank;         // [T][k]
  uint8_t* kept;         // [T][k]
  int64_t* dest_row;     // [T][k], -1 when dropped
  int64_t dropped;
  int64_t capacity;      // -1: no limit
  double aux, z;
  double balance[3];     // aux over all choices, CV of counts, cv^2 of P
  double* y;             // [n_rows][d]
};

void orc_router_logits(int64_t T, int64_t d, int64_t E, const void* x, int x_type, const void* W_r, int w_type,
                       const void* b_r, int b_type, int round_f32, double* h) {
  const View X{x, x_type}, W{W_r, w_type}, B{b_r, b_type};
  for (int64_t t = 0; t < T; ++t) router_logits_row(X, t, d, E, W, B, round_f32, h + t * E);
}

void orc_softmax_lse(int64_t T, int64_t E, const double* h, double* p, double* lse) {
  for (int64_t t = 0; t < T; ++t) softmax_lse_row(h + t * E, E, p + t * E, lse + t);
}

void orc_top_k(int64_t T, int64_t E, int64_t k, const double* h, int64_t* idx) {
  for (int64_t t = 0; t < T; ++t) top_k_row(h + t * E, E, k, idx + t * k);
}

void orc_gates(int64_t T, int64_t E, int64_t k, const double* h, const double* p, const int64_t* idx,
               int gate_mode, double* g) {
  for (int64_t t = 0; t < T; ++t) gates_row(h + t * E, p + t * E, idx + t * k, k, gate_mode, g + t * k);
}

// "Capacity and dropped tokens": tokens/experts x factor, with the T k
// assignments of top-k counted: C = ceil(cf * T * k / E); -1 for cf <= 0.
int64_t orc_expert_capacity(double capacity_factor, int64_t T, int64_t k, int64_t E) {
  if (!(capacity_factor > 0.0)) return -1;
  return static_cast<int64_t>(std::ceil(capacity_factor * static_cast<double>(T) * static_cast<double>(k) /
                                        static_cast<double>(E)));
}

void orc_assign_slots(int64_t T, int64_t k, int64_t E, const int64_t* idx, int64_t C, int64_t* counts,
                      int64_t* kept_counts, int64_t* offsets, int64_t* rank, uint8_t* kept, int64_t* dest,
                      int64_t* dropped) {
  assign_slots_impl(T, k, E, idx, C, counts, kept_counts, offsets, rank, kept, dest, dropped);
}

void orc_expert_ffn(int64_t n, int64_t d, int64_t d_ff, int act, const double* xr, const void* W1, const void* W3,
                    const void* W2, int w_type, double* out, int threads) {
  const View V1{W1, w_type}, V3{W3, w_type}, V2{W2, w_type};
  for_each_index(n, threads, [&](int64_t r) { expert_row(xr + r * d, d, d_ff, act, V1, V3, V2, 0, 0, out + r * d); });
}

void orc_aux_and_z(int64_t T, int64_t E, int64_t k, const double* p, const double* lse, const int64_t* idx,
                   double* out2) {
  aux_and_z_impl(T, E, k, p, lse, idx, &out2[0], &out2[1]);
}

void orc_balance_losses(int64_t T, int64_t E, int64_t k, const double* p, const int64_t* idx, double* out3) {
  balance_impl(T, E, k, p, idx, out3);
}

/*
 * The whole layer.  Routing, capacity and the losses always cover all T
 * tokens; y is computed for the n_rows tokens listed in rows (all T when rows
 * is NULL), since y_t depends only on x_t and the global routing.
 *   x [T][d]; W_r [E][d]; b_r [E] or NULL; logits_in [T][E] (double) or NULL:
 *   route from these values instead of W_r x + b.
 *   W1, W3 [E][d_ff][d] (W3 NULL for ReLU); W2 [E][d][d_ff];
 *   W1s, W3s, W2s: n_shared shared experts of the same shapes (or NULL).
 * y_t = sum over kept (t, j), in slot order j, of g_tj E_{idx_tj}(x_t), then
 * plus sum_s S_s(x_t) in shared-expert order.  Returns 0, or 1 on bad sizes.
 */
int orc_moe_forward(int64_t T, int64_t d, int64_t E, int64_t k, int64_t d_ff, int act, int gate_mode,
                    double capacity_factor, const void* x, int x_type, const void* W_r, int wr_type,
                    const void* b_r, int br_type, const double* logits_in, int round_f32, const void* W1,
                    const void* W3, const void* W2, int w_type, int64_t n_shared, const void* W1s, const void* W3s,
                    const void* W2s, const int64_t* rows, int64_t n_rows, int threads, orc_result* r) {
  if (T < 0 || d < 1 || E < 1 || k < 1 || k > E || d_ff < 1 || n_shared < 0) return 1;
  const View X{x, x_type}, WR{W_r, wr_type}, BR{b_r, br_type};
  const View V1{W1, w_type}, V3{W3, w_type}, V2{W2, w_type};
  const View S1{W1s, w_type}, S3{W3s, w_type}, S2{W2s, w_type};

  for_each_index(T, threads, [&](int64_t t) {
    double* h = r->logits + t * E;
    if (logits_in != nullptr) {
      for (int64_t e = 0; e < E; ++e) h[e] = logits_in[t * E + e];
    } else {
      router_logits_row(X, t, d, E, WR, BR, round_f32, h);
    }
    softmax_lse_row(h, E, r->p + t * E, r->lse + t);
    top_k_row(h, E, k, r->idx + t * k);
    gates_row(h, r->p + t * E, r->idx + t * k, k, gate_mode, r->gate + t * k);
  });
  r->capacity = orc_expert_capacity(capacity_factor, T, k, E);
  assign_slots_impl(T, k, E, r->idx, r->capacity, r->counts, r->kept_counts, r->offsets, r->rank, r->kept,
                    r->dest_row, &r->dropped);
  aux_and_z_impl(T, E, k, r->p, r->lse, r->idx, &r->aux, &r->z);
  balance_impl(T, E, k, r->p, r->idx, r->balance);

  const int64_t n = rows == nullptr ? T : n_rows;
  for_each_index(n, threads, [&](int64_t i) {
    const int64_t t = rows == nullptr ? i : rows[i];
    std::vector<double> xr(d), out(d);
    for (int64_t c = 0; c < d; ++c) xr[c] = X.at(t * d + c);
    double* y = r->y + i * d;
    for (int64_t c = 0; c < d; ++c) y[c] = 0.0;
    for (int64_t j = 0; j < k; ++j) {  // slot order
      const int64_t a = t * k + j;
      if (!r->kept[a]) continue;
      const int64_t e = r->idx[a];
      expert_row(xr.data(), d, d_ff, act, V1, V3, V2, e * d_ff * d, e * d * d_ff, out.data());
      for (int64_t c = 0; c < d; ++c) y[c] += r->gate[a] * out[c];
    }
    for (int64_t s = 0; s < n_shared; ++s) {  // shared experts, after the routed sum
      expert_row(xr.data(), d, d_ff, act, S1, S3, S2, s * d_ff * d, s * d * d_ff, out.data());
      for (int64_t c = 0; c < d; ++c) y[c] += out[c];
    }
  });
  return 0;
}

int orc_hardware_threads(void) { return static_cast<int>(std::thread::hardware_concurrency()); }

}  // extern "C"
