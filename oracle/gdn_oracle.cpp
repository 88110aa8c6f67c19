// Gated DeltaNet token mixer -- CPU oracle, fp64.
//
// TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously-correct
// reference that the CUDA library is checked against.  Only the test suite,
// the smoke check and the CPU-baseline leg of the benchmark load it; the
// product path (the CUDA library and its Python binding) never does, and the
// two share no code.
//
// What it computes, in the order the layer applies it:
//   1. causal depthwise conv1d, kernel 4, no bias, over the mixed q|k|v
//      projection ("Qwen3.5 (Qwen3-Next)", API table: linear_conv_kernel_dim 4;
//      "Qwen/Qwen3.5-9B", module tree: conv1d 8192x1x4 with 32.8K parameters,
//      i.e. no bias term);
//   2. SiLU;
//   3. split into q (Hk heads), k (Hk heads), v (Hv heads), each head dk or dv
//      wide; q and k L2-normalised per head, q multiplied by `scale`;
//   4. gates per value head: g = -exp(A_log) * softplus(a + dt_bias),
//      alpha = exp(g), beta = sigmoid(b)  ("Qwen/Qwen3.5-9B", module tree:
//      the two direct parameter vectors "32, 32" of the GDN block and the
//      in_proj_a / in_proj_b projections to 32 = Hv values);
//   5. the gated delta rule per value head h, key head h / (Hv/Hk):
//         S_t = alpha_t * S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
//         o_t = S_t q_t
//      S is dv x dk ("Qwen (text & vision-language)", Architecture notes:
//      Gated-DeltaNet = conv1d + delta rule; Generation: the per-layer conv
//      state and recurrent state are carried across steps);
//   6. gated RMSNorm over dv with one dv-wide weight shared by every head:
//         out = o / sqrt(mean(o^2) + eps) * w * silu(z)
//      ("Qwen/Qwen3.5-9B", module tree: norm Qwen3_5RMSNormGated, 128 params);
//   7. the conv tail: the last 3 raw (pre-conv) inputs per channel.
//
// Every quantity is double.  Inputs are the exact values the GPU consumes
// (bf16-rounded on the host), widened to double by the caller.
//
// A second core implements the chunked (WY / UT-transform) form of step 5
// in fp64; the two are algebraically identical ("Qwen (text &
// vision-language)", Verified parity: chunked and recurrent Gated-DeltaNet
// differ only by floating-point accumulation), which the tests check.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>
#include <algorithm>
#include <functional>

namespace {

struct Dims {
  int Hk, Hv, dk, dv;
  int Cc() const { return 2 * Hk * dk + Hv * dv; }
  int G() const { return Hv / Hk; }
};

// Run f(i) for i in [0, n) over `nthreads` host threads (static blocking).
void parallel_for(int n, int nthreads, const std::function<void(int)>& f) {
  if (nthreads <= 1 || n <= 1) {
    for (int i = 0; i < n; ++i) f(i);
    return;
  }
  nthreads = std::min(nthreads, n);
  std::vector<std::thread> pool;
  pool.reserve(nthreads);
  for (int w = 0; w < nthreads; ++w) {
    pool.emplace_back([&, w]() {
      for (int i = w; i < n; i += nthreads) f(i);
    });
  }
  for (auto& t : pool) t.join();
}

double silu(double x) { return x / (1.0 + std::exp(-x)); }
double sigmoid(double x) { return 1.0 / (1.0 + std::exp(-x)); }
// softplus(x) = log(1 + e^x), written in a form that neither overflows nor
// loses the small-x tail.
double softplus(double x) { return std::max(x, 0.0) + std::log1p(std::exp(-std::fabs(x))); }

// Step 1-4 for all tokens of one sequence.
//   x      [T_tot, Cc] raw mixed projection
//   y_pre  [T_tot, Cc] conv output before SiLU (optional)
//   q,k    [T_tot, Hk, dk] normalised (q scaled)
//   v      [T_tot, Hv, dv]
//   g,beta [T_tot, Hv]
void prep_sequence(const Dims& D, double scale, double eps_l2, int64_t bos, int64_t eos,
                   const double* x, const double* conv_w, const double* hist /*[Cc,3] or null*/,
                   const double* a, const double* b, const double* A_log, const double* dt_bias,
                   double* y_pre, double* q, double* k, double* v, double* g, double* beta,
                   double* conv_tail /*[Cc,3] or null*/) {
  const int Cc = D.Cc();
  const int KW = 4;
  std::vector<double> y(Cc);
  for (int64_t t = bos; t < eos; ++t) {
    // 1. causal depthwise conv: tap j multiplies the input at t - 3 + j, so
    //    tap 3 is the current token and tap 0 the oldest.
    for (int c = 0; c < Cc; ++c) {
      double acc = 0.0;
      for (int j = 0; j < KW; ++j) {
        int64_t tau = t - (KW - 1) + j;
        double xv;
        if (tau >= bos) {
          xv = x[tau * Cc + c];
        } else {
          int64_t back = bos - tau;  // 1..3 positions before the start
          xv = hist ? hist[(int64_t)c * 3 + (3 - back)] : 0.0;
        }
        acc += conv_w[c * KW + j] * xv;
      }
      if (y_pre) y_pre[t * Cc + c] = acc;
      // 2. SiLU
      y[c] = silu(acc);
    }
    // 3. split q | k | v, head-major inside each block
    for (int hk = 0; hk < D.Hk; ++hk) {
      const double* yq = &y[hk * D.dk];
      const double* yk = &y[D.Hk * D.dk + hk * D.dk];
      double sq = 0.0, sk = 0.0;
      for (int i = 0; i < D.dk; ++i) { sq += yq[i] * yq[i]; sk += yk[i] * yk[i]; }
      double rq = 1.0 / std::sqrt(sq + eps_l2), rk = 1.0 / std::sqrt(sk + eps_l2);
      double* qo = q + (t * D.Hk + hk) * D.dk;
      double* ko = k + (t * D.Hk + hk) * D.dk;
      for (int i = 0; i < D.dk; ++i) { qo[i] = yq[i] * rq * scale; ko[i] = yk[i] * rk; }
    }
    for (int h = 0; h < D.Hv; ++h) {
      const double* yv = &y[2 * D.Hk * D.dk + h * D.dv];
      double* vo = v + (t * D.Hv + h) * D.dv;
      for (int i = 0; i < D.dv; ++i) vo[i] = yv[i];
    }
    // 4. gates
    for (int h = 0; h < D.Hv; ++h) {
      double gg = -std::exp(A_log[h]) * softplus(a[t * D.Hv + h] + dt_bias[h]);
      g[t * D.Hv + h] = gg;
      beta[t * D.Hv + h] = sigmoid(b[t * D.Hv + h]);
    }
  }
  // 7. conv tail: the last three raw inputs of the history [hist ; x[bos:eos]]
  if (conv_tail) {
    int64_t len = eos - bos;
    for (int c = 0; c < Cc; ++c) {
      for (int s = 0; s < 3; ++s) {
        // position s of the tail is history index len - 3 + s
        int64_t idx = len - 3 + s;
        double val;
        if (idx >= 0) val = x[(bos + idx) * Cc + c];
        else val = hist ? hist[(int64_t)c * 3 + (3 + idx)] : 0.0;
        conv_tail[(int64_t)c * 3 + s] = val;
      }
    }
  }
}

// Step 5, recurrent form, for one (sequence, value head).
//   S (dv x dk, row = value channel) is updated in place.
void core_recurrent_head(const Dims& D, int h, int64_t bos, int64_t eos, const double* q,
                         const double* k, const double* v, const double* g, const double* beta,
                         double* S, double* o) {
  const int hk = h / D.G();
  std::vector<double> u(D.dv);
  for (int64_t t = bos; t < eos; ++t) {
    const double* kt = k + (t * D.Hk + hk) * D.dk;
    const double* qt = q + (t * D.Hk + hk) * D.dk;
    const double* vt = v + (t * D.Hv + h) * D.dv;
    const double alpha = std::exp(g[t * D.Hv + h]);
    const double bt = beta[t * D.Hv + h];
    // S (I - b k k^T) = S - b (S k) k^T
    for (int r = 0; r < D.dv; ++r) {
      double acc = 0.0;
      for (int j = 0; j < D.dk; ++j) acc += S[r * D.dk + j] * kt[j];
      u[r] = acc;
    }
    for (int r = 0; r < D.dv; ++r)
      for (int j = 0; j < D.dk; ++j)
        S[r * D.dk + j] = alpha * (S[r * D.dk + j] - bt * u[r] * kt[j]) + bt * vt[r] * kt[j];
    double* ot = o + (t * D.Hv + h) * D.dv;
    for (int r = 0; r < D.dv; ++r) {
      double acc = 0.0;
      for (int j = 0; j < D.dk; ++j) acc += S[r * D.dk + j] * qt[j];
      ot[r] = acc;
    }
  }
}

// Plain dense helpers for the chunked form (row-major).
// C[m x n] = A[m x p] * B[p x n]
void matmul(int m, int p, int n, const double* A, const double* B, double* C) {
  for (int i = 0; i < m; ++i)
    for (int j = 0; j < n; ++j) {
      double acc = 0.0;
      for (int l = 0; l < p; ++l) acc += A[i * p + l] * B[l * n + j];
      C[i * n + j] = acc;
    }
}

// Step 5, chunked form, for one (sequence, value head).  Within a chunk of
// L <= C tokens, with gamma_i = g_1 + ... + g_i (cumulative log decay):
//   A_ij = beta_i exp(gamma_i - gamma_j) k_i . k_j        (i > j), else 0
//   T    = (I + A)^-1                                      (unit lower triangular)
//   W    = T diag(beta exp(gamma)) K
//   U    = T diag(beta) V
//   Vn   = U - W S0^T
//   O    = diag(exp(gamma)) Q S0^T + ((Q K^T) o M[i >= j] exp(gamma_i - gamma_j)) Vn
//   S_L  = exp(gamma_L) S0 + Vn^T diag(exp(gamma_L - gamma)) K
// Only differences gamma_i - gamma_j with i >= j (never positive) are
// exponentiated, besides gamma_i itself (never positive).
void core_chunked_head(const Dims& D, int h, int C, int64_t bos, int64_t eos, const double* q,
                       const double* k, const double* v, const double* g, const double* beta,
                       double* S, double* o) {
  const int hk = h / D.G();
  const int dk = D.dk, dv = D.dv;
  std::vector<double> Kc, Qc, Vc, gam, bet, Amat, T, X, W, U, Vn, tmp, St, QK, O;
  for (int64_t c0 = bos; c0 < eos; c0 += C) {
    const int L = (int)std::min<int64_t>(C, eos - c0);
    Kc.assign((size_t)L * dk, 0.0); Qc.assign((size_t)L * dk, 0.0); Vc.assign((size_t)L * dv, 0.0);
    gam.assign(L, 0.0); bet.assign(L, 0.0);
    double run = 0.0;
    for (int i = 0; i < L; ++i) {
      const int64_t t = c0 + i;
      for (int j = 0; j < dk; ++j) {
        Kc[i * dk + j] = k[(t * D.Hk + hk) * dk + j];
        Qc[i * dk + j] = q[(t * D.Hk + hk) * dk + j];
      }
      for (int j = 0; j < dv; ++j) Vc[i * dv + j] = v[(t * D.Hv + h) * dv + j];
      run += g[t * D.Hv + h];
      gam[i] = run;
      bet[i] = beta[t * D.Hv + h];
    }
    // A and T = (I + A)^-1 by forward substitution, row by row:
    //   T_i = e_i - sum_{j<i} A_ij T_j
    Amat.assign((size_t)L * L, 0.0);
    for (int i = 0; i < L; ++i)
      for (int j = 0; j < i; ++j) {
        double kk = 0.0;
        for (int l = 0; l < dk; ++l) kk += Kc[i * dk + l] * Kc[j * dk + l];
        Amat[i * L + j] = bet[i] * std::exp(gam[i] - gam[j]) * kk;
      }
    T.assign((size_t)L * L, 0.0);
    for (int i = 0; i < L; ++i) {
      T[i * L + i] = 1.0;
      for (int j = 0; j < i; ++j) {
        const double aij = Amat[i * L + j];
        if (aij == 0.0) continue;
        for (int m = 0; m < L; ++m) T[i * L + m] -= aij * T[j * L + m];
      }
    }
    // W = T diag(beta e^gamma) K ; U = T diag(beta) V
    X.assign((size_t)L * dk, 0.0);
    for (int i = 0; i < L; ++i)
      for (int l = 0; l < dk; ++l) X[i * dk + l] = bet[i] * std::exp(gam[i]) * Kc[i * dk + l];
    W.assign((size_t)L * dk, 0.0);
    matmul(L, L, dk, T.data(), X.data(), W.data());
    X.assign((size_t)L * dv, 0.0);
    for (int i = 0; i < L; ++i)
      for (int l = 0; l < dv; ++l) X[i * dv + l] = bet[i] * Vc[i * dv + l];
    U.assign((size_t)L * dv, 0.0);
    matmul(L, L, dv, T.data(), X.data(), U.data());
    // S0^T (dk x dv)
    St.assign((size_t)dk * dv, 0.0);
    for (int r = 0; r < dv; ++r)
      for (int j = 0; j < dk; ++j) St[j * dv + r] = S[r * dk + j];
    // Vn = U - W S0^T
    tmp.assign((size_t)L * dv, 0.0);
    matmul(L, dk, dv, W.data(), St.data(), tmp.data());
    Vn.assign((size_t)L * dv, 0.0);
    for (size_t e = 0; e < Vn.size(); ++e) Vn[e] = U[e] - tmp[e];
    // O = diag(e^gamma) Q S0^T + (QK^T o decay mask) Vn
    O.assign((size_t)L * dv, 0.0);
    matmul(L, dk, dv, Qc.data(), St.data(), O.data());
    for (int i = 0; i < L; ++i)
      for (int r = 0; r < dv; ++r) O[i * dv + r] *= std::exp(gam[i]);
    QK.assign((size_t)L * L, 0.0);
    for (int i = 0; i < L; ++i)
      for (int j = 0; j <= i; ++j) {
        double qk = 0.0;
        for (int l = 0; l < dk; ++l) qk += Qc[i * dk + l] * Kc[j * dk + l];
        QK[i * L + j] = qk * std::exp(gam[i] - gam[j]);
      }
    tmp.assign((size_t)L * dv, 0.0);
    matmul(L, L, dv, QK.data(), Vn.data(), tmp.data());
    for (int i = 0; i < L; ++i)
      for (int r = 0; r < dv; ++r) o[((c0 + i) * D.Hv + h) * dv + r] = O[i * dv + r] + tmp[i * dv + r];
    // S_L = e^{gamma_L} S0 + Vn^T diag(e^{gamma_L - gamma}) K
    const double gL = gam[L - 1];
    for (int r = 0; r < dv; ++r)
      for (int j = 0; j < dk; ++j) {
        double acc = std::exp(gL) * S[r * dk + j];
        for (int i = 0; i < L; ++i) acc += Vn[i * dv + r] * std::exp(gL - gam[i]) * Kc[i * dk + j];
        S[r * dk + j] = acc;
      }
  }
}

// Step 6 for one (token, value head).
void gated_rmsnorm(int dv, double eps, const double* o, const double* z, const double* w, double* out) {
  double ss = 0.0;
  for (int r = 0; r < dv; ++r) ss += o[r] * o[r];
  const double inv = 1.0 / std::sqrt(ss / dv + eps);
  for (int r = 0; r < dv; ++r) out[r] = o[r] * inv * w[r] * silu(z[r]);
}

bool dims_ok(const Dims& D) {
  return D.Hk > 0 && D.Hv > 0 && D.dk > 0 && D.dv > 0 && D.Hv % D.Hk == 0;
}

// Core runner shared by both core entry points.
int run_core(const Dims& D, int N, const int64_t* cu, const double* q, const double* k,
             const double* v, const double* g, const double* beta, const double* S0, double* o,
             double* S_final, int chunk, int nthreads) {
  const size_t SS = (size_t)D.dv * D.dk;
  parallel_for(N * D.Hv, nthreads, [&](int idx) {
    const int n = idx / D.Hv, h = idx % D.Hv;
    std::vector<double> S(SS, 0.0);
    if (S0) std::memcpy(S.data(), S0 + ((size_t)n * D.Hv + h) * SS, SS * sizeof(double));
    if (chunk <= 0)
      core_recurrent_head(D, h, cu[n], cu[n + 1], q, k, v, g, beta, S.data(), o);
    else
      core_chunked_head(D, h, chunk, cu[n], cu[n + 1], q, k, v, g, beta, S.data(), o);
    if (S_final) std::memcpy(S_final + ((size_t)n * D.Hv + h) * SS, S.data(), SS * sizeof(double));
  });
  return 0;
}

}  // namespace

extern "C" {

// Whole mixer (steps 1-7), recurrent core.  Returns 0, or -1 on bad dims.
// Optional outputs (may be NULL): final_state, conv_state_out, y_pre, q_hat,
// k_hat, v_act, g_out, beta_out, o_core.
int gdn_oracle_prefill(int Hk, int Hv, int dk, int dv, double scale, double eps_l2,
                       double eps_norm, int N, const int64_t* cu_seqlens, const double* mixed_qkv,
                       const double* conv_w, const double* a, const double* b,
                       const double* A_log, const double* dt_bias, const double* z,
                       const double* norm_w, const double* initial_state,
                       const double* conv_state_in, double* out, double* final_state,
                       double* conv_state_out, double* y_pre, double* q_hat, double* k_hat,
                       double* v_act, double* g_out, double* beta_out, double* o_core,
                       int nthreads) {
  Dims D{Hk, Hv, dk, dv};
  if (!dims_ok(D) || N < 0) return -1;
  const int64_t T = cu_seqlens[N];
  const int Cc = D.Cc();
  std::vector<double> qv, kv, vv, gv, bv, ov;
  double* q = q_hat; double* k = k_hat; double* v = v_act; double* g = g_out; double* be = beta_out;
  double* o = o_core;
  if (!q) { qv.assign((size_t)T * Hk * dk, 0.0); q = qv.data(); }
  if (!k) { kv.assign((size_t)T * Hk * dk, 0.0); k = kv.data(); }
  if (!v) { vv.assign((size_t)T * Hv * dv, 0.0); v = vv.data(); }
  if (!g) { gv.assign((size_t)T * Hv, 0.0); g = gv.data(); }
  if (!be) { bv.assign((size_t)T * Hv, 0.0); be = bv.data(); }
  if (!o) { ov.assign((size_t)T * Hv * dv, 0.0); o = ov.data(); }
  parallel_for(N, nthreads, [&](int n) {
    prep_sequence(D, scale, eps_l2, cu_seqlens[n], cu_seqlens[n + 1], mixed_qkv, conv_w,
                  conv_state_in ? conv_state_in + (size_t)n * Cc * 3 : nullptr, a, b, A_log,
                  dt_bias, y_pre, q, k, v, g, be,
                  conv_state_out ? conv_state_out + (size_t)n * Cc * 3 : nullptr);
  });
  run_core(D, N, cu_seqlens, q, k, v, g, be, initial_state, o, final_state, 0, nthreads);
  parallel_for((int)std::min<int64_t>(T, 1 << 30), nthreads, [&](int t) {
    for (int h = 0; h < Hv; ++h)
      gated_rmsnorm(dv, eps_norm, o + ((size_t)t * Hv + h) * dv, z + ((size_t)t * Hv + h) * dv,
                    norm_w, out + ((size_t)t * Hv + h) * dv);
  });
  return 0;
}

// One recurrent step for a batch of B independent sequences: the same code
// path as the prefill, run with one token per sequence, the conv cache as the
// conv history and the state as the initial state.  state and conv_state are
// read and then overwritten with the updated values.
int gdn_oracle_decode(int Hk, int Hv, int dk, int dv, double scale, double eps_l2,
                      double eps_norm, int B, const double* mixed_qkv, const double* conv_w,
                      const double* a, const double* b, const double* A_log,
                      const double* dt_bias, const double* z, const double* norm_w,
                      double* state, double* conv_state, double* out, int nthreads) {
  Dims D{Hk, Hv, dk, dv};
  if (!dims_ok(D) || B < 0) return -1;
  std::vector<int64_t> cu(B + 1);
  for (int i = 0; i <= B; ++i) cu[i] = i;
  std::vector<double> S_in(state, state + (size_t)B * Hv * dv * dk);
  std::vector<double> cs_in(conv_state, conv_state + (size_t)B * D.Cc() * 3);
  return gdn_oracle_prefill(Hk, Hv, dk, dv, scale, eps_l2, eps_norm, B, cu.data(), mixed_qkv,
                            conv_w, a, b, A_log, dt_bias, z, norm_w, S_in.data(), cs_in.data(),
                            out, state, conv_state, nullptr, nullptr, nullptr, nullptr, nullptr,
                            nullptr, nullptr, nthreads);
}

// Step 5 alone on given q, k, v, g (log decay), beta.
//   q, k [T, Hk, dk]; v [T, Hv, dv]; g, beta [T, Hv]; S0 [N, Hv, dv, dk] or NULL.
//   chunk <= 0 selects the recurrent form, chunk > 0 the chunked form.
int gdn_oracle_core(int Hk, int Hv, int dk, int dv, int N, const int64_t* cu_seqlens,
                    const double* q, const double* k, const double* v, const double* g,
                    const double* beta, const double* S0, double* o, double* S_final, int chunk,
                    int nthreads) {
  Dims D{Hk, Hv, dk, dv};
  if (!dims_ok(D) || N < 0) return -1;
  return run_core(D, N, cu_seqlens, q, k, v, g, beta, S0, o, S_final, chunk, nthreads);
}

// The element-wise pieces on their own, so that the tests can pin them at
// hand-evaluated points: y[i] = silu(x[i]) (step 2), and step 6 over `rows`
// independent (token, value head) rows of width dv with one dv-wide weight.
void gdn_oracle_silu(int n, const double* x, double* y) {
  for (int i = 0; i < n; ++i) y[i] = silu(x[i]);
}
void gdn_oracle_gated_rmsnorm(int rows, int dv, double eps, const double* o, const double* z,
                              const double* w, double* out) {
  for (int r = 0; r < rows; ++r)
    gated_rmsnorm(dv, eps, o + (size_t)r * dv, z + (size_t)r * dv, w, out + (size_t)r * dv);
}

}  // extern "C"
