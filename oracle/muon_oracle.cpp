// Plain fp64 reference of the Muon optimizer step (and of the AdamW step for the
// parameters Muon leaves out): TEST INFRASTRUCTURE ONLY.
//
// Only the tests, the smoke check and the benchmark's CPU-baseline leg may
// load this library. The product path (the CUDA library) never calls it and
// shares no code, header or table with it.
//
// Everything is computed in IEEE double, step by step in the order the pages
// give it, with no blocking, fusion or re-association:
//
//   * "Muon optimizer: matrix-aware LLM training" (airosetta.com), the
//     `newtonschulz5` and `Muon.step` listings: bf16 working copy, divide by
//     (||X||_F + eps), transpose when rows > cols, `steps` iterations of
//     A = X X^T, B = b A + c A A, X = a X + B X, transpose back; momentum
//     buf = mu buf + (1 - mu) g; Nesterov select; p -= lr * O.
//     (This oracle keeps double precision throughout instead of bf16.)
//   * "Muon meets Mamba" (wmrh.cn), section 2.1 `zerocenter`: g minus its
//     mean over dim 0, taken before the momentum buffer (section 4.2 order);
//     section 2.2: the cubic iteration X = 1.5 X - 0.5 X X^T X; section 4.2:
//     decoupled weight decay p *= (1 - lr wd) before the update.
//   * "Muon meets Mamba" section 4.2 `_step_adamw` (and the moment equations of
//     section 1.3): the AdamW step, with bias correction and decoupled decay,
//     for the parameters that do not go to Muon.
//   * "AdamW vs Muon" (adg.csdn.net), part 3 "scaling and update": RMS rescale
//     by matrix shape, then times lr, then weight decay and subtraction; the
//     quintic written as M_k = a M + b (M M^T) M + c (M M^T)^2 M; the
//     normalisation M0 = M / ||M||_F.
//
// Readings where the pages are silent or garbled (each also listed in the
// design notes): Nesterov is u = mu m_t + (1 - mu) g_t (the `Muon.step`
// listing's select line is garbled); eps is added to the norm; rows > cols is
// the transpose test; the RMS factor is sqrt(max(1, rows/cols)) when
// requested, else 1; a zero update matrix gives O = 0.
//
// Threads only split the rows of each matrix product; every output element is
// still the sum over k in increasing k order, so the result does not depend
// on the thread count.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

using i64 = int64_t;

int resolve_threads(int nthreads) {
  if (nthreads > 0) return nthreads;
  unsigned h = std::thread::hardware_concurrency();
  return h == 0 ? 1 : (int)h;
}

// Run body(i0, i1) over [0, rows) split into contiguous row ranges.
template <class F>
void parallel_rows(i64 rows, int nthreads, F body) {
  int t = (int)std::min<i64>(std::max<i64>(rows, 1), nthreads);
  if (t <= 1) { body((i64)0, rows); return; }
  std::vector<std::thread> pool;
  i64 per = (rows + t - 1) / t;
  for (int w = 0; w < t; ++w) {
    i64 i0 = w * per, i1 = std::min(rows, i0 + per);
    if (i0 >= i1) break;
    pool.emplace_back([=] { body(i0, i1); });
  }
  for (auto& th : pool) th.join();
}

// C = A B with A: M x K, B: K x N, all row-major.
// C[i][j] = sum_{k=0}^{K-1} A[i][k] B[k][j], accumulated for k = 0, 1, ... in order.
void matmul(const double* A, const double* B, double* C, i64 M, i64 K, i64 N, int nthreads) {
  parallel_rows(M, nthreads, [=](i64 i0, i64 i1) {
    for (i64 i = i0; i < i1; ++i) {
      double* c = C + i * N;
      for (i64 j = 0; j < N; ++j) c[j] = 0.0;
      for (i64 k = 0; k < K; ++k) {
        const double a = A[i * K + k];
        const double* b = B + k * N;
        for (i64 j = 0; j < N; ++j) c[j] += a * b[j];
      }
    }
  });
}

// T = X^T, X: r x c row-major.
void transpose(const double* X, double* T, i64 r, i64 c) {
  for (i64 i = 0; i < r; ++i)
    for (i64 j = 0; j < c; ++j) T[j * r + i] = X[i * c + j];
}

// g <- g - 1 * mean_over_dim0(g)^T  (subtract each column's mean).
void zero_center_rows(double* g, i64 r, i64 c) {
  std::vector<double> mean(c, 0.0);
  for (i64 i = 0; i < r; ++i)
    for (i64 j = 0; j < c; ++j) mean[j] += g[i * c + j];
  for (i64 j = 0; j < c; ++j) mean[j] /= (double)r;
  for (i64 i = 0; i < r; ++i)
    for (i64 j = 0; j < c; ++j) g[i * c + j] -= mean[j];
}

double frobenius(const double* x, i64 n) {
  double s = 0.0;
  for (i64 e = 0; e < n; ++e) s += x[e] * x[e];
  return std::sqrt(s);
}

// The Newton-Schulz map applied to an update matrix u (r x c), result in O (r x c).
// coeffs holds steps triples (a_k, b_k, c_k).
void newton_schulz(const double* u, double* O, i64 r, i64 c, int steps, const double* coeffs,
                   double eps, int nthreads) {
  const i64 n_el = r * c;
  const bool tall = r > c;
  const i64 m = tall ? c : r;   // rows of the oriented iterate
  const i64 n = tall ? r : c;   // columns of the oriented iterate

  // X0 = u / (||u||_F + eps), oriented so that it is m x n with m <= n.
  const double scale = 1.0 / (frobenius(u, n_el) + eps);
  std::vector<double> X(n_el), Xt(n_el), A(m * m), AA(m * m), B(m * m), BX(n_el);
  if (tall) {
    transpose(u, X.data(), r, c);
  } else {
    std::memcpy(X.data(), u, sizeof(double) * n_el);
  }
  for (i64 e = 0; e < n_el; ++e) X[e] *= scale;

  for (int k = 0; k < steps; ++k) {
    const double a = coeffs[3 * k + 0], b = coeffs[3 * k + 1], cc = coeffs[3 * k + 2];
    transpose(X.data(), Xt.data(), m, n);               // X^T: n x m
    matmul(X.data(), Xt.data(), A.data(), m, n, m, nthreads);   // A = X X^T
    matmul(A.data(), A.data(), AA.data(), m, m, m, nthreads);   // A A
    for (i64 e = 0; e < m * m; ++e) B[e] = b * A[e] + cc * AA[e];   // B = b A + c A A
    matmul(B.data(), X.data(), BX.data(), m, m, n, nthreads);   // B X
    for (i64 e = 0; e < n_el; ++e) X[e] = a * X[e] + BX[e];     // X = a X + B X
  }

  if (tall) {
    transpose(X.data(), O, m, n);
  } else {
    std::memcpy(O, X.data(), sizeof(double) * n_el);
  }
}

}  // namespace

extern "C" {

// Newton-Schulz orthogonalisation of G (rows x cols, row-major) into O (same shape).
// zero_center != 0 first subtracts the mean over dim 0. Returns 0, or -1 on bad arguments.
int oracle_newton_schulz(const double* G, double* O, i64 rows, i64 cols, int steps,
                         const double* coeffs, int zero_center, double eps, int nthreads) {
  if (!G || !O || rows <= 0 || cols <= 0 || steps < 0 || (steps > 0 && !coeffs)) return -1;
  nthreads = resolve_threads(nthreads);
  std::vector<double> u(G, G + rows * cols);
  if (zero_center) zero_center_rows(u.data(), rows, cols);
  newton_schulz(u.data(), O, rows, cols, steps, coeffs, eps, nthreads);
  return 0;
}

// One Muon step over `count` matrices (all arrays row-major doubles, updated in place):
//   g  <- g - mean_dim0(g)                       (if zero_center)
//   m  <- mu m + (1 - mu) g
//   u  <- nesterov ? mu m + (1 - mu) g : m
//   O  <- NewtonSchulz(u)
//   p  <- p (1 - lr wd) - lr s O,  s = sqrt(max(1, rows/cols)) if rms_mode == 1 else 1
// grads[i] == NULL skips matrix i. O_out (optional, entries may be NULL) receives O.
int oracle_muon_step(int count, double* const* params, const double* const* grads,
                     double* const* momentum, const i64* rows, const i64* cols, double lr,
                     double mu, int nesterov, double weight_decay, int rms_mode, int steps,
                     const double* coeffs, int zero_center, double eps, int nthreads,
                     double* const* O_out) {
  if (count < 0 || (count > 0 && (!params || !grads || !momentum || !rows || !cols))) return -1;
  if (steps < 0 || (steps > 0 && !coeffs)) return -1;
  nthreads = resolve_threads(nthreads);
  for (int i = 0; i < count; ++i) {
    if (!grads[i]) continue;
    const i64 r = rows[i], c = cols[i], n_el = r * c;
    if (r <= 0 || c <= 0 || !params[i] || !momentum[i]) return -1;
    std::vector<double> g(grads[i], grads[i] + n_el), u(n_el), O(n_el);
    if (zero_center) zero_center_rows(g.data(), r, c);
    double* m = momentum[i];
    for (i64 e = 0; e < n_el; ++e) m[e] = mu * m[e] + (1.0 - mu) * g[e];
    for (i64 e = 0; e < n_el; ++e) u[e] = nesterov ? mu * m[e] + (1.0 - mu) * g[e] : m[e];
    newton_schulz(u.data(), O.data(), r, c, steps, coeffs, eps, nthreads);
    const double s = (rms_mode == 1) ? std::sqrt(std::max(1.0, (double)r / (double)c)) : 1.0;
    double* p = params[i];
    for (i64 e = 0; e < n_el; ++e) p[e] = p[e] * (1.0 - lr * weight_decay) - lr * s * O[e];
    if (O_out && O_out[i]) std::memcpy(O_out[i], O.data(), sizeof(double) * n_el);
  }
  return 0;
}

// One AdamW step over `count` tensors of numel[i] elements (the `_step_adamw` routine of
// "Muon meets Mamba" section 4.2, for the parameters that do not go to Muon: embeddings, head,
// norms, biases), in this order:
//   p  <- p (1 - lr wd)                            (decoupled weight decay, first)
//   m  <- beta1 m + (1 - beta1) g
//   v  <- beta2 v + (1 - beta2) g^2
//   p  <- p - (lr / (1 - beta1^t)) m / (sqrt(v) / sqrt(1 - beta2^t) + eps)
// with t = step, the step count after this step (t >= 1). grads[i] == NULL skips tensor i.
int oracle_adamw_step(int count, double* const* params, const double* const* grads,
                      double* const* exp_avg, double* const* exp_avg_sq, const i64* numel, i64 step,
                      double lr, double beta1, double beta2, double eps, double weight_decay) {
  if (count < 0 || step < 1) return -1;
  if (count > 0 && (!params || !grads || !exp_avg || !exp_avg_sq || !numel)) return -1;
  const double bias_corr1 = 1.0 - std::pow(beta1, (double)step);
  const double bias_corr2 = 1.0 - std::pow(beta2, (double)step);
  const double step_size = lr / bias_corr1;
  for (int i = 0; i < count; ++i) {
    if (!grads[i]) continue;
    if (numel[i] < 0 || !params[i] || !exp_avg[i] || !exp_avg_sq[i]) return -1;
    double* p = params[i];
    double* m = exp_avg[i];
    double* v = exp_avg_sq[i];
    const double* g = grads[i];
    for (i64 e = 0; e < numel[i]; ++e) {
      if (weight_decay != 0.0) p[e] = p[e] * (1.0 - lr * weight_decay);
      m[e] = beta1 * m[e] + (1.0 - beta1) * g[e];
      v[e] = beta2 * v[e] + (1.0 - beta2) * g[e] * g[e];
      const double denom = std::sqrt(v[e]) / std::sqrt(bias_corr2) + eps;
      p[e] = p[e] - step_size * m[e] / denom;
    }
  }
  return 0;
}

}  // extern "C"
