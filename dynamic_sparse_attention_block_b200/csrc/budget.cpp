// budget.cpp -- profiling-guided speculation budget (host code; no kernel).
//
// PRR sizes its speculation from profiling (PRR abstract: a profiling-guided
// speculation budget keeps speculative work off the critical path).  Its
// limitations list says the overheads at context lengths off the profiled grid
// (between or beyond its points) come from polynomial regressions in the context length.  So a budget model here is:
//   select_us(x) and, for every profiled budget p_j, spec_us_j(x),
// each a least-squares polynomial in x = context_tokens / 65536 (a scale that keeps
// the normal equations well conditioned at 4K-1M tokens).  The budget for a context
// is the largest profiled p_j whose predicted speculation time does not exceed the
// predicted selection time, so speculation finishes while selection is still running.
#include <cmath>
#include <cstddef>

#include "prr.h"

namespace {

constexpr int kMaxDegree = 3;
constexpr double kTokensPerUnit = 65536.0;

double poly(const double* c, int degree, double x) {
  double y = 0.0;
  for (int k = degree; k >= 0; --k) y = y * x + c[k];
  return y;
}

}  // namespace

extern "C" prr_status prr_budget_fit(const double* context_tokens, const double* us, int32_t n, int32_t degree,
                                     double* coef) {
  if (!context_tokens || !us || !coef) return PRR_ERR_INVALID_ARG;
  if (degree < 0 || degree > kMaxDegree || n <= degree) return PRR_ERR_SHAPE;
  const int m = degree + 1;
  // normal equations  (V^T V) c = V^T y  with V[i][k] = x_i^k, solved by Gaussian
  // elimination with partial pivoting (at most 4 x 4)
  double a[kMaxDegree + 1][kMaxDegree + 2] = {};
  for (int i = 0; i < n; ++i) {
    const double x = context_tokens[i] / kTokensPerUnit;
    double pw[2 * kMaxDegree + 1];
    pw[0] = 1.0;
    for (int k = 1; k <= 2 * degree; ++k) pw[k] = pw[k - 1] * x;
    for (int r = 0; r < m; ++r) {
      for (int c = 0; c < m; ++c) a[r][c] += pw[r + c];
      a[r][m] += pw[r] * us[i];
    }
  }
  double scale = 0.0;
  for (int r = 0; r < m; ++r) scale = std::fmax(scale, std::fabs(a[r][r]));
  for (int col = 0; col < m; ++col) {
    int piv = col;
    for (int r = col + 1; r < m; ++r)
      if (std::fabs(a[r][col]) > std::fabs(a[piv][col])) piv = r;
    // (numerically) singular: fewer distinct contexts than coefficients
    if (!(std::fabs(a[piv][col]) > 1e-12 * scale)) return PRR_ERR_INVALID_ARG;
    if (piv != col)
      for (int c = 0; c <= m; ++c) {
        const double t = a[col][c];
        a[col][c] = a[piv][c];
        a[piv][c] = t;
      }
    for (int r = 0; r < m; ++r) {
      if (r == col) continue;
      const double f = a[r][col] / a[col][col];
      for (int c = col; c <= m; ++c) a[r][c] -= f * a[col][c];
    }
  }
  for (int k = 0; k < m; ++k) coef[k] = a[k][m] / a[k][k];
  return PRR_OK;
}

extern "C" prr_status prr_budget_choose(const double* sel_coef, const double* spec_coef, const int32_t* p_grid,
                                        int32_t np, int32_t degree, int32_t context_tokens, int32_t* p_out) {
  if (!sel_coef || !spec_coef || !p_grid || !p_out) return PRR_ERR_INVALID_ARG;
  if (degree < 0 || degree > kMaxDegree || np < 1 || context_tokens < 1) return PRR_ERR_SHAPE;
  for (int j = 1; j < np; ++j)
    if (p_grid[j] <= p_grid[j - 1]) return PRR_ERR_SHAPE;
  const double x = context_tokens / kTokensPerUnit;
  const double sel_us = poly(sel_coef, degree, x);
  int32_t best = 0;
  for (int j = 0; j < np; ++j)
    if (poly(spec_coef + static_cast<size_t>(j) * (degree + 1), degree, x) <= sel_us) best = p_grid[j];
  *p_out = best;
  return PRR_OK;
}
