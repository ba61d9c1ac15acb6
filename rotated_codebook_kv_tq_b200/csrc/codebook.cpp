// Host Lloyd-Max solver for the coordinate law of a randomly rotated unit vector.
//
// "Google presenta TurboQuant ..." (7minutos.es), "La mecanica geometrica de
// TurboQuant": after the random rotation each coordinate follows a Beta law on
// [-1, 1]; the b-bit scalar quantizer minimises the MSE cost C(f_X, b) and is
// solved once offline.  The law used is (1 + X) / 2 ~ Beta(a, a) with
// a = (d - 1) / 2, i.e. f_d(x) = C_d (1 - x^2)^((d-3)/2).
//
// Cell masses come from the regularized incomplete Beta function, evaluated
// with its continued fraction (DLMF 8.17.22) by the modified Lentz method;
// first moments from the closed form
//   int_a^b x f_d(x) dx = C_d / (d - 1) [(1 - a^2)^((d-1)/2) - (1 - b^2)^((d-1)/2)].
// Lloyd's two conditions (centroid = conditional mean, threshold = midpoint)
// are iterated from evenly spaced centroids; each step is made exactly odd,
// since f_d is even.
#include <cmath>
#include <vector>

namespace tqhost {

namespace {

// Continued fraction of I_x(a, b) (DLMF 8.17.22), modified Lentz evaluation.
double ibeta_cf(double a, double b, double x) {
  const double tiny = 1e-300;
  double c = 1.0;
  double dd = 1.0 - (a + b) * x / (a + 1.0);
  if (std::fabs(dd) < tiny) dd = tiny;
  dd = 1.0 / dd;
  double f = dd;
  for (int m = 1; m < 100000; ++m) {
    // even step: d_{2m} = m (b - m) x / ((a + 2m - 1)(a + 2m))
    double num = m * (b - m) * x / ((a + 2.0 * m - 1.0) * (a + 2.0 * m));
    dd = 1.0 + num * dd;
    if (std::fabs(dd) < tiny) dd = tiny;
    c = 1.0 + num / c;
    if (std::fabs(c) < tiny) c = tiny;
    dd = 1.0 / dd;
    f *= dd * c;
    // odd step: d_{2m+1} = -(a + m)(a + b + m) x / ((a + 2m)(a + 2m + 1))
    num = -(a + m) * (a + b + m) * x / ((a + 2.0 * m) * (a + 2.0 * m + 1.0));
    dd = 1.0 + num * dd;
    if (std::fabs(dd) < tiny) dd = tiny;
    c = 1.0 + num / c;
    if (std::fabs(c) < tiny) c = tiny;
    dd = 1.0 / dd;
    const double delta = dd * c;
    f *= delta;
    if (std::fabs(delta - 1.0) < 1e-16) break;
  }
  return f;
}

// Regularized incomplete Beta I_x(a, b).
double ibeta(double a, double b, double x) {
  if (x <= 0.0) return 0.0;
  if (x >= 1.0) return 1.0;
  const double lpre = std::lgamma(a + b) - std::lgamma(a) - std::lgamma(b) +
                      a * std::log(x) + b * std::log1p(-x);
  const double pre = std::exp(lpre);
  if (x < (a + 1.0) / (a + b + 2.0)) return pre * ibeta_cf(a, b, x) / a;
  return 1.0 - pre * ibeta_cf(b, a, 1.0 - x) / b;
}

// P(X <= t) for the coordinate law; symmetric evaluation keeps the argument
// of the continued fraction at or below one half.
double coord_cdf(int d, double t) {
  const double a = 0.5 * (d - 1);
  if (t <= 0.0) return ibeta(a, a, 0.5 * (1.0 + t));
  return 1.0 - ibeta(a, a, 0.5 * (1.0 - t));
}

double log_norm_const(int d) {
  return std::lgamma(0.5 * d) - 0.5 * std::log(M_PI) - std::lgamma(0.5 * (d - 1));
}

double pow_term(int d, double x) {  // (1 - x^2)^((d-1)/2), zero at |x| >= 1
  if (std::fabs(x) >= 1.0) return 0.0;
  return std::exp(0.5 * (d - 1) * std::log1p(-x * x));
}

}  // namespace

// Returns false on invalid arguments.
bool lloyd_max(int d, int bits, std::vector<double> &c, std::vector<double> &t,
               double &mse) {
  if (d < 4 || bits < 1 || bits > 8) return false;
  const int n = 1 << bits;
  const double sigma = 1.0 / std::sqrt(static_cast<double>(d));
  c.assign(n, 0.0);
  for (int m = 0; m < n; ++m)
    c[m] = n == 2 ? (m ? sigma : -sigma) : sigma * (-2.0 + 4.0 * m / (n - 1));
  const double cmom = std::exp(log_norm_const(d)) / (d - 1);
  std::vector<double> edges(n + 1), cdf(n + 1), cn(n);
  for (int it = 0; it < 500000; ++it) {
    edges[0] = -1.0;
    edges[n] = 1.0;
    for (int k = 1; k < n; ++k) edges[k] = 0.5 * (c[k - 1] + c[k]);
    for (int k = 0; k <= n; ++k) cdf[k] = coord_cdf(d, edges[k]);
    for (int m = 0; m < n; ++m) {
      const double mass = cdf[m + 1] - cdf[m];
      const double mom = cmom * (pow_term(d, edges[m]) - pow_term(d, edges[m + 1]));
      cn[m] = mom / mass;
    }
    double moved = 0.0;
    for (int m = 0; m < n; ++m) {
      const double v = 0.5 * (cn[m] - cn[n - 1 - m]);
      moved = std::fmax(moved, std::fabs(v - c[m]));
      c[m] = v;
    }
    if (moved < 1e-14) break;
  }
  t.assign(n - 1, 0.0);
  for (int k = 1; k < n; ++k) t[k - 1] = 0.5 * (c[k - 1] + c[k]);
  // MSE at the fixed point: E[X^2] - sum_m P_m c_m^2, with E[X^2] = 1/d.
  edges[0] = -1.0;
  edges[n] = 1.0;
  for (int k = 1; k < n; ++k) edges[k] = t[k - 1];
  double acc = 0.0;
  for (int m = 0; m < n; ++m)
    acc += (coord_cdf(d, edges[m + 1]) - coord_cdf(d, edges[m])) * c[m] * c[m];
  mse = 1.0 / d - acc;
  return true;
}

}  // namespace tqhost
