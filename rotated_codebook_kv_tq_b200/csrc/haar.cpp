// Host construction of a dense Haar rotation: the orthogonal factor Q of a
// square Gaussian matrix G = Q R with every diagonal entry of R made positive
// (each column of Q scaled by the sign of R's diagonal entry), which makes Q
// Haar distributed.  The shared random rotation of the theory ("Google
// presenta TurboQuant ...", "La mecanica geometrica de TurboQuant"; "FibQuant
// ...", section 2.1).  Householder reflections in fp64.
#include <cmath>
#include <vector>

namespace tqhost {

bool haar_rotation(int d, const float *g, std::vector<double> &pi) {
  if (d < 1 || !g) return false;
  const size_t n = static_cast<size_t>(d);
  // column-major working copy: a[i + j n] = G[i][j]
  std::vector<double> a(n * n), v(n * n, 0.0), vv(n, 0.0), rdiag(n, 0.0);
  for (size_t i = 0; i < n; ++i)
    for (size_t j = 0; j < n; ++j) a[i + j * n] = static_cast<double>(g[i * n + j]);
  for (size_t k = 0; k < n; ++k) {
    double nrm = 0.0;
    for (size_t i = k; i < n; ++i) nrm += a[i + k * n] * a[i + k * n];
    nrm = std::sqrt(nrm);
    const double alpha = a[k + k * n] >= 0.0 ? -nrm : nrm;   // the new R_kk
    double s2 = 0.0;
    for (size_t i = k; i < n; ++i) {
      const double vi = a[i + k * n] - (i == k ? alpha : 0.0);
      v[i + k * n] = vi;
      s2 += vi * vi;
    }
    vv[k] = s2;
    if (s2 > 0.0)
      for (size_t j = k; j < n; ++j) {   // a[k:, j] -= 2 v (v . a[k:, j]) / (v . v)
        double dot = 0.0;
        for (size_t i = k; i < n; ++i) dot += v[i + k * n] * a[i + j * n];
        const double f = 2.0 * dot / s2;
        for (size_t i = k; i < n; ++i) a[i + j * n] -= f * v[i + k * n];
      }
    rdiag[k] = a[k + k * n];
  }
  // Q = H_0 H_1 ... H_{n-1}, built by applying H_{n-1} first to the identity
  std::vector<double> q(n * n, 0.0);
  for (size_t i = 0; i < n; ++i) q[i + i * n] = 1.0;
  for (size_t kk = n; kk-- > 0;) {
    if (vv[kk] <= 0.0) continue;
    for (size_t j = 0; j < n; ++j) {
      double dot = 0.0;
      for (size_t i = kk; i < n; ++i) dot += v[i + kk * n] * q[i + j * n];
      const double f = 2.0 * dot / vv[kk];
      for (size_t i = kk; i < n; ++i) q[i + j * n] -= f * v[i + kk * n];
    }
  }
  pi.assign(n * n, 0.0);
  for (size_t j = 0; j < n; ++j) {
    const double sgn = rdiag[j] < 0.0 ? -1.0 : 1.0;
    for (size_t i = 0; i < n; ++i) pi[i * n + j] = q[i + j * n] * sgn;
  }
  return true;
}

}  // namespace tqhost
