// Host construction of the FibQuant k = 2 pair codebook.
//
// "FibQuant: Quantizzazione Vettoriale Universale ..." section 2.1: two
// consecutive coordinates of a randomly rotated unit vector follow
// f_{d,2}(x) = (d-2)/(2 pi) (1 - |x|^2)^((d-4)/2) on the unit disk, so
// T = |x|^2 ~ Beta(1, b), b = (d-2)/2, with CDF 1 - (1 - t)^b.
// Section 2.2: the start puts codeword n of N on the golden-angle spiral,
// angle n pi (3 - sqrt 5), at the radius where the Bennett-Gersho point density
// f^(1/2) has radial CDF (n + delta)/N, r_n^2 = 1 - (1 - (n + delta)/N)^(4/d);
// Lloyd-Max steps then refine it for the finite N, restarted from several
// deltas.
//
// The Lloyd steps run on a fixed quadrature of f: NU shells of T of equal
// probability, each at its conditional mean of T (closed form for the
// Beta(1, b) law), times NA equally spaced angles, all of equal weight.  Each
// step assigns every point to its nearest codeword (first one on a tie) and
// moves each codeword to the mean of its points (an empty cell stays put).
// The restart with the smallest quadrature MSE is kept; a later restart
// replaces an earlier one only when lower by more than a relative 1e-9.
#include <cmath>
#include <map>
#include <mutex>
#include <utility>
#include <vector>

namespace tqhost {

namespace {

constexpr int kShells = 256;
constexpr int kAngles = 256;
constexpr int kSteps = 100;
constexpr double kDeltas[3] = {0.25, 0.5, 0.75};
constexpr double kMargin = 1e-9;

struct Grid {
  std::vector<double> x, y;
};

Grid make_grid(int d) {
  const double b = (d - 2) / 2.0;
  std::vector<double> r(kShells);
  for (int i = 0; i < kShells; ++i) {
    // shell between CDF values p0 = i/NU and p1 = (i+1)/NU of T
    const double p0 = static_cast<double>(i) / kShells, p1 = static_cast<double>(i + 1) / kShells;
    const double t0 = 1.0 - std::pow(1.0 - p0, 1.0 / b), t1 = 1.0 - std::pow(1.0 - p1, 1.0 / b);
    // int_{t0}^{t1} t dF(t) by parts, with (1 - t)^b = 1 - p
    const double part = t0 * (1.0 - p0) - t1 * (1.0 - p1) +
                        (std::pow(1.0 - p0, (b + 1) / b) - std::pow(1.0 - p1, (b + 1) / b)) / (b + 1);
    r[i] = std::sqrt(part * kShells);
  }
  Grid g;
  g.x.resize(static_cast<size_t>(kShells) * kAngles);
  g.y.resize(g.x.size());
  const double two_pi = 2.0 * M_PI;
  for (int j = 0; j < kAngles; ++j) {
    const double ph = two_pi * (j + 0.5) / kAngles;
    const double cs = std::cos(ph), sn = std::sin(ph);
    for (int i = 0; i < kShells; ++i) {
      g.x[static_cast<size_t>(i) * kAngles + j] = r[i] * cs;
      g.y[static_cast<size_t>(i) * kAngles + j] = r[i] * sn;
    }
  }
  return g;
}

// Nearest codeword of point (px, py); writes the squared distance.
inline int nearest(double px, double py, const std::vector<double> &cx,
                   const std::vector<double> &cy, double &dist) {
  int best = 0;
  double bd = 0.0;
  for (size_t n = 0; n < cx.size(); ++n) {
    const double dx = px - cx[n], dy = py - cy[n];
    const double dd = dx * dx + dy * dy;
    if (n == 0 || dd < bd) {
      bd = dd;
      best = static_cast<int>(n);
    }
  }
  dist = bd;
  return best;
}

double refine(const Grid &g, std::vector<double> &cx, std::vector<double> &cy) {
  const size_t N = cx.size(), P = g.x.size();
  std::vector<double> sx(N), sy(N);
  std::vector<long> cnt(N);
  double dist = 0.0;
  for (int s = 0; s < kSteps; ++s) {
    std::fill(sx.begin(), sx.end(), 0.0);
    std::fill(sy.begin(), sy.end(), 0.0);
    std::fill(cnt.begin(), cnt.end(), 0L);
    for (size_t p = 0; p < P; ++p) {
      const int n = nearest(g.x[p], g.y[p], cx, cy, dist);
      sx[n] += g.x[p];
      sy[n] += g.y[p];
      ++cnt[n];
    }
    for (size_t n = 0; n < N; ++n)
      if (cnt[n] > 0) {
        cx[n] = sx[n] / static_cast<double>(cnt[n]);
        cy[n] = sy[n] / static_cast<double>(cnt[n]);
      }
  }
  double tot = 0.0;
  for (size_t p = 0; p < P; ++p) {
    nearest(g.x[p], g.y[p], cx, cy, dist);
    tot += dist;
  }
  return tot / static_cast<double>(P);
}

struct Solved {
  std::vector<double> c;   // x0, y0, x1, y1, ...
  double mse;
};

std::mutex g_mu;
std::map<std::pair<int, int>, Solved> g_solved;

}  // namespace

bool fq_pair_codebook(int d, int bits, std::vector<double> &c, double &mse) {
  if (d < 4 || bits < 1 || bits > 8) return false;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_solved.find({d, bits});
    if (it != g_solved.end()) {
      c = it->second.c;
      mse = it->second.mse;
      return true;
    }
  }
  const Grid g = make_grid(d);
  const int N = 1 << bits;
  const double golden = M_PI * (3.0 - std::sqrt(5.0));
  Solved best{{}, 0.0};
  bool have = false;
  for (double delta : kDeltas) {
    std::vector<double> cx(N), cy(N);
    for (int n = 0; n < N; ++n) {
      const double r = std::sqrt(1.0 - std::pow(1.0 - (n + delta) / N, 4.0 / d));
      const double th = n * golden;
      cx[n] = r * std::cos(th);
      cy[n] = r * std::sin(th);
    }
    const double m = refine(g, cx, cy);
    if (!have || m < best.mse * (1.0 - kMargin)) {
      best.c.assign(2 * static_cast<size_t>(N), 0.0);
      for (int n = 0; n < N; ++n) {
        best.c[2 * n] = cx[n];
        best.c[2 * n + 1] = cy[n];
      }
      best.mse = m;
      have = true;
    }
  }
  std::lock_guard<std::mutex> lk(g_mu);
  g_solved[{d, bits}] = best;
  c = best.c;
  mse = best.mse;
  return true;
}

}  // namespace tqhost
