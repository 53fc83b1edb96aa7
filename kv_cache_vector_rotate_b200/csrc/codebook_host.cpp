// Host-side (float64) construction of the codec constants.
//
// Method source: "TurboQuant explained" (a2a-mcp.org), §Stage 1 (rotation by
// the Q factor of a Gaussian matrix; Beta((d-1)/2,(d-1)/2) coordinate law;
// Lloyd-Max quantizer) and §Stage 2 (Gaussian QJL projection).  This runs once
// per codebook, off the hot path; all transcendental math stays on the host.

#include "codebook_host.h"

#include <algorithm>
#include <cmath>
#include <vector>

namespace tqhost {

// SplitMix64 (Steele, Lea & Flood 2014) in counter form: output i is the
// published mix of seed + (i + 1) * gamma.
static inline uint64_t splitmix_at(uint64_t seed, uint64_t i) {
  uint64_t z = seed + (i + 1) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

void gaussian_fill(uint64_t seed, size_t n, double* out) {
  // Box-Muller on uniform pairs (2k, 2k+1); a uniform is the top 53 bits.
  const double two_pi = 6.283185307179586476925286766559;
  for (size_t k = 0; 2 * k < n; ++k) {
    double u1 = (double)(splitmix_at(seed, 2 * k) >> 11) * 0x1.0p-53;
    double u2 = (double)(splitmix_at(seed, 2 * k + 1) >> 11) * 0x1.0p-53;
    double rho = std::sqrt(-2.0 * std::log1p(-u1));
    out[2 * k] = rho * std::cos(two_pi * u2);
    if (2 * k + 1 < n) out[2 * k + 1] = rho * std::sin(two_pi * u2);
  }
}

// Householder QR of a row-major n x n matrix A.  Returns Q (row-major) with
// the sign of each column chosen so that diag(R) > 0.
std::vector<double> orthogonal_factor(const std::vector<double>& A_in, int n) {
  std::vector<double> A(A_in);                // working copy, becomes R
  std::vector<std::vector<double>> vs;        // reflector vectors
  vs.reserve(n);
  for (int k = 0; k < n; ++k) {
    std::vector<double> v(n - k);
    double norm2 = 0.0;
    for (int i = k; i < n; ++i) {
      v[i - k] = A[(size_t)i * n + k];
      norm2 += v[i - k] * v[i - k];
    }
    double alpha = std::sqrt(norm2);
    if (v[0] > 0) alpha = -alpha;             // R_kk = alpha, avoids cancellation
    v[0] -= alpha;
    double vn2 = 0.0;
    for (double e : v) vn2 += e * e;
    if (vn2 > 0.0) {
      double inv = 1.0 / std::sqrt(vn2);
      for (double& e : v) e *= inv;
      for (int j = k; j < n; ++j) {           // A[k:, j] -= 2 v (v . A[k:, j])
        double dot = 0.0;
        for (int i = k; i < n; ++i) dot += v[i - k] * A[(size_t)i * n + j];
        for (int i = k; i < n; ++i) A[(size_t)i * n + j] -= 2.0 * v[i - k] * dot;
      }
    }
    vs.push_back(std::move(v));
  }
  // Q = H_0 H_1 ... H_{n-1}: apply the reflectors to I in reverse order.
  std::vector<double> Q((size_t)n * n, 0.0);
  for (int i = 0; i < n; ++i) Q[(size_t)i * n + i] = 1.0;
  for (int k = n - 1; k >= 0; --k) {
    const std::vector<double>& v = vs[k];
    for (int j = 0; j < n; ++j) {
      double dot = 0.0;
      for (int i = k; i < n; ++i) dot += v[i - k] * Q[(size_t)i * n + j];
      for (int i = k; i < n; ++i) Q[(size_t)i * n + j] -= 2.0 * v[i - k] * dot;
    }
  }
  for (int k = 0; k < n; ++k) {
    if (A[(size_t)k * n + k] < 0.0)
      for (int i = 0; i < n; ++i) Q[(size_t)i * n + k] = -Q[(size_t)i * n + k];
  }
  return Q;
}

// ---- Lloyd-Max for f(t) = C_d (1 - t^2)^((d-3)/2) on [-1, 1] -------------
// Integrals are taken in theta = asin t, where the integrand
// C_d cos^(d-2)(theta) is smooth for every d >= 2.  Gauss-Legendre nodes are
// found by Newton's method on the Legendre polynomial (three-term recurrence).

namespace {

struct Gauss {
  std::vector<double> x, w;
  explicit Gauss(int n) : x(n), w(n) {
    const double pi = 3.14159265358979323846;
    for (int i = 0; i < n; ++i) {
      double z = std::cos(pi * (i + 0.75) / (n + 0.5));
      double dp = 1.0;
      for (int it = 0; it < 100; ++it) {
        double p0 = 1.0, p1 = z;
        for (int k = 2; k <= n; ++k) {
          double p2 = ((2.0 * k - 1.0) * z * p1 - (k - 1.0) * p0) / k;
          p0 = p1;
          p1 = p2;
        }
        dp = n * (z * p1 - p0) / (z * z - 1.0);   // P_n'(z)
        double dz = p1 / dp;
        z -= dz;
        if (std::fabs(dz) < 1e-16) break;
      }
      x[i] = z;
      w[i] = 2.0 / ((1.0 - z * z) * dp * dp);
    }
  }
};

struct Moments {
  double p, m1, m2;
};

// The coordinate law of §Stage 1.  Start cells: equal probability, from a
// trapezoid CDF in theta.
class BetaLaw {
 public:
  explicit BetaLaw(int d) : d_(d), gauss_(24) {
    c_ = std::exp(std::lgamma(d / 2.0) - 0.5 * std::log(3.14159265358979323846) -
                  std::lgamma((d - 1) / 2.0));
  }
  double lo() const { return -1.0; }
  double hi() const { return 1.0; }
  double centre() const { return 0.0; }
  double density(double t) const {
    double s = 1.0 - t * t;
    if (s <= 0.0) return 0.0;
    return c_ * std::pow(s, (d_ - 3) / 2.0);
  }
  Moments cell(double lo, double hi) const {
    const int panels = 48;
    double a = std::asin(std::max(-1.0, std::min(1.0, lo)));
    double b = std::asin(std::max(-1.0, std::min(1.0, hi)));
    double h = (b - a) / panels;
    Moments r{0.0, 0.0, 0.0};
    for (int p = 0; p < panels; ++p) {
      double mid = a + (p + 0.5) * h, half = 0.5 * h;
      for (size_t i = 0; i < gauss_.x.size(); ++i) {
        double th = mid + half * gauss_.x[i];
        double g = half * gauss_.w[i] * std::pow(std::cos(th), d_ - 2);
        double s = std::sin(th);
        r.p += g;
        r.m1 += g * s;
        r.m2 += g * s * s;
      }
    }
    r.p *= c_;
    r.m1 *= c_;
    r.m2 *= c_;
    return r;
  }
  std::vector<double> equiprobable_edges(int K) const {
    const int G = 20001;
    const double half_pi = 1.57079632679489661923;
    std::vector<double> th(G), cdf(G, 0.0);
    for (int i = 0; i < G; ++i) th[i] = -half_pi + 2.0 * half_pi * i / (G - 1);
    for (int i = 1; i < G; ++i)
      cdf[i] = cdf[i - 1] + 0.5 * (std::pow(std::cos(th[i]), d_ - 2) +
                                   std::pow(std::cos(th[i - 1]), d_ - 2)) * (th[i] - th[i - 1]);
    std::vector<double> qe(K + 1);
    qe[0] = -1.0;
    qe[K] = 1.0;
    int j = 0;
    for (int k = 1; k < K; ++k) {
      double target = (double)k / K * cdf[G - 1];
      while (j < G - 2 && cdf[j + 1] < target) ++j;
      double fr = (target - cdf[j]) / (cdf[j + 1] - cdf[j]);
      qe[k] = std::sin(th[j] + fr * (th[j + 1] - th[j]));
    }
    return qe;
  }

 private:
  int d_;
  double c_;
  Gauss gauss_;
};

// The law of a level-`level` angle of the recursive polar form of §Stage 1
// for a uniform unit vector: level 1 uniform on [-pi, pi]; level l > 1, whose
// radii each cover k = 2^(l-1) coordinates, 2 (sin phi cos phi)^(k-1) /
// B(k/2, k/2) on [0, pi/2] (sin^2 phi follows Beta(k/2, k/2)).  Smooth on its
// support, so cells are integrated in phi directly.
class AngleLaw {
 public:
  explicit AngleLaw(int level) : level_(level), gauss_(24) {
    const double pi = 3.14159265358979323846;
    if (level == 1) {
      lo_ = -pi;
      hi_ = pi;
      logc_ = -std::log(2.0 * pi);
    } else {
      const double k = std::ldexp(1.0, level - 1);
      lo_ = 0.0;
      hi_ = 0.5 * pi;
      logc_ = std::log(2.0) + std::lgamma(k) - 2.0 * std::lgamma(0.5 * k);
    }
  }
  double lo() const { return lo_; }
  double hi() const { return hi_; }
  double centre() const { return 0.5 * (lo_ + hi_); }
  double density(double phi) const {
    if (phi < lo_ || phi > hi_) return 0.0;
    if (level_ == 1) return std::exp(logc_);
    const double s = std::sin(phi) * std::cos(phi);
    if (s <= 0.0) return 0.0;
    return std::exp(logc_ + (std::ldexp(1.0, level_ - 1) - 1.0) * std::log(s));
  }
  Moments cell(double a, double b) const {
    const int panels = 48;
    const double h = (b - a) / panels;
    Moments r{0.0, 0.0, 0.0};
    for (int p = 0; p < panels; ++p) {
      const double mid = a + (p + 0.5) * h, half = 0.5 * h;
      for (size_t i = 0; i < gauss_.x.size(); ++i) {
        const double x = mid + half * gauss_.x[i];
        const double g = half * gauss_.w[i] * density(x);
        r.p += g;
        r.m1 += g * x;
        r.m2 += g * x * x;
      }
    }
    return r;
  }
  std::vector<double> equiprobable_edges(int K) const {
    const int G = 20001;
    std::vector<double> x(G), cdf(G, 0.0);
    for (int i = 0; i < G; ++i) x[i] = lo_ + (hi_ - lo_) * i / (G - 1);
    for (int i = 1; i < G; ++i) cdf[i] = cdf[i - 1] + 0.5 * (density(x[i]) + density(x[i - 1])) * (x[i] - x[i - 1]);
    std::vector<double> qe(K + 1);
    qe[0] = lo_;
    qe[K] = hi_;
    int j = 0;
    for (int k = 1; k < K; ++k) {
      const double target = (double)k / K * cdf[G - 1];
      while (j < G - 2 && cdf[j + 1] < target) ++j;
      const double fr = (target - cdf[j]) / (cdf[j + 1] - cdf[j]);
      qe[k] = x[j] + fr * (x[j + 1] - x[j]);
    }
    return qe;
  }

 private:
  int level_;
  double lo_, hi_, logc_;
  Gauss gauss_;
};

// Lloyd-Max quantizer of a law symmetric about its centre (Lloyd 1957/1982,
// Max 1960): centroids are the conditional means of their cells, boundaries
// the midpoints.  Lloyd sweeps from the equal-probability cells, then Newton
// on F_i(c) = c_i - mean_i(c) (tridiagonal Jacobian); the laws here are
// log-concave, so the fixed point is unique.  The result is made exactly
// symmetric about the centre.
template <class Law>
LloydMax lloyd_max_law(const Law& law, int K) {
  std::vector<double> c(K), e(K + 1);
  {
    const std::vector<double> qe = law.equiprobable_edges(K);
    for (int k = 0; k < K; ++k) {
      Moments m = law.cell(qe[k], qe[k + 1]);
      c[k] = m.m1 / m.p;
    }
  }
  auto edges = [&](const std::vector<double>& cc) {
    e[0] = law.lo();
    e[K] = law.hi();
    for (int i = 1; i < K; ++i) e[i] = 0.5 * (cc[i - 1] + cc[i]);
  };
  std::vector<Moments> mo(K);
  auto moments = [&]() {
    edges(c);
    for (int i = 0; i < K; ++i) mo[i] = law.cell(e[i], e[i + 1]);
  };
  for (int it = 0; it < 300; ++it) {
    moments();
    double step = 0.0;
    for (int i = 0; i < K; ++i) {
      double nc = mo[i].m1 / mo[i].p;
      step = std::max(step, std::fabs(nc - c[i]));
      c[i] = nc;
    }
    if (step < 1e-15) break;
  }
  for (int it = 0; it < 60; ++it) {
    moments();
    std::vector<double> F(K), lower(K, 0.0), diag(K, 1.0), upper(K, 0.0);
    double fmax = 0.0;
    for (int i = 0; i < K; ++i) {
      double mu = mo[i].m1 / mo[i].p;
      F[i] = c[i] - mu;
      fmax = std::max(fmax, std::fabs(F[i]));
      double flo = (i > 0) ? law.density(e[i]) : 0.0;
      double fhi = (i < K - 1) ? law.density(e[i + 1]) : 0.0;
      double dlo = flo * (mu - e[i]) / mo[i].p;       // d mean_i / d e_i
      double dhi = fhi * (e[i + 1] - mu) / mo[i].p;   // d mean_i / d e_{i+1}
      diag[i] = 1.0 - 0.5 * (dlo + dhi);
      if (i > 0) lower[i] = -0.5 * dlo;
      if (i < K - 1) upper[i] = -0.5 * dhi;
    }
    if (fmax < 1e-15) break;
    // Thomas algorithm for the tridiagonal system J delta = F.
    std::vector<double> cp(K), dp(K);
    cp[0] = upper[0] / diag[0];
    dp[0] = F[0] / diag[0];
    for (int i = 1; i < K; ++i) {
      double den = diag[i] - lower[i] * cp[i - 1];
      cp[i] = (i < K - 1) ? upper[i] / den : 0.0;
      dp[i] = (F[i] - lower[i] * dp[i - 1]) / den;
    }
    std::vector<double> delta(K);
    delta[K - 1] = dp[K - 1];
    for (int i = K - 2; i >= 0; --i) delta[i] = dp[i] - cp[i] * delta[i + 1];
    for (int i = 0; i < K; ++i) c[i] -= delta[i];
  }
  const double ctr = law.centre();
  std::vector<double> cs(K);
  for (int i = 0; i < K; ++i) cs[i] = ctr + 0.5 * ((c[i] - ctr) - (c[K - 1 - i] - ctr));
  LloydMax out;
  out.centroids = cs;
  out.boundaries.resize(K - 1);
  for (int i = 1; i < K; ++i) out.boundaries[i - 1] = 0.5 * (cs[i - 1] + cs[i]);
  out.distortion = 0.0;
  e[0] = law.lo();
  e[K] = law.hi();
  for (int i = 1; i < K; ++i) e[i] = out.boundaries[i - 1];
  for (int i = 0; i < K; ++i) {
    Moments m = law.cell(e[i], e[i + 1]);
    out.distortion += m.m2 - 2.0 * cs[i] * m.m1 + cs[i] * cs[i] * m.p;
  }
  return out;
}

}  // namespace

LloydMax lloyd_max(int d, int bits) { return lloyd_max_law(BetaLaw(d), 1 << bits); }

LloydMax polar_angle_lloyd_max(int level, int bits) { return lloyd_max_law(AngleLaw(level), 1 << bits); }

}  // namespace tqhost
