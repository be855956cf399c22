// Host-side Lloyd-Max codebook (fp64) for one coordinate of a randomly rotated unit vector.
//
// Density ("谷歌 TurboQuant 深度拆解", 第六部分 "为什么随机旋转这么关键"):
//   f_X(x) = C_d (1 - x^2)^((d-3)/2) on [-1, 1].
// Quantizer ("TurboQuant 学习路径", 三.4 Lloyd-Max; same juejin page, 第二部分 第一步): Lloyd's
// iteration, thresholds = midpoints of neighbouring centroids, centroids = conditional means.
//
// Integrals are evaluated in closed form.  With x = sin(theta) the density element becomes
// cos^(d-2)(theta) d(theta); for even d write d - 2 = 2n and use the stable recursion
//   J_k(phi) = int_0^phi cos^(2k) = cos^(2k-1)(phi) sin(phi) / (2k) + (2k-1)/(2k) J_(k-1)(phi),
//   J_0(phi) = phi.
// Then F(x) = 1/2 + J_n(asin x) / (2 J_n(pi/2)) (so C_d = 1 / (2 J_n(pi/2))), the first moment
// of a cell is C_d [(1-a^2)^((d-1)/2) - (1-b^2)^((d-1)/2)] / (d-1), and the second moment is
// P_d - (d-1)/d P_(d+2) (the density of dimension d+2 is proportional to (1-x^2)^((d-1)/2)).
#include <cmath>
#include <vector>

#include "tq_internal.h"

namespace {

struct CoordLaw {
  int n;          // (d - 2) / 2
  double jhalf;   // J_n(pi/2)
  double d;

  explicit CoordLaw(int d_) : n((d_ - 2) / 2), d(d_) { jhalf = J(M_PI / 2); }

  double J(double phi) const {
    const double c = std::cos(phi), s = std::sin(phi);
    double j = phi;
    double cp = c;  // cos^(2k-1)
    for (int k = 1; k <= n; ++k) {
      j = cp * s / (2.0 * k) + (2.0 * k - 1.0) / (2.0 * k) * j;
      cp *= c * c;
    }
    return j;
  }
  double phi(double x) const { return std::asin(std::fmax(-1.0, std::fmin(1.0, x))); }
  // P(a <= X < b)
  double mass(double a, double b) const { return (J(phi(b)) - J(phi(a))) / (2.0 * jhalf); }
  // int_a^b x f(x) dx
  double moment1(double a, double b) const {
    const double e = (d - 1.0) / 2.0;
    return (std::pow(1.0 - a * a, e) - std::pow(1.0 - b * b, e)) / (2.0 * jhalf * (d - 1.0));
  }
};

}  // namespace

tq_status tq_codebook_fp64(int d, int bits, double *centroids, double *thresholds, double *mse) {
  const int L = 1 << bits;
  CoordLaw law(d);
  std::vector<double> c(L), cn(L), e(L + 1);
  // start: evenly spaced over +-3 standard deviations of X (variance 1/d)
  for (int i = 0; i < L; ++i) c[i] = (2.0 * (i + 0.5) / L - 1.0) * 3.0 / std::sqrt((double)d);
  for (int it = 0; it < 2000000; ++it) {
    e[0] = -1.0;
    e[L] = 1.0;
    for (int i = 1; i < L; ++i) e[i] = 0.5 * (c[i - 1] + c[i]);
    double move = 0.0;
    for (int i = 0; i < L; ++i) {
      cn[i] = law.moment1(e[i], e[i + 1]) / law.mass(e[i], e[i + 1]);
      move = std::fmax(move, std::fabs(cn[i] - c[i]));
    }
    c.swap(cn);
    if (move < 1e-13) break;
  }
  // the density is even, so the exact codebook is antisymmetric: impose c_i = -c_(L-1-i), which
  // makes the middle threshold exactly 0
  for (int i = 0; i < L / 2; ++i) {
    const double a = 0.5 * (c[L - 1 - i] - c[i]);
    c[i] = -a;
    c[L - 1 - i] = a;
  }
  for (int i = 0; i < L; ++i) centroids[i] = c[i];
  for (int i = 1; i < L; ++i) thresholds[i - 1] = 0.5 * (c[i - 1] + c[i]);
  if (mse) {
    CoordLaw law2(d + 2);
    e[0] = -1.0;
    e[L] = 1.0;
    for (int i = 1; i < L; ++i) e[i] = thresholds[i - 1];
    double acc = 0.0;
    for (int i = 0; i < L; ++i) {
      const double p = law.mass(e[i], e[i + 1]);
      const double m1 = law.moment1(e[i], e[i + 1]);
      const double m2 = p - (d - 1.0) / d * law2.mass(e[i], e[i + 1]);
      acc += m2 - 2.0 * c[i] * m1 + c[i] * c[i] * p;
    }
    *mse = acc;
  }
  return TQ_OK;
}

// ------------------------------------------------------------------ PolarQuant angle codebooks
// ("谷歌 TurboQuant 深度拆解" 第二部分 第一步: the rotated vector in recursive polar form; the angle
// laws are known in advance.)  Level 1 angles of a uniformly random direction are uniform on
// (-pi, pi]: 2^b equal cells from -pi, centroids at the cell middles.  A level-l angle (l >= 2) is
// atan2 of two independent radii of k = 2^(l-1) coordinates each, with density
//   f_l(a) = 2 (sin a cos a)^(k-1) / B(k/2, k/2) on [0, pi/2];
// its Lloyd-Max codebook is iterated with composite Gauss-Legendre quadrature of each cell.
namespace {

// 16-point Gauss-Legendre nodes and weights on [-1, 1], by Newton's method on P_16.
struct GaussLegendre16 {
  double x[16], w[16];
  GaussLegendre16() {
    const int n = 16;
    for (int i = 0; i < n; ++i) {
      double z = std::cos(M_PI * (i + 0.75) / (n + 0.5)), dp = 0.0;
      for (int it = 0; it < 100; ++it) {
        double p0 = 1.0, p1 = z;
        for (int k = 2; k <= n; ++k) {
          const double p2 = ((2.0 * k - 1.0) * z * p1 - (k - 1.0) * p0) / k;
          p0 = p1;
          p1 = p2;
        }
        dp = n * (z * p1 - p0) / (z * z - 1.0);
        const double dz = p1 / dp;
        z -= dz;
        if (std::fabs(dz) < 1e-16) break;
      }
      x[i] = z;
      w[i] = 2.0 / ((1.0 - z * z) * dp * dp);
    }
  }
};

struct AngleLaw {
  double k, lognorm;
  explicit AngleLaw(int level) : k(std::ldexp(1.0, level - 1)) {
    // log(2 / B(k/2, k/2))
    lognorm = std::log(2.0) - (2.0 * std::lgamma(k / 2.0) - std::lgamma(k));
  }
  double f(double a) const {
    const double sc = std::sin(a) * std::cos(a);
    return sc <= 0.0 ? 0.0 : std::exp(lognorm + (k - 1.0) * std::log(sc));
  }
  // int_lo^hi f and int_lo^hi a f, 64 panels of 16-point Gauss-Legendre
  void moments(double lo, double hi, double &m0, double &m1) const {
    static const GaussLegendre16 gl;
    m0 = m1 = 0.0;
    const int panels = 64;
    const double h = (hi - lo) / panels;
    for (int p = 0; p < panels; ++p) {
      const double a0 = lo + p * h, mid = a0 + 0.5 * h;
      for (int i = 0; i < 16; ++i) {
        const double a = mid + 0.5 * h * gl.x[i], wv = 0.5 * h * gl.w[i] * f(a);
        m0 += wv;
        m1 += wv * a;
      }
    }
  }
};

}  // namespace

tq_status tq_polar_codebook_fp64(int level, int bits, double *centroids, double *thresholds) {
  const int L = 1 << bits;
  if (level == 1) {
    const double w = 2.0 * M_PI / L;
    for (int i = 0; i < L; ++i) centroids[i] = -M_PI + w * (i + 0.5);
    for (int i = 1; i < L; ++i) thresholds[i - 1] = -M_PI + w * i;
    return TQ_OK;
  }
  AngleLaw law(level);
  std::vector<double> c(L), cn(L), e(L + 1);
  // start at evenly spaced points over +-3 standard deviations around pi/4 (sd ~ 1 / (2 sqrt(k)))
  const double sd = 0.5 / std::sqrt(law.k);
  for (int i = 0; i < L; ++i)
    c[i] = std::fmin(M_PI / 2 - 1e-6, std::fmax(1e-6, M_PI / 4 + (2.0 * (i + 0.5) / L - 1.0) * 3.0 * sd));
  for (int it = 0; it < 200000; ++it) {
    e[0] = 0.0;
    e[L] = M_PI / 2;
    for (int i = 1; i < L; ++i) e[i] = 0.5 * (c[i - 1] + c[i]);
    double move = 0.0;
    for (int i = 0; i < L; ++i) {
      double m0, m1;
      law.moments(e[i], e[i + 1], m0, m1);
      cn[i] = m0 > 0.0 ? m1 / m0 : 0.5 * (e[i] + e[i + 1]);
      move = std::fmax(move, std::fabs(cn[i] - c[i]));
    }
    c.swap(cn);
    if (move < 1e-13) break;
  }
  // the law is symmetric about pi/4: impose it exactly
  for (int i = 0; i < L / 2; ++i) {
    const double a = 0.5 * ((M_PI / 2 - c[L - 1 - i]) + c[i]);
    c[i] = a;
    c[L - 1 - i] = M_PI / 2 - a;
  }
  for (int i = 0; i < L; ++i) centroids[i] = c[i];
  for (int i = 1; i < L; ++i) thresholds[i - 1] = 0.5 * (c[i - 1] + c[i]);
  return TQ_OK;
}
