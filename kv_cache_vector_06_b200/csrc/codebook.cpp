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
