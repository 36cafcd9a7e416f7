// Host-side Lloyd-Max codebook builder for N(0,1) ("Qwen3.6-35B-A3B -- HLWQ Q5"
// model card, Method step [4]: Lloyd-Max quantization with 32 centroids for
// N(0,1); "Qwen3.6-35B-A3B-TQ3-native", Files: loaders rebuild the codebook
// deterministically instead of storing it).
//
// The quantizer is symmetric, so only the L/2 non-negative centroids are
// iterated.  For a cell (a, b] on the positive half-line the conditional mean of
// Z ~ N(0,1) is (phi(a) - phi(b)) / (Q(a) - Q(b)) with Q the upper tail, which
// is evaluated through erfc so that no difference of numbers close to 1 occurs.
// The iteration runs until the centroids stop moving (the fp64 noise floor);
// the fixed point is unique for the Gaussian (log-concave density), so the
// result does not depend on the starting point.

#include <cmath>
#include <cstdint>
#include <vector>

#include "hlwq.h"

namespace {

constexpr double kInvSqrt2 = 0.70710678118654752440;
constexpr double kInvSqrt2Pi = 0.39894228040143267794;

double density(double x) { return std::isinf(x) ? 0.0 : kInvSqrt2Pi * std::exp(-0.5 * x * x); }

double tail(double x) {  // P(Z > x), x >= 0 here
  return std::isinf(x) ? 0.0 : 0.5 * std::erfc(x * kInvSqrt2);
}

// One Lloyd step on the positive half: cells (t_k, t_{k+1}] with t_0 = 0,
// t_k = (p_{k-1} + p_k) / 2, t_half = inf.
void lloyd_step(const std::vector<double>& p, std::vector<double>& out) {
  const size_t n = p.size();
  double lo = 0.0;
  for (size_t k = 0; k < n; ++k) {
    const double hi = (k + 1 < n) ? 0.5 * (p[k] + p[k + 1]) : INFINITY;
    out[k] = (density(lo) - density(hi)) / (tail(lo) - tail(hi));
    lo = hi;
  }
}

double mse_of(const std::vector<double>& c) {
  // E[(Z - q(Z))^2] with nearest-neighbour cells, summed over both halves.
  const size_t L = c.size();
  double d = 0.0;
  for (size_t k = 0; k < L; ++k) {
    const double a = (k == 0) ? -INFINITY : 0.5 * (c[k - 1] + c[k]);
    const double b = (k + 1 == L) ? INFINITY : 0.5 * (c[k] + c[k + 1]);
    // P(a < Z <= b), int z phi, int z^2 phi over the cell.
    double pr;
    if (a >= 0) pr = tail(a) - tail(b);
    else if (b <= 0) pr = tail(-b) - tail(-a);
    else pr = 1.0 - tail(-a) - tail(b);
    const double m1 = density(a) - density(b);
    const double m2 = pr + (std::isinf(a) ? 0.0 : a * density(a)) - (std::isinf(b) ? 0.0 : b * density(b));
    d += m2 - 2.0 * c[k] * m1 + c[k] * c[k] * pr;
  }
  return d;
}

}  // namespace

extern "C" int hlwq_lloyd_codebook(int levels, float* centroids, float* midpoints, double* mse) {
  if (!centroids) return HLWQ_EINVAL;
  if (levels != 2 && levels != 4 && levels != 8 && levels != 16 && levels != 32) return HLWQ_EINVAL;
  const int half = levels / 2;
  // Start from an even spacing on [0, 3]; any start converges to the same point.
  std::vector<double> p(half), q(half);
  for (int k = 0; k < half; ++k) p[k] = 3.0 * (k + 0.5) / half;
  double last = INFINITY;
  int stalled = 0;
  for (int it = 0; it < 1000000; ++it) {
    lloyd_step(p, q);
    double step = 0.0;
    for (int k = 0; k < half; ++k) step = std::fmax(step, std::fabs(q[k] - p[k]));
    p.swap(q);
    if (step == 0.0) break;
    if (step < last) {
      last = step;
      stalled = 0;
    } else if (++stalled > 200) {
      break;
    }
  }
  std::vector<double> c(levels);
  for (int k = 0; k < half; ++k) {
    c[half + k] = p[k];
    c[half - 1 - k] = -p[k];
  }
  for (int k = 0; k < levels; ++k) centroids[k] = static_cast<float>(c[k]);
  if (midpoints) {
    for (int k = 0; k + 1 < levels; ++k)
      midpoints[k] = static_cast<float>(0.5 * (static_cast<double>(centroids[k]) + centroids[k + 1]));
  }
  if (mse) *mse = mse_of(c);
  return HLWQ_OK;
}
