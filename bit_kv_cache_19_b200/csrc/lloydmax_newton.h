// Gaussian Lloyd-Max codebooks by Newton's method on the thresholds.
//
// TQ-MSE ("RoPE-Aware Bit Allocation for KV-Cache Quantization", abstract:
// Block-GTQ is built on TurboQuant-MSE) codes each normalised coordinate with
// an MSE-optimal scalar codebook; the reading adopted is the Lloyd-Max
// quantizer of a unit Gaussian with 2^b levels, b = 1..8.
//
// The optimum satisfies t_i = (c_i + c_{i+1}) / 2 for the L-1 thresholds,
// with c_i the conditional mean of cell (t_{i-1}, t_i]:
//   c(a, b) = (phi(a) - phi(b)) / (Phi(b) - Phi(a)),
//   dc/da = phi(a) (c - a) / P,   dc/db = phi(b) (b - c) / P.
// F_i(t) = t_i - (c_i + c_{i+1}) / 2 has a tridiagonal Jacobian, so each
// Newton step is one Thomas solve. Start: centroids at the Gaussian
// quantiles (m + 1/2) / L. Converges quadratically to fp64 accuracy.
//
// Frozen codebook: centroids rounded once to fp16 (round to nearest even,
// directly from fp64), thresholds = exact midpoints of adjacent frozen
// centroids (exact in fp32).
#pragma once

#include <cmath>
#include <cstdint>
#include <vector>

namespace kvq_lm {

inline double pdf(double x) {
  if (!std::isfinite(x)) return 0.0;
  return 0.3989422804014326779399461 * std::exp(-0.5 * x * x);
}

// P(a < X <= b), accurate in both tails.
inline double cell_prob(double a, double b) {
  const double r = 0.7071067811865475244008444;
  if (a >= 0.0) return 0.5 * (std::erfc(a * r) - std::erfc(b * r));
  if (b <= 0.0) return 0.5 * (std::erfc(-b * r) - std::erfc(-a * r));
  return 1.0 - 0.5 * std::erfc(-a * r) - 0.5 * std::erfc(b * r);
}

inline double inv_cdf(double p) {  // bisection on the CDF; only for the start point
  double lo = -12.0, hi = 12.0;
  const double r = 0.7071067811865475244008444;
  for (int it = 0; it < 200; ++it) {
    double mid = 0.5 * (lo + hi);
    double c = 0.5 * std::erfc(-mid * r);
    (c < p ? lo : hi) = mid;
  }
  return 0.5 * (lo + hi);
}

struct Codebook {
  std::vector<double> c;  // fp64 centroids, ascending
  double D = 1.0;         // distortion per unit variance
};

inline void centroids_of(const std::vector<double>& t, std::vector<double>& c,
                         std::vector<double>& P) {
  const size_t L = t.size() + 1;
  c.assign(L, 0.0);
  P.assign(L, 0.0);
  for (size_t i = 0; i < L; ++i) {
    double a = i == 0 ? -INFINITY : t[i - 1];
    double b = i == L - 1 ? INFINITY : t[i];
    P[i] = cell_prob(a, b);
    c[i] = (pdf(a) - pdf(b)) / P[i];
  }
}

// Distortion of centroids c with midpoint cells: per cell (a, b] with mean c,
// E[(X - c)^2; cell] = (1 + c^2) P - 2 c (phi(a) - phi(b)) + a phi(a) - b phi(b).
inline double distortion(const std::vector<double>& c) {
  const size_t L = c.size();
  double D = 0.0;
  for (size_t i = 0; i < L; ++i) {
    double a = i == 0 ? -INFINITY : 0.5 * (c[i - 1] + c[i]);
    double b = i == L - 1 ? INFINITY : 0.5 * (c[i] + c[i + 1]);
    double P = cell_prob(a, b), fa = pdf(a), fb = pdf(b);
    double afa = std::isfinite(a) ? a * fa : 0.0, bfb = std::isfinite(b) ? b * fb : 0.0;
    D += (1.0 + c[i] * c[i]) * P - 2.0 * c[i] * (fa - fb) + afa - bfb;
  }
  return D;
}

inline Codebook solve(int bits) {
  const int L = 1 << bits;
  Codebook cb;
  std::vector<double> c(L), t(L - 1), P, F(L - 1), lo(L - 1), di(L - 1), up(L - 1);
  for (int m = 0; m < L; ++m) c[m] = inv_cdf((m + 0.5) / L);
  for (int i = 0; i < L - 1; ++i) t[i] = 0.5 * (c[i] + c[i + 1]);
  for (int it = 0; it < 200; ++it) {
    centroids_of(t, c, P);
    double fmax = 0.0;
    for (int i = 0; i < L - 1; ++i) {
      F[i] = t[i] - 0.5 * (c[i] + c[i + 1]);
      fmax = std::fmax(fmax, std::fabs(F[i]));
    }
    if (fmax < 1e-15) break;
    // Jacobian rows i: dF_i/dt_{i-1}, dF_i/dt_i, dF_i/dt_{i+1}
    for (int i = 0; i < L - 1; ++i) {
      // cell i is (t_{i-1}, t_i], cell i+1 is (t_i, t_{i+1}]
      double dci_dti = pdf(t[i]) * (t[i] - c[i]) / P[i];
      double dcj_dti = pdf(t[i]) * (c[i + 1] - t[i]) / P[i + 1];
      di[i] = 1.0 - 0.5 * (dci_dti + dcj_dti);
      lo[i] = i > 0 ? -0.5 * pdf(t[i - 1]) * (c[i] - t[i - 1]) / P[i] : 0.0;
      up[i] = i < L - 2 ? -0.5 * pdf(t[i + 1]) * (t[i + 1] - c[i + 1]) / P[i + 1] : 0.0;
    }
    // Thomas algorithm for J dx = -F
    std::vector<double> cp(L - 1), dp(L - 1);
    for (int i = 0; i < L - 1; ++i) {
      double den = di[i] - (i > 0 ? lo[i] * cp[i - 1] : 0.0);
      cp[i] = up[i] / den;
      dp[i] = (-F[i] - (i > 0 ? lo[i] * dp[i - 1] : 0.0)) / den;
    }
    for (int i = L - 3; i >= 0; --i) dp[i] -= cp[i] * dp[i + 1];
    for (int i = 0; i < L - 1; ++i) t[i] += dp[i];
  }
  centroids_of(t, c, P);
  cb.c.resize(L);
  for (int m = 0; m < L; ++m) cb.c[m] = 0.5 * (c[m] - c[L - 1 - m]);  // exact symmetry
  cb.D = distortion(cb.c);
  return cb;
}

// fp64 -> fp16 bits, round to nearest even, directly (no fp32 step).
inline uint16_t to_half_bits(double x) {
  uint16_t sign = std::signbit(x) ? 0x8000u : 0u;
  double a = std::fabs(x);
  if (std::isnan(x)) return 0x7E00u;
  if (a >= 65520.0) return sign | 0x7C00u;
  int e;
  std::frexp(a, &e);          // a = f 2^e, f in [0.5, 1)
  int ue = e - 1;             // a in [2^ue, 2^(ue+1))
  if (ue < -14) ue = -14;     // subnormal spacing 2^-24
  double ulp = std::ldexp(1.0, ue - 10);
  double q = std::nearbyint(a / ulp);  // default rounding: to nearest even
  double v = q * ulp;
  // encode
  if (v == 0.0) return sign;
  int ve;
  std::frexp(v, &ve);
  int ex = ve - 1;
  if (ex < -14) return sign | (uint16_t)(v / std::ldexp(1.0, -24));
  uint16_t mant = (uint16_t)(v / std::ldexp(1.0, ex - 10)) - 1024;
  return sign | (uint16_t)((ex + 15) << 10) | mant;
}

inline double half_bits_to_double(uint16_t h) {
  int ex = (h >> 10) & 31, mant = h & 1023;
  double v = ex == 0 ? std::ldexp((double)mant, -24) : std::ldexp(1024.0 + mant, ex - 25);
  return (h & 0x8000u) ? -v : v;
}

}  // namespace kvq_lm
