// Constant tables of libkvq, computed on the host in fp64 at first use:
//   * Lloyd-Max codebooks for N(0,1), widths 1..8 (TQ-MSE base quantizer of
//     "RoPE-aware bit allocation for KV cache quantization", abstract),
//   * the NF4 levels (QLoRA construction, cited by the NQKV review as reference [20]).
// Stored forms: centroids rounded to fp16, thresholds = fp32 midpoints of adjacent fp16
// centroids, delta(w) = fp32 MSE of that stored quantizer on N(0,1), delta(0) = 1.
#include "tables.h"

#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

namespace kvq {
namespace {

constexpr double kInvSqrt2Pi = 0.398942280401432677939946059934;
constexpr double kSqrt1_2 = 0.707106781186547524400844362105;

double npdf(double x) { return std::isfinite(x) ? kInvSqrt2Pi * std::exp(-0.5 * x * x) : 0.0; }
double ncdf(double x) { return 0.5 * std::erfc(-x * kSqrt1_2); }
double nsf(double x) { return 0.5 * std::erfc(x * kSqrt1_2); }

// P(a < X < b), taken from the tail that keeps precision.
double mass(double a, double b) {
  if (a >= 0.0) return nsf(a) - nsf(b);
  if (b <= 0.0) return ncdf(b) - ncdf(a);
  return 1.0 - ncdf(a) - nsf(b);
}

// Inverse of the standard normal CDF: bisection to a bracket, then Newton steps. For
// p > 1/2 the residual is taken on the upper tail, (1 - p) - Q(x), which is exact to form
// there (1 - p is exact for p in [1/2, 1]); otherwise Phi(x) - p.
double norm_quantile(double p) {
  double lo = -40.0, hi = 40.0;
  for (int i = 0; i < 200 && hi - lo > 1e-3; ++i) {
    double mid = 0.5 * (lo + hi);
    if (ncdf(mid) < p) lo = mid; else hi = mid;
  }
  double x = 0.5 * (lo + hi);
  const bool upper = p > 0.5;
  const double q = 1.0 - p;
  for (int i = 0; i < 100; ++i) {
    double f = upper ? (q - nsf(x)) : (ncdf(x) - p);
    double step = f / npdf(x);
    x -= step;
    if (std::fabs(step) <= 1e-17 * std::fmax(1.0, std::fabs(x))) break;
  }
  return x;
}

// Round a double to the nearest fp16 value (ties to even); returns the IEEE half bit pattern.
uint16_t to_half_bits(double v) {
  uint16_t sign = std::signbit(v) ? 0x8000u : 0u;
  double a = std::fabs(v);
  if (std::isnan(v)) return 0x7e00u;
  if (a == 0.0) return sign;
  int e;
  std::frexp(a, &e);                 // a = m * 2^e, m in [0.5, 1)
  int exp_unb = e - 1;               // a in [2^exp_unb, 2^(exp_unb+1))
  if (exp_unb < -14) {               // subnormal: multiples of 2^-24
    double q = std::nearbyint(std::ldexp(a, 24));
    if (q >= 1024.0) return static_cast<uint16_t>(sign | 0x0400u);
    return static_cast<uint16_t>(sign | static_cast<uint16_t>(q));
  }
  double q = std::nearbyint(std::ldexp(a, 10 - exp_unb));  // in [1024, 2048]
  if (q >= 2048.0) { q = 1024.0; ++exp_unb; }
  if (exp_unb > 15) return static_cast<uint16_t>(sign | 0x7c00u);
  uint16_t bits = static_cast<uint16_t>(((exp_unb + 15) << 10) | (static_cast<int>(q) - 1024));
  return static_cast<uint16_t>(sign | bits);
}

double half_bits_to_double(uint16_t h) {
  int s = (h >> 15) & 1, e = (h >> 10) & 0x1f, m = h & 0x3ff;
  double v;
  if (e == 0) v = std::ldexp(static_cast<double>(m), -24);
  else if (e == 31) v = m ? NAN : INFINITY;
  else v = std::ldexp(1024.0 + m, e - 25);
  return s ? -v : v;
}

// Lloyd map: conditional mean of each cell bounded by the midpoints of c.
void lloyd_map(const std::vector<double>& c, std::vector<double>& m, std::vector<double>& a,
               std::vector<double>& b, std::vector<double>& p) {
  const size_t n = c.size();
  for (size_t i = 0; i < n; ++i) {
    a[i] = (i == 0) ? -INFINITY : 0.5 * (c[i - 1] + c[i]);
    b[i] = (i + 1 == n) ? INFINITY : 0.5 * (c[i] + c[i + 1]);
    p[i] = mass(a[i], b[i]);
    m[i] = (npdf(a[i]) - npdf(b[i])) / p[i];
  }
}

// Fixed point of the Lloyd conditions for 2^w levels: Lloyd sweeps from the N(0,3)
// quantile start, then Newton with the tridiagonal Jacobian (Thomas algorithm).
std::vector<double> lloyd_max(int w) {
  const size_t n = size_t(1) << w;
  std::vector<double> c(n), m(n), a(n), b(n), p(n);
  for (size_t i = 0; i < n; ++i) c[i] = std::sqrt(3.0) * norm_quantile((i + 0.5) / double(n));
  for (int it = 0; it < 200; ++it) {
    lloyd_map(c, m, a, b, p);
    c = m;
  }
  std::vector<double> lo(n), di(n), up(n), r(n);
  for (int it = 0; it < 100; ++it) {
    lloyd_map(c, m, a, b, p);
    double worst = 0.0;
    for (size_t i = 0; i < n; ++i) {
      r[i] = c[i] - m[i];
      worst = std::fmax(worst, std::fabs(r[i]));
    }
    if (worst < 1e-15) break;
    for (size_t i = 0; i < n; ++i) {
      double dma = std::isfinite(a[i]) ? npdf(a[i]) * (m[i] - a[i]) / p[i] : 0.0;
      double dmb = std::isfinite(b[i]) ? npdf(b[i]) * (b[i] - m[i]) / p[i] : 0.0;
      lo[i] = (i > 0) ? -0.5 * dma : 0.0;
      up[i] = (i + 1 < n) ? -0.5 * dmb : 0.0;
      di[i] = 1.0 - ((i > 0) ? 0.5 * dma : 0.0) - ((i + 1 < n) ? 0.5 * dmb : 0.0);
    }
    // Thomas algorithm for J * delta = r.
    std::vector<double> cp(n), dp(n);
    cp[0] = up[0] / di[0];
    dp[0] = r[0] / di[0];
    for (size_t i = 1; i < n; ++i) {
      double den = di[i] - lo[i] * cp[i - 1];
      cp[i] = up[i] / den;
      dp[i] = (r[i] - lo[i] * dp[i - 1]) / den;
    }
    std::vector<double> delta(n);
    delta[n - 1] = dp[n - 1];
    for (size_t i = n - 1; i-- > 0;) delta[i] = dp[i] - cp[i] * delta[i + 1];
    for (size_t i = 0; i < n; ++i) c[i] -= delta[i];
  }
  // The solution is odd-symmetric; remove rounding asymmetry.
  std::vector<double> s(n);
  for (size_t i = 0; i < n; ++i) s[i] = 0.5 * (c[i] - c[n - 1 - i]);
  return s;
}

double stored_mse(const std::vector<double>& cent, const std::vector<double>& thr) {
  const size_t n = cent.size();
  double acc = 0.0;
  for (size_t i = 0; i < n; ++i) {
    double a = (i == 0) ? -INFINITY : thr[i - 1];
    double b = (i + 1 == n) ? INFINITY : thr[i];
    double p0 = mass(a, b);
    double p1 = npdf(a) - npdf(b);
    double apa = std::isfinite(a) ? a * npdf(a) : 0.0;
    double bpb = std::isfinite(b) ? b * npdf(b) : 0.0;
    double p2 = p0 + apa - bpb;
    acc += p2 - 2.0 * cent[i] * p1 + cent[i] * cent[i] * p0;
  }
  return acc;
}

Tables g_tables;
std::once_flag g_once;

void build() {
  Tables& t = g_tables;
  std::memset(&t, 0, sizeof(t));
  t.delta[0] = 1.0f;
  for (int w = 1; w <= 8; ++w) {
    const int n = 1 << w;
    std::vector<double> c = lloyd_max(w);
    std::vector<double> c16(n), thr(n - 1);
    for (int i = 0; i < n; ++i) {
      uint16_t hb = to_half_bits(c[i]);
      t.centroid_f16[centroid_offset(w) + i] = hb;
      c16[i] = half_bits_to_double(hb);
    }
    for (int i = 0; i + 1 < n; ++i) {
      float tf = static_cast<float>(0.5 * (c16[i] + c16[i + 1]));
      t.threshold[threshold_offset(w) + i] = tf;
      thr[i] = static_cast<double>(tf);
    }
    t.delta[w] = static_cast<float>(stored_mse(c16, thr));
  }
  // NF4: quantiles at probabilities evenly spaced from `off` toward 1/2 (excluded):
  // 8 on the positive side, 7 mirrored on the negative side, plus an exact 0; the
  // outermost probability `off` is the mean of 1 - 1/30 and 1 - 1/32.
  const double off = 0.5 * ((1.0 - 1.0 / 30.0) + (1.0 - 1.0 / 32.0));
  const double step8 = (0.5 - off) / 8.0, step7 = (0.5 - off) / 7.0;
  double lv[16];
  int k = 0;
  for (int i = 0; i <= 6; ++i) lv[k++] = -norm_quantile(i * step7 + off);     // ascending negatives
  lv[k++] = 0.0;
  for (int i = 7; i >= 0; --i) lv[k++] = norm_quantile(i * step8 + off);      // ascending positives
  const double top = norm_quantile(off);
  for (int i = 0; i < 16; ++i) t.nf4[i] = static_cast<float>(lv[i] / top);
  for (int i = 0; i < 15; ++i)
    t.nf4_mid[i] = static_cast<float>(0.5 * (double(t.nf4[i]) + double(t.nf4[i + 1])));
}

}  // namespace

const Tables& tables() {
  std::call_once(g_once, build);
  return g_tables;
}

}  // namespace kvq
