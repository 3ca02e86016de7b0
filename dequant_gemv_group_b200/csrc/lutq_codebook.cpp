// Host-side codebook construction (once per layer).
//
// Sources: the FLUTE abstract ("Daily Papers", query "group-128": NormalFloat
// lookup tables, 3-bit widths), the Log_bQuant abstract (catalyzex author page:
// logarithmic levels with an adjustable base) and "TurboQuant: A
// first-principles walkthrough" (the Lloyd-Max algorithm).  Every table is
// computed in double precision, normalised to max |level| = 1 and rounded once
// to bf16 (round to nearest, ties to even).
#include <cfenv>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>
#include <algorithm>

#include "lutq.h"
#include "lutq_trace.h"

namespace {

double normal_cdf(double z) { return 0.5 * std::erfc(-z / std::sqrt(2.0)); }
double normal_pdf(double z) { return std::exp(-0.5 * z * z) / std::sqrt(2.0 * M_PI); }

// Inverse normal CDF by bisection on the erfc-based CDF (monotone, so the
// bracket always holds the root); 200 halvings reach the double-precision
// resolution of the CDF.
double normal_quantile(double p) {
  double lo = -40.0, hi = 40.0;
  for (int it = 0; it < 200; ++it) {
    double mid = 0.5 * (lo + hi);
    if (normal_cdf(mid) < p) lo = mid; else hi = mid;
  }
  return 0.5 * (lo + hi);
}

// P(a < Z < b), taking the upper tail when both ends are positive.
double normal_mass(double a, double b) {
  if (a >= 0.0) return 0.5 * std::erfc(a / std::sqrt(2.0)) - 0.5 * std::erfc(b / std::sqrt(2.0));
  return normal_cdf(b) - normal_cdf(a);
}

// Round a double once to bf16, ties to even; returns the bit pattern.
uint16_t to_bf16_rne(double v) {
  if (v == 0.0) return std::signbit(v) ? 0x8000 : 0x0000;
  int e = 0;
  double m = std::frexp(v, &e);                  // v = m * 2^e, |m| in [0.5, 1)
  std::fesetround(FE_TONEAREST);
  double q = std::nearbyint(m * 256.0);          // 8 significant bits, ties to even
  float f = static_cast<float>(std::ldexp(q, e - 8));   // exact
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return static_cast<uint16_t>(u >> 16);
}

std::vector<double> nf4() {
  const double delta = 0.5 * ((1.0 - 1.0 / 30.0) + (1.0 - 1.0 / 32.0));
  std::vector<double> lv;
  lv.push_back(0.0);
  for (int i = 0; i < 8; ++i) {                  // 9 points from delta to 1/2, drop 1/2
    double p = delta + (0.5 - delta) * i / 8.0;
    lv.push_back(normal_quantile(p));
  }
  for (int i = 0; i < 7; ++i) {                  // 8 points from delta to 1/2, drop 1/2
    double p = delta + (0.5 - delta) * i / 7.0;
    lv.push_back(-normal_quantile(p));
  }
  std::sort(lv.begin(), lv.end());
  const double top = normal_quantile(delta);
  for (double& v : lv) v /= top;
  return lv;
}

std::vector<double> log_base_levels(double base) {
  std::vector<double> lv;
  for (int k = 0; k < 8; ++k) {
    double m = std::pow(base, -static_cast<double>(k));
    lv.push_back(m);
    lv.push_back(-m);
  }
  std::sort(lv.begin(), lv.end());
  return lv;
}

// Lloyd-Max for N(0,1): thresholds at midpoints, levels at cell centroids
// (pdf(a) - pdf(b)) / P(a < Z < b), repeated until the levels stop moving.
std::vector<double> lloyd_max(int n) {
  std::vector<double> y(n), t(n + 1), y2(n);
  for (int i = 0; i < n; ++i) y[i] = -2.0 + 4.0 * i / (n - 1);
  for (int it = 0; it < 100000; ++it) {
    t[0] = -INFINITY;
    t[n] = INFINITY;
    for (int i = 1; i < n; ++i) t[i] = 0.5 * (y[i - 1] + y[i]);
    double step = 0.0;
    for (int i = 0; i < n; ++i) {
      double pa = std::isinf(t[i]) ? 0.0 : normal_pdf(t[i]);
      double pb = std::isinf(t[i + 1]) ? 0.0 : normal_pdf(t[i + 1]);
      y2[i] = (pa - pb) / normal_mass(t[i], t[i + 1]);
      step = std::max(step, std::fabs(y2[i] - y[i]));
    }
    y = y2;
    if (step < 1e-13) break;
  }
  double top = 0.0;
  for (double v : y) top = std::max(top, std::fabs(v));
  for (double& v : y) v /= top;
  return y;
}

}  // namespace

extern "C" lutq_status lutq_codebook(int kind, int bits, uint16_t* out_bf16) {
  LUTQ_TRACE_RANGE("lutq_codebook");
  if (out_bf16 == nullptr) return LUTQ_ERR_INVALID_ARG;
  std::vector<double> lv;
  switch (kind) {
    case LUTQ_CODEBOOK_NF4:
      if (bits != 4) return LUTQ_ERR_BITS;
      lv = nf4();
      break;
    case LUTQ_CODEBOOK_LOGB:
      if (bits != 4) return LUTQ_ERR_BITS;
      lv = log_base_levels(1.6);
      break;
    case LUTQ_CODEBOOK_LLOYD_MAX3:
      if (bits != 3) return LUTQ_ERR_BITS;
      lv = lloyd_max(8);
      break;
    case LUTQ_CODEBOOK_UNIFORM4:
      if (bits != 4) return LUTQ_ERR_BITS;
      for (int i = 0; i < 16; ++i) lv.push_back((2.0 * i - 15.0) / 15.0);
      break;
    default:
      return LUTQ_ERR_INVALID_ARG;
  }
  for (size_t i = 0; i < lv.size(); ++i) out_bf16[i] = to_bf16_rne(lv[i]);
  return LUTQ_OK;
}

// Asymmetric linear codebook (Log_bQuant abstract: the asymmetric linear
// quantization it compares with): the 2^bits evenly spaced values from w_min
// to w_max, divided by S = max(|w_min|, |w_max|) (the matrix's scale, as
// lutq_quantize_tensorscale writes it), fp64, rounded once to bf16.
extern "C" lutq_status lutq_codebook_asym_linear(double w_min, double w_max, int bits,
                                                 uint16_t* out_bf16) {
  LUTQ_TRACE_RANGE("lutq_codebook_asym_linear");
  if (out_bf16 == nullptr) return LUTQ_ERR_INVALID_ARG;
  if (bits != 3 && bits != 4) return LUTQ_ERR_BITS;
  if (!std::isfinite(w_min) || !std::isfinite(w_max) || !(w_min <= w_max))
    return LUTQ_ERR_INVALID_ARG;
  const int n = 1 << bits;
  const double s = std::max(std::fabs(w_min), std::fabs(w_max));
  for (int i = 0; i < n; ++i) {
    const double v = s == 0.0 ? 0.0 : (w_min + i * (w_max - w_min) / (n - 1)) / s;
    out_bf16[i] = to_bf16_rne(v);
  }
  return LUTQ_OK;
}

// Lloyd-Max on a histogram of normalised weights (kHistBins bins over
// [-1, 1], centre of bin b = (2 b + 1 - kHistBins) / kHistBins): alternately
// give every bin to its nearest level (fp64 distance, ties to the lower
// level) and move every level to the count-weighted mean of its bins' centres
// (an exact integer ratio: |numerator| < 2^59 for fewer than 2^31 weights; a
// level whose cell is empty stays), until the assignment repeats or max_iter
// passes; the levels are rounded once to bf16.  The method is the Lloyd-Max
// algorithm ("TurboQuant: A first-principles walkthrough") applied to the
// layer's own weights.
extern "C" lutq_status lutq_fit_codebook(const uint64_t* hist, int bits, const uint16_t* init_bf16,
                                         int max_iter, uint16_t* out_bf16) {
  LUTQ_TRACE_RANGE("lutq_fit_codebook");
  constexpr int kHistBins = 16384;
  if (hist == nullptr || init_bf16 == nullptr || out_bf16 == nullptr || max_iter < 0)
    return LUTQ_ERR_INVALID_ARG;
  if (bits != 3 && bits != 4) return LUTQ_ERR_BITS;
  uint64_t total = 0;
  for (int b = 0; b < kHistBins; ++b) {
    total += hist[b];
    if (hist[b] >= (uint64_t(1) << 31) || total >= (uint64_t(1) << 31)) return LUTQ_ERR_INVALID_ARG;
  }
  const int n = 1 << bits;
  std::vector<double> levels(n);
  for (int i = 0; i < n; ++i) {
    const uint32_t u = uint32_t(init_bf16[i]) << 16;
    float f;
    std::memcpy(&f, &u, 4);
    if (!std::isfinite(f)) return LUTQ_ERR_INVALID_ARG;
    levels[i] = f;
  }
  std::vector<int> assign(kHistBins, -1), next(kHistBins);
  for (int it = 0; it < max_iter; ++it) {
    for (int b = 0; b < kHistBins; ++b) {
      const double c = double(2 * b + 1 - kHistBins) / double(kHistBins);
      int best = 0;
      double best_d = std::fabs(c - levels[0]);
      for (int i = 1; i < n; ++i) {
        const double d = std::fabs(c - levels[i]);
        if (d < best_d) {
          best = i;
          best_d = d;
        }
      }
      next[b] = best;
    }
    if (it > 0 && next == assign) break;
    assign.swap(next);
    std::vector<int64_t> num(n, 0), den(n, 0);
    for (int b = 0; b < kHistBins; ++b) {
      if (hist[b] == 0) continue;
      num[assign[b]] += int64_t(hist[b]) * int64_t(2 * b + 1 - kHistBins);
      den[assign[b]] += int64_t(hist[b]);
    }
    for (int i = 0; i < n; ++i)
      if (den[i] != 0) levels[i] = double(num[i]) / double(den[i] * kHistBins);
  }
  for (int i = 0; i < n; ++i) out_bf16[i] = to_bf16_rne(levels[i]);
  return LUTQ_OK;
}
