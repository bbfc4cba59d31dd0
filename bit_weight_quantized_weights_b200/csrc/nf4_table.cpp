// NF4 codebook, computed on the host once per process.
//
// Construction: QLoRA's 4-bit NormalFloat ("QLoRA: Efficient Finetuning of
// Quantized LLMs", cited by title on "DecDEC: A Systems Approach to Advancing
// Low-Bit LLM Quantization"; the format is the subject of "Fast NF4
// Dequantization Kernels for Large Language Model Inference", Abstract):
// eight positive values at standard-normal quantiles of probabilities evenly
// spaced from delta down towards 1/2, seven negative values the same way with
// one step fewer, an exact zero, all divided by the largest. delta is the mean
// of 1 - 1/30 and 1 - 1/32. Each value is computed in double and rounded once
// to float.
//
// The inverse normal CDF is computed here from std::erfc alone: bisection to
// bracket the root of Phi(t) = p, then Newton steps with Phi'(t) = phi(t).
#include <cmath>
#include <mutex>

#include "common.cuh"

namespace wq {
namespace {

double normal_cdf(double t) { return 0.5 * std::erfc(-t / std::sqrt(2.0)); }

double normal_quantile(double p) {
  double lo = -12.0, hi = 12.0;
  for (int i = 0; i < 200 && hi - lo > 1e-13; ++i) {
    double mid = 0.5 * (lo + hi);
    if (normal_cdf(mid) < p) lo = mid; else hi = mid;
  }
  double t = 0.5 * (lo + hi);
  const double inv_sqrt_2pi = 0.39894228040143267794;
  for (int i = 0; i < 4; ++i) {
    double f = normal_cdf(t) - p;
    double d = inv_sqrt_2pi * std::exp(-0.5 * t * t);
    t -= f / d;
  }
  return t;
}

Nf4Table build_table() {
  const double delta = 0.5 * ((1.0 - 1.0 / 30.0) + (1.0 - 1.0 / 32.0));
  double vals[16];
  int n = 0;
  // seven negative values, ascending: probabilities delta - j*(delta - 1/2)/7,
  // j = 0..6, negated (j = 0 is the most negative)
  for (int j = 0; j <= 6; ++j) {
    double p = delta - j * (delta - 0.5) / 7.0;
    vals[n++] = -normal_quantile(p);
  }
  vals[n++] = 0.0;
  // eight positive values, ascending: probabilities delta - j*(delta - 1/2)/8,
  // j = 7..0
  for (int j = 7; j >= 0; --j) {
    double p = delta - j * (delta - 0.5) / 8.0;
    vals[n++] = normal_quantile(p);
  }
  const double top = normal_quantile(delta);
  Nf4Table t;
  for (int i = 0; i < 16; ++i) t.v[i] = static_cast<float>(vals[i] / top);
  return t;
}

}  // namespace

const Nf4Table& nf4_table() {
  static Nf4Table table;
  static std::once_flag once;
  std::call_once(once, [] { table = build_table(); });
  return table;
}

}  // namespace wq
