// Host-side level tables of the library.
//
// NF4 ("QLoRA技术从入门到精通", 2(3)2) NF4非均匀格点; "LoRA 与 QLoRA：用一块
// GPU 微调大模型", 量化/NF4): split N(0,1) into equal-probability intervals,
// take the median of each, keep an exact 0, dense near 0.  Built per half:
// 8 intervals of [0, inf) (median at p = 1/2 + (j - 1/2)/16) and 7 of
// (-inf, 0] (median at p = 1/2 - (j - 1/2)/14), each half divided by its
// extreme so the table spans [-1, 1] exactly, plus 0.
//
// The normal quantile is solved here by Newton's method on
// Phi(z) = erfc(-z/sqrt 2)/2 from a log-based starting point, in double, then
// rounded once to float.
#include <cmath>
#include <cstring>

#include "internal.cuh"

namespace qlora {
namespace {

double normal_cdf(double z) { return 0.5 * std::erfc(-z * M_SQRT1_2); }

double normal_pdf(double z) { return std::exp(-0.5 * z * z) / std::sqrt(2.0 * M_PI); }

double normal_quantile(double p) {
  // Starting point from the tail behaviour Phi^-1(p) ~ -sqrt(-2 ln p).
  double t = (p < 0.5) ? p : 1.0 - p;
  double z = std::sqrt(-2.0 * std::log(t));
  z = (p < 0.5) ? -0.5 * z : 0.5 * z;
  for (int it = 0; it < 100; ++it) {
    double step = (normal_cdf(z) - p) / normal_pdf(z);
    if (step > 1.0) step = 1.0;
    if (step < -1.0) step = -1.0;
    double zn = z - step;
    if (zn == z) break;
    z = zn;
    if (std::fabs(step) < 1e-17 * (1.0 + std::fabs(z))) break;
  }
  return z;
}

void fill_nf4(float* lv) {
  double pos[8], neg[7];
  for (int j = 1; j <= 8; ++j) pos[j - 1] = normal_quantile(0.5 + (j - 0.5) / 16.0);
  for (int j = 1; j <= 7; ++j) neg[j - 1] = normal_quantile(0.5 - (j - 0.5) / 14.0);
  // ascending: neg[6] (most negative) ... neg[0], 0, pos[0] ... pos[7]
  for (int j = 0; j < 7; ++j) lv[j] = static_cast<float>(neg[6 - j] / -neg[6]);
  lv[7] = 0.0f;
  for (int j = 0; j < 8; ++j) lv[8 + j] = static_cast<float>(pos[j] / pos[7]);
}

void fill_uniform(float* lv) {
  for (int k = 0; k < 16; ++k) lv[k] = static_cast<float>(-1.0 + k * (2.0 / 15.0));
}

}  // namespace

qlora_status make_level_table(int32_t table, LevelTable* out) {
  std::memset(out, 0, sizeof(*out));
  if (table == QLORA_TABLE_NF4) {
    fill_nf4(out->level);
  } else if (table == QLORA_TABLE_UNIFORM) {
    fill_uniform(out->level);
  } else {
    return QLORA_ERR_UNSUPPORTED;
  }
  for (int k = 0; k < 15; ++k) {
    // exact midpoint (sum of two floats is exact in double, halving is exact)
    double mid = (static_cast<double>(out->level[k]) + out->level[k + 1]) * 0.5;
    float t = static_cast<float>(mid);
    if (static_cast<double>(t) > mid) t = std::nextafter(t, -INFINITY);
    out->thr[k] = t;
  }
  out->thr[15] = INFINITY;
  return QLORA_OK;
}

}  // namespace qlora
