// YaRN frequency table (host, float64) and the rotation of one rotary pair
// (device), shared by the RoPE kernel and the query-absorb kernel.
//
// [P1] "256K 长上下文真能本地用：Xing4.0 原生长上下文的工程代价拆解", section 一:
//      rope_scaling yarn, factor 64 from 4096, beta_fast 32, beta_slow 1,
//      mscale = mscale_all_dim = 1.0.
// The table follows the NTK-by-parts interpolation of the YaRN paper (Peng et
// al. 2023, section 3.2); rope_theta is not printed on the pages.
#pragma once

#include <cmath>
#include <cstdint>

#include "xmla_device.cuh"

namespace xmla {

struct RopeTable {
  double inv_freq[kDRope / 2];
  double magnitude;  // mscale(factor, mscale) / mscale(factor, mscale_all_dim)
};

inline double mscale_of(double s, double m) { return s <= 1.0 ? 1.0 : 0.1 * m * std::log(s) + 1.0; }

inline bool yarn_cfg_ok(const xmla_yarn_cfg* c) {
  return c != nullptr && c->rope_theta > 1.0 && c->factor > 0.0 &&
         c->original_max_position_embeddings > 0 && c->beta_fast > 0.0 && c->beta_slow > 0.0;
}

// Inverse frequency of each rotary pair.  A pair whose wavelength turns more
// than beta_fast times over the original context keeps its frequency, one
// turning fewer than beta_slow times is slowed by `factor`, and pairs between
// the two (band edges rounded outward) are blended linearly.
inline void yarn_table(const xmla_yarn_cfg* c, double* out) {
  const int half = c->rotary_dim / 2;
  const double d = (double)c->rotary_dim;
  const double L = (double)c->original_max_position_embeddings;
  const double two_pi = 6.283185307179586476925286766559;
  auto pair_for_rotations = [&](double turns) {
    return d * std::log(L / (turns * two_pi)) / (2.0 * std::log(c->rope_theta));
  };
  double lo = std::floor(pair_for_rotations(c->beta_fast));
  double hi = std::ceil(pair_for_rotations(c->beta_slow));
  if (lo < 0.0) lo = 0.0;
  if (hi > d - 1.0) hi = d - 1.0;
  if (lo == hi) hi += 0.001;
  for (int i = 0; i < half; ++i) {
    const double f = std::pow(c->rope_theta, -2.0 * (double)i / d);
    if (c->factor == 1.0) {
      out[i] = f;
      continue;
    }
    double t = ((double)i - lo) / (hi - lo);
    t = t < 0.0 ? 0.0 : (t > 1.0 ? 1.0 : t);
    out[i] = (f / c->factor) * t + f * (1.0 - t);
  }
}

inline RopeTable make_rope_table(const xmla_yarn_cfg* c) {
  RopeTable t;
  yarn_table(c, t.inv_freq);
  t.magnitude = mscale_of(c->factor, c->mscale) / mscale_of(c->factor, c->mscale_all_dim);
  return t;
}

// Rotate pair (x1, x2) = (x[i], x[i + 32]) at an integer position.  The angle
// is formed in float64 from the exact position, so it stays accurate at
// positions of 2^19 and beyond.
__device__ __forceinline__ void rope_pair(double x1, double x2, int64_t pos, int i,
                                          const RopeTable& tab, double* y1, double* y2) {
  double s, c;
  sincos((double)pos * tab.inv_freq[i], &s, &c);
  s *= tab.magnitude;
  c *= tab.magnitude;
  *y1 = x1 * c - x2 * s;
  *y2 = x2 * c + x1 * s;
}

}  // namespace xmla
