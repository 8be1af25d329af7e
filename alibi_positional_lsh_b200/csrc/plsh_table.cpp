// Host-side (delta, u) table sampler: plsh_draw_table.
//
// Random Binning Features for the Laplace kernel applied to integer
// positions (Positional LSH technical summary, Methodology 1) with s i.i.d.
// hashes per head (Methodology 2). The pitch law Gamma(shape 2, scale sigma)
// is the one whose binning has P(same bin) = e^{-|i-j|/sigma}: with
// density p(delta) = delta e^{-delta/sigma} / sigma^2,
//   int_{D}^{inf} (1 - D/delta) p(delta) d delta = e^{-D/sigma}.
// A Gamma(2, sigma) variate is sigma times the sum of two Exp(1) variates,
// i.e. -sigma (ln U1 + ln U2).
//
// Uniforms come from SplitMix64 (Steele, Lea & Flood, OOPSLA 2014) used as
// a counter-based generator: output number x of the stream seeded with
// `seed` is mix(seed + (x + 1) * 0x9E3779B97F4A7C15). This file is built
// with floating-point contraction off so the arithmetic is the plain IEEE
// sequence written below.
#include <cmath>
#include <cstdint>

#include "plsh_internal.h"

namespace {

constexpr uint64_t kGoldenGamma = 0x9E3779B97F4A7C15ull;
constexpr int kHeadShift = 16;

inline uint64_t splitmix64_output(uint64_t seed, uint64_t index) {
  uint64_t z = seed + (index + 1u) * kGoldenGamma;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// (0, 1): the top 52 bits plus one half, times 2^-52 (exact in double).
inline double unit_open(uint64_t z) { return (static_cast<double>(z >> 12) + 0.5) * 0x1p-52; }
// [0, 1): the top 53 bits times 2^-53 (exact in double).
inline double unit_closed_open(uint64_t z) { return static_cast<double>(z >> 11) * 0x1p-53; }

}  // namespace

// Rows of global heads h0 .. h0 + H - 1 of the table; row h is drawn from the counters of head
// h0 + h, so the slices of a head partition concatenate to the whole table.
static int draw_heads(const char* fn, uint64_t seed, int h0, int H, int s, const double* sigma_host,
                      double* table_host) {
  if (H < 1 || s < 1 || s > PLSH_MAX_S)
    return plsh::fail(PLSH_ERR_INVALID_ARG, "%s: need H >= 1 and 1 <= s <= %d (H=%d s=%d)", fn, PLSH_MAX_S, H, s);
  if (h0 < 0 || static_cast<int64_t>(h0) + H > PLSH_MAX_HEADS)
    return plsh::fail(PLSH_ERR_INVALID_ARG, "%s: need 0 <= h0 and h0 + H <= %d (h0=%d H=%d)", fn, PLSH_MAX_HEADS,
                      h0, H);
  if (!sigma_host || !table_host) return plsh::fail(PLSH_ERR_INVALID_ARG, "%s: null pointer", fn);
  for (int h = 0; h < H; ++h) {
    const double sg = sigma_host[h];
    if (!(std::isfinite(sg) && sg > 0.0))
      return plsh::fail(PLSH_ERR_INVALID_ARG, "%s: sigma[%d] = %g is not finite and > 0", fn, h, sg);
  }
  for (int h = 0; h < H; ++h) {
    const double neg_sigma = -sigma_host[h];
    const uint64_t hg = static_cast<uint64_t>(h0) + static_cast<uint64_t>(h);
    for (int k = 0; k < s; ++k) {
      const uint64_t base = ((hg << kHeadShift) | static_cast<uint64_t>(k)) * 3u;
      const double u1 = unit_open(splitmix64_output(seed, base));
      const double u2 = unit_open(splitmix64_output(seed, base + 1));
      const double u3 = unit_closed_open(splitmix64_output(seed, base + 2));
      const double delta = neg_sigma * (std::log(u1) + std::log(u2));
      double* e = table_host + (static_cast<size_t>(h) * s + k) * 2;
      e[0] = delta;
      e[1] = u3 * delta;
    }
  }
  return PLSH_OK;
}

extern "C" int plsh_draw_table(uint64_t seed, int H, int s, const double* sigma_host, double* table_host) {
  return draw_heads("plsh_draw_table", seed, 0, H, s, sigma_host, table_host);
}

extern "C" int plsh_draw_table_heads(uint64_t seed, int h0, int H, int s, const double* sigma_host,
                                     double* table_host) {
  return draw_heads("plsh_draw_table_heads", seed, h0, H, s, sigma_host, table_host);
}
