// Bin ids of the random binnings, shared by K1 (plsh_sample_bins) and the fused window path
// (plsh_window_from_table), so that both evaluate every id with the same IEEE float64 steps.
//
// Positional LSH technical summary, Methodology 1 (mechanism): a hash splits the integer positions
// into contiguous bins, bin(i) = floor((i + u) / delta); ids are stored relative to position 0,
//   id(i) = floor(RN(RN(i + u) / delta)) - floor(RN(u / delta)),
// with IEEE float64 round-to-nearest add and divide.
#pragma once

#include <cmath>
#include <cstdint>

#include "plsh_internal.h"

namespace plsh {

// floor(RN((pos + u) / delta)) without a division for almost every position. With
// a = RN(pos + u) and rcp = RN(1 / delta), xa = RN(a * rcp) is within 3 * 2^-53 * xa of
// q = RN(a / delta) (each of the three roundings is relative 2^-53). If xa lies more than
// 2^-50 * xa from both integers around it, q lies strictly between them too and
// floor(q) = floor(xa); otherwise the exact quotient is taken.
__device__ __forceinline__ double floor_quotient(double pos, double u, double delta, double rcp) {
  const double a = __dadd_rn(pos, u);
  const double xa = __dmul_rn(a, rcp);
  const double fl = floor(xa);
  const double tol = xa * 0x1p-50;
  if (xa - fl > tol && (fl + 1.0) - xa > tol) return fl;
  return floor(__ddiv_rn(a, delta));
}

// The id of position pos relative to position 0 (base = floor(RN(u / delta))); an id outside
// [0, 2^31) sets PLSH_DEVERR_RANGE in flags and reads as 2^31 - 1.
__device__ __forceinline__ int32_t bin_id(double pos, double u, double delta, double rcp, double base,
                                          uint32_t& flags) {
  const double id = floor_quotient(pos, u, delta, rcp) - base;
  if (!(id >= 0.0 && id <= 2147483647.0)) {
    flags |= PLSH_DEVERR_RANGE;
    return 2147483647;
  }
  return static_cast<int32_t>(id);
}

// One hash's binning, ready to evaluate ids: (delta, u) from the table, with 1/delta and the base.
// A table entry with delta not finite and > 0, or u not finite, gives id 0 everywhere (as K1 writes).
struct Binning {
  double u, delta, rcp, base;
  bool ok;
  __device__ __forceinline__ static Binning from_table(const double* entry) {
    Binning b;
    b.delta = entry[0];
    b.u = entry[1];
    b.ok = isfinite(b.delta) && b.delta > 0.0 && isfinite(b.u);
    b.base = b.ok ? floor(__ddiv_rn(b.u, b.delta)) : 0.0;
    b.rcp = b.ok ? __drcp_rn(b.delta) : 0.0;
    return b;
  }
  __device__ __forceinline__ int32_t at(int p) const {
    uint32_t f = 0;
    return ok ? bin_id(static_cast<double>(p), u, delta, rcp, base, f) : 0;
  }
  // the device error bits K1 would report for positions [0, n): ids are non-decreasing from 0, so
  // only the last one can overflow
  __device__ __forceinline__ uint32_t flags(int n) const {
    if (!ok) return PLSH_DEVERR_TABLE;
    uint32_t f = 0;
    (void)bin_id(static_cast<double>(n - 1), u, delta, rcp, base, f);
    return f;
  }
};

}  // namespace plsh
