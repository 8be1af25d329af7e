// K1: bin ids of every (head, hash, position) -- plsh_sample_bins.
//
// Positional LSH technical summary, Methodology 1 (mechanism): a hash h
// splits the integer positions into contiguous bins. With the random
// binning form bin(i) = floor((i + u)/delta), this kernel writes
//   id_{h,k}(i) = floor((i + u_k)/delta_k) - floor(u_k/delta_k)
// using explicitly rounded IEEE float64 add and divide (round to nearest),
// so the ids agree bit for bit with any IEEE float64 evaluation of the same
// expression. Ids are stored relative to position 0 so they fit int32.
//
// HBM-bound: 4 bytes written per (head, hash, position), no reads beyond
// the 16-byte table entry; the quotient is a multiply by the reciprocal with
// an exactness test (floor_quotient in plsh_binid.cuh, shared with the fused
// window path), so the float64 divide runs only near bin boundaries. Each thread writes 4 consecutive ids (one 16-byte
// store) when the row is 16-byte aligned.
#include <cmath>

#include "plsh_binid.cuh"
#include "plsh_internal.h"

namespace plsh {
namespace {

constexpr int kThreads = 256;
constexpr int kPerThread = 4;

__global__ void __launch_bounds__(kThreads) sample_bins_kernel(const double* __restrict__ table, int s,
                                                               int n, int32_t* __restrict__ ids,
                                                               uint32_t* __restrict__ err) {
  const int k = blockIdx.y;
  const int h = blockIdx.z;
  const double delta = table[(static_cast<size_t>(h) * s + k) * 2];
  const double u = table[(static_cast<size_t>(h) * s + k) * 2 + 1];
  uint32_t flags = 0;
  const bool ok = isfinite(delta) && delta > 0.0 && isfinite(u);
  if (!ok) flags |= PLSH_DEVERR_TABLE;
  const double base = ok ? floor(__ddiv_rn(u, delta)) : 0.0;
  const double rcp = ok ? __drcp_rn(delta) : 0.0;
  int32_t* row = ids + (static_cast<size_t>(h) * s + k) * n;
  const bool vec = (n % kPerThread) == 0;  // rows start 16-byte aligned when n % 4 == 0
  const int stride = gridDim.x * kThreads * kPerThread;
  for (int i0 = (blockIdx.x * kThreads + threadIdx.x) * kPerThread; i0 < n; i0 += stride) {
    int32_t v[kPerThread];
#pragma unroll
    for (int e = 0; e < kPerThread; ++e) {
      const int i = i0 + e;
      v[e] = (ok && i < n) ? bin_id(static_cast<double>(i), u, delta, rcp, base, flags) : 0;
    }
    if (vec && i0 + kPerThread <= n) {
      *reinterpret_cast<int4*>(row + i0) = make_int4(v[0], v[1], v[2], v[3]);
    } else {
#pragma unroll
      for (int e = 0; e < kPerThread; ++e)
        if (i0 + e < n) row[i0 + e] = v[e];
    }
  }
  if (flags) atomicOr(err, flags);
}

}  // namespace

int launch_sample_bins(const double* table, int H, int s, int n, int32_t* ids, uint32_t* err,
                       cudaStream_t st) {
  const int per_block = kThreads * kPerThread;
  int gx = ceil_div(n, per_block);
  if (gx > 4096) gx = 4096;
  dim3 grid(gx, s, H);
  sample_bins_kernel<<<grid, kThreads, 0, st>>>(table, s, n, ids, err);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? PLSH_OK : cuda_fail(e, "sample_bins_kernel launch");
}

}  // namespace plsh
