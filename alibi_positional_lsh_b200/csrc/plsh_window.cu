// K2: window reduction -- plsh_window.
//
// Positional LSH technical summary, Methodology 1 (structure: the bins of
// one hash are contiguous, non-overlapping blocks) and Methodology 2
// (block-size control, b_max ~ sigma log log n). From the bin ids this
// computes, per head:
//   * bmask[p]: bit k set iff hash k opens a block at position p
//     (position 0 opens a block for every hash);
//   * b_max: the longest block over the s hashes;
//   * for each 128-row query tile, the key window [lo, hi] of every key
//     with a nonzero weight for some row of the tile.
// Because blocks are contiguous, the count of hashes putting i and j in one
// bin is s - popcount(OR of bmask over (min(i,j), max(i,j)]), which is how
// the attention kernels read the weights.
//
// Block ends and starts are found by an exponential-then-binary search on
// the non-decreasing ids, so each block costs O(log length) reads.
#include "plsh_internal.h"

namespace plsh {
namespace {

constexpr int kThreads = 256;

// First position of the run of value `a` that contains position p (row[p] == a).
__device__ __forceinline__ int block_start(const int32_t* __restrict__ row, int p, int32_t a) {
  int good = p, bad = -1, step = 1;
  while (true) {
    const int q = p - step;
    if (q < 0) { bad = -1; break; }
    if (row[q] != a) { bad = q; break; }
    good = q;
    if (step > (1 << 29)) { bad = -1; break; }
    step <<= 1;
  }
  while (good - bad > 1) {
    const int mid = bad + (good - bad) / 2;
    if (row[mid] == a) good = mid; else bad = mid;
  }
  return good;
}

// Last position of the run of value `a` that contains position p (row[p] == a).
__device__ __forceinline__ int block_end(const int32_t* __restrict__ row, int p, int32_t a, int n) {
  int good = p, bad = n, step = 1;
  while (true) {
    const int q = p + step;
    if (q >= n) { bad = n; break; }
    if (row[q] != a) { bad = q; break; }
    good = q;
    if (step > (1 << 29)) { bad = n; break; }
    step <<= 1;
  }
  while (bad - good > 1) {
    const int mid = good + (bad - good) / 2;
    if (row[mid] == a) good = mid; else bad = mid;
  }
  return good;
}

template <typename MaskT>
__global__ void __launch_bounds__(kThreads) mask_bmax_kernel(const int32_t* __restrict__ ids, int s, int n,
                                                             MaskT* __restrict__ bmask,
                                                             int32_t* __restrict__ bmax) {
  const int h = blockIdx.y;
  const int p = blockIdx.x * kThreads + threadIdx.x;
  int longest = 0;
  if (p < n) {
    MaskT m = 0;
    const int32_t* base = ids + static_cast<size_t>(h) * s * n;
    for (int k = 0; k < s; ++k) {
      const int32_t* row = base + static_cast<size_t>(k) * n;
      const int32_t a = row[p];
      if (p == 0 || row[p - 1] != a) m |= static_cast<MaskT>(1) << k;
      const bool ends_here = (p == n - 1) || (row[p + 1] != a);
      if (ends_here) {
        const int len = p - block_start(row, p, a) + 1;
        longest = len > longest ? len : longest;
      }
    }
    bmask[static_cast<size_t>(h) * n + p] = m;
  }
  longest = __reduce_max_sync(0xffffffffu, longest);
  if ((threadIdx.x & 31) == 0 && longest > 0) atomicMax(bmax + h, longest);
}

// One warp per (head, query tile); lanes walk the hashes.
__global__ void __launch_bounds__(kThreads) spans_kernel(const int32_t* __restrict__ ids, int H, int s, int n,
                                                         int causal, int32_t* __restrict__ spans) {
  const int T = (n + PLSH_TILE - 1) / PLSH_TILE;
  const int warp = (blockIdx.x * kThreads + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= H * T) return;
  const int h = warp / T, t = warp % T;
  const int i0 = t * PLSH_TILE;
  const int i1 = min(n, i0 + PLSH_TILE) - 1;
  int lo = i0, hi = i1;
  for (int k = lane; k < s; k += 32) {
    const int32_t* row = ids + (static_cast<size_t>(h) * s + k) * n;
    lo = min(lo, block_start(row, i0, row[i0]));
    if (!causal) hi = max(hi, block_end(row, i1, row[i1], n));
  }
  lo = __reduce_min_sync(0xffffffffu, lo);
  hi = __reduce_max_sync(0xffffffffu, hi);
  if (lane == 0) {
    spans[(static_cast<size_t>(h) * T + t) * 2] = lo;
    spans[(static_cast<size_t>(h) * T + t) * 2 + 1] = hi;
  }
}

}  // namespace

int launch_window(const int32_t* ids, int H, int s, int n, int causal, int32_t* bmax,
                  int32_t* spans, void* bmask, uint32_t* err, cudaStream_t st) {
  (void)err;
  cudaError_t e = cudaMemsetAsync(bmax, 0, sizeof(int32_t) * H, st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(bmax)");
  dim3 g1(ceil_div(n, kThreads), H);
  if (s <= 32)
    mask_bmax_kernel<uint32_t><<<g1, kThreads, 0, st>>>(ids, s, n, static_cast<uint32_t*>(bmask), bmax);
  else
    mask_bmax_kernel<unsigned long long><<<g1, kThreads, 0, st>>>(
        ids, s, n, static_cast<unsigned long long*>(bmask), bmax);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "mask_bmax_kernel launch");
  const long long warps = static_cast<long long>(H) * ceil_div(n, PLSH_TILE);
  const int g2 = static_cast<int>((warps * 32 + kThreads - 1) / kThreads);
  spans_kernel<<<g2, kThreads, 0, st>>>(ids, H, s, n, causal, spans);
  e = cudaGetLastError();
  return e == cudaSuccess ? PLSH_OK : cuda_fail(e, "spans_kernel launch");
}

}  // namespace plsh
