// Per-hash key windows for the per-sample comparator (K4).
//
// Theorem 2.2's construction attends, for each sample k, only inside the
// blocks of that sample's binning (Positional LSH technical summary,
// Methodology 3). For query tile t (rows [128t, min(n, 128t + 128))) and
// hash k, the keys that share a hash-k block with some row of the tile are
// the contiguous range from the start of the block holding row 128t to the
// end of the block holding the tile's last row (blocks are contiguous,
// Methodology 1, structure); when causal the range ends at the tile's last
// row. Bin ids are non-decreasing in the position, so both ends are binary
// searches over the ids of (h, k).
#include "plsh_internal.h"

namespace plsh {
namespace {

__global__ void varlen_spans_kernel(const int32_t* __restrict__ ids, int H, int s, int n, int causal, int T,
                                    int32_t* __restrict__ spans) {
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<long long>(H) * s * T) return;
  const int t = static_cast<int>(idx % T);
  const int32_t* id = ids + (idx / T) * static_cast<long long>(n);   // ids of (h, k) = idx / T
  const int i0 = t * PLSH_TILE;
  const int last = min(n, i0 + PLSH_TILE) - 1;
  const int32_t a = id[i0], z = id[last];
  int L = 0, R = i0;                 // first j in [0, i0] with id[j] >= a
  while (L < R) {
    const int mid = (L + R) >> 1;
    if (id[mid] < a) L = mid + 1;
    else R = mid;
  }
  int hi = last;
  if (!causal) {                     // last j in [last, n - 1] with id[j] <= z
    int L2 = last, R2 = n - 1;
    while (L2 < R2) {
      const int mid = (L2 + R2 + 1) >> 1;
      if (id[mid] > z) R2 = mid - 1;
      else L2 = mid;
    }
    hi = L2;
  }
  spans[2 * idx] = L;
  spans[2 * idx + 1] = hi;
}

}  // namespace

int launch_varlen_spans(const int32_t* ids, int H, int s, int n, int causal, int32_t* spans, cudaStream_t st) {
  const int T = ceil_div(n, PLSH_TILE);
  const long long total = static_cast<long long>(H) * s * T;
  if (total > (1ll << 31) - 1) return fail(PLSH_ERR_RANGE, "per-hash windows: H * s * tiles too large");
  const int threads = 256;
  const int blocks = static_cast<int>((total + threads - 1) / threads);
  varlen_spans_kernel<<<blocks, threads, 0, st>>>(ids, H, s, n, causal, T, spans);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? PLSH_OK : cuda_fail(e, "varlen_spans_kernel launch");
}

}  // namespace plsh
