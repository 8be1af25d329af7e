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
// The masks and block lengths come from one coalesced pass over the ids
// (block lengths via a CTA-wide scan of block starts); only the block
// holding each CTA's first position, and the window ends, are found by an
// exponential-then-binary search on the non-decreasing ids.
//
// The ids come either from memory (plsh_window, after K1) or straight from
// the (delta, u) table (plsh_window_from_table): each id is then evaluated
// where it is needed with K1's own float64 steps (plsh_binid.cuh), so the
// outputs are the same bit for bit and the [H][s][n] ids are never written
// or read.
#include "plsh_binid.cuh"
#include "plsh_internal.h"

namespace plsh {
namespace {

constexpr int kThreads = 256;

// The ids of one (head, hash) read from memory; Binning (plsh_binid.cuh) evaluates them from the table.
struct MemRow {
  const int32_t* row;
  __device__ __forceinline__ int32_t at(int p) const { return row[p]; }
};

// First position of the run of value `a` that contains position p (row.at(p) == a).
template <typename Row>
__device__ __forceinline__ int block_start(const Row& row, int p, int32_t a) {
  int good = p, bad = -1, step = 1;
  while (true) {
    const int q = p - step;
    if (q < 0) { bad = -1; break; }
    if (row.at(q) != a) { bad = q; break; }
    good = q;
    if (step > (1 << 29)) { bad = -1; break; }
    step <<= 1;
  }
  while (good - bad > 1) {
    const int mid = bad + (good - bad) / 2;
    if (row.at(mid) == a) good = mid; else bad = mid;
  }
  return good;
}

// Last position of the run of value `a` that contains position p (row.at(p) == a).
template <typename Row>
__device__ __forceinline__ int block_end(const Row& row, int p, int32_t a, int n) {
  int good = p, bad = n, step = 1;
  while (true) {
    const int q = p + step;
    if (q >= n) { bad = n; break; }
    if (row.at(q) != a) { bad = q; break; }
    good = q;
    if (step > (1 << 29)) { bad = n; break; }
    step <<= 1;
  }
  while (bad - good > 1) {
    const int mid = good + (bad - good) / 2;
    if (row.at(mid) == a) good = mid; else bad = mid;
  }
  return good;
}

// Boundary masks and longest blocks for 1024 positions of one head per CTA, all s hashes.
// Per hash a thread holds 4 consecutive ids; a block starts where the id changes and ends
// before the next change. Each block's length is taken at its last position, from the latest
// block start at or before it: within the thread, else from earlier threads of the CTA (a
// CTA-wide max-scan of the threads' last starts), else the block began before the CTA's first
// position p0 and its start is carry[k], found once per CTA and hash by a search.
template <typename MaskT, bool kFromTable>
__global__ void __launch_bounds__(kThreads) mask_bmax_kernel(const int32_t* __restrict__ ids,
                                                             const double* __restrict__ table, int s, int n,
                                                             MaskT* __restrict__ bmask,
                                                             int32_t* __restrict__ bmax, uint32_t* __restrict__ err) {
  constexpr int kPer = 4;
  constexpr int kSpan = kThreads * kPer;
  constexpr int kWarps = kThreads / 32;
  __shared__ int carry[PLSH_MAX_S];
  __shared__ int warp_last[kWarps];
  __shared__ Binning bins[kFromTable ? PLSH_MAX_S : 1];
  const int h = blockIdx.y;
  const int p0 = blockIdx.x * kSpan;
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  const int32_t* base = kFromTable ? nullptr : ids + static_cast<size_t>(h) * s * n;
  if (t < s) {
    if constexpr (kFromTable) {
      const Binning b = Binning::from_table(table + (static_cast<size_t>(h) * s + t) * 2);
      bins[t] = b;
      if (blockIdx.x == 0) {
        const uint32_t f = b.flags(n);
        if (f) atomicOr(err, f);
      }
      carry[t] = block_start(b, p0, b.at(p0));
    } else {
      const MemRow row{base + static_cast<size_t>(t) * n};
      carry[t] = block_start(row, p0, row.at(p0));
    }
  }
  __syncthreads();
  const int pb = p0 + kPer * t;                     // this thread's first position
  const bool vec = (n % 4 == 0) && (pb + kPer <= n);  // 16-byte aligned full int4
  MaskT m[kPer] = {0, 0, 0, 0};
  int longest = 0;
  for (int k = 0; k < s; ++k) {
    int32_t id[kPer], prev, next;
    if constexpr (kFromTable) {
      const Binning b = bins[k];
#pragma unroll
      for (int e = 0; e < kPer; ++e) id[e] = (pb + e < n) ? b.at(pb + e) : 0;
      prev = (pb > 0 && pb < n) ? b.at(pb - 1) : 0;
      next = (pb + kPer < n) ? b.at(pb + kPer) : 0;
    } else {
      const int32_t* row = base + static_cast<size_t>(k) * n;
      if (vec) {
        const int4 v = *reinterpret_cast<const int4*>(row + pb);
        id[0] = v.x; id[1] = v.y; id[2] = v.z; id[3] = v.w;
      } else {
#pragma unroll
        for (int e = 0; e < kPer; ++e) id[e] = (pb + e < n) ? row[pb + e] : 0;
      }
      prev = (pb > 0 && pb < n) ? row[pb - 1] : 0;
      next = (pb + kPer < n) ? row[pb + kPer] : 0;
    }
    bool st[kPer], en[kPer];
    int mylast = -1;
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      const int p = pb + e;
      const bool ok = p < n;
      st[e] = ok && (p == 0 || id[e] != (e > 0 ? id[e - 1] : prev));
      en[e] = ok && (p == n - 1 || id[e] != (e + 1 < kPer ? id[e + 1] : next));
      if (st[e]) {
        m[e] |= static_cast<MaskT>(1) << k;
        mylast = p;
      }
    }
    // latest block start before this thread's positions, over the CTA
    int incl = mylast;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl = max(incl, y);
    }
    if (lane == 31) warp_last[w] = incl;
    __syncthreads();
    int before = __shfl_up_sync(0xffffffffu, incl, 1);
    if (lane == 0) before = -1;
    for (int w2 = 0; w2 < w; ++w2) before = max(before, warp_last[w2]);
    __syncthreads();  // warp_last is rewritten for the next hash
    int cur = before >= 0 ? before : carry[k];
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      if (st[e]) cur = pb + e;
      if (en[e]) longest = max(longest, pb + e - cur + 1);
    }
  }
  MaskT* out = bmask + static_cast<size_t>(h) * n;
  if (vec && sizeof(MaskT) == 4) {
    *reinterpret_cast<uint4*>(out + pb) = make_uint4(static_cast<uint32_t>(m[0]), static_cast<uint32_t>(m[1]),
                                                     static_cast<uint32_t>(m[2]), static_cast<uint32_t>(m[3]));
  } else {
#pragma unroll
    for (int e = 0; e < kPer; ++e)
      if (pb + e < n) out[pb + e] = m[e];
  }
  longest = __reduce_max_sync(0xffffffffu, longest);
  if (lane == 0 && longest > 0) atomicMax(bmax + h, longest);
}

// One warp per (head, query tile); lanes walk the hashes.
template <bool kFromTable>
__global__ void __launch_bounds__(kThreads) spans_kernel(const int32_t* __restrict__ ids,
                                                         const double* __restrict__ table, int H, int s, int n,
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
    if constexpr (kFromTable) {
      const Binning b = Binning::from_table(table + (static_cast<size_t>(h) * s + k) * 2);
      lo = min(lo, block_start(b, i0, b.at(i0)));
      if (!causal) hi = max(hi, block_end(b, i1, b.at(i1), n));
    } else {
      const MemRow row{ids + (static_cast<size_t>(h) * s + k) * n};
      lo = min(lo, block_start(row, i0, row.at(i0)));
      if (!causal) hi = max(hi, block_end(row, i1, row.at(i1), n));
    }
  }
  lo = __reduce_min_sync(0xffffffffu, lo);
  hi = __reduce_max_sync(0xffffffffu, hi);
  if (lane == 0) {
    spans[(static_cast<size_t>(h) * T + t) * 2] = lo;
    spans[(static_cast<size_t>(h) * T + t) * 2 + 1] = hi;
  }
}

template <bool kFromTable>
int launch_window_impl(const int32_t* ids, const double* table, int H, int s, int n, int causal, int32_t* bmax,
                       int32_t* spans, void* bmask, uint32_t* err, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(bmax, 0, sizeof(int32_t) * H, st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(bmax)");
  dim3 g1(ceil_div(n, 4 * kThreads), H);
  if (s <= 32)
    mask_bmax_kernel<uint32_t, kFromTable><<<g1, kThreads, 0, st>>>(ids, table, s, n, static_cast<uint32_t*>(bmask),
                                                                    bmax, err);
  else
    mask_bmax_kernel<unsigned long long, kFromTable><<<g1, kThreads, 0, st>>>(
        ids, table, s, n, static_cast<unsigned long long*>(bmask), bmax, err);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "mask_bmax_kernel launch");
  const long long warps = static_cast<long long>(H) * ceil_div(n, PLSH_TILE);
  const int g2 = static_cast<int>((warps * 32 + kThreads - 1) / kThreads);
  spans_kernel<kFromTable><<<g2, kThreads, 0, st>>>(ids, table, H, s, n, causal, spans);
  e = cudaGetLastError();
  return e == cudaSuccess ? PLSH_OK : cuda_fail(e, "spans_kernel launch");
}

}  // namespace

int launch_window(const int32_t* ids, int H, int s, int n, int causal, int32_t* bmax,
                  int32_t* spans, void* bmask, uint32_t* err, cudaStream_t st) {
  return launch_window_impl<false>(ids, nullptr, H, s, n, causal, bmax, spans, bmask, err, st);
}

int launch_window_from_table(const double* table, int H, int s, int n, int causal, int32_t* bmax,
                             int32_t* spans, void* bmask, uint32_t* err, cudaStream_t st) {
  return launch_window_impl<true>(nullptr, table, H, s, n, causal, bmax, spans, bmask, err, st);
}

}  // namespace plsh
