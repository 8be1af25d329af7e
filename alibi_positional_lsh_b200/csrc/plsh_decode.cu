// Decode: single query rows against the cached keys -- plsh_decode_fwd.
//
// For query row t of (batch b, head h) at position i = pos[t], the output is
// row i of T~ = D~^{-1} (exp(Q K^T / sqrt d) o M~) V (Positional LSH technical
// summary, Methodology 2 and 3), with the key range ending at i when causal:
//   O = sum_j c_ij e^{S_ij} V_j / sum_j c_ij e^{S_ij},  S_ij = q . K_j / sqrt d,
// c_ij = s - popcount(OR of the boundary masks over (min(i,j), max(i,j)]).
// Blocks are contiguous (Methodology 1, structure), so walking away from i
// the OR only grows and c_ij only falls: the keys with weight form one run
// below i (i included) and, when not causal, one run above it. Only their K
// and V rows are read.
//
// Two kernels. decode_range_kernel gives every row (one CTA each) the length
// of both runs -- an OR-scan of the masks along the walk, 2048 keys a step, to
// the first key whose OR holds every hash -- cuts each run into segments of
// 16 KB of K rows, hands the segments to at most 8 work units per row, and
// stores for each unit the OR of the masks between i and its first key (the
// carry), appending the units to a work list. decode_unit_kernel runs
// persistent CTAs over the list, each a small pipeline of warp roles: a
// producer warp turns each segment's masks into counts and bulk-copies its K
// and V rows into shared memory two segments ahead, eight compute warps score
// the keys and fold them into running maxima, sums and output rows, and a
// merger warp combines the warps of a finished unit and writes its partial
// result to caller scratch. The last unit of a row to finish (a ticket from a
// per-row counter in the same scratch) merges the partials into O and row_sum
// and resets the counter.
//
// Every wait on a copy is bounded in time (PLSH_DEVERR_TIMEOUT); a CTA that
// gives up waits (again bounded) for the copies it issued and returns, and its
// rows' outputs are left unwritten. A test hook (plsh_test_withhold_mma) makes
// the producer issue nothing, so that the compute warps' waits run out.
#include <algorithm>
#include <cmath>

#include <cuda_bf16.h>

#include "plsh_internal.h"
#include "plsh_sm100.cuh"

namespace plsh {
namespace {

using namespace sm100;

constexpr int kRangeThreads = 128;       // decode_range_kernel: one CTA per row
constexpr int kUnits = kDecodeMaxSplit;  // work units per row
constexpr int kSegBytes = 16384;         // bytes of K rows (and of V rows) in one segment
constexpr int kScan = 16;                // range scan: keys per lane per step
constexpr int kMinSegs = 2;              // segments per work unit, at least (when the run has them)
constexpr uint64_t kDrainLimitNs = 100000000ull;  // bound of the wait for copies in flight at an abort

// A work unit, written by decode_range_kernel for decode_unit_kernel (32 bytes): segments
// [e0, e1) of the walk of query row `row` on one side of its position i.
struct UnitDesc {
  int row;   // (b H + h) m + t
  int i;     // the row's position
  int meta;  // side (bit 0: 0 below, 1 above), the unit's slot u (bits 1-4), the row's unit count U (bits 5-8)
  int e0, e1;
  int len;   // keys with weight on that side: walk offsets [0, len)
  unsigned long long carry;  // OR of the masks between i and the unit's first key
};
static_assert(sizeof(UnitDesc) == 32, "UnitDesc layout");

template <typename MaskT>
__device__ __forceinline__ int popc_mask(MaskT m) {
  if constexpr (sizeof(MaskT) == 8) return __popcll(static_cast<unsigned long long>(m));
  else return __popc(static_cast<unsigned>(m));
}

// The mask that the walk's key at offset w from i contributes on `side` (0: i and below, 1: above).
// Below, key j = i - w needs the masks over (j, i], so it adds bm[j + 1] (nothing for j = i, whose
// count is s); above, key j = i + 1 + w adds bm[j]. Keys outside [0, n) add every hash.
template <typename MaskT>
__device__ __forceinline__ MaskT walk_mask(const MaskT* bm, int i, int n, int side, int w, MaskT full) {
  const int j = side == 0 ? i - w : i + 1 + w;
  if (j < 0 || j >= n) return full;
  return side == 1 ? bm[j] : (j == i ? static_cast<MaskT>(0) : bm[j + 1]);
}

template <typename MaskT>
__device__ __forceinline__ MaskT warp_or(MaskT v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v |= __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Exclusive OR-prefix over the lanes (lane 0 gets 0).
template <typename MaskT>
__device__ __forceinline__ MaskT warp_excl_or(MaskT v, int lane) {
  MaskT x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const MaskT y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x |= y;
  }
  const MaskT e = __shfl_up_sync(0xffffffffu, x, 1);
  return lane == 0 ? static_cast<MaskT>(0) : e;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// The lane's N consecutive values of a row in shared memory (N = 2 or 4), as floats.
template <int N>
__device__ __forceinline__ void row_n(const float* p, float* out) {
  if constexpr (N == 4) {
    const float4 x = *reinterpret_cast<const float4*>(p);
    out[0] = x.x; out[1] = x.y; out[2] = x.z; out[3] = x.w;
  } else {
    const float2 x = *reinterpret_cast<const float2*>(p);
    out[0] = x.x; out[1] = x.y;
  }
}
template <int N>
__device__ __forceinline__ void row_n(const __nv_bfloat16* p, float* out) {
  if constexpr (N == 4) {
    const uint2 x = *reinterpret_cast<const uint2*>(p);
    out[0] = __uint_as_float(x.x << 16); out[1] = __uint_as_float(x.x & 0xFFFF0000u);
    out[2] = __uint_as_float(x.y << 16); out[3] = __uint_as_float(x.y & 0xFFFF0000u);
  } else {
    const uint32_t x = *reinterpret_cast<const uint32_t*>(p);
    out[0] = __uint_as_float(x << 16); out[1] = __uint_as_float(x & 0xFFFF0000u);
  }
}
__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void from_f(float& y, float x) { y = x; }
__device__ __forceinline__ void from_f(__nv_bfloat16& y, float x) { y = __float2bfloat16_rn(x); }

// One CTA per query row: the lengths of the runs of keys with weight on both sides of i, their
// split into at most kUnits work units of whole segments (seg keys each; seg a multiple of kScan),
// and each unit's carry; the row's units are appended to the call's work list. The masks are
// scanned along the walk kRangeThreads * kScan keys a step (warp w takes the step's keys
// 512 w .. 512 w + 511, lane l sixteen of them). A position outside [0, n)
// gives the row no units and sets PLSH_DEVERR_POSITION.
template <typename MaskT>
__global__ void __launch_bounds__(kRangeThreads) decode_range_kernel(const int32_t* __restrict__ pos, int m, int H, int n,
                                                                int s, int causal, const MaskT* __restrict__ bmask,
                                                                int seg, UnitDesc* __restrict__ units,
                                                                unsigned* __restrict__ unit_count,
                                                                uint32_t* __restrict__ err) {
  constexpr int kRW = kRangeThreads / 32;
  __shared__ MaskT tile[kRW][32 * kScan + kScan];
  __shared__ MaskT wt[kRW];
  __shared__ int wh[kRW];
  __shared__ unsigned long long carry_s[kUnits];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = blockIdx.x;
  const int t = static_cast<int>(row % m);
  const int h = static_cast<int>((row / m) % H);
  const int i = pos[t];
  if (i < 0 || i >= n) {  // the row gets no units
    if (threadIdx.x == 0) atomicOr(err, PLSH_DEVERR_POSITION);
    return;
  }
  const MaskT FULL = (s >= static_cast<int>(8 * sizeof(MaskT))) ? static_cast<MaskT>(~static_cast<MaskT>(0))
                                                              : static_cast<MaskT>((static_cast<MaskT>(1) << s) - 1);
  const MaskT* bm = bmask + static_cast<size_t>(h) * n;
  constexpr int kStep = kRangeThreads * kScan;

  // One step of the walk from offset `base`: the thread's sixteen walk masks (offsets >= wend count as
  // empty), and the OR of the walk masks before the thread's first offset (from the carry before the
  // step). Returns the OR over the whole step.
  auto step = [&](int side, int base, int wend, MaskT carry, MaskT (&v)[kScan], MaskT& before) -> MaskT {
    // the warp's 512 masks, loaded 32 consecutive at a time and handed to the lanes through shared
    // memory (a padded tile: element x at x + x / 32)
    const int wb = base + 32 * kScan * warp;
#pragma unroll
    for (int e = 0; e < kScan; ++e) {
      const int x = lane + 32 * e, w = wb + x;
      tile[warp][x + (x >> 5)] = w < wend ? walk_mask(bm, i, n, side, w, FULL) : static_cast<MaskT>(0);
    }
    __syncwarp();
    MaskT tot = 0;
#pragma unroll
    for (int e = 0; e < kScan; ++e) {
      const int x = kScan * lane + e;
      v[e] = tile[warp][x + (x >> 5)];
      tot |= v[e];
    }
    __syncwarp();
    const MaskT xl = warp_excl_or(tot, lane);
    const MaskT wtot = warp_or(tot);
    __syncthreads();  // the previous step's readers of wt are done
    if (lane == 0) wt[warp] = wtot;
    __syncthreads();
    MaskT pw = carry, all = carry;
#pragma unroll
    for (int w2 = 0; w2 < kRW; ++w2) {
      if (w2 < warp) pw |= wt[w2];
      all |= wt[w2];
    }
    before = pw | xl;
    return all;
  };

  // walk offsets [0, len) carry weight; the key at offset len is the first whose OR holds every hash
  // (keys outside [0, n) hold every hash, so the scan ends)
  auto run_length = [&](int side) -> int {
    MaskT carry = 0;
    for (int base = 0;; base += kStep) {
      MaskT v[kScan], before;
      const MaskT all = step(side, base, 0x7fffffff, carry, v, before);
      MaskT R = before;
      int fe = kScan;
#pragma unroll
      for (int e = 0; e < kScan; ++e) {
        R |= v[e];
        if (fe == kScan && R == FULL) fe = e;
      }
      const unsigned hit = __ballot_sync(0xffffffffu, fe < kScan);
      int first = 0x7fffffff;  // the warp's first offset whose OR holds every hash
      if (hit) {
        const int fl = __ffs(hit) - 1;
        first = base + kScan * (32 * warp + fl) + __shfl_sync(0xffffffffu, fe, fl);
      }
      if (lane == 0) wh[warp] = first;
      __syncthreads();
      int len = 0x7fffffff;
#pragma unroll
      for (int w2 = 0; w2 < kRW; ++w2) len = min(len, wh[w2]);
      __syncthreads();  // every thread has read wh
      if (len != 0x7fffffff) return len;
      carry = all;
    }
  };
  const int len_lo = run_length(0);  // >= 1: key i has count s
  const int len_hi = causal ? 0 : run_length(1);
  const int ns_lo = (len_lo + seg - 1) / seg, ns_hi = (len_hi + seg - 1) / seg;
  // units: shared between the sides in proportion to their segments, at least one for each side
  // with keys; then as few units as carry the same number of segments each
  int u_hi = 0;
  if (ns_hi > 0) u_hi = min(ns_hi, max(1, min(kUnits - 1, (kUnits * ns_hi) / (ns_lo + ns_hi))));
  int u_lo = min(ns_lo, kUnits - u_hi);
  const int k_lo = max((ns_lo + u_lo - 1) / u_lo, min(ns_lo, kMinSegs));
  u_lo = (ns_lo + k_lo - 1) / k_lo;
  int k_hi = 1;
  if (u_hi > 0) {
    k_hi = max((ns_hi + u_hi - 1) / u_hi, min(ns_hi, kMinSegs));
    u_hi = (ns_hi + k_hi - 1) / k_hi;
  }

  // the carry of each unit of one side: the OR of the walk masks at offsets [0, W) for a unit whose
  // first offset is W (a multiple of seg, so some thread's first offset in some step)
  auto carries = [&](int side, int nu, int kk, int slot0) {
    if (threadIdx.x == 0) carry_s[slot0] = 0ull;
    if (nu <= 1) return;
    const int unit = kk * seg;
    const int wmax = (nu - 1) * unit;  // the last unit's first offset
    MaskT carry = 0;
    for (int base = 0; base <= wmax; base += kStep) {
      MaskT v[kScan], before;
      carry = step(side, base, wmax, carry, v, before);
      const int w0 = base + kScan * threadIdx.x;
      if (w0 > 0 && w0 <= wmax && w0 % unit == 0) carry_s[slot0 + w0 / unit] = static_cast<unsigned long long>(before);
    }
  };
  carries(0, u_lo, k_lo, 0);
  if (u_hi > 0) carries(1, u_hi, k_hi, u_lo);
  __syncthreads();
  if (threadIdx.x == 0) {
    // the row's units join the call's work list (in no particular order)
    const int U = u_lo + u_hi;
    const unsigned base = atomicAdd(unit_count, static_cast<unsigned>(U));
    for (int u = 0; u < U; ++u) {
      const int side = u < u_lo ? 0 : 1;
      const int kk = side ? k_hi : k_lo;
      const int ns = side ? ns_hi : ns_lo;
      UnitDesc ud;
      ud.row = static_cast<int>(row);
      ud.i = i;
      ud.meta = side | (u << 1) | (U << 5);
      ud.e0 = (side ? u - u_lo : u) * kk;
      ud.e1 = min(ud.e0 + kk, ns);
      ud.len = side ? len_hi : len_lo;
      ud.carry = carry_s[u];
      units[base + u] = ud;
    }
  }
}

constexpr int kComputeWarps = 8;  // warps 0-7: the segments' arithmetic
constexpr int kWarpProducer = 8, kWarpMerger = 9;
constexpr int kUnitThreads = 32 * (kComputeWarps + 2);

template <typename T, int D, typename MaskT>
struct UnitSmem {
  static constexpr int kSeg = kSegBytes / (D * static_cast<int>(sizeof(T)));  // keys per segment
  T k[2][kSegBytes / sizeof(T)];  // the segments' K rows, two stages
  T v[2][kSegBytes / sizeof(T)];  // and V rows
  T q[2][D];                      // the query row, with the first segment of each unit
  int cnt[3][kSeg];               // the segments' counts, in walk order (by segment % 3)
  float wm[kComputeWarps], wl[kComputeWarps];
  float wo[kComputeWarps][D];     // a finished unit's per-warp partial results, for the merger
  int res_unit[3];                // and its row, slot u and the row's unit count U
  UnitDesc ring[4];               // the units the producer has started, by ordinal % 4
  uint64_t full[2], empty[2];     // a stage's copies landed / all compute warps done with it
  uint64_t rfull, rempty;         // a unit's partials written / taken by the merger
  int abort_flag;
};

// Persistent CTAs over the call's work list: CTA c takes units c, c + G, c + 2G, ... (G CTAs); its
// segments, unit after unit, form one stream, and the roles meet only at barriers in shared memory.
// The producer warp loads each segment's walk masks, turns them into counts (an OR-scan from the
// unit's carry) and starts bulk copies of its K rows, V rows and (first segment of a unit) the query
// row, two segments ahead. Each compute warp scores its keys of the segment (lanes over dims, a
// transpose-reduce of the partial dot products) and folds them into its running maximum, sum and
// output row in log2 units. The merger warp combines a finished unit's warps and writes its partial
// result to part slot u of its row; the row's last unit to finish merges the slots into O and
// row_sum.
template <typename T, int D, typename MaskT>
__global__ void __launch_bounds__(kUnitThreads) decode_unit_kernel(
    const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V, int m, int H, int H_kv, int n, int s,
    const MaskT* __restrict__ bmask, const UnitDesc* __restrict__ units, const unsigned* __restrict__ unit_count,
    float* __restrict__ part, unsigned* __restrict__ done, T* __restrict__ O, float* __restrict__ row_sum,
    uint32_t* __restrict__ err, uint64_t wait_ns, int withhold) {
  using Smem = UnitSmem<T, D, MaskT>;
  constexpr int SEG = Smem::kSeg;
  constexpr int KPW = SEG / kComputeWarps;  // keys per compute warp per segment
  constexpr int KPL = SEG / 32;             // keys per producer lane per segment
  constexpr int DPL = D / 32;               // dims per lane
  static_assert(KPW >= 2 && KPW <= 16 && (KPW & (KPW - 1)) == 0 && KPL >= 1 && KPL * 32 == SEG, "segment geometry");
  extern __shared__ __align__(128) uint8_t smem_raw[];
  const uint32_t pad = (128u - (static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw)) & 127u)) & 127u;
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw + pad);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned total = *unit_count;
  const unsigned G = gridDim.x;
  if (blockIdx.x >= total) return;
  const MaskT FULL = (s >= static_cast<int>(8 * sizeof(MaskT))) ? static_cast<MaskT>(~static_cast<MaskT>(0))
                                                              : static_cast<MaskT>((static_cast<MaskT>(1) << s) - 1);
  auto has_unit = [&](int ord) { return blockIdx.x + static_cast<unsigned>(ord) * G < total; };
  // segment e of unit ud: walk offsets [e SEG, min((e + 1) SEG, len)); its keys jmin .. jmin + nk - 1
  auto seg_keys = [&](const UnitDesc& ud, int e, int& jmin, int& nk) {
    const int w0 = e * SEG, w1 = min(w0 + SEG, ud.len);
    nk = w1 - w0;
    jmin = (ud.meta & 1) == 0 ? ud.i - (w1 - 1) : ud.i + 1 + w0;
  };
  if (tid == 0) {
    sm.abort_flag = 0;
    for (int b2 = 0; b2 < 2; ++b2) {
      mbar_init(&sm.full[b2], 1);
      mbar_init(&sm.empty[b2], kComputeWarps);
    }
    mbar_init(&sm.rfull, kComputeWarps);
    mbar_init(&sm.rempty, 1);
    fence_mbarrier_init();
  }
  __syncthreads();

  if (warp == kWarpProducer) {
    // ------------------------------------------------------------ producer
    // (a failure-detection test can tell it to issue nothing, so that the compute warps' waits run out)
    int issued = 0;
    bool ok = withhold == 0;
    UnitDesc nxt;  // the next unit's descriptor, loaded one unit ahead
    if (ok && has_unit(0)) nxt = units[blockIdx.x];
    for (int ord = 0; ok && has_unit(ord); ++ord) {
      const UnitDesc pd = nxt;
      if (has_unit(ord + 1)) nxt = units[blockIdx.x + static_cast<unsigned>(ord + 1) * G];
      const int h = (pd.row / m) % H, b = pd.row / (m * H);
      const MaskT* bm = bmask + static_cast<size_t>(h) * n;
      const size_t kv0 = (static_cast<size_t>(b) * H_kv + h / (H / H_kv)) * static_cast<size_t>(n) * D;
      MaskT carry = static_cast<MaskT>(pd.carry);
      for (int e = pd.e0; e < pd.e1; ++e, ++issued) {
        int jmin, nk;
        seg_keys(pd, e, jmin, nk);
        const int st = issued & 1;
        // counts of the segment's keys: lane l takes walk offsets KPL l .. KPL l + KPL - 1 of it
        MaskT wmk[KPL];
#pragma unroll
        for (int r = 0; r < KPL; ++r) {
          const int tt = KPL * lane + r;
          wmk[r] = tt < nk ? walk_mask(bm, pd.i, n, pd.meta & 1, e * SEG + tt, FULL) : static_cast<MaskT>(0);
        }
        MaskT loc = 0;
#pragma unroll
        for (int r = 0; r < KPL; ++r) loc |= wmk[r];
        MaskT R = carry | warp_excl_or(loc, lane);
        int* cnt = sm.cnt[issued % 3];  // last read for segment issued - 3, whose stage has been released
#pragma unroll
        for (int r = 0; r < KPL; ++r) {
          R |= wmk[r];
          cnt[KPL * lane + r] = s - popc_mask(R);
        }
        carry |= warp_or(loc);
        if (issued >= 2 && !__all_sync(0xffffffffu, mbar_wait(&sm.empty[st], static_cast<uint32_t>((issued - 2) >> 1) & 1u,
                                                             &sm.abort_flag, err, wait_ns))) {
          ok = false;
          break;
        }
        if (lane == 0 && e == pd.e0) sm.ring[ord & 3] = pd;
        __syncwarp();
        if (lane == 0) {
          const uint32_t bytes = static_cast<uint32_t>(nk) * D * sizeof(T);
          const bool first = e == pd.e0;
          mbar_arrive_expect_tx(&sm.full[st], 2u * bytes + (first ? static_cast<uint32_t>(D * sizeof(T)) : 0u));
          bulk_load(sm.k[st], K + kv0 + static_cast<size_t>(jmin) * D, bytes, &sm.full[st]);
          bulk_load(sm.v[st], V + kv0 + static_cast<size_t>(jmin) * D, bytes, &sm.full[st]);
          if (first) bulk_load(sm.q[st], Q + static_cast<size_t>(pd.row) * D, D * sizeof(T), &sm.full[st]);
        }
      }
    }
    if (!ok && lane == 0) {
      // the copies still in flight land before the CTA exits
      for (int x2 = max(0, issued - 2); x2 < issued; ++x2)
        mbar_wait_drain(&sm.full[x2 & 1], static_cast<uint32_t>(x2 >> 1) & 1u, kDrainLimitNs);
    }
  } else if (warp == kWarpMerger) {
    // ------------------------------------------------------------ merger
    for (int ord = 0; has_unit(ord); ++ord) {
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.rfull, static_cast<uint32_t>(ord) & 1u, &sm.abort_flag, err, wait_ns)))
        break;
      const int row = sm.res_unit[0], u = sm.res_unit[1], U = sm.res_unit[2];
      float mt = -INFINITY;
#pragma unroll
      for (int w2 = 0; w2 < kComputeWarps; ++w2) mt = fmaxf(mt, sm.wm[w2]);
      float lt = 0.0f, ot[DPL];
#pragma unroll
      for (int d2 = 0; d2 < DPL; ++d2) ot[d2] = 0.0f;
#pragma unroll
      for (int w2 = 0; w2 < kComputeWarps; ++w2) {
        const float f = ex2_approx(sm.wm[w2] - mt);  // 0 for a warp without keys
        lt += sm.wl[w2] * f;
#pragma unroll
        for (int d2 = 0; d2 < DPL; ++d2) ot[d2] += sm.wo[w2][lane * DPL + d2] * f;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.rempty);  // the compute warps may write the next unit's partials
      float* pr = part + (static_cast<size_t>(row) * kUnits + u) * (D + 2);
#pragma unroll
      for (int d2 = 0; d2 < DPL; ++d2) pr[2 + lane * DPL + d2] = ot[d2];
      if (lane == 0) {
        pr[0] = mt;
        pr[1] = lt;
      }
      // the row's last unit to finish merges the U partial results (the others' writes are visible
      // to it once its ticket shows they have all been published) and leaves the row's counter at zero
      __threadfence();
      __syncwarp();
      unsigned ticket = 0;
      if (lane == 0) ticket = atomicAdd(&done[row], 1u);
      ticket = __shfl_sync(0xffffffffu, ticket, 0);
      if (ticket != static_cast<unsigned>(U - 1)) continue;
      __threadfence();
      const float* p0 = part + static_cast<size_t>(row) * kUnits * (D + 2);
      float M = -INFINITY;
      for (int g2 = 0; g2 < U; ++g2) M = fmaxf(M, __ldcg(p0 + g2 * (D + 2)));
      float L = 0.0f, acc[DPL];
#pragma unroll
      for (int d2 = 0; d2 < DPL; ++d2) acc[d2] = 0.0f;
      for (int g2 = 0; g2 < U; ++g2) {
        const float* q2 = p0 + g2 * (D + 2);
        const float m2 = __ldcg(q2);
        if (m2 == -INFINITY) continue;
        const float f = ex2_approx(m2 - M);
        L += __ldcg(q2 + 1) * f;
#pragma unroll
        for (int d2 = 0; d2 < DPL; ++d2) acc[d2] += __ldcg(q2 + 2 + lane * DPL + d2) * f;
      }
      const float inv = 1.0f / L;
      T* orow = O + static_cast<size_t>(row) * D;
#pragma unroll
      for (int d2 = 0; d2 < DPL; ++d2) from_f(orow[lane * DPL + d2], acc[d2] * inv);
      if (lane == 0) {
        row_sum[row] = (log2f(L) + M) * 0.6931471805599453f - logf(static_cast<float>(s));
        done[row] = 0u;
      }
    }
  } else {
    // ------------------------------------------------------------ compute warps
    const float sc2 = 1.4426950408889634f / sqrtf(static_cast<float>(D));  // log2(e) / sqrt(d)
    // after the transpose-reduce, lane l holds the score of the warp's key kidx (lanes that differ only
    // in bits 0 .. 4 - log2(KPW) hold the same one); `rep` is the lowest lane holding key k
    int kidx = 0;
#pragma unroll
    for (int o = 16, c2 = KPW; c2 > 1; o >>= 1, c2 >>= 1) kidx += ((lane & o) != 0) ? c2 / 2 : 0;
    auto rep = [&](int k2) {
      int l2 = 0;
#pragma unroll
      for (int o = 16, c2 = KPW; c2 > 1; o >>= 1, c2 >>= 1)
        if (k2 & (c2 / 2)) {
          l2 |= o;
          k2 -= c2 / 2;
        }
      return l2;
    };
    int c_ord = 0, x = 0;
    UnitDesc cd;
    int ce = 0;
    float qv[DPL];
    float mw = -INFINITY, lw = 0.0f, ow[DPL];
    bool start = true;
    for (;;) {
      const int st = x & 1;
      if (!mbar_wait(&sm.full[st], static_cast<uint32_t>(x >> 1) & 1u, &sm.abort_flag, err, wait_ns)) break;
      if (start) {
        cd = sm.ring[c_ord & 3];
        ce = cd.e0;
        mw = -INFINITY;
        lw = 0.0f;
#pragma unroll
        for (int d2 = 0; d2 < DPL; ++d2) {
          ow[d2] = 0.0f;
          qv[d2] = to_f(sm.q[st][lane * DPL + d2]);
        }
        start = false;
      }
      int jmin, nk;
      seg_keys(cd, ce, jmin, nk);
      const int side = cd.meta & 1;
      const int* cnt = sm.cnt[x % 3];
      // partial dot products of the warp's KPW keys (walk offsets warp KPW + j), lanes over dims
      float a[KPW];
#pragma unroll
      for (int j = 0; j < KPW; ++j) {
        const int tt = warp * KPW + j;
        const int r = side == 0 ? nk - 1 - tt : tt;  // the key's row in the stage
        float acc = 0.0f;
        if (tt < nk) {
          float kv[DPL];
          row_n<DPL>(sm.k[st] + static_cast<size_t>(r) * D + lane * DPL, kv);
#pragma unroll
          for (int d2 = 0; d2 < DPL; ++d2) acc = fmaf(qv[d2], kv[d2], acc);
        }
        a[j] = acc;
      }
      // transpose-reduce: halve the values per lane at each of the first log2(KPW) steps
#pragma unroll
      for (int o = 16, c2 = KPW; c2 > 1; o >>= 1, c2 >>= 1) {
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int j = 0; j < c2 / 2; ++j) {
          const float send = up ? a[j] : a[j + c2 / 2];
          const float keep = up ? a[j + c2 / 2] : a[j];
          a[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
#pragma unroll
      for (int o = 16 / KPW; o >= 1; o >>= 1) a[0] += __shfl_xor_sync(0xffffffffu, a[0], o);
      const int tk = warp * KPW + kidx;
      const bool valid = tk < nk;
      const float sl = valid ? a[0] * sc2 : -INFINITY;  // the score in log2 units
      float mx = sl;
#pragma unroll
      for (int o = 16, c2 = KPW; c2 > 1; o >>= 1, c2 >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      if (mx > -INFINITY) {
        const float m_new = fmaxf(mw, mx);
        const float corr = ex2_approx(mw - m_new);
        mw = m_new;
        const float p = valid ? static_cast<float>(cnt[tk]) * ex2_approx(sl - m_new) : 0.0f;
        float ps = p;
#pragma unroll
        for (int o = 16, c2 = KPW; c2 > 1; o >>= 1, c2 >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
        lw = lw * corr + ps;
#pragma unroll
        for (int d2 = 0; d2 < DPL; ++d2) ow[d2] *= corr;
#pragma unroll
        for (int j = 0; j < KPW; ++j) {
          const float pj = __shfl_sync(0xffffffffu, p, rep(j));
          const int tt = warp * KPW + j;
          if (tt < nk) {
            const int r = side == 0 ? nk - 1 - tt : tt;
            float vv[DPL];
            row_n<DPL>(sm.v[st] + static_cast<size_t>(r) * D + lane * DPL, vv);
#pragma unroll
            for (int d2 = 0; d2 < DPL; ++d2) ow[d2] = fmaf(pj, vv[d2], ow[d2]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[st]);  // this warp is done with the stage
      ++x;
      if (++ce < cd.e1) continue;

      // ---- the unit is done: this warp's partial result for the merger
      if (c_ord >= 1 &&
          !mbar_wait(&sm.rempty, static_cast<uint32_t>(c_ord - 1) & 1u, &sm.abort_flag, err, wait_ns))
        break;
      if (lane == 0) {
        sm.wm[warp] = mw;
        sm.wl[warp] = lw;
      }
#pragma unroll
      for (int d2 = 0; d2 < DPL; ++d2) sm.wo[warp][lane * DPL + d2] = ow[d2];
      if (warp == 0 && lane == 0) {
        sm.res_unit[0] = cd.row;
        sm.res_unit[1] = (cd.meta >> 1) & 15;
        sm.res_unit[2] = (cd.meta >> 5) & 15;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.rfull);
      start = true;
      if (!has_unit(++c_ord)) break;
    }
  }
}

// Scratch layout: part [rows][kUnits][D + 2] floats, the work list [rows * kUnits] UnitDesc, its
// counter (zeroed by each call) padded to 16 bytes, then one merge counter per row.
struct DecodeScratch {
  UnitDesc* units;
  unsigned* unit_count;
  unsigned* done;
};
DecodeScratch decode_scratch(float* part, long long rows, int d) {
  DecodeScratch sc;
  sc.units = reinterpret_cast<UnitDesc*>(part + rows * kUnits * (d + 2));
  sc.unit_count = reinterpret_cast<unsigned*>(sc.units + rows * kUnits);
  sc.done = sc.unit_count + 4;
  return sc;
}

template <typename T, int D, typename MaskT>
int launch_decode_typed(const DecodeArgs& a, cudaStream_t st) {
  const long long rows = static_cast<long long>(a.B) * a.H * a.m;
  if (rows * kUnits > 0x7fffffffLL) return fail(PLSH_ERR_RANGE, "plsh_decode_fwd: too many rows");
  const DecodeScratch sc = decode_scratch(a.part, rows, a.d);
  constexpr int SEG = UnitSmem<T, D, MaskT>::kSeg;
  cudaError_t e = cudaMemsetAsync(sc.unit_count, 0, sizeof(unsigned), st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(decode work-list counter)");
  decode_range_kernel<MaskT><<<static_cast<unsigned>(rows), kRangeThreads, 0, st>>>(
      a.pos, a.m, a.H, a.n, a.s, a.causal, static_cast<const MaskT*>(a.bmask), SEG, sc.units, sc.unit_count, a.err);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "decode_range_kernel launch");
  auto kern = decode_unit_kernel<T, D, MaskT>;
  const size_t smem = sizeof(UnitSmem<T, D, MaskT>) + 128;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(decode_unit_kernel)");
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kUnitThreads, smem);
  if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor(decode_unit_kernel)");
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    sms = 148;
  // at most one CTA per unit; CTAs past the list's length return at once
  const long long grid = std::min<long long>(rows * kUnits, static_cast<long long>(std::max(per_sm, 1)) * sms);
  kern<<<static_cast<unsigned>(grid), kUnitThreads, smem, st>>>(
      static_cast<const T*>(a.Q), static_cast<const T*>(a.K), static_cast<const T*>(a.V), a.m, a.H, a.H_kv, a.n, a.s,
      static_cast<const MaskT*>(a.bmask), sc.units, sc.unit_count, a.part, sc.done, static_cast<T*>(a.O),
      a.row_sum, a.err, wait_limit_ns(), withhold_mma() ? 1 : 0);
  e = cudaGetLastError();
  return e == cudaSuccess ? PLSH_OK : cuda_fail(e, "decode_unit_kernel launch");
}

template <typename T, int D>
int launch_decode_mask(const DecodeArgs& a, cudaStream_t st) {
  return a.s <= 32 ? launch_decode_typed<T, D, uint32_t>(a, st) : launch_decode_typed<T, D, unsigned long long>(a, st);
}

}  // namespace

int launch_decode(const DecodeArgs& a, cudaStream_t st) {
  if (a.dtype == PLSH_F32)
    return a.d == 64 ? launch_decode_mask<float, 64>(a, st) : launch_decode_mask<float, 128>(a, st);
  return a.d == 64 ? launch_decode_mask<__nv_bfloat16, 64>(a, st) : launch_decode_mask<__nv_bfloat16, 128>(a, st);
}

size_t decode_scratch_bytes(long long rows, int d) {
  return static_cast<size_t>(rows) * (sizeof(float) * kUnits * (static_cast<size_t>(d) + 2) +
                                      sizeof(UnitDesc) * kUnits + sizeof(unsigned)) +
         4 * sizeof(unsigned);
}

}  // namespace plsh
