// Tile machinery shared by the tensor-core attention kernels (the fused forward and the tensor-core
// backward): tile geometry, the boundary-mask stage a mask warp publishes per key tile, the
// diagonal-tile scan that turns masks into counts, and the host-side tensor maps.
//
// Hash-match counts come from boundary masks: Bm(p) has bit k set where hash k opens a block at
// position p. Blocks are contiguous (Positional LSH technical summary, Methodology 1, structure),
// so the number of hashes that put i and j in one bin is c_ij = s - popcount(OR of Bm over
// (min(i, j), max(i, j)]), and the OR over such a range splits into a part that depends on one
// end only and a part that depends on the other end only.
#pragma once

#include <cstdint>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "plsh_internal.h"

namespace plsh {
namespace tiles {

constexpr int kTile = PLSH_TILE;
constexpr int kD = 128;
constexpr int kChunkBytes = kTile * 64 * 2;  // 128 rows x 64 bf16 = 16 KB (one SW128 box)
constexpr int kTileBytes = 2 * kChunkBytes;  // 128 x 128 bf16 = 32 KB
constexpr int kMaxSortedHeads = 256;
constexpr uint64_t kDrainNs = 100000000ull;

template <typename MaskT>
struct alignas(16) MaskStage {
  MaskT bm[kTile + 4];  // bm[c]  = boundary mask of key j0 + c, c = 0..128 (all ones outside [0, n))
  MaskT pre[kTile];     // pre[c] = OR bm[1 .. c]        (pre[0] = 0)
  MaskT suf[kTile];     // suf[c] = OR bm[c + 1 .. 127]  (suf[127] = 0)
  // range ORs against the 32-row block of warp q (diagonal tile only):
  // dq[q][c] = OR bm[c + 1 .. 32q] for c < 32q, OR bm[32q + 32 .. c] for c >= 32q + 32
  MaskT dq[4][kTile];
  // the tile as the softmax needs it: valid (0 = end of the CTA's work), kind (0 diagonal,
  // 1 below, 2 above), first / last tile of its item,
  // item index x, first key j0, and the comparator's hash of the sub-item
  int valid, kind, first, last, x, j0, sub, pad;
};

struct Params {
  int B, H, H_kv, n, s, causal, T, items;
  // [H][T][2] union windows (K3), or [H][s][T][2] per-hash windows for the comparator (K4, the
  // kVarlen instantiations, which walk every item once per hash)
  const int32_t* spans;
  // exact banded ALiBi (the kAlibi instantiations): per-head length scales and ln(1/eps); the
  // window of a query tile reaches W_h = ceil(sigma_h ln(1/eps)) keys past its rows
  const double* sigma;
  double log_inv_eps;
  // wall-clock limit of every barrier wait; for failure-detection tests, the MMA issuer can be
  // told to issue nothing, so that every wait for a score tile runs out
  uint64_t wait_ns;
  int withhold_mma;
};

// Keys past which exp(-|i - j| / sigma) < eps, clamped to [0, n].
__device__ __forceinline__ int alibi_reach(double sigma, double log_inv_eps, int n) {
  const double w = ceil(sigma * log_inv_eps);
  return (w >= static_cast<double>(n) || !(w >= 0.0)) ? n : static_cast<int>(w);
}

// The key tiles of a CTA's work items, in the order every role walks them:
// items x0, x0 + stride, ...; within an item the diagonal tile, then the tiles
// below, then (non-causal) the tiles above. For the per-sample comparator an
// item is walked once per hash k (a sub-item), each time over that hash's
// window. The next (sub-)item's window is fetched one ahead.
template <bool kVarlen, bool kAlibi = false>
struct TileIter {
  const Params* p;
  const int16_t* order;
  int x, stride;
  int k;        // items started so far by this CTA
  int sub;      // sub-item (hash) within the item: 0 for K3
  int it;       // key tile within the sub-item
  int total;    // key tiles of the sub-item
  int n_below;
  int b, h, i0;
  int g;        // key tiles so far by this CTA
  bool valid;
  bool bad_window;  // the window read for this sub-item was out of range (and was clamped)
  int nx_lo, nx_hi;

  __device__ __forceinline__ int n_sub() const { return kVarlen ? p->s : 1; }
  __device__ __forceinline__ int head_of(int xx) const {
    const int hr = xx / (p->B * p->T);
    return (p->H <= kMaxSortedHeads) ? static_cast<int>(order[hr]) : hr;
  }
  __device__ __forceinline__ void fetch(int xx, int sb, int& lo, int& hi) const {
    if (xx < p->items) {
      const int hh = head_of(xx);
      const int tt = (xx % (p->B * p->T)) % p->T;
      if constexpr (kAlibi) {
        const int reach = alibi_reach(p->sigma[hh], p->log_inv_eps, p->n);
        const int i0 = tt * kTile, last_row = min(p->n, i0 + kTile) - 1;
        lo = max(0, i0 - reach);
        hi = p->causal ? last_row : min(p->n - 1, last_row + reach);
        return;
      }
      const size_t at = kVarlen ? ((static_cast<size_t>(hh) * p->s + sb) * p->T + tt) * 2
                                : (static_cast<size_t>(hh) * p->T + tt) * 2;
      lo = p->spans[at];
      hi = p->spans[at + 1];
    }
  }
  __device__ __forceinline__ void load_sub(int lo, int hi) {
    if (kVarlen && sub + 1 < n_sub()) fetch(x, sub + 1, nx_lo, nx_hi);
    else fetch(x + stride, 0, nx_lo, nx_hi);
    const int last_row = min(p->n, i0 + kTile) - 1;
    bad_window = lo < 0 || lo > i0 || hi >= p->n || hi < last_row;
    lo = max(0, min(lo, i0));
    hi = min(p->n - 1, max(hi, last_row));
    n_below = (i0 - lo + kTile - 1) / kTile;
    total = 1 + n_below + (p->causal ? 0 : (hi - i0) / kTile);
    it = 0;
  }
  __device__ __forceinline__ void load_item(int lo, int hi) {
    valid = x < p->items;
    if (!valid) return;
    const int rem = x % (p->B * p->T);
    h = head_of(x);
    b = rem / p->T;
    i0 = (rem % p->T) * kTile;
    sub = 0;
    load_sub(lo, hi);
  }
  __device__ __forceinline__ void start(const Params* pp, const int16_t* ord) {
    p = pp;
    order = ord;
    x = blockIdx.x;
    stride = gridDim.x;
    k = 0;
    g = 0;
    nx_lo = nx_hi = 0;
    int lo = 0, hi = 0;
    fetch(x, 0, lo, hi);
    load_item(lo, hi);
  }
  __device__ __forceinline__ void next() {
    ++g;
    if (++it >= total) {
      if (kVarlen && sub + 1 < n_sub()) {
        ++sub;
        load_sub(nx_lo, nx_hi);
      } else {
        x += stride;
        ++k;
        load_item(nx_lo, nx_hi);
      }
    }
  }
  __device__ __forceinline__ int kind() const { return it == 0 ? 0 : (it <= n_below ? 1 : 2); }
  __device__ __forceinline__ int j0() const {
    const int kd = kind();
    return kd == 0 ? i0 : (kd == 1 ? i0 - kTile * it : i0 + kTile * (it - n_below));
  }
  __device__ __forceinline__ bool first() const { return it == 0 && (!kVarlen || sub == 0); }
  __device__ __forceinline__ bool last() const { return it == total - 1 && (!kVarlen || sub == n_sub() - 1); }
};

template <typename MaskT>
__device__ __forceinline__ int popc_m(MaskT m) {
  if constexpr (sizeof(MaskT) == 8) return __popcll(static_cast<unsigned long long>(m));
  else return __popc(static_cast<unsigned>(m));
}

template <typename MaskT>
__device__ __forceinline__ void load4(const MaskT* p, MaskT (&b)[4]) {
  if constexpr (sizeof(MaskT) == 8) {
    const ulonglong2 a = reinterpret_cast<const ulonglong2*>(p)[0];
    const ulonglong2 c = reinterpret_cast<const ulonglong2*>(p)[1];
    b[0] = a.x; b[1] = a.y; b[2] = c.x; b[3] = c.y;
  } else {
    const uint4 a = *reinterpret_cast<const uint4*>(p);
    b[0] = a.x; b[1] = a.y; b[2] = a.z; b[3] = a.w;
  }
}

template <typename MaskT>
__device__ __forceinline__ MaskT warp_prefix_or(MaskT v, int lane) {  // inclusive over lanes 0..lane
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const MaskT y = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v |= y;
  }
  return v;
}

template <typename MaskT>
__device__ __forceinline__ MaskT warp_suffix_or(MaskT v, int lane) {  // inclusive over lanes lane..31
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const MaskT y = __shfl_down_sync(0xffffffffu, v, o);
    if (lane + o < 32) v |= y;
  }
  return v;
}

// Orders every later use of r after the preceding tcgen05.wait::ld (the registers of an
// asynchronous TMEM load are only valid after the wait).
template <int N>
__device__ __forceinline__ void regs_after_wait(uint32_t (&r)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

// Diagonal tile, one 32-row block (rows [32q, 32q + 32) of the tile, row r): counts of the block's own 32 keys,
// as bytes (key 32q + 4j + e in byte e of word j), written to this thread's column cw[j * ld] of
// shared memory, and the carries for the other keys. Keys c < r: R = OR bm[c + 1 .. r], scanned
// from the row down (count 0 unless kBelow); the row's own key: count s; keys c > r:
// R = OR bm[r + 1 .. c], scanned from the row up (count 0 unless kAbove). On return
// lo = OR bm[32q + 1 .. r] and hi = OR bm[r + 1 .. 32q + 31] (0 unless kAbove).
// bq[c] = mask of the block's key c (c = 0..32), rr = the row within the block (0..31).
template <typename MaskT, bool kBelow, bool kAbove>
__device__ __forceinline__ void diag_scan_block(const MaskT* bq, int rr, int s, uint32_t* cw, int ld, MaskT& lo,
                                                MaskT& hi) {
  MaskT R = 0;
#pragma unroll 1
  for (int j = 7; j >= 0; --j) {
    uint32_t acc = 0;
#pragma unroll
    for (int e = 3; e >= 0; --e) {
      const int cc = 4 * j + e;
      if (cc < rr) R |= bq[cc + 1];
      acc = (acc << 8) | ((cc == rr || (kBelow && cc < rr)) ? static_cast<uint32_t>(s - popc_m(R)) : 0u);
    }
    cw[j * ld] = acc;
  }
  lo = R;
  MaskT R2 = 0;
  if (kAbove) {
#pragma unroll 1
    for (int j = 0; j < 8; ++j) {
      uint32_t acc = cw[j * ld];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int cc = 4 * j + e;
        if (cc > rr) {
          R2 |= bq[cc];
          acc |= static_cast<uint32_t>(s - popc_m(R2)) << (8 * e);
        }
      }
      cw[j * ld] = acc;
    }
  }
  hi = R2;
}
// The same for row r of the published stage's 32-row block q (bm[c] = mask of key j0 + c, c = 0..128).
template <typename MaskT, bool kBelow, bool kAbove>
__device__ __forceinline__ void diag_scan(const MaskStage<MaskT>& ms, int q, int r, int s, uint32_t* cw, int ld,
                                          MaskT& lo, MaskT& hi) {
  diag_scan_block<MaskT, kBelow, kAbove>(ms.bm + 32 * q, r - 32 * q, s, cw, ld, lo, hi);
}

// The masks of a key tile as the mask warp publishes them: xv[e] is the mask of key 4 lane + e,
// x128 (lane 0) the mask of the key just past the tile. Writes bm, the in-tile prefix and suffix
// ORs and, on the diagonal tile, the range ORs against each 32-row block: below the block when
// kBelow (dq[q][c] = OR bm[c + 1 .. 32q], c < 32q), above it when kAbove
// (dq[q][c] = OR bm[32q + 32 .. c], c >= 32q + 32).
template <typename MaskT, bool kBelow, bool kAbove>
__device__ __forceinline__ void publish_masks(MaskStage<MaskT>& ms, const MaskT (&xv)[4], MaskT x128, bool diag,
                                              int lane) {
  MaskT pre_v[4], suf_v[4];
  {  // pre[c] = OR bm[1..c]
    const MaskT p0 = lane == 0 ? static_cast<MaskT>(0) : xv[0];
    const MaskT p1 = p0 | xv[1], p2 = p1 | xv[2], p3 = p2 | xv[3];
    MaskT before = __shfl_up_sync(0xffffffffu, warp_prefix_or<MaskT>(p3, lane), 1);
    if (lane == 0) before = 0;
    pre_v[0] = before | p0;
    pre_v[1] = before | p1;
    pre_v[2] = before | p2;
    pre_v[3] = before | p3;
  }
  {  // suf[c] = OR bm[c+1..127]
    const MaskT u2 = xv[3], u1 = u2 | xv[2], u0 = u1 | xv[1];
    MaskT after = __shfl_down_sync(0xffffffffu, warp_suffix_or<MaskT>(u0 | xv[0], lane), 1);
    if (lane == 31) after = 0;
    suf_v[0] = after | u0;
    suf_v[1] = after | u1;
    suf_v[2] = after | u2;
    suf_v[3] = after;
  }
  if (diag) {
    if (kBelow) {
#pragma unroll 1
      for (int q = 1; q < 4; ++q) {  // dq[q][c] = OR bm[c + 1 .. 32q], c < 32q
        MaskT v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) v[e] = (4 * lane + e <= 32 * q) ? xv[e] : static_cast<MaskT>(0);
        const MaskT u2 = v[3], u1 = u2 | v[2], u0 = u1 | v[1];
        MaskT after = __shfl_down_sync(0xffffffffu, warp_suffix_or<MaskT>(u0 | v[0], lane), 1);
        if (lane == 31) after = 0;
        if (4 * lane < 32 * q) {
          ms.dq[q][4 * lane] = after | u0;
          ms.dq[q][4 * lane + 1] = after | u1;
          ms.dq[q][4 * lane + 2] = after | u2;
          ms.dq[q][4 * lane + 3] = after;
        }
      }
    }
    if (kAbove) {
#pragma unroll 1
      for (int q = 0; q < 3; ++q) {  // dq[q][c] = OR bm[32q + 32 .. c], c >= 32q + 32
        MaskT v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) v[e] = (4 * lane + e >= 32 * q + 32) ? xv[e] : static_cast<MaskT>(0);
        const MaskT p0 = v[0], p1 = p0 | v[1], p2 = p1 | v[2], p3 = p2 | v[3];
        MaskT before = __shfl_up_sync(0xffffffffu, warp_prefix_or<MaskT>(p3, lane), 1);
        if (lane == 0) before = 0;
        if (4 * lane >= 32 * q + 32) {
          ms.dq[q][4 * lane] = before | p0;
          ms.dq[q][4 * lane + 1] = before | p1;
          ms.dq[q][4 * lane + 2] = before | p2;
          ms.dq[q][4 * lane + 3] = before | p3;
        }
      }
    }
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int c = 4 * lane + e;
    ms.bm[c] = xv[e];
    ms.pre[c] = pre_v[e];
    ms.suf[c] = suf_v[e];
  }
  if (lane == 0) ms.bm[kTile] = x128;
}

// ---------------------------------------------------------------- host side

inline PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  // looked up once per process (thread-safe static initialisation)
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    return nullptr;
  }();
  return fn;
}

// [planes][rows][128] bf16, boxes of 64 x 128 x 1 with 128-byte swizzle; rows past `rows` read as zero.
inline int make_map(CUtensorMap* map, const void* base, int rows, int planes) {
  auto enc = get_encode_fn();
  if (!enc) return fail(PLSH_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(planes)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(kD) * 2, static_cast<cuuint64_t>(rows) * kD * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(kTile), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PLSH_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return PLSH_OK;
}

// [planes][rows][128] bf16, boxes of 32 x 32 x 1 without swizzle (an output tile of 32 rows and
// 32 columns staged row-major, 64 bytes a row); elements past `rows` are not written.
inline int make_map_o(CUtensorMap* map, void* base, int rows, int planes) {
  auto enc = get_encode_fn();
  if (!enc) return fail(PLSH_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(planes)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(kD) * 2, static_cast<cuuint64_t>(rows) * kD * 2};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PLSH_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return PLSH_OK;
}

inline int sm_count() {
  static const int count = []() {
    int dev = 0, c = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || c <= 0) return 148;
    return c;
  }();
  return count;
}

}  // namespace tiles
}  // namespace plsh
