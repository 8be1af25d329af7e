// K3: fused banded Positional-LSH attention on the sm_100a tensor cores.
//
// For every (batch, query head, 128-row query tile) it computes
//   O_i = sum_j c_ij e^{S_ij} V_j / sum_j c_ij e^{S_ij},   S = Q K^T / sqrt(d),
// where c_ij counts the hashes that put i and j in one bin (Positional LSH
// technical summary, Methodology 2: M~ = (1/s) sum_k M(h_k); the 1/s cancels
// in O and is restored in row_sum). Blocks are contiguous (Methodology 1,
// structure), so c_ij = s - popcount(OR of the boundary masks over
// (min(i,j), max(i,j)]); only keys in the tile's window [lo, hi] can have
// c_ij > 0 (Methodology 2, block-size control), and only those key tiles are
// visited (Methodology 3: attention restricted to short random blocks).
//
// Persistent CTAs (one per SM) walk a static list of work items, heads with
// the widest windows first. Warp roles (352 threads):
//   warps 0-7    softmax: warps 0-3 own key columns 0-63 and warps 4-7 key
//                columns 64-127 of query row (warp % 4) * 32 + lane
//   warp 8       TMA producer: Q per item (2 buffers), K and V per key tile (2-stage rings)
//   warp 9       TMEM owner and single-thread tcgen05.mma issuer
//   warp 10      mask warp: the key tile's boundary masks and their in-tile
//                prefix / suffix ORs; for 32-bit masks also the tile's table
//                of log2 weights (below)
// Per key tile g (counted across items): S_g = Q K_g^T (SS MMA into TMEM,
// double-buffered); the softmax warps turn S_g into bf16 P_g written over
// the first 64 columns of S_g; then O += P_g V_g (TS MMA, P from TMEM, fp32 O
// in TMEM, one O buffer per item parity). S_{g+1} is issued before PV_g so
// the tensor core works while the softmax runs. An item's epilogue (O / l)
// runs after the next item's first tile, when its last PV has long finished.
//
// Weights. The logit is x = S * log2(e)/sqrt(d) + log2(c_ij) (-inf where
// c_ij = 0), so P = 2^(x - m) = c_ij 2^(S log2(e)/sqrt(d) - m). Key tiles are
// visited diagonal first, then downward, then upward. Below the diagonal
// the OR over (j, i] splits into SUF[c] (inside the key tile) and the row's
// carry Y = OR over [j0 + 128, i]; above it into the row's carry
// Z = OR over (i, j0] and PRE[c]. The carries of a query tile's rows form a
// chain of nested sets, so a tile has few distinct carries; the mask warp
// writes one row of log2 weights per distinct carry (indexed by its
// popcount) and each softmax thread reads its row: one shared load and one
// FMA per key. On the diagonal tile (and for 64-bit masks everywhere) a row
// scans its keys away from itself with a running OR instead, recomputing
// log2(s - popcount) only where some hash opens a block.
// The reference maximum m moves only when a tile's maximum exceeds it by
// more than 8 (then O and the row sum are rescaled), so every P <= 256.
//
// Every barrier wait is bounded in time (PLSH_DEVERR_TIMEOUT); on timeout all
// roles leave their loops, in-flight copies and MMAs are drained and TMEM is
// freed before the CTA returns.
#include <cmath>
#include <type_traits>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "plsh_internal.h"
#include "plsh_sm100.cuh"

namespace plsh {
namespace {

using namespace sm100;

constexpr int kTile = PLSH_TILE;
constexpr int kD = 128;
constexpr int kThreads = 352;         // 11 warps
constexpr int kSoftmaxWarps = 8;      // warps 0-7
constexpr int kWarpTma = 8, kWarpMma = 9, kWarpMask = 10;
constexpr int kHalf = 64;             // key columns per softmax thread
constexpr int kStages = 2;
constexpr int kChunkBytes = kTile * 64 * 2;         // 128 rows x 64 bf16 = 16 KB (one SW128 box)
constexpr int kTileBytes = 2 * kChunkBytes;         // 128 x 128 bf16 = 32 KB
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;      // S buffers at columns 0 and 128 (P overwrites their first 64 columns)
constexpr uint32_t kColO = 256;    // O buffers at columns 256 and 384
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr int kMaxSortedHeads = 256;
constexpr int kTblRows = 33;       // table rows: popcounts 0..32
constexpr int kTblStride = 132;    // floats per table row (spreads rows over banks)

template <typename MaskT>
struct alignas(16) MaskStage {
  MaskT bm[kTile + 4];   // bm[c]   = boundary mask of key j0 + c, c = 0..128 (all ones outside [0, n))
  MaskT bmn[kTile];      // bmn[c]  = bm[c + 1]
  MaskT pre[kTile];      // pre[c]  = OR bm[1 .. c]        (pre[0] = 0)
  MaskT suf[kTile];      // suf[c]  = OR bm[c + 1 .. 127]  (suf[127] = 0)
  MaskT preh[kHalf];     // preh[q] = OR bm[64 .. 64 + q]
  MaskT sufl[kHalf];     // sufl[c] = OR bm[c + 1 .. 63]   (sufl[63] = 0)
};

// Log2-weight table of one key tile (32-bit masks only).
struct alignas(16) WeightTable {
  float w[kTblRows][kTblStride];
};
struct NoTable {};

template <typename MaskT>
constexpr bool kUseTable = sizeof(MaskT) == 4;

template <typename MaskT>
struct __align__(1024) TcSmem {
  uint8_t q[2][kTileBytes];
  uint8_t k[kStages][kTileBytes];
  uint8_t v[kStages][kTileBytes];
  MaskStage<MaskT> m[kStages];
  typename std::conditional<kUseTable<MaskT>, WeightTable, NoTable>::type tbl;
  MaskT pfxq[kTile];                   // mask warp: OR over [i0, i0 + r] of the current item
  MaskT sfxq[kTile];                   // mask warp: OR over (i0 + r, i0 + 127]
  MaskT ykey[kTblRows + 3];            // mask warp: carry set of each popcount present
  float pmax[2][2][kTile];             // [tile parity][half][row] partial row maxima
  float psum[2][2][kTile];             // [item parity][half][row] partial row sums
  float lg[PLSH_MAX_S + 4];            // lg[w] = log2(w), lg[0] = -inf
  int16_t order[kMaxSortedHeads];      // heads by decreasing window width
  int32_t width[kMaxSortedHeads];
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[kStages], k_empty[kStages];
  uint64_t v_full[kStages], v_empty[kStages];
  uint64_t m_full[kStages], m_empty[kStages];
  uint64_t t_full, t_empty;            // weight table handoff
  uint64_t s_full[2], p_full[2], pv_done[2];
  uint64_t xmax[2], xsum[2];           // softmax half exchange: row maxima per tile, row sums per item
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

struct Params {
  int B, H, H_kv, n, s, causal, T, items;
  const int32_t* spans;
};

// One key tile of one work item, in the order every role walks them. The
// window of the next item is fetched one item ahead.
struct TileIter {
  const Params* p;
  const int16_t* order;
  int x;        // work item index
  int k;        // work items started by this CTA so far (Q and O buffer = k & 1)
  int it;       // key tile within the item
  int total;    // key tiles of the item
  int n_below;
  int b, h, t, i0;
  int g;        // key tile counted across this CTA's items
  int u;        // table tiles (below / above the diagonal) counted across this CTA's items
  bool valid;
  bool bad_window;  // the window read for this item was out of range (and was clamped)
  int nx_lo, nx_hi; // window of item x + gridDim.x

  __device__ __forceinline__ int head_of(int xx) const {
    const int hr = xx / (p->B * p->T);
    return (p->H <= kMaxSortedHeads) ? static_cast<int>(order[hr]) : hr;
  }
  __device__ __forceinline__ void fetch(int xx, int& lo, int& hi) const {
    if (xx < p->items) {
      const int hh = head_of(xx);
      const int tt = (xx - (xx / (p->B * p->T)) * (p->B * p->T)) % p->T;
      lo = p->spans[(static_cast<size_t>(hh) * p->T + tt) * 2];
      hi = p->spans[(static_cast<size_t>(hh) * p->T + tt) * 2 + 1];
    }
  }
  __device__ __forceinline__ void load_item(int lo, int hi) {
    valid = x < p->items;
    if (!valid) return;
    const int BT = p->B * p->T;
    const int rem = x - (x / BT) * BT;
    h = head_of(x);
    b = rem / p->T;
    t = rem - b * p->T;
    i0 = t * kTile;
    fetch(x + gridDim.x, nx_lo, nx_hi);
    const int last_row = min(p->n, i0 + kTile) - 1;
    bad_window = lo < 0 || lo > i0 || hi >= p->n || hi < last_row;
    lo = max(0, min(lo, i0));
    hi = min(p->n - 1, max(hi, last_row));
    n_below = (i0 - lo + kTile - 1) / kTile;
    total = 1 + n_below + (p->causal ? 0 : (hi - i0) / kTile);
    it = 0;
  }
  __device__ __forceinline__ void start(const Params* pp, const int16_t* ord) {
    p = pp;
    order = ord;
    x = blockIdx.x;
    k = 0;
    g = 0;
    u = 0;
    nx_lo = nx_hi = 0;
    int lo = 0, hi = 0;
    fetch(x, lo, hi);
    load_item(lo, hi);
  }
  __device__ __forceinline__ void next() {
    ++g;
    if (it > 0) ++u;
    if (++it >= total) {
      x += gridDim.x;
      ++k;
      load_item(nx_lo, nx_hi);
    }
  }
  __device__ __forceinline__ int kind() const { return it == 0 ? 0 : (it <= n_below ? 1 : 2); }
  __device__ __forceinline__ int j0() const {
    const int kd = kind();
    return kd == 0 ? i0 : (kd == 1 ? i0 - kTile * it : i0 + kTile * (it - n_below));
  }
  __device__ __forceinline__ bool first() const { return it == 0; }
  __device__ __forceinline__ bool last() const { return it == total - 1; }
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
__device__ __forceinline__ MaskT warp_prefix_or(MaskT v, int lane) {   // inclusive over lanes 0..lane
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const MaskT y = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v |= y;
  }
  return v;
}

template <typename MaskT>
__device__ __forceinline__ MaskT warp_suffix_or(MaskT v, int lane) {   // inclusive over lanes lane..31
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const MaskT y = __shfl_down_sync(0xffffffffu, v, o);
    if (lane + o < 32) v |= y;
  }
  return v;
}

__device__ __forceinline__ int lg_index(int s, int popcount) { return max(0, s - popcount); }

// x[cc] <- x[cc] * sc + table row, for the 64 columns of this half (loads issued four at a time
// so that at most 16 table values are live next to the 64 logits).
__device__ __forceinline__ void logits_from_table(float (&x)[kHalf], const float* row, float sc) {
#pragma unroll
  for (int g4 = 0; g4 < kHalf / 4; ++g4) {
    if ((g4 & 3) == 0) asm volatile("" ::: "memory");
    const float4 t4 = reinterpret_cast<const float4*>(row)[g4];
    x[4 * g4 + 0] = fmaf(x[4 * g4 + 0], sc, t4.x);
    x[4 * g4 + 1] = fmaf(x[4 * g4 + 1], sc, t4.y);
    x[4 * g4 + 2] = fmaf(x[4 * g4 + 2], sc, t4.z);
    x[4 * g4 + 3] = fmaf(x[4 * g4 + 3], sc, t4.w);
  }
}

// Scans for one row's half of a key tile: x[cc] <- S[c] * sc + log2(c_ij) for c = 64*half + cc.
// kind 0: diagonal tile (row r is column r); kind 1: below the diagonal; kind 2: above.
// R is the OR over the gap between the row and the current key, carried in from Y / Z.
template <typename MaskT, bool kCausal>
__device__ __forceinline__ void logits_by_scan(float (&x)[kHalf], const MaskStage<MaskT>& ms, const float* lg,
                                               int kind, int r, int half, int s, float sc, MaskT Y, MaskT Z) {
  const int c0 = kHalf * half;
  if (kind == 1) {
    // R(127) = Y, R(63) = Y | OR bm[64..127], R(c) = R(c + 1) | bm[c + 1]
    MaskT R = half ? Y : static_cast<MaskT>(Y | ms.suf[kHalf - 1]);
    float lw = lg[lg_index(s, popc_m(R))];
#pragma unroll
    for (int g4 = kHalf / 4 - 1; g4 >= 0; --g4) {
      MaskT bb[4];
      load4(&ms.bmn[c0 + 4 * g4], bb);
      if (g4 == kHalf / 4 - 1 && half) bb[3] = 0;
      if ((bb[0] | bb[1] | bb[2] | bb[3]) != 0) {
#pragma unroll
        for (int e = 3; e >= 0; --e) {
          R |= bb[e];
          lw = lg[lg_index(s, popc_m(R))];
          x[4 * g4 + e] = fmaf(x[4 * g4 + e], sc, lw);
        }
      } else {
#pragma unroll
        for (int e = 3; e >= 0; --e) x[4 * g4 + e] = fmaf(x[4 * g4 + e], sc, lw);
      }
    }
  } else if (!kCausal && kind == 2) {
    // R(0) = Z (holds bm[0]), R(63) = Z | OR bm[1..63], R(c) = R(c - 1) | bm[c]
    MaskT R = half ? static_cast<MaskT>(Z | ms.pre[kHalf - 1]) : Z;
    float lw = lg[lg_index(s, popc_m(R))];
#pragma unroll
    for (int g4 = 0; g4 < kHalf / 4; ++g4) {
      MaskT bb[4];
      load4(&ms.bm[c0 + 4 * g4], bb);
      if (g4 == 0 && !half) bb[0] = 0;
      if ((bb[0] | bb[1] | bb[2] | bb[3]) != 0) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          R |= bb[e];
          lw = lg[lg_index(s, popc_m(R))];
          x[4 * g4 + e] = fmaf(x[4 * g4 + e], sc, lw);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) x[4 * g4 + e] = fmaf(x[4 * g4 + e], sc, lw);
      }
    }
  } else {
    // columns c <= r: R(c) = OR bm[c+1 .. r]; in the low half a row r >= 64 starts from OR bm[64..r]
    MaskT R = (!half && r >= kHalf) ? ms.preh[r - kHalf] : static_cast<MaskT>(0);
    float lw = lg[lg_index(s, popc_m(R))];
#pragma unroll
    for (int g4 = kHalf / 4 - 1; g4 >= 0; --g4) {
      MaskT bb[4];
      load4(&ms.bmn[c0 + 4 * g4], bb);
      if ((bb[0] | bb[1] | bb[2] | bb[3]) != 0) {
#pragma unroll
        for (int e = 3; e >= 0; --e) {
          const int cc = 4 * g4 + e, c = c0 + cc;
          if (c < r) R |= bb[e];
          lw = lg[lg_index(s, popc_m(R))];
          x[cc] = (c <= r) ? fmaf(x[cc], sc, lw) : (kCausal ? -INFINITY : x[cc]);
        }
      } else {
#pragma unroll
        for (int e = 3; e >= 0; --e) {
          const int cc = 4 * g4 + e, c = c0 + cc;
          x[cc] = (c <= r) ? fmaf(x[cc], sc, lw) : (kCausal ? -INFINITY : x[cc]);
        }
      }
    }
    if (!kCausal) {
      // columns c > r: R(c) = OR bm[r+1 .. c]; in the high half a row r < 64 starts from OR bm[r+1..63]
      MaskT R2 = (half && r < kHalf) ? ms.sufl[r] : static_cast<MaskT>(0);
      float lw2 = lg[lg_index(s, popc_m(R2))];
#pragma unroll
      for (int g4 = 0; g4 < kHalf / 4; ++g4) {
        MaskT bb[4];
        load4(&ms.bm[c0 + 4 * g4], bb);
        if ((bb[0] | bb[1] | bb[2] | bb[3]) != 0) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int cc = 4 * g4 + e, c = c0 + cc;
            if (c > r) R2 |= bb[e];
            lw2 = lg[lg_index(s, popc_m(R2))];
            if (c > r) x[cc] = fmaf(x[cc], sc, lw2);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int cc = 4 * g4 + e, c = c0 + cc;
            if (c > r) x[cc] = fmaf(x[cc], sc, lw2);
          }
        }
      }
    }
  }
}

template <typename MaskT, bool kCausal>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
               const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ Params prm,
               const double* __restrict__ sigma,
               const double* __restrict__ table, const MaskT* __restrict__ bmask, __nv_bfloat16* __restrict__ O,
               float* __restrict__ row_sum, uint32_t* __restrict__ err) {
  constexpr bool kTable = kUseTable<MaskT>;
  extern __shared__ uint8_t smem_raw[];
  auto& sm = *reinterpret_cast<TcSmem<MaskT>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  volatile int* abort_flag = &sm.abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = prm.n, s = prm.s, H = prm.H;
  const MaskT FULL = (s >= static_cast<int>(8 * sizeof(MaskT))) ? static_cast<MaskT>(~static_cast<MaskT>(0))
                                                              : static_cast<MaskT>((static_cast<MaskT>(1) << s) - 1);

  // table and sigma checks, one head per thread of CTA 0
  if (blockIdx.x == 0) {
    uint32_t flags = 0;
    for (int h = threadIdx.x; h < H; h += kThreads) {
      if (sigma && !(isfinite(sigma[h]) && sigma[h] > 0.0)) flags |= PLSH_DEVERR_SIGMA;
      if (table)
        for (int k = 0; k < s; ++k) {
          const double dl = table[(static_cast<size_t>(h) * s + k) * 2];
          if (!(isfinite(dl) && dl > 0.0)) flags |= PLSH_DEVERR_TABLE;
        }
    }
    if (flags) atomicOr(err, flags);
  }
  // heads by decreasing window width of their middle query tile, ties by head index (the same order in every CTA)
  if (H <= kMaxSortedHeads) {
    const int tm = prm.T / 2;
    for (int h = threadIdx.x; h < H; h += kThreads)
      sm.width[h] = prm.spans[(static_cast<size_t>(h) * prm.T + tm) * 2 + 1] -
                    prm.spans[(static_cast<size_t>(h) * prm.T + tm) * 2];
  }
  if (threadIdx.x < PLSH_MAX_S + 4)
    sm.lg[threadIdx.x] = threadIdx.x == 0 ? -INFINITY : log2f(static_cast<float>(threadIdx.x));
  __syncthreads();
  if (H <= kMaxSortedHeads) {
    for (int h = threadIdx.x; h < H; h += kThreads) {
      const int wh = sm.width[h];
      int rank = 0;
      for (int o = 0; o < H; ++o) {
        const int wo = sm.width[o];
        rank += (wo > wh) || (wo == wh && o < h);
      }
      sm.order[rank] = static_cast<int16_t>(h);
    }
  }
  if (threadIdx.x == 0) {
    sm.abort_flag = 0;
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.q_full[i], 1);
      mbar_init(&sm.q_empty[i], 1);
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.p_full[i], kSoftmaxWarps);
      mbar_init(&sm.pv_done[i], 1);
      mbar_init(&sm.xmax[i], kSoftmaxWarps);
      mbar_init(&sm.xsum[i], kSoftmaxWarps);
    }
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sm.k_full[i], 1);
      mbar_init(&sm.k_empty[i], 1);
      mbar_init(&sm.v_full[i], 1);
      mbar_init(&sm.v_empty[i], 1);
      mbar_init(&sm.m_full[i], 1);
      mbar_init(&sm.m_empty[i], kSoftmaxWarps);
    }
    mbar_init(&sm.t_full, 1);
    mbar_init(&sm.t_empty, kSoftmaxWarps);
    mbar_init(&sm.drain, 1);
    fence_mbarrier_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == kWarpTma) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmap_q);
      tma_prefetch_desc(&tmap_k);
      tma_prefetch_desc(&tmap_v);
      TileIter ti;
      ti.start(&prm, sm.order);
      int issued_g = 0, issued_k = 0;
      bool ok = true;
      while (ok && ti.valid) {
        const int zkv = ti.b * prm.H_kv + ti.h / (H / prm.H_kv);
        if (ti.first()) {
          const int qb = ti.k & 1;
          if (ti.k >= 2 && !mbar_wait(&sm.q_empty[qb], ((ti.k >> 1) & 1) ^ 1, abort_flag, err)) break;
          mbar_arrive_expect_tx(&sm.q_full[qb], kTileBytes);
          tma_load_3d(sm.q[qb], &tmap_q, 0, ti.i0, ti.b * H + ti.h, &sm.q_full[qb]);
          tma_load_3d(sm.q[qb] + kChunkBytes, &tmap_q, 64, ti.i0, ti.b * H + ti.h, &sm.q_full[qb]);
          issued_k = ti.k + 1;
        }
        const int st = ti.g % kStages;
        const uint32_t ph = static_cast<uint32_t>(ti.g / kStages) & 1u;
        const int j0 = ti.j0();
        if (ti.g >= kStages && !mbar_wait(&sm.k_empty[st], ph ^ 1u, abort_flag, err)) break;
        mbar_arrive_expect_tx(&sm.k_full[st], kTileBytes);
        tma_load_3d(sm.k[st], &tmap_k, 0, j0, zkv, &sm.k_full[st]);
        tma_load_3d(sm.k[st] + kChunkBytes, &tmap_k, 64, j0, zkv, &sm.k_full[st]);
        ok = !(ti.g >= kStages && !mbar_wait(&sm.v_empty[st], ph ^ 1u, abort_flag, err));
        if (ok) {
          mbar_arrive_expect_tx(&sm.v_full[st], kTileBytes);
          tma_load_3d(sm.v[st], &tmap_v, 0, j0, zkv, &sm.v_full[st]);
          tma_load_3d(sm.v[st] + kChunkBytes, &tmap_v, 64, j0, zkv, &sm.v_full[st]);
        }
        issued_g = ti.g + 1;
        ti.next();
      }
      if (*abort_flag) {
        // let every copy already issued land before the CTA can exit
        for (int kk = (issued_k > 2 ? issued_k - 2 : 0); kk < issued_k; ++kk)
          mbar_wait_drain(&sm.q_full[kk & 1], (kk >> 1) & 1, 100000000ull);
        for (int gg = (issued_g > kStages ? issued_g - kStages : 0); gg < issued_g; ++gg) {
          const int st = gg % kStages;
          const uint32_t ph = static_cast<uint32_t>(gg / kStages) & 1u;
          mbar_wait_drain(&sm.k_full[st], ph, 100000000ull);
          mbar_wait_drain(&sm.v_full[st], ph, 100000000ull);
        }
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 128, 1);
      auto issue_s = [&](const TileIter& ti) -> bool {
        const int qb = ti.k & 1;
        if (ti.first() && !mbar_wait(&sm.q_full[qb], (ti.k >> 1) & 1, abort_flag, err)) return false;
        const int st = ti.g % kStages;
        if (!mbar_wait(&sm.k_full[st], static_cast<uint32_t>(ti.g / kStages) & 1u, abort_flag, err)) return false;
        tc_fence_after();
        const uint32_t q_addr = smem_u32(sm.q[qb]);
        const uint32_t k_addr = smem_u32(sm.k[st]);
        const uint32_t d_tmem = tmem + kColS + 128u * static_cast<uint32_t>(ti.g & 1);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = static_cast<uint32_t>((kk >> 2) * kChunkBytes + (kk & 3) * 32);
          mma_ss(d_tmem, smem_desc_sw128(q_addr + off, 16, 1024), smem_desc_sw128(k_addr + off, 16, 1024),
                 idesc_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit(&sm.s_full[ti.g & 1]);
        mma_commit(&sm.k_empty[st]);
        if (ti.last()) mma_commit(&sm.q_empty[qb]);
        return true;
      };
      auto issue_pv = [&](const TileIter& ti) -> bool {
        const int st = ti.g % kStages;
        if (!mbar_wait(&sm.p_full[ti.g & 1], static_cast<uint32_t>(ti.g >> 1) & 1u, abort_flag, err)) return false;
        if (!mbar_wait(&sm.v_full[st], static_cast<uint32_t>(ti.g / kStages) & 1u, abort_flag, err)) return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(sm.v[st]);
        const uint32_t p_tmem = tmem + kColS + 128u * static_cast<uint32_t>(ti.g & 1);
        const uint32_t o_tmem = tmem + kColO + 128u * static_cast<uint32_t>(ti.k & 1);
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk) {
          // 16 keys = two 8-row groups of the MN-major V tile; the two d halves sit kChunkBytes apart
          mma_ts(o_tmem, p_tmem + 8u * kk, smem_desc_sw128(v_addr + kk * 2048, kChunkBytes, 1024), idesc_pv,
                 (ti.it > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&sm.pv_done[ti.g & 1]);
        mma_commit(&sm.v_empty[st]);
        return true;
      };
      // `nxt` runs one tile ahead of `cur`: S of the next tile is issued before PV of the current one
      TileIter cur, nxt;
      cur.start(&prm, sm.order);
      nxt.start(&prm, sm.order);
      bool ok = !cur.valid || issue_s(cur);
      if (nxt.valid) nxt.next();
      while (ok && cur.valid) {
        if (nxt.valid) ok = issue_s(nxt);
        if (ok) ok = issue_pv(cur);
        cur.next();
        if (nxt.valid) nxt.next();
      }
      // every MMA issued so far completes before `drain` arrives
      mma_commit(&sm.drain);
      mbar_wait_drain(&sm.drain, 0, 100000000ull);
    }
  } else if (warp == kWarpMask) {
    // ------------------------------------------------------------ mask warp
    TileIter ti;
    ti.start(&prm, sm.order);
    MaskT mid_b = 0;   // below the diagonal: OR over [j0 + 128, i0)
    MaskT mid_a = 0;   // above the diagonal: OR over [i0 + 128, j0]
    while (ti.valid) {
      const int st = ti.g % kStages;
      if (ti.g >= kStages &&
          !mbar_wait(&sm.m_empty[st], (static_cast<uint32_t>(ti.g / kStages) & 1u) ^ 1u, abort_flag, err))
        break;
      const MaskT* bm_h = bmask + static_cast<size_t>(ti.h) * n;
      MaskStage<MaskT>& ms = sm.m[st];
      const int j0 = ti.j0();
      const int kind = ti.kind();
      MaskT xv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = 4 * lane + e, j = j0 + c;
        xv[e] = (j >= 0 && j < n) ? bm_h[j] : FULL;
        ms.bm[c] = xv[e];
        if (c >= 1) ms.bmn[c - 1] = xv[e];
      }
      if (lane == 0) {
        const int j = j0 + kTile;
        const MaskT v = (j >= 0 && j < n) ? bm_h[j] : FULL;
        ms.bm[kTile] = v;
        ms.bmn[kTile - 1] = v;
      }
      MaskT pre_v[4], suf_v[4];
      {  // pre[c] = OR bm[1..c]
        const MaskT p0 = lane == 0 ? static_cast<MaskT>(0) : xv[0];
        const MaskT p1 = p0 | xv[1], p2 = p1 | xv[2], p3 = p2 | xv[3];
        MaskT before = __shfl_up_sync(0xffffffffu, warp_prefix_or<MaskT>(p3, lane), 1);
        if (lane == 0) before = 0;
        pre_v[0] = before | p0; pre_v[1] = before | p1; pre_v[2] = before | p2; pre_v[3] = before | p3;
      }
      {  // suf[c] = OR bm[c+1..127]
        const MaskT u2 = xv[3], u1 = u2 | xv[2], u0 = u1 | xv[1];
        MaskT after = __shfl_down_sync(0xffffffffu, warp_suffix_or<MaskT>(u0 | xv[0], lane), 1);
        if (lane == 31) after = 0;
        suf_v[0] = after | u0; suf_v[1] = after | u1; suf_v[2] = after | u2; suf_v[3] = after;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        ms.pre[4 * lane + e] = pre_v[e];
        ms.suf[4 * lane + e] = suf_v[e];
      }
      {  // preh[q] = OR bm[64..64+q] (lanes 16..31 hold columns 64..127)
        const bool hiL = lane >= 16;
        const MaskT h0 = xv[0], h1 = h0 | xv[1], h2 = h1 | xv[2], h3 = h2 | xv[3];
        MaskT before = __shfl_up_sync(0xffffffffu, warp_prefix_or<MaskT>(hiL ? h3 : static_cast<MaskT>(0), lane), 1);
        if (lane <= 16) before = 0;
        if (hiL) {
          const int q = 4 * (lane - 16);
          ms.preh[q + 0] = before | h0;
          ms.preh[q + 1] = before | h1;
          ms.preh[q + 2] = before | h2;
          ms.preh[q + 3] = before | h3;
        }
      }
      {  // sufl[c] = OR bm[c+1..63] (lanes 0..15 hold columns 0..63)
        const bool loL = lane < 16;
        const MaskT u2 = xv[3], u1 = u2 | xv[2], u0 = u1 | xv[1];
        MaskT after = __shfl_down_sync(0xffffffffu, warp_suffix_or<MaskT>(loL ? static_cast<MaskT>(u0 | xv[0])
                                                                              : static_cast<MaskT>(0), lane), 1);
        if (lane >= 15) after = 0;
        if (loL) {
          ms.sufl[4 * lane + 0] = after | u0;
          ms.sufl[4 * lane + 1] = after | u1;
          ms.sufl[4 * lane + 2] = after | u2;
          ms.sufl[4 * lane + 3] = after;
        }
      }
      if constexpr (kTable) {
        if (kind == 0) {
          // the query tile's own prefix / suffix ORs, for this item's table tiles
          const MaskT bm0 = __shfl_sync(0xffffffffu, xv[0], 0);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            sm.pfxq[4 * lane + e] = static_cast<MaskT>(bm0 | pre_v[e]);
            sm.sfxq[4 * lane + e] = suf_v[e];
          }
          mid_b = 0;
          mid_a = 0;
        } else {
          // the distinct carries of the tile's rows, then one table row per distinct carry
          const MaskT bm0 = __shfl_sync(0xffffffffu, xv[0], 0);
          if (kind == 2) mid_a |= bm0;
          const MaskT mid = kind == 1 ? mid_b : mid_a;
          __syncwarp();
          uint32_t pres_lo = 0, pres_hi = 0;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int r = lane + 32 * e;
            const MaskT cy = static_cast<MaskT>(mid | (kind == 1 ? sm.pfxq[r] : sm.sfxq[r]));
            const int key = popc_m(cy);
            if (key < 32) pres_lo |= 1u << key; else pres_hi |= 1u << (key - 32);
          }
          pres_lo = __reduce_or_sync(0xffffffffu, pres_lo);
          pres_hi = __reduce_or_sync(0xffffffffu, pres_hi);
          bool ok = true;
          if (ti.u >= 1) ok = mbar_wait(&sm.t_empty, static_cast<uint32_t>((ti.u - 1) & 1), abort_flag, err);
          if (!__all_sync(0xffffffffu, ok)) break;
          // rows with the same popcount hold the same carry (the carries of a tile are nested)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int r = lane + 32 * e;
            const MaskT cy = static_cast<MaskT>(mid | (kind == 1 ? sm.pfxq[r] : sm.sfxq[r]));
            sm.ykey[popc_m(cy)] = cy;
          }
          __syncwarp();
          for (int key = 0; key < kTblRows; ++key) {
            const bool present = key < 32 ? ((pres_lo >> key) & 1u) : ((pres_hi >> (key - 32)) & 1u);
            if (!present) continue;
            const MaskT cy = sm.ykey[key];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c = lane + 32 * e;
              const MaskT Rc = kind == 1 ? static_cast<MaskT>(ms.suf[c] | cy) : static_cast<MaskT>(cy | ms.pre[c]);
              sm.tbl.w[key][c] = sm.lg[lg_index(s, popc_m(Rc))];
            }
          }
          if (kind == 1) mid_b |= static_cast<MaskT>(bm0 | __shfl_sync(0xffffffffu, suf_v[0], 0));
          else mid_a |= __shfl_sync(0xffffffffu, pre_v[3], 31);
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.t_full);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.m_full[st]);
      ti.next();
    }
  } else if (warp < kSoftmaxWarps) {
    // ------------------------------------------------------------ softmax
    const int half = warp >= 4 ? 1 : 0;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;   // row within the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t col_off = static_cast<uint32_t>(kHalf * half);
    const float sc = 1.4426950408889634f / sqrtf(static_cast<float>(kD));
    float m2 = -INFINITY, l = 0.0f;
    MaskT Y = 0, Z = 0;
    // epilogue still owed for the previous item
    // (always the item just before the current tile's item: index x - gridDim.x, tile g - 1, count k - 1)
    bool pend = false;
    float pend_l = 0.0f, pend_m = 0.0f;
    auto epilogue = [&](int pend_x, int pend_g, int pend_k) -> bool {
      const int BT = prm.B * prm.T;
      const int pend_h = (H <= kMaxSortedHeads) ? static_cast<int>(sm.order[pend_x / BT]) : pend_x / BT;
      const int rem = pend_x % BT;
      const int pend_b = rem / prm.T;
      const int pend_i0 = (rem % prm.T) * kTile;
      bool okw = mbar_wait(&sm.pv_done[pend_g & 1], static_cast<uint32_t>(pend_g >> 1) & 1u, abort_flag, err);
      okw = __all_sync(0xffffffffu, okw && mbar_wait(&sm.xsum[pend_k & 1], static_cast<uint32_t>(pend_k >> 1) & 1u,
                                                     abort_flag, err));
      if (!okw) return false;
      tc_fence_after();
      const float ltot = pend_l + sm.psum[pend_k & 1][half ^ 1][r];
      const int i = pend_i0 + r;
      const float inv = 1.0f / ltot;
      const uint32_t ob = tmem + lane_off + kColO + 128u * static_cast<uint32_t>(pend_k & 1) + col_off;
      __nv_bfloat16* orow = O + ((static_cast<size_t>(pend_b) * H + pend_h) * n + (i < n ? i : 0)) * kD + col_off;
#pragma unroll 1
      for (int q2 = 0; q2 < 2; ++q2) {
        uint32_t raw[32];
        tmem_ld32(ob + 32u * q2, raw);
        tmem_wait_ld();
        if (i < n) {
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * q2);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            uint32_t pk[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
              pk[u] = pack_bf16x2(__uint_as_float(raw[8 * e + 2 * u]) * inv, __uint_as_float(raw[8 * e + 2 * u + 1]) * inv);
            dst[e] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        }
      }
      tc_fence_before();
      if (i < n) {
        if (half == 0)
          row_sum[(static_cast<size_t>(pend_b) * H + pend_h) * n + i] =
              (log2f(ltot) + pend_m) * 0.6931471805599453f - logf(static_cast<float>(s));
      }
      pend = false;
      return true;
    };
    TileIter ti;
    ti.start(&prm, sm.order);
    bool ok = true;
    while (ti.valid) {
      const int g = ti.g;
      const int st = g % kStages;
      const int kind = ti.kind();
      if (ti.first()) {
        m2 = -INFINITY;
        l = 0.0f;
        if (ti.bad_window && r == 0 && half == 0) atomicOr(err, PLSH_DEVERR_WINDOW);
      }
      ok = mbar_wait(&sm.m_full[st], static_cast<uint32_t>(g / kStages) & 1u, abort_flag, err);
      ok = ok && mbar_wait(&sm.s_full[g & 1], static_cast<uint32_t>(g >> 1) & 1u, abort_flag, err);
      if (kTable && kind != 0) ok = ok && mbar_wait(&sm.t_full, static_cast<uint32_t>(ti.u & 1), abort_flag, err);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      float x[kHalf];
      {
        const uint32_t base = tmem + lane_off + kColS + 128u * static_cast<uint32_t>(g & 1) + col_off;
        uint32_t raw[2][32];
        tmem_ld32(base, raw[0]);
        tmem_ld32(base + 32u, raw[1]);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          x[e] = __uint_as_float(raw[0][e]);
          x[32 + e] = __uint_as_float(raw[1][e]);
        }
      }
      const MaskStage<MaskT>& ms = sm.m[st];
      if (kind == 2) Z |= ms.bm[0];   // now OR over (i, j0]
      if constexpr (kTable) {
        if (kind != 0) {
          const MaskT cy = kind == 1 ? Y : Z;
          logits_from_table(x, &sm.tbl.w[popc_m(cy)][col_off], sc);
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.t_empty);
        } else {
          logits_by_scan<MaskT, kCausal>(x, ms, sm.lg, kind, r, half, s, sc, Y, Z);
        }
      } else {
        logits_by_scan<MaskT, kCausal>(x, ms, sm.lg, kind, r, half, s, sc, Y, Z);
      }
      // carries past this tile
      if (kind == 0) {
        Y = static_cast<MaskT>(ms.bm[0] | ms.pre[r]);       // OR over [i0, i]
        Z = kCausal ? static_cast<MaskT>(0) : ms.suf[r];     // OR over (i, i0 + 127]
      } else if (kind == 1) {
        Y = static_cast<MaskT>(Y | ms.bm[0] | ms.suf[0]);   // OR over [j0, i]
      } else {
        Z = static_cast<MaskT>(Z | ms.pre[kTile - 1]);      // OR over (i, j0 + 127]
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.m_empty[st]);

      // ---- tile maximum (both halves) and reference update
      float mx[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) mx[u] = x[u];
#pragma unroll
      for (int c = 8; c < kHalf; ++c) mx[c & 7] = fmaxf(mx[c & 7], x[c]);
      float mt = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      sm.pmax[g & 1][half][r] = mt;
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.xmax[g & 1]);
      ok = __all_sync(0xffffffffu, mbar_wait(&sm.xmax[g & 1], static_cast<uint32_t>(g >> 1) & 1u, abort_flag, err));
      if (!ok) break;
      mt = fmaxf(mt, sm.pmax[g & 1][half ^ 1][r]);
      float alpha = 1.0f;
      bool need_rescale = false;
      if (mt > m2 + kRescaleThreshold) {
        if (m2 != -INFINITY) {
          alpha = ex2_approx(m2 - mt);
          need_rescale = true;
        }
        m2 = mt;
      }
      const float neg_m = (m2 == -INFINITY) ? 0.0f : -m2;

      // ---- rescale this half of the item's O when some row of the warp moved its reference
      if (__any_sync(0xffffffffu, need_rescale)) {
        ok = __all_sync(0xffffffffu, mbar_wait(&sm.pv_done[(g - 1) & 1], static_cast<uint32_t>((g - 1) >> 1) & 1u,
                                               abort_flag, err));
        if (!ok) break;
        tc_fence_after();
#pragma unroll 1
        for (int q4 = 0; q4 < 4; ++q4) {
          uint32_t raw[16];
          const uint32_t addr = tmem + lane_off + kColO + 128u * static_cast<uint32_t>(ti.k & 1) + col_off + 16u * q4;
          tmem_ld16(addr, raw);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) raw[e] = __float_as_uint(__uint_as_float(raw[e]) * alpha);
          tmem_st16(addr, raw);
        }
        tmem_wait_st();
      }

      // ---- P = 2^(x - m) as bf16 over the first 64 columns of S_g, partial row sum
      const uint32_t p_base = tmem + lane_off + kColS + 128u * static_cast<uint32_t>(g & 1) + col_off / 2;
      float ls[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) ls[u] = 0.0f;
#pragma unroll
      for (int q2 = 0; q2 < 2; ++q2) {
        uint32_t packed[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const float p0 = ex2_approx(x[32 * q2 + e] + neg_m);
          const float p1 = ex2_approx(x[32 * q2 + e + 1] + neg_m);
          ls[e & 7] += p0;
          ls[(e + 1) & 7] += p1;
          packed[e >> 1] = pack_bf16x2(p0, p1);
        }
        tmem_st16(p_base + 16u * q2, packed);
      }
      tmem_wait_st();
      l = l * alpha + (((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7])));
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.p_full[g & 1]);

      // ---- the previous item's epilogue, now that its last PV has had a tile's time to finish
      if (pend && !epilogue(ti.x - static_cast<int>(gridDim.x), g - 1, ti.k - 1)) {
        ok = false;
        break;
      }
      if (ti.last()) {
        sm.psum[ti.k & 1][half][r] = l;
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.xsum[ti.k & 1]);
        pend = true;
        pend_l = l;
        pend_m = m2;
      }
      ti.next();
    }
    // the CTA's last item: ti has moved past it
    if (ok && pend) epilogue(ti.x - static_cast<int>(gridDim.x), ti.g - 1, ti.k - 1);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
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
int make_map(CUtensorMap* map, const void* base, int rows, int planes) {
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

int sm_count() {
  static const int count = []() {
    int dev = 0, c = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || c <= 0) return 148;
    return c;
  }();
  return count;
}

template <typename MaskT, bool kCausal>
int launch_tc_typed(const AttnArgs& a, cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  if (int rc = make_map(&mq, a.Q, a.n, a.B * a.H)) return rc;
  if (int rc = make_map(&mk, a.K, a.n, a.B * a.H_kv)) return rc;
  if (int rc = make_map(&mv, a.V, a.n, a.B * a.H_kv)) return rc;
  Params prm;
  prm.B = a.B;
  prm.H = a.H;
  prm.H_kv = a.H_kv;
  prm.n = a.n;
  prm.s = a.s;
  prm.causal = a.causal;
  prm.T = ceil_div(a.n, kTile);
  prm.items = a.B * a.H * prm.T;
  prm.spans = a.spans;
  auto kern = attn_tc_kernel<MaskT, kCausal>;
  const size_t smem = sizeof(TcSmem<MaskT>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(attn_tc_kernel)");
  const int grid = prm.items < sm_count() ? prm.items : sm_count();
  kern<<<grid, kThreads, smem, st>>>(mq, mk, mv, prm, a.sigma, a.table, static_cast<const MaskT*>(a.bmask),
                                     static_cast<__nv_bfloat16*>(a.O), a.row_sum, a.err);
  e = cudaGetLastError();
  return e == cudaSuccess ? PLSH_OK : cuda_fail(e, "attn_tc_kernel launch");
}

}  // namespace

int launch_attention_tc(const AttnArgs& a, cudaStream_t st) {
  if (static_cast<long long>(a.B) * a.H * ceil_div(a.n, kTile) > 0x7fffffffLL)
    return fail(PLSH_ERR_RANGE, "plsh_attention_fwd: too many query tiles");
  if (a.causal)
    return a.s <= 32 ? launch_tc_typed<uint32_t, true>(a, st) : launch_tc_typed<unsigned long long, true>(a, st);
  return a.s <= 32 ? launch_tc_typed<uint32_t, false>(a, st) : launch_tc_typed<unsigned long long, false>(a, st);
}

}  // namespace plsh
