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
// the widest windows first. Warp roles (256 threads):
//   warp 0      TMA producer: Q per item (2 buffers), K and V per key tile (2-stage rings)
//   warp 1      TMEM owner and single-thread tcgen05.mma issuer
//   warp 2      mask producer: the key tile's boundary masks into shared memory
//   warps 4-7   softmax: one query row per thread (TMEM lane = row)
// Per key tile g (counted across items): S_g = Q K_g^T (SS MMA into TMEM,
// double-buffered); the softmax warps turn S_g into bf16 P_g in TMEM; then
// O += P_g V_g (TS MMA: P from TMEM, fp32 O in TMEM). S_{g+1} is issued
// before PV_g so the tensor core works while the softmax runs.
//
// Weights: a row keeps a running OR R of the boundary masks between itself
// and the current key while it walks the tile's columns away from itself;
// log2(s - popcount(R)) is only recomputed where some hash opens a block
// (checked four keys at a time, the same for the whole warp). The logit is
// x = S * log2(e)/sqrt(d) + log2(c_ij) (-inf where c_ij = 0), so
// P = 2^(x - m) = c_ij 2^(S log2(e)/sqrt(d) - m). Key tiles are visited
// diagonal first, then downward, then upward, so the OR passed so far carries
// from tile to tile. The reference maximum m moves only when a tile's
// maximum exceeds it by more than 8 (then O and the row sum are rescaled),
// which keeps every P <= 256.
//
// Every barrier wait is bounded in time (PLSH_DEVERR_TIMEOUT); on timeout all
// roles leave their loops, in-flight copies and MMAs are drained and TMEM is
// freed before the CTA returns.
#include <cmath>

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
constexpr int kThreads = 256;
constexpr int kStages = 2;
constexpr int kChunkBytes = kTile * 64 * 2;         // 128 rows x 64 bf16 = 16 KB (one SW128 box)
constexpr int kTileBytes = 2 * kChunkBytes;         // 128 x 128 bf16 = 32 KB
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;      // S buffers at columns 0 and 128
constexpr uint32_t kColO = 256;    // O accumulator, 128 fp32 columns
constexpr uint32_t kColP = 384;    // P buffers at 384 and 448 (bf16 pairs)
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr int kMaxSortedHeads = 256;

template <typename MaskT>
struct alignas(16) MaskStage {
  MaskT bm[kTile + 4];   // bm[c]  = boundary mask of key j0 + c, c = 0..128 (all ones outside [0, n))
  MaskT bmn[kTile];      // bmn[c] = bm[c + 1]
};

template <typename MaskT>
struct __align__(1024) TcSmem {
  uint8_t q[2][kTileBytes];
  uint8_t k[kStages][kTileBytes];
  uint8_t v[kStages][kTileBytes];
  MaskStage<MaskT> m[kStages];
  float lg[PLSH_MAX_S + 4];            // lg[w] = log2(w), lg[0] = -inf
  int16_t order[kMaxSortedHeads];      // heads by decreasing window width
  int32_t width[kMaxSortedHeads];
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[kStages], k_empty[kStages];
  uint64_t v_full[kStages], v_empty[kStages];
  uint64_t m_full[kStages], m_empty[kStages];
  uint64_t s_full[2], p_full[2], pv_done[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

struct Params {
  int B, H, H_kv, n, s, causal, T, items;
  const int32_t* spans;
};

// One key tile of one work item, in the order every role walks them.
struct TileIter {
  const Params* p;
  const int16_t* order;
  int x;        // work item index
  int k;        // work items started by this CTA so far (Q buffer = k & 1)
  int it;       // key tile within the item
  int total;    // key tiles of the item
  int n_below;
  int b, h, t, i0;
  int g;        // key tile counted across this CTA's items
  bool valid;
  bool bad_window;  // the window read for this item was out of range (and was clamped)

  __device__ __forceinline__ void load_item() {
    valid = x < p->items;
    if (!valid) return;
    const int BT = p->B * p->T;
    const int hr = x / BT, rem = x - hr * BT;
    h = (p->H <= kMaxSortedHeads) ? static_cast<int>(order[hr]) : hr;
    b = rem / p->T;
    t = rem - b * p->T;
    i0 = t * kTile;
    int lo = p->spans[(static_cast<size_t>(h) * p->T + t) * 2];
    int hi = p->spans[(static_cast<size_t>(h) * p->T + t) * 2 + 1];
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
    load_item();
  }
  __device__ __forceinline__ void next() {
    ++g;
    if (++it >= total) {
      x += gridDim.x;
      ++k;
      load_item();
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

// Logits of one key tile for one row: x[c] <- S[c] * sc + log2(c_ij), with the running OR carried in/out.
// kind 0: diagonal tile (row r = column r); kind 1: below the diagonal; kind 2: above.
template <typename MaskT, bool kCausal>
__device__ __forceinline__ void tile_logits(float (&x)[kTile], const MaskStage<MaskT>& ms, const float* lg, int kind,
                                            int r, int s, float sc, MaskT& Y, MaskT& Z) {
  constexpr bool causal = kCausal;
  if (kind == 1) {
    // R(127) = Y; R(c) = R(c + 1) | bm[c + 1]
    MaskT R = Y;
    float lw = lg[max(0, s - popc_m(R))];
#pragma unroll
    for (int g4 = kTile / 4 - 1; g4 >= 0; --g4) {
      MaskT bb[4];
      load4(&ms.bmn[4 * g4], bb);
      if (g4 == kTile / 4 - 1) bb[3] = 0;
      if ((bb[0] | bb[1] | bb[2] | bb[3]) != 0) {
#pragma unroll
        for (int e = 3; e >= 0; --e) {
          R |= bb[e];
          lw = lg[max(0, s - popc_m(R))];
          x[4 * g4 + e] = fmaf(x[4 * g4 + e], sc, lw);
        }
      } else {
#pragma unroll
        for (int e = 3; e >= 0; --e) x[4 * g4 + e] = fmaf(x[4 * g4 + e], sc, lw);
      }
    }
    Y = R | ms.bm[0];   // OR over [j0, i]
  } else if (!kCausal && kind == 2) {
    // R(0) = Z (already holds bm[0]); R(c) = R(c - 1) | bm[c]
    MaskT R = Z;
    float lw = lg[max(0, s - popc_m(R))];
#pragma unroll
    for (int g4 = 0; g4 < kTile / 4; ++g4) {
      MaskT bb[4];
      load4(&ms.bm[4 * g4], bb);
      if (g4 == 0) bb[0] = 0;
      if ((bb[0] | bb[1] | bb[2] | bb[3]) != 0) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          R |= bb[e];
          lw = lg[max(0, s - popc_m(R))];
          x[4 * g4 + e] = fmaf(x[4 * g4 + e], sc, lw);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) x[4 * g4 + e] = fmaf(x[4 * g4 + e], sc, lw);
      }
    }
    Z = R;              // OR over (i, j0 + 127]
  } else {
    // columns c <= r: R(r) = 0; R(c) = R(c + 1) | bm[c + 1] for c < r
    MaskT R = 0;
    float lw = lg[s];
#pragma unroll
    for (int g4 = kTile / 4 - 1; g4 >= 0; --g4) {
      MaskT bb[4];
      load4(&ms.bmn[4 * g4], bb);
      if ((bb[0] | bb[1] | bb[2] | bb[3]) != 0) {
#pragma unroll
        for (int e = 3; e >= 0; --e) {
          const int c = 4 * g4 + e;
          if (c < r) R |= bb[e];
          lw = lg[max(0, s - popc_m(R))];
          x[c] = (c <= r) ? fmaf(x[c], sc, lw) : (causal ? -INFINITY : x[c]);
        }
      } else {
#pragma unroll
        for (int e = 3; e >= 0; --e) {
          const int c = 4 * g4 + e;
          x[c] = (c <= r) ? fmaf(x[c], sc, lw) : (causal ? -INFINITY : x[c]);
        }
      }
    }
    Y = R | ms.bm[0];   // OR over [i0, i]
    MaskT R2 = 0;
    if (!causal) {
      // columns c > r: R(r) = 0; R(c) = R(c - 1) | bm[c]
      float lw2 = lg[s];
#pragma unroll
      for (int g4 = 0; g4 < kTile / 4; ++g4) {
        MaskT bb[4];
        load4(&ms.bm[4 * g4], bb);
        if ((bb[0] | bb[1] | bb[2] | bb[3]) != 0) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = 4 * g4 + e;
            if (c > r) R2 |= bb[e];
            lw2 = lg[max(0, s - popc_m(R2))];
            if (c > r) x[c] = fmaf(x[c], sc, lw2);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = 4 * g4 + e;
            if (c > r) x[c] = fmaf(x[c], sc, lw2);
          }
        }
      }
    }
    Z = R2;             // OR over (i, i0 + 127]
  }
}

template <typename MaskT, bool kCausal>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
               const __grid_constant__ CUtensorMap tmap_v, Params prm, const double* __restrict__ sigma,
               const double* __restrict__ table, const MaskT* __restrict__ bmask, __nv_bfloat16* __restrict__ O,
               float* __restrict__ row_sum, uint32_t* __restrict__ err) {
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
      mbar_init(&sm.p_full[i], 4);
      mbar_init(&sm.pv_done[i], 1);
    }
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sm.k_full[i], 1);
      mbar_init(&sm.k_empty[i], 1);
      mbar_init(&sm.v_full[i], 1);
      mbar_init(&sm.v_empty[i], 1);
      mbar_init(&sm.m_full[i], 1);
      mbar_init(&sm.m_empty[i], 4);
    }
    mbar_init(&sm.drain, 1);
    fence_mbarrier_init();
  }
  if (threadIdx.x < PLSH_MAX_S + 4) sm.lg[threadIdx.x] = threadIdx.x == 0 ? -INFINITY : log2f(static_cast<float>(threadIdx.x));
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
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
  } else if (warp == 1) {
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
        const uint32_t p_tmem = tmem + kColP + 64u * static_cast<uint32_t>(ti.g & 1);
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk) {
          // 16 keys = two 8-row groups of the MN-major V tile; the two d halves sit kChunkBytes apart
          mma_ts(tmem + kColO, p_tmem + 8u * kk, smem_desc_sw128(v_addr + kk * 2048, kChunkBytes, 1024), idesc_pv,
                 (ti.it > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&sm.pv_done[ti.g & 1]);
        mma_commit(&sm.v_empty[st]);
        return true;
      };
      TileIter cur, nxt;
      cur.start(&prm, sm.order);
      bool ok = !cur.valid || issue_s(cur);
      while (ok && cur.valid) {
        nxt = cur;
        nxt.next();
        if (nxt.valid) ok = issue_s(nxt);
        if (ok) ok = issue_pv(cur);
        cur = nxt;
      }
      // every MMA issued so far completes before `drain` arrives
      mma_commit(&sm.drain);
      mbar_wait_drain(&sm.drain, 0, 100000000ull);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ mask producer
    TileIter ti;
    ti.start(&prm, sm.order);
    while (ti.valid) {
      const int st = ti.g % kStages;
      if (ti.g >= kStages &&
          !mbar_wait(&sm.m_empty[st], (static_cast<uint32_t>(ti.g / kStages) & 1u) ^ 1u, abort_flag, err))
        break;
      const MaskT* bm_h = bmask + static_cast<size_t>(ti.h) * n;
      MaskStage<MaskT>& ms = sm.m[st];
      const int j0 = ti.j0();
#pragma unroll
      for (int e = 0; e < 5; ++e) {
        const int c = lane + 32 * e;
        if (c <= kTile) {
          const int j = j0 + c;
          const MaskT v = (j >= 0 && j < n) ? bm_h[j] : FULL;
          ms.bm[c] = v;
          if (c >= 1) ms.bmn[c - 1] = v;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.m_full[st]);
      ti.next();
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int quarter = warp - 4;
    const int r = quarter * 32 + lane;   // row within the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float sc = 1.4426950408889634f / sqrtf(static_cast<float>(kD));
    float m2 = -INFINITY, l = 0.0f;
    MaskT Y = 0, Z = 0;
    TileIter ti;
    ti.start(&prm, sm.order);
    bool ok = true;
    while (ti.valid) {
      const int g = ti.g;
      const int st = g % kStages;
      if (ti.first()) {
        m2 = -INFINITY;
        l = 0.0f;
        if (ti.bad_window && r == 0) atomicOr(err, PLSH_DEVERR_WINDOW);
      }
      ok = mbar_wait(&sm.m_full[st], static_cast<uint32_t>(g / kStages) & 1u, abort_flag, err);
      ok = __all_sync(0xffffffffu, ok && mbar_wait(&sm.s_full[g & 1], static_cast<uint32_t>(g >> 1) & 1u,
                                                   abort_flag, err));
      if (!ok) break;
      tc_fence_after();
      float x[kTile];
      {
        const uint32_t base = tmem + lane_off + kColS + 128u * static_cast<uint32_t>(g & 1);
        uint32_t raw[4][32];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) tmem_ld32(base + 32u * q4, raw[q4]);
        tmem_wait_ld();
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
#pragma unroll
          for (int e = 0; e < 32; ++e) x[32 * q4 + e] = __uint_as_float(raw[q4][e]);
      }
      const MaskStage<MaskT>& ms = sm.m[st];
      const int kind = ti.kind();
      if (kind == 2) Z |= ms.bm[0];   // now OR over (i, j0]
      tile_logits<MaskT, kCausal>(x, ms, sm.lg, kind, r, s, sc, Y, Z);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.m_empty[st]);

      // ---- tile maximum and reference update
      float mx[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) mx[u] = x[u];
#pragma unroll
      for (int c = 8; c < kTile; ++c) mx[c & 7] = fmaxf(mx[c & 7], x[c]);
      const float mt = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                             fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
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

      // ---- P buffer g&1 must be free: PV of tile g-2 done
      if (g >= 2) {
        ok = __all_sync(0xffffffffu, mbar_wait(&sm.pv_done[g & 1], static_cast<uint32_t>((g - 2) >> 1) & 1u,
                                               abort_flag, err));
        if (!ok) break;
      }
      // ---- rescale O when some row of the warp moved its reference (never on an item's first tile)
      if (__any_sync(0xffffffffu, need_rescale)) {
        ok = __all_sync(0xffffffffu, mbar_wait(&sm.pv_done[(g - 1) & 1], static_cast<uint32_t>((g - 1) >> 1) & 1u,
                                               abort_flag, err));
        if (!ok) break;
        tc_fence_after();
        uint32_t raw[32];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const uint32_t addr = tmem + lane_off + kColO + 32u * q4;
          tmem_ld32(addr, raw);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) raw[e] = __float_as_uint(__uint_as_float(raw[e]) * alpha);
          tmem_st32(addr, raw);
        }
        tmem_wait_st();
      }

      // ---- P = 2^(x - m) as bf16 into TMEM, row sum
      const uint32_t p_base = tmem + lane_off + kColP + 64u * static_cast<uint32_t>(g & 1);
      float ls[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) ls[u] = 0.0f;
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        uint32_t packed[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const float p0 = ex2_approx(x[32 * q4 + e] + neg_m);
          const float p1 = ex2_approx(x[32 * q4 + e + 1] + neg_m);
          ls[e & 7] += p0;
          ls[(e + 1) & 7] += p1;
          packed[e >> 1] = pack_bf16x2(p0, p1);
        }
        tmem_st16(p_base + 16u * q4, packed);
      }
      tmem_wait_st();
      l = l * alpha + (((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7])));
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.p_full[g & 1]);

      // ---- epilogue of the item: O / l and row_sum
      if (ti.last()) {
        ok = __all_sync(0xffffffffu, mbar_wait(&sm.pv_done[g & 1], static_cast<uint32_t>(g >> 1) & 1u,
                                               abort_flag, err));
        if (!ok) break;
        tc_fence_after();
        const int i = ti.i0 + r;
        const float inv = 1.0f / l;
        __nv_bfloat16* orow = O + ((static_cast<size_t>(ti.b) * H + ti.h) * n + (i < n ? i : 0)) * kD;
#pragma unroll 1
        for (int q4 = 0; q4 < 4; ++q4) {
          uint32_t raw[32];
          tmem_ld32(tmem + lane_off + kColO + 32u * q4, raw);
          tmem_wait_ld();
          if (i < n) {
            uint4* dst = reinterpret_cast<uint4*>(orow + 32 * q4);
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
          row_sum[(static_cast<size_t>(ti.b) * H + ti.h) * n + i] =
              (log2f(l) + m2) * 0.6931471805599453f - logf(static_cast<float>(s));
        }
      }
      ti.next();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
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
