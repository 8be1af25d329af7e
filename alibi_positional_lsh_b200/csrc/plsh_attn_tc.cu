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
// Persistent CTAs (one per SM) walk a static list of items, heads with the
// widest windows first. Warp roles (352 threads):
//   warps 0-7    softmax: warp w owns rows 32 (w % 4) + 16 (w / 4) .. + 15 of
//                every tile (16 lanes of its TMEM lane quarter w % 4); inside
//                the warp, threads t and t + 16 share row t % 16 and split each
//                pair of 16-key chunks (the 16x32bx2 TMEM access shape), so a
//                row's maximum and sum combine with one shuffle
//   warp 8       TMA producer: Q per item (two buffers), K and V per key tile
//                (two stages each)
//   warp 9       TMEM owner and single-thread tcgen05.mma issuer
//   warp 10      mask warp: the key tile's boundary masks, their in-tile
//                prefix / suffix ORs and the tile's descriptor
// TMEM holds S twice (tiles of even and odd index) and O twice (items of even
// and odd index): S(g+1) = Q K^T is issued before O += P(g) V, so the tensor
// core computes the next tile's scores while the softmax works on the
// current one; the softmax turns S into bf16 P written back over S, and the
// PV MMA reads P from TMEM. An item's epilogue (O / l to global memory) runs
// after the next tile's mask-only work (the diagonal scan), so that work
// overlaps the item's last PV on the tensor core.
//
// Weights. P_ij = c_ij 2^(S_ij log2(e)/sqrt(d) - m): the count multiplies the
// exponential as an exact small-integer float, so no logarithm is taken.
// With R_ij the OR of the boundary masks strictly after min(i,j) up to
// max(i,j), c_ij = s - popcount(R_ij), and R_ij splits into a part that
// depends on the row only (a carry) and a part that depends on the key only,
// the same for a whole warp: below the diagonal R = Y | suf[c] with Y the OR
// from the tile's end to the row; above it R = Z | pre[c] with Z the OR from
// the row to the tile's start. On the diagonal tile the rows of each 32-row
// block (one TMEM lane quarter) scan the keys of the block's own 32 keys from
// the row outwards (before S is ready), which yields the carries for the rest
// of the tile, whose keys take range ORs that end (or start) at that block. Key tiles are
// visited diagonal first, then downward, then upward, so the carries pass
// from tile to tile.
// The reference m is a running upper bound: the largest S log2(e)/sqrt(d)
// over the tile's live keys raises it when it exceeds m by more than 8, and O
// and the row sum are then rescaled; so P <= s 2^8, and the row's own key
// (c = s) keeps the sum away from zero. A pair of chunks whose key nearest to
// the warp's rows has count 0 for all of them has count 0 throughout (the OR of
// the masks only grows moving away from a row): its S is neither read nor
// exponentiated and its P is written as zeros. Per tile a softmax thread reads
// its live S twice (the maximum, then P, chunk by chunk) and writes P of keys
// [16ch, 16ch + 16) as bf16 pairs to columns [8ch, 8ch + 8) of the S region,
// over columns already read.
//
// The per-sample comparator (K4) runs the same machinery with each item walked
// once per hash k over that hash's own window, the boundary masks reduced to
// bit k and the weight count s replaced by 1: each pass adds hash k's 0/1
// block-diagonal attention, and the passes share one online softmax, so the
// result is the same T~ (Methodology 3, Theorem 2.2's construction).
//
// Exact banded ALiBi (the kAlibi instantiations, the competitor Positional LSH
// approximates) runs on the same machinery with weights computed from the
// positions: x = S log2(e)/sqrt(d) - |i - j| log2(e)/sigma_h - m over the keys
// within W_h = ceil(sigma_h ln(1/eps)) of the tile's rows; the mask warp then
// only publishes each tile's descriptor.
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
#include "plsh_tile_common.cuh"

namespace plsh {
namespace {

using namespace sm100;
using namespace tiles;

constexpr int kThreads = 352;  // 11 warps
constexpr int kSoftmaxWarps = 8;
constexpr int kWarpTma = 8, kWarpMma = 9, kWarpMask = 10;
constexpr int kStages = 2;     // K and V buffers
constexpr int kMaskStages = 2;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;              // S (then P) of tile g at columns 128 (g % 2)
constexpr uint32_t kColO = 256;            // O of item k at columns 256 + 128 (k % 2)
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <typename MaskT>
struct __align__(1024) TcSmem {
  uint8_t q[2][kTileBytes];
  uint8_t k[kStages][kTileBytes];
  uint8_t v[kStages][kTileBytes];
  MaskStage<MaskT> m[kMaskStages];
  uint32_t cw[8][kSoftmaxWarps * 32];  // diagonal tile: own-block counts, one column per softmax thread
  int16_t order[kMaxSortedHeads];  // heads by decreasing window width
  int32_t width[kMaxSortedHeads];
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[kStages], k_empty[kStages];
  uint64_t v_full[kStages], v_empty[kStages];
  uint64_t m_full[kMaskStages], m_empty[kMaskStages];
  uint64_t s_full[2], p_full[2], pv_done[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

static_assert(kStages == 2, "the descriptor selects assume two K/V stages");
static_assert(sizeof(TcSmem<unsigned long long>) + 1024 <= 232448, "shared memory budget");

// The largest of m and 32 raw fp32 values (four independent chains of three-input maxima).
__device__ __forceinline__ float max32(const uint32_t (&v)[32], float m) {
  float mx[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const uint32_t* w = v + 8 * u;
    float x = max3(__uint_as_float(w[0]), __uint_as_float(w[1]), __uint_as_float(w[2]));
    x = max3(x, __uint_as_float(w[3]), __uint_as_float(w[4]));
    x = max3(x, __uint_as_float(w[5]), __uint_as_float(w[6]));
    mx[u] = fmaxf(x, __uint_as_float(w[7]));
  }
  return max3(m, max3(mx[0], mx[1], mx[2]), mx[3]);
}

// Constants of the softmax, each as a packed pair: the scale log2(e)/sqrt(d), -m, and -2^23 (which
// turns the float with the bits of 2^23 + c back into c).
struct SoftmaxK {
  uint64_t sc2, negm2, neg2p23;
};

// Exact ALiBi: P = 2^(S sc - m - lam |i - j|) for 16 keys, with t0 = lam (i - j) at the first key
// (i - j falls by one per key) and keys k > lim dropped (the causal mask, and keys past n, which
// the tensor map reads as zeros). Returns the sum of P.
__device__ __forceinline__ float p16_alibi(const uint32_t (&sv)[16], float t0, float lam, int lim, float sc,
                                           float neg_m, uint32_t (&pk)[8]) {
  float ls[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
  for (int g4 = 0; g4 < 4; ++g4) {
    float p[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int k = 4 * g4 + e;
      const float t = fmaf(-lam, static_cast<float>(k), t0);
      const float x = fmaf(__uint_as_float(sv[k]), sc, neg_m) - fabsf(t);
      p[e] = k > lim ? 0.0f : ex2_approx(x);
      ls[e] += p[e];
    }
    pk[2 * g4] = pack_bf16x2(p[0], p[1]);
    pk[2 * g4 + 1] = pack_bf16x2(p[2], p[3]);
  }
  return (ls[0] + ls[1]) + (ls[2] + ls[3]);
}

// P = c 2^(S sc - m) for 16 keys (S as raw fp32 bits), with cf[k] the float bits of 2^23 + c_k;
// packed as 8 bf16 pairs. Returns the sum of P.
__device__ __forceinline__ float p16_cf(const uint32_t (&sv)[16], const uint32_t (&cf)[16], const SoftmaxK& k2,
                                        uint32_t (&pk)[8]) {
  uint64_t ls2[2] = {0ull, 0ull};
#pragma unroll
  for (int g4 = 0; g4 < 4; ++g4) {
#pragma unroll
    for (int e2 = 0; e2 < 2; ++e2) {
      const int kk = 4 * g4 + 2 * e2;
      float x0, x1;
      f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[kk]), __uint_as_float(sv[kk + 1])), k2.sc2, k2.negm2), x0, x1);
      const uint64_t w2 = f2_add(f2_pack(__uint_as_float(cf[kk]), __uint_as_float(cf[kk + 1])), k2.neg2p23);
      const uint64_t p2 = f2_mul(f2_pack(ex2_approx(x0), ex2_approx(x1)), w2);
      ls2[e2] = f2_add(ls2[e2], p2);
      float p0, p1;
      f2_unpack(p2, p0, p1);
      pk[2 * g4 + e2] = pack_bf16x2(p0, p1);
    }
  }
  float a0, a1, b0, b1;
  f2_unpack(ls2[0], a0, a1);
  f2_unpack(ls2[1], b0, b1);
  return (a0 + a1) + (b0 + b1);
}

template <typename MaskT, bool kCausal, bool kVarlen, bool kAlibi>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
               const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ Params prm,
               const double* __restrict__ sigma, const double* __restrict__ table, const MaskT* __restrict__ bmask,
               __nv_bfloat16* __restrict__ O, float* __restrict__ row_sum, uint32_t* __restrict__ err) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t smem_pad = (1024u - (static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw)) & 1023u)) & 1023u;
  auto& sm = *reinterpret_cast<TcSmem<MaskT>*>(smem_raw + smem_pad);
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
    const int nsub = kVarlen ? s : 1;
    for (int h = threadIdx.x; h < H; h += kThreads) {
      int w = 0;
      if constexpr (kAlibi) {
        w = alibi_reach(prm.sigma[h], prm.log_inv_eps, n);
      } else {
        for (int sb = 0; sb < nsub; ++sb) {
          const size_t at = (static_cast<size_t>(h) * nsub + sb) * prm.T + tm;
          w += prm.spans[at * 2 + 1] - prm.spans[at * 2];
        }
      }
      sm.width[h] = w;
    }
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
      mbar_init(&sm.k_full[i], 1);
      mbar_init(&sm.k_empty[i], 1);
      mbar_init(&sm.v_full[i], 1);
      mbar_init(&sm.v_empty[i], 1);
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.p_full[i], kSoftmaxWarps);
      mbar_init(&sm.pv_done[i], 1);
    }
    for (int i = 0; i < kMaskStages; ++i) {
      mbar_init(&sm.m_full[i], 1);
      mbar_init(&sm.m_empty[i], kSoftmaxWarps);
    }
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
    // Q per item (two buffers by item parity), K and V per key tile (two stages each).
    if (lane == 0) {
      tma_prefetch_desc(&tmap_q);
      tma_prefetch_desc(&tmap_k);
      tma_prefetch_desc(&tmap_v);
      TileIter<kVarlen, kAlibi> ti;
      ti.start(&prm, sm.order);
      int issued_g = 0, issued_v = 0, issued_k = 0;  // K tiles, V tiles and Q items issued
      while (ti.valid) {
        const int zkv = ti.b * prm.H_kv + ti.h / (H / prm.H_kv);
        if (ti.first()) {
          const int qb = ti.k & 1;
          if (ti.k >= 2 && !mbar_wait(&sm.q_empty[qb], ((ti.k >> 1) & 1) ^ 1, abort_flag, err, prm.wait_ns)) break;
          mbar_arrive_expect_tx(&sm.q_full[qb], kTileBytes);
          tma_load_3d(sm.q[qb], &tmap_q, 0, ti.i0, ti.b * H + ti.h, &sm.q_full[qb]);
          tma_load_3d(sm.q[qb] + kChunkBytes, &tmap_q, 64, ti.i0, ti.b * H + ti.h, &sm.q_full[qb]);
          issued_k = ti.k + 1;
        }
        const int st = ti.g % kStages;
        const uint32_t ph = static_cast<uint32_t>(ti.g / kStages) & 1u;
        const int j0 = ti.j0();
        if (ti.g >= kStages && !mbar_wait(&sm.k_empty[st], ph ^ 1u, abort_flag, err, prm.wait_ns)) break;
        mbar_arrive_expect_tx(&sm.k_full[st], kTileBytes);
        tma_load_3d(sm.k[st], &tmap_k, 0, j0, zkv, &sm.k_full[st]);
        tma_load_3d(sm.k[st] + kChunkBytes, &tmap_k, 64, j0, zkv, &sm.k_full[st]);
        issued_g = ti.g + 1;
        if (ti.g >= kStages && !mbar_wait(&sm.v_empty[st], ph ^ 1u, abort_flag, err, prm.wait_ns)) break;
        mbar_arrive_expect_tx(&sm.v_full[st], kTileBytes);
        tma_load_3d(sm.v[st], &tmap_v, 0, j0, zkv, &sm.v_full[st]);
        tma_load_3d(sm.v[st] + kChunkBytes, &tmap_v, 64, j0, zkv, &sm.v_full[st]);
        issued_v = ti.g + 1;
        ti.next();
      }
      if (*abort_flag) {
        // let every copy already issued land before the CTA can exit
        for (int kk = (issued_k > 2 ? issued_k - 2 : 0); kk < issued_k; ++kk)
          mbar_wait_drain(&sm.q_full[kk & 1], (kk >> 1) & 1, kDrainNs);
        for (int gg = (issued_g > kStages ? issued_g - kStages : 0); gg < issued_g; ++gg)
          mbar_wait_drain(&sm.k_full[gg % kStages], static_cast<uint32_t>(gg / kStages) & 1u, kDrainNs);
        for (int gg = (issued_v > kStages ? issued_v - kStages : 0); gg < issued_v; ++gg)
          mbar_wait_drain(&sm.v_full[gg % kStages], static_cast<uint32_t>(gg / kStages) & 1u, kDrainNs);
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    // S of the next tile is issued before PV of the current one: S is double-buffered in TMEM
    // and S(g+1) computes while the softmax works on S(g). P(g-1) lives in S(g+1)'s buffer; it is
    // read by PV(g-1), which was issued before S(g+1), and the tensor core runs them in order.
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 128, 1);
      uint64_t q_desc[2], k_desc[kStages], v_desc[kStages];
      for (int i = 0; i < 2; ++i) q_desc[i] = smem_desc_sw128(smem_u32(sm.q[i]), 16, 1024);
      for (int i = 0; i < kStages; ++i) {
        k_desc[i] = smem_desc_sw128(smem_u32(sm.k[i]), 16, 1024);
        v_desc[i] = smem_desc_sw128(smem_u32(sm.v[i]), kChunkBytes, 1024);
      }
      auto issue_s = [&](const TileIter<kVarlen, kAlibi>& ti) -> bool {
        const int qb = ti.k & 1;
        if (ti.first() && !mbar_wait(&sm.q_full[qb], (ti.k >> 1) & 1, abort_flag, err, prm.wait_ns)) return false;
        const int st = ti.g % kStages;
        if (!mbar_wait(&sm.k_full[st], static_cast<uint32_t>(ti.g / kStages) & 1u, abort_flag, err, prm.wait_ns)) return false;
        tc_fence_after();
        const uint32_t d_tmem = tmem + kColS + 128u * static_cast<uint32_t>(ti.g & 1);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          // the descriptors' start address field counts 16-byte units
          const uint64_t off = static_cast<uint64_t>(((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4);
          mma_ss(d_tmem, (qb ? q_desc[1] : q_desc[0]) + off, (st ? k_desc[1] : k_desc[0]) + off, idesc_qk,
                 kk > 0 ? 1u : 0u);
        }
        mma_commit(&sm.s_full[ti.g & 1]);
        mma_commit(&sm.k_empty[st]);
        if (ti.last()) mma_commit(&sm.q_empty[qb]);
        return true;
      };
      auto issue_pv = [&](const TileIter<kVarlen, kAlibi>& ti) -> bool {
        const int st = ti.g % kStages;
        if (!mbar_wait(&sm.p_full[ti.g & 1], static_cast<uint32_t>(ti.g >> 1) & 1u, abort_flag, err, prm.wait_ns)) return false;
        if (!mbar_wait(&sm.v_full[st], static_cast<uint32_t>(ti.g / kStages) & 1u, abort_flag, err, prm.wait_ns)) return false;
        tc_fence_after();
        const uint32_t p_tmem = tmem + kColS + 128u * static_cast<uint32_t>(ti.g & 1);
        const uint32_t o_tmem = tmem + kColO + 128u * static_cast<uint32_t>(ti.k & 1);
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk) {
          // keys 16kk..16kk+15: P at columns 8kk; the keys are two 8-row groups of the MN-major V
          // tile, whose two d halves sit kChunkBytes apart
          mma_ts(o_tmem, p_tmem + 8u * kk,
                 (st ? v_desc[1] : v_desc[0]) + static_cast<uint64_t>((kk * 2048) >> 4), idesc_pv,
                 (!ti.first() || kk > 0) ? 1u : 0u);
        }
        mma_commit(&sm.pv_done[ti.g & 1]);
        mma_commit(&sm.v_empty[st]);
        return true;
      };
      TileIter<kVarlen, kAlibi> cur, nxt;
      cur.start(&prm, sm.order);
      nxt.start(&prm, sm.order);
      if (prm.withhold_mma) cur.valid = nxt.valid = false;  // failure-detection tests only
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
      mbar_wait_drain(&sm.drain, 0, kDrainNs);
    }
  } else if (warp == kWarpMask) {
    // ------------------------------------------------------------ mask warp
    if constexpr (kAlibi) {
      // exact banded ALiBi needs no masks: the warp only publishes each tile's descriptor
      TileIter<kVarlen, kAlibi> ti;
      ti.start(&prm, sm.order);
      int g_end = 0;
      bool ok = true;
      while (ti.valid) {
        const int st = ti.g % kMaskStages;
        if (ti.g >= kMaskStages) {
          ok = mbar_wait(&sm.m_empty[st], (static_cast<uint32_t>(ti.g / kMaskStages) & 1u) ^ 1u, abort_flag, err, prm.wait_ns);
          if (!__all_sync(0xffffffffu, ok)) {
            ok = false;
            break;
          }
        }
        if (lane == 0) {
          MaskStage<MaskT>& ms = sm.m[st];
          ms.valid = 1;
          ms.kind = ti.kind();
          ms.first = ti.first() ? 1 : 0;
          ms.last = ti.last() ? 1 : 0;
          ms.x = ti.x;
          ms.j0 = ti.j0();
          mbar_arrive(&sm.m_full[st]);
        }
        __syncwarp();
        g_end = ti.g + 1;
        ti.next();
      }
      if (ok && !*abort_flag) {
        const int st = g_end % kMaskStages;
        ok = g_end < kMaskStages ||
             mbar_wait(&sm.m_empty[st], (static_cast<uint32_t>(g_end / kMaskStages) & 1u) ^ 1u, abort_flag, err, prm.wait_ns);
        if (__all_sync(0xffffffffu, ok) && lane == 0) {
          sm.m[st].valid = 0;
          mbar_arrive(&sm.m_full[st]);
        }
      }
    } else {
    TileIter<kVarlen, kAlibi> ti, nx;
    ti.start(&prm, sm.order);
    nx.start(&prm, sm.order);
    if (nx.valid) nx.next();
    // the masks of a tile; a comparator sub-item keeps only its own hash's bit
    auto load_masks = [&](const TileIter<kVarlen, kAlibi>& t, MaskT (&v)[4], MaskT& v128) {
      const MaskT* bm_h = bmask + static_cast<size_t>(t.h) * n;
      const MaskT bits = kVarlen ? static_cast<MaskT>(static_cast<MaskT>(1) << t.sub) : FULL;
      const int j0 = t.j0();
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = j0 + 4 * lane + e;
        v[e] = static_cast<MaskT>(((j >= 0 && j < n) ? bm_h[j] : FULL) & bits);
      }
      const int j = j0 + kTile;
      v128 = static_cast<MaskT>(((lane == 0 && j >= 0 && j < n) ? bm_h[j] : FULL) & bits);
    };
    MaskT xv[4] = {FULL, FULL, FULL, FULL}, x128 = FULL;
    if (ti.valid) load_masks(ti, xv, x128);
    int g_end = 0;
    bool ok = true;
    while (ti.valid) {
      const int st = ti.g % kMaskStages;
      MaskT nv[4] = {FULL, FULL, FULL, FULL}, n128 = FULL;
      if (nx.valid) load_masks(nx, nv, n128);  // lands while this tile is processed
      if (ti.g >= kMaskStages) {
        ok = mbar_wait(&sm.m_empty[st], (static_cast<uint32_t>(ti.g / kMaskStages) & 1u) ^ 1u, abort_flag, err, prm.wait_ns);
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
      }
      MaskStage<MaskT>& ms = sm.m[st];
      publish_masks<MaskT, true, !kCausal>(ms, xv, x128, ti.kind() == 0, lane);
      if (lane == 0) {
        ms.valid = 1;
        ms.kind = ti.kind();
        ms.first = ti.first() ? 1 : 0;
        ms.last = ti.last() ? 1 : 0;
        ms.x = ti.x;
        ms.j0 = ti.j0();
        ms.sub = ti.sub;
        if (ti.first() && ti.bad_window) atomicOr(err, PLSH_DEVERR_WINDOW);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.m_full[st]);
      g_end = ti.g + 1;
      ti.next();
      if (nx.valid) nx.next();
#pragma unroll
      for (int e = 0; e < 4; ++e) xv[e] = nv[e];
      x128 = n128;
    }
    // the end marker for the softmax warps
    if (ok && !*abort_flag) {
      const int st = g_end % kMaskStages;
      ok = g_end < kMaskStages ||
           mbar_wait(&sm.m_empty[st], (static_cast<uint32_t>(g_end / kMaskStages) & 1u) ^ 1u, abort_flag, err, prm.wait_ns);
      if (__all_sync(0xffffffffu, ok) && lane == 0) {
        sm.m[st].valid = 0;
        mbar_arrive(&sm.m_full[st]);
      }
    }
    }  // masks (PLSH) or descriptors only (exact ALiBi)
  } else {
    // ------------------------------------------------------------ softmax
    // Warp w owns rows 32 (w % 4) + 16 (w / 4) .. + 15 of every tile (16 lanes of its TMEM
    // quarter). Inside the warp, threads t and t + 16 share row t % 16: of each pair of 16-key
    // chunks (keys 32m .. 32m + 31) thread t takes the even chunk and thread t + 16 the odd one
    // (the 16x32bx2 TMEM access shape), so a row's maximum and sum combine with one shuffle.
    const int quarter = warp & 3;
    const int hq = warp >> 2;   // which 16 rows of the quarter
    const int kh = lane >> 4;   // which chunk of each pair
    const int r = quarter * 32 + hq * 16 + (lane & 15);  // row within the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32 + hq * 16) << 16;
    const float sc = 1.4426950408889634f / sqrtf(static_cast<float>(kD));
    // weights count hashes: all s of them, or (comparator) the one hash of the sub-item
    const int sw = kVarlen ? 1 : s;
    float m2 = -INFINITY, l = 0.0f;
    MaskT Y = 0, Z = 0;
    float lam = 0.0f;  // exact ALiBi: log2(e) / sigma of the item's head
    int a_i0 = 0;      // exact ALiBi: the item's first row
    int items = 0;     // items finished by this warp
    bool pend = false;  // an item's epilogue is pending
    int pend_tx = 0, pend_g = 0;  // its item index and last tile
    for (int g = 0;; ++g) {
      const int st = g % kMaskStages;
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.m_full[st], static_cast<uint32_t>(g / kMaskStages) & 1u,
                                             abort_flag, err, prm.wait_ns)))
        break;
      const MaskStage<MaskT>& ms = sm.m[st];
      const bool valid = ms.valid != 0;
      const int kind = ms.kind, first = ms.first, last = ms.last, tx = ms.x;
      // weights that need only the masks: the diagonal's own block and its carries (before the
      // previous item's epilogue, whose last PV is still running on the tensor core)
      MaskT lo = 0, hi = 0;
      if (!kAlibi && valid && kind == 0) diag_scan<MaskT, true, !kCausal>(ms, quarter, r, sw, &sm.cw[0][threadIdx.x], kSoftmaxWarps * 32, lo, hi);
      // ---- the previous item's epilogue: O / l once its last PV has completed, stored four rows
      // at a time by each lane quad (thread t: columns 0..63 of its row, thread t + 16: 64..127)
      if (pend) {
        pend = false;
        const int kb = items & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&sm.pv_done[pend_g & 1], static_cast<uint32_t>(pend_g >> 1) & 1u, abort_flag, err, prm.wait_ns)))
          break;
        tc_fence_after();
        const float ltot = l + __shfl_xor_sync(0xffffffffu, l, 16);
        const int BT = prm.B * prm.T;
        const int hh = (H <= kMaxSortedHeads) ? static_cast<int>(sm.order[pend_tx / BT]) : pend_tx / BT;
        const int rem = pend_tx % BT;
        const int bb = rem / prm.T, i0 = (rem % prm.T) * kTile;
        const float inv = 1.0f / ltot;
        const int p4 = lane & 3;
        const int quad_row = quarter * 32 + hq * 16 + ((lane & 15) & ~3);  // first of the quad's four rows
        const uint32_t o_row = tmem + lane_off + kColO + 128u * static_cast<uint32_t>(kb);
        __nv_bfloat16* obase = O + (static_cast<size_t>(bb) * H + hh) * static_cast<size_t>(n) * kD + 64 * kh;
#pragma unroll 1
        for (int blk = 0; blk < 2; ++blk) {
          uint32_t raw[32];
          tmem_ld16x2_32<64>(o_row + 32u * blk, raw);
          tmem_wait_ld();
          regs_after_wait(raw);
          uint32_t a[4][4];  // [16-byte chunk][word] of this row's 32 columns
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int w = 0; w < 4; ++w)
              a[c][w] = pack_bf16x2(__uint_as_float(raw[8 * c + 2 * w]) * inv,
                                    __uint_as_float(raw[8 * c + 2 * w + 1]) * inv);
          // 4x4 transpose of 16-byte chunks inside the quad: lane p then holds chunk p of the quad's rows
#pragma unroll
          for (int msk = 2; msk >= 1; msk >>= 1) {
            const bool lo_lane = (p4 & msk) == 0;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              if (c & msk) continue;
#pragma unroll
              for (int w = 0; w < 4; ++w) {
                const uint32_t send = lo_lane ? a[c | msk][w] : a[c][w];
                const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, msk);
                if (lo_lane) a[c | msk][w] = recv;
                else a[c][w] = recv;
              }
            }
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int row = i0 + quad_row + e;
            if (row < n)
              *reinterpret_cast<uint4*>(obase + static_cast<size_t>(row) * kD + 32 * blk + 8 * p4) =
                  make_uint4(a[e][0], a[e][1], a[e][2], a[e][3]);
          }
        }
        tc_fence_before();
        const int i = i0 + r;
        if (kh == 0 && i < n)
          row_sum[(static_cast<size_t>(bb) * H + hh) * n + i] =
              (log2f(ltot) + m2) * 0.6931471805599453f - (kAlibi ? 0.0f : logf(static_cast<float>(s)));
        ++items;
      }
      if (!valid) break;
      if (first) {
        m2 = -INFINITY;
        l = 0.0f;
        if constexpr (kAlibi) {
          const int BT = prm.B * prm.T;
          const int hh = (H <= kMaxSortedHeads) ? static_cast<int>(sm.order[tx / BT]) : tx / BT;
          lam = static_cast<float>(1.4426950408889634 / prm.sigma[hh]);
          a_i0 = ((tx % BT) % prm.T) * kTile;
        }
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full[g & 1], static_cast<uint32_t>(g >> 1) & 1u, abort_flag, err, prm.wait_ns)))
        break;
      tc_fence_after();
      const uint32_t s_base = tmem + lane_off + kColS + 128u * static_cast<uint32_t>(g & 1);

      // ---- the chunk pairs that carry weight for some row of the warp. Moving away from the row
      // the OR of the boundary masks only grows (blocks are contiguous), so a pair whose key
      // nearest to the rows has count 0 for every row of the warp has count 0 throughout: its S
      // is neither read nor exponentiated, and its P is written as zeros. (When causal, the
      // diagonal tile's pairs past the warp's own block are dead as well.)
      const int n_pairs = (kCausal && kind == 0) ? quarter + 1 : kTile / 32;
      const MaskT Zc = static_cast<MaskT>(Z | ms.bm[0]);
      // the hashes without a boundary in the row's part of the gap, below and above the rows, and
      // the per-key part: below Y | suf[c], above Z | bm[0] | pre[c], diagonal lo | dq[c] below
      // the warp's block and hi | dq[c] above it (the comparator's sub-item counts its own hash)
      const MaskT hashes = kVarlen ? static_cast<MaskT>(static_cast<MaskT>(1) << ms.sub) : FULL;
      const MaskT keep_lo = static_cast<MaskT>(hashes & ~(kind == 1 ? Y : lo));
      const MaskT keep_hi = static_cast<MaskT>(hashes & ~(kind == 2 ? Zc : hi));
      const MaskT* km_tile = kind == 1 ? ms.suf : (kind == 2 ? ms.pre : ms.dq[quarter]);
      uint32_t live = 0;  // bit m: pair m
#pragma unroll
      for (int m = 0; m < kTile / 32; ++m) {
        bool lv = m < n_pairs;
        if (!kAlibi && lv && !(kind == 0 && m == quarter)) {
          const bool below = kind == 1 || (kind == 0 && m < quarter);
          const MaskT kn = km_tile[below ? 32 * m + 31 : 32 * m];  // the key nearest to the rows
          lv = static_cast<MaskT>((below ? keep_lo : keep_hi) & ~kn) != 0;
        }
        if (__any_sync(0xffffffffu, lv)) live |= 1u << m;
      }

      // ---- pass 1: the row's maximum of S over the live 64-key halves (thread t reads columns
      // [64h, 64h + 32), thread t + 16 [64h + 32, 64h + 64)), combined over the row's two threads
      float mraw = -INFINITY;
      {
        uint32_t sa[32], sb[32];
        if (live & 3u) tmem_ld16x2_32<32>(s_base, sa);
        if (live & 12u) tmem_ld16x2_32<32>(s_base + 64u, sb);
        tmem_wait_ld();
        regs_after_wait(sa);
        regs_after_wait(sb);
        if (live & 3u) mraw = max32(sa, mraw);
        if (live & 12u) mraw = max32(sb, mraw);
      }
      mraw = fmaxf(mraw, __shfl_xor_sync(0xffffffffu, mraw, 16));
      const float mt = mraw * sc;

      // ---- reference update (the same in the row's two threads); O is rescaled in place once
      // PV(g-1) has completed
      float alpha = 1.0f;
      bool need_rescale = false;
      if (mt > m2 + kRescaleThreshold) {
        if (m2 != -INFINITY) {
          alpha = ex2_approx(m2 - mt);
          need_rescale = true;
        }
        m2 = mt;
      }
      const float neg_m = -m2;
      if (__any_sync(0xffffffffu, need_rescale)) {
        if (!__all_sync(0xffffffffu, mbar_wait(&sm.pv_done[(g - 1) & 1], static_cast<uint32_t>((g - 1) >> 1) & 1u,
                                               abort_flag, err, prm.wait_ns)))
          break;
        tc_fence_after();
        // thread t: columns [16 q4, 16 q4 + 16), thread t + 16 the same 64 columns further
        const uint32_t o_row = tmem + lane_off + kColO + 128u * static_cast<uint32_t>(items & 1);
#pragma unroll 1
        for (int q4 = 0; q4 < 4; ++q4) {
          uint32_t raw[16];
          tmem_ld16x2_16<64>(o_row + 16u * q4, raw);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) raw[e] = __float_as_uint(__uint_as_float(raw[e]) * alpha);
          tmem_st16x2_16<64>(o_row + 16u * q4, raw);
        }
      }

      // ---- pass 2: P = c 2^(S sc - m), one chunk pair at a time; P of chunk ch goes to columns
      // 8 ch, over S columns already read (S of chunk ch sits at columns 16 ch)
      SoftmaxK k2;
      k2.sc2 = f2_pack(sc, sc);
      k2.negm2 = f2_pack(neg_m, neg_m);
      k2.neg2p23 = f2_pack(-8388608.0f, -8388608.0f);
      float lsum = 0.0f;
#pragma unroll 1
      for (int m = 0; m < kTile / 32; ++m) {
        uint32_t pk[8];
        if (live & (1u << m)) {
          uint32_t sv[16];
          tmem_ld16x2_16<16>(s_base + 32u * m, sv);  // this thread's chunk 2m + kh
          tmem_wait_ld();
          regs_after_wait(sv);
          const int ch = 2 * m + kh;
          if constexpr (kAlibi) {
            // i - j for the chunk's first key; keys past the row (when causal) and past n are dropped
            const int jc = ms.j0 + 16 * ch;
            const int d0 = a_i0 + r - jc;
            lsum += p16_alibi(sv, lam * static_cast<float>(d0), lam, min(kCausal ? d0 : 16, n - 1 - jc), sc, neg_m, pk);
          } else {
            // the chunk's counts as the float bits of 2^23 + c, from the diagonal scan's bytes or
            // from the masks, then one P body for both (a second copy of it in the loop costs more
            // in instruction fetch than the extra integer work here)
            uint32_t cf[16];
            if (kind == 0 && m == quarter) {
              // the warp's own block on the diagonal: counts from the scan (words 4 kh .. 4 kh + 3)
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const uint32_t c4 = sm.cw[4 * kh + u][threadIdx.x];
#pragma unroll
                for (int e = 0; e < 4; ++e) cf[4 * u + e] = __byte_perm(c4, 0x4B000000u, 0x7540u | e);
              }
            } else {
              // c = popcount(keep & ~km[k]): the hashes with no block boundary between the row and key k
              const bool below = kind == 1 || (kind == 0 && m < quarter);
              const MaskT keep = below ? keep_lo : keep_hi;
              const MaskT* km = km_tile + 16 * ch;
#pragma unroll
              for (int g4 = 0; g4 < 4; ++g4) {
                MaskT bb[4];
                load4(km + 4 * g4, bb);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                  cf[4 * g4 + e] = 0x4B000000u | static_cast<uint32_t>(popc_m(static_cast<MaskT>(keep & ~bb[e])));
              }
            }
            lsum += p16_cf(sv, cf, k2, pk);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) pk[e] = 0u;
        }
        tmem_st16x2_8<8>(s_base + 16u * m, pk);
      }
      if (kAlibi) {
      } else if (kind == 1) {
        Y = static_cast<MaskT>(Y | ms.bm[0] | ms.suf[0]);  // OR over [j0, i]
      } else if (kind == 2) {
        Z = static_cast<MaskT>(Zc | ms.pre[kTile - 1]);    // OR over (i, j0 + 127]
      } else {
        Y = static_cast<MaskT>(ms.bm[0] | ms.pre[r]);      // OR over [i0, i]
        if (!kCausal) Z = ms.suf[r];                        // OR over (i, i0 + 127]
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.m_empty[st]);
      tmem_wait_st();
      l = l * alpha + lsum;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.p_full[g & 1]);

      if (last) {  // the item's epilogue runs at the top of the next iteration
        pend = true;
        pend_tx = tx;
        pend_g = g;
      }
    }
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

template <typename MaskT, bool kCausal, bool kVarlen, bool kAlibi>
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
  prm.sigma = a.sigma;
  prm.log_inv_eps = a.log_inv_eps;
  prm.wait_ns = wait_limit_ns();
  prm.withhold_mma = withhold_mma() ? 1 : 0;
  auto kern = attn_tc_kernel<MaskT, kCausal, kVarlen, kAlibi>;
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
  if (a.alibi)
    return a.causal ? launch_tc_typed<uint32_t, true, false, true>(a, st)
                    : launch_tc_typed<uint32_t, false, false, true>(a, st);
  if (a.varlen) {
    if (a.causal)
      return a.s <= 32 ? launch_tc_typed<uint32_t, true, true, false>(a, st)
                       : launch_tc_typed<unsigned long long, true, true, false>(a, st);
    return a.s <= 32 ? launch_tc_typed<uint32_t, false, true, false>(a, st)
                     : launch_tc_typed<unsigned long long, false, true, false>(a, st);
  }
  if (a.causal)
    return a.s <= 32 ? launch_tc_typed<uint32_t, true, false, false>(a, st)
                     : launch_tc_typed<unsigned long long, true, false, false>(a, st);
  return a.s <= 32 ? launch_tc_typed<uint32_t, false, false, false>(a, st)
                   : launch_tc_typed<unsigned long long, false, false, false>(a, st);
}

}  // namespace plsh
