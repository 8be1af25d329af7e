// Tensor-core backward of T~ for bf16 with d = 128: dQ, dK, dV with the (delta, u) table held
// fixed (plsh_attention_bwd_tc).
//
// T~ = P V with P_ij = c_ij e^{S_ij} / sum_l c_il e^{S_il} (Positional LSH technical summary,
// Methodology 2 and 3; the pages train and fine-tune models with this attention, Results,
// experimental validation). With the forward's row_sum L_i = ln(sum_j (c_ij / s) e^{S_ij}) the
// weights are recomputed exactly, P_ij = (c_ij / s) e^{S_ij - L_i}, and
//   dV = P^T dO,  dP = dO V^T,  D_i = dO_i . O_i,  dS = P o (dP - D),
//   dQ = dS K / sqrt d,  dK = dS^T Q / sqrt d.
// c_ij comes from the boundary masks exactly as in the fused forward kernel: blocks are
// contiguous (Methodology 1, structure), so c_ij = s - popcount(OR of the masks over
// (min(i, j), max(i, j)]), split into a per-row carry and a per-key part.
//
// Two kernels in the fused forward kernel's mould (a TMA warp, a single-thread tcgen05.mma
// issuer, a mask warp and eight elementwise warps; every wait bounded in time):
//   bwd_dq_tc_kernel    one item per (batch, query head, 128-row query tile), walking the key
//                       tiles of the forward's window: S = Q K^T and dP = dO V^T (SS MMAs), the
//                       elementwise warps write dS over S in Tensor Memory, dQ += dS K (TS MMA).
//   bwd_dkdv_tc_kernel  one item per (batch, KV head, 128-key tile), walking, for every query
//                       head of the group, the query tiles whose rows reach the key tile (the
//                       same windows by the symmetry of c_ij; only rows at or after the keys when
//                       causal): S^T = K Q^T and dP^T = V dO^T, the elementwise warps write P^T and
//                       dS^T over them, dV += P^T dO and dK += dS^T Q (TS MMAs).
// Tensor Memory holds S, dP and the accumulators (dQ; dV and dK): the score MMAs of a tile wait
// for the previous tile's gradient MMAs to read the elementwise results (one thread's MMAs run in
// order). An item's epilogue (the accumulators to global memory) runs after the next tile's
// mask-only work (the diagonal scan), so that the scan overlaps the item's last gradient MMAs.
// D_i comes from the existing row-dot kernel before both.
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
constexpr int kElemWarps = 8;
constexpr int kWarpTma = 8, kWarpMma = 9, kWarpMask = 10;
constexpr int kStages = 2;
constexpr int kMaskStages = 2;
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

struct BwdTcParams {
  int B, H, H_kv, n, s, causal, T, items;
  const int32_t* spans;  // [H][T][2]: dQ kernel, the forward's windows; dK/dV kernel, the non-causal ones
  uint64_t wait_ns;
};

// The query tiles of a dK/dV item (x = (g B + b) T + t: KV head g, batch b, key tile t), in the
// order every role walks them: the item is walked once per query head of its group (sub-item j:
// head g group + j) over that head's window: the key tile's own tile, then (non-causal only) the
// tiles before it, then the tiles after it.
struct KvIter {
  const BwdTcParams* p;
  int x, stride;
  int k;        // items started so far by this CTA
  int sub;      // query head of the group
  int it, total, n_below;
  int b, g, h, j0;  // batch, KV head, query head, the key tile's first key
  int gt;       // walked tiles so far by this CTA
  bool valid, bad_window;

  __device__ __forceinline__ int group() const { return p->H / p->H_kv; }
  __device__ __forceinline__ void load_sub() {
    h = g * group() + sub;
    const size_t at = (static_cast<size_t>(h) * p->T + j0 / kTile) * 2;
    int lo = p->spans[at], hi = p->spans[at + 1];
    const int last_key = min(p->n, j0 + kTile) - 1;
    bad_window = lo < 0 || lo > j0 || hi >= p->n || hi < last_key;
    lo = max(0, min(lo, j0));
    hi = min(p->n - 1, max(hi, last_key));
    n_below = p->causal ? 0 : (j0 - lo + kTile - 1) / kTile;
    total = 1 + n_below + (hi - j0) / kTile;
    it = 0;
  }
  __device__ __forceinline__ void load_item() {
    valid = x < p->items;
    if (!valid) return;
    const int BT = p->B * p->T;
    g = x / BT;
    b = (x % BT) / p->T;
    j0 = (x % p->T) * kTile;
    sub = 0;
    load_sub();
  }
  __device__ __forceinline__ void start(const BwdTcParams* pp) {
    p = pp;
    x = blockIdx.x;
    stride = gridDim.x;
    k = 0;
    gt = 0;
    load_item();
  }
  __device__ __forceinline__ void next() {
    ++gt;
    if (++it >= total) {
      if (sub + 1 < group()) {
        ++sub;
        load_sub();
      } else {
        x += stride;
        ++k;
        load_item();
      }
    }
  }
  __device__ __forceinline__ int kind() const { return it == 0 ? 0 : (it <= n_below ? 1 : 2); }
  // first query row of the walked tile
  __device__ __forceinline__ int i0() const {
    const int kd = kind();
    return kd == 0 ? j0 : (kd == 1 ? j0 - kTile * it : j0 + kTile * (it - n_below));
  }
  __device__ __forceinline__ bool first() const { return it == 0 && sub == 0; }
  __device__ __forceinline__ bool last() const { return it == total - 1 && sub == group() - 1; }
};

// dS = P (dP - D) for 16 keys with P = c 2^(S sc - bias) (S, dP as raw fp32 bits; cf[k] the float
// bits of 2^23 + c_k), packed as 8 bf16 pairs.
__device__ __forceinline__ void ds16_cf(const uint32_t (&sv)[16], const uint32_t (&dv)[16], const uint32_t (&cf)[16],
                                        uint64_t sc2, uint64_t nbias2, uint64_t nD2, uint32_t (&pk)[8]) {
  const uint64_t n2p23 = f2_pack(-8388608.0f, -8388608.0f);
#pragma unroll
  for (int g4 = 0; g4 < 4; ++g4) {
#pragma unroll
    for (int e2 = 0; e2 < 2; ++e2) {
      const int kk = 4 * g4 + 2 * e2;
      float x0, x1;
      f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[kk]), __uint_as_float(sv[kk + 1])), sc2, nbias2), x0, x1);
      const uint64_t w2 = f2_add(f2_pack(__uint_as_float(cf[kk]), __uint_as_float(cf[kk + 1])), n2p23);
      const uint64_t p2 = f2_mul(f2_pack(ex2_approx(x0), ex2_approx(x1)), w2);
      const uint64_t d2 = f2_add(f2_pack(__uint_as_float(dv[kk]), __uint_as_float(dv[kk + 1])), nD2);
      float s0, s1;
      f2_unpack(f2_mul(p2, d2), s0, s1);
      pk[2 * g4 + e2] = pack_bf16x2(s0, s1);
    }
  }
}

// Transposed form for the dK/dV kernel (rows are keys, columns query rows): p = c 2^(S sc -
// bias[col]) and ds = p (dP - D[col]) for 16 columns, with the per-column bias and D from shared
// memory; P and dS packed as bf16 pairs. w16: the 16 counts as floats.
__device__ __forceinline__ void pds16_cols(const uint32_t (&sv)[16], const uint32_t (&dv)[16], const float (&w16)[16],
                                           const float* nbias, const float* nD, uint64_t sc2, uint32_t (&pp)[8],
                                           uint32_t (&pd)[8]) {
#pragma unroll
  for (int g4 = 0; g4 < 4; ++g4) {
    const float4 nb = *reinterpret_cast<const float4*>(nbias + 4 * g4);
    const float4 nd = *reinterpret_cast<const float4*>(nD + 4 * g4);
#pragma unroll
    for (int e2 = 0; e2 < 2; ++e2) {
      const int kk = 4 * g4 + 2 * e2;
      const uint64_t nb2 = e2 ? f2_pack(nb.z, nb.w) : f2_pack(nb.x, nb.y);
      const uint64_t nd2 = e2 ? f2_pack(nd.z, nd.w) : f2_pack(nd.x, nd.y);
      float x0, x1;
      f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[kk]), __uint_as_float(sv[kk + 1])), sc2, nb2), x0, x1);
      const uint64_t p2 = f2_mul(f2_pack(ex2_approx(x0), ex2_approx(x1)), f2_pack(w16[kk], w16[kk + 1]));
      const uint64_t d2 = f2_add(f2_pack(__uint_as_float(dv[kk]), __uint_as_float(dv[kk + 1])), nd2);
      float p0, p1, s0, s1;
      f2_unpack(p2, p0, p1);
      f2_unpack(f2_mul(p2, d2), s0, s1);
      pp[2 * g4 + e2] = pack_bf16x2(p0, p1);
      pd[2 * g4 + e2] = pack_bf16x2(s0, s1);
    }
  }
}

// Counts of 16 keys as floats: popcount(keep & ~km[k]) (carry form) ...
template <typename MaskT>
__device__ __forceinline__ void w16_carry(const MaskT* km, MaskT keep, float (&w)[16]) {
#pragma unroll
  for (int g4 = 0; g4 < 4; ++g4) {
    MaskT bb[4];
    load4(km + 4 * g4, bb);
#pragma unroll
    for (int e = 0; e < 4; ++e)
      w[4 * g4 + e] = __int_as_float(0x4B000000u | static_cast<uint32_t>(popc_m(static_cast<MaskT>(keep & ~bb[e])))) -
                      8388608.0f;
  }
}

// ... or from bytes (the diagonal's own block).
__device__ __forceinline__ void w16_counts(const uint32_t (&c4)[4], float (&w)[16]) {
#pragma unroll
  for (int g4 = 0; g4 < 4; ++g4)
#pragma unroll
    for (int e = 0; e < 4; ++e)
      w[4 * g4 + e] = __int_as_float(__byte_perm(c4[g4], 0x4B000000u, 0x7540u | static_cast<uint32_t>(e))) -
                      8388608.0f;
}

// Epilogue of an accumulator: this thread's 64 columns of its row (threads t: columns 0..63,
// t + 16: 64..127; 16x32bx2 loads with a 64-column split) times `scale`, stored as bf16 four rows
// at a time by each lane quad.
__device__ __forceinline__ void store_rows(uint32_t acc_row, float scale, __nv_bfloat16* out, int row0, int quad_row,
                                          int n, int kh, int lane) {
  const int p4 = lane & 3;
  __nv_bfloat16* obase = out + 64 * kh;
#pragma unroll 1
  for (int blk = 0; blk < 2; ++blk) {
    uint32_t raw[32];
    tmem_ld16x2_32<64>(acc_row + 32u * blk, raw);
    tmem_wait_ld();
    regs_after_wait(raw);
    uint32_t a[4][4];
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
      for (int w = 0; w < 4; ++w)
        a[c][w] = pack_bf16x2(__uint_as_float(raw[8 * c + 2 * w]) * scale, __uint_as_float(raw[8 * c + 2 * w + 1]) * scale);
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
      const int row = row0 + quad_row + e;
      if (row < n)
        *reinterpret_cast<uint4*>(obase + static_cast<size_t>(row) * kD + 32 * blk + 8 * p4) =
            make_uint4(a[e][0], a[e][1], a[e][2], a[e][3]);
    }
  }
}

// ================================================================ dQ

template <typename MaskT>
struct __align__(1024) DqSmem {
  uint8_t q[kTileBytes];
  uint8_t dO[kTileBytes];
  uint8_t k[kStages][kTileBytes];
  uint8_t v[kStages][kTileBytes];
  MaskStage<MaskT> m[kMaskStages];
  uint32_t cw[8][kElemWarps * 32];
  int16_t order[kMaxSortedHeads];
  int32_t width[kMaxSortedHeads];
  uint64_t q_full, q_empty;
  uint64_t k_full[kStages], k_empty[kStages], v_full[kStages], v_empty[kStages];
  uint64_t m_full[kMaskStages], m_empty[kMaskStages];
  uint64_t s_full, p_full, g_done;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

static_assert(sizeof(DqSmem<unsigned long long>) + 1024 <= 232448, "shared memory budget");

// Heads by decreasing window width of their middle tile, ties by head index (the same order in every
// CTA), into order[] (the item list starts with the widest heads).
__device__ __forceinline__ void sort_heads(const int32_t* spans, int H, int T, int16_t* order, int32_t* width) {
  if (H > kMaxSortedHeads) return;
  const int tm = T / 2;
  for (int h = threadIdx.x; h < H; h += kThreads) {
    const size_t at = (static_cast<size_t>(h) * T + tm) * 2;
    width[h] = spans[at + 1] - spans[at];
  }
  __syncthreads();
  for (int h = threadIdx.x; h < H; h += kThreads) {
    const int wh = width[h];
    int rank = 0;
    for (int o = 0; o < H; ++o) {
      const int wo = width[o];
      rank += (wo > wh) || (wo == wh && o < h);
    }
    order[rank] = static_cast<int16_t>(h);
  }
}

template <typename MaskT, bool kCausal>
__global__ void __launch_bounds__(kThreads, 1)
bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_do,
                 const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                 const __grid_constant__ Params prm, const MaskT* __restrict__ bmask,
                 const float* __restrict__ row_sum, const float* __restrict__ delta,
                 __nv_bfloat16* __restrict__ dQ, uint32_t* __restrict__ err) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t smem_pad = (1024u - (static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw)) & 1023u)) & 1023u;
  auto& sm = *reinterpret_cast<DqSmem<MaskT>*>(smem_raw + smem_pad);
  volatile int* abort_flag = &sm.abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = prm.n, s = prm.s, H = prm.H;
  const uint64_t wait_ns = prm.wait_ns;
  const MaskT FULL = (s >= static_cast<int>(8 * sizeof(MaskT))) ? static_cast<MaskT>(~static_cast<MaskT>(0))
                                                              : static_cast<MaskT>((static_cast<MaskT>(1) << s) - 1);
  sort_heads(prm.spans, H, prm.T, sm.order, sm.width);
  if (threadIdx.x == 0) {
    sm.abort_flag = 0;
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_empty, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sm.k_full[i], 1);
      mbar_init(&sm.k_empty[i], 1);
      mbar_init(&sm.v_full[i], 1);
      mbar_init(&sm.v_empty[i], 1);
    }
    for (int i = 0; i < kMaskStages; ++i) {
      mbar_init(&sm.m_full[i], 1);
      mbar_init(&sm.m_empty[i], kElemWarps);
    }
    mbar_init(&sm.s_full, 1);
    mbar_init(&sm.p_full, kElemWarps);
    mbar_init(&sm.g_done, 1);
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
  // S (then dS) of tile g at columns 0 or 384 by g's parity, dP at 128, the dQ accumulator at 256
  constexpr uint32_t kColS = 0, kColDP = 128, kColAcc = 256, kColS1 = 384;

  if (warp == kWarpTma) {
    // ------------------------------------------------------------ TMA: Q and dO per item, K and V per tile
    if (lane == 0) {
      tma_prefetch_desc(&tmap_q);
      tma_prefetch_desc(&tmap_do);
      tma_prefetch_desc(&tmap_k);
      tma_prefetch_desc(&tmap_v);
      TileIter<false, false> ti;
      ti.start(&prm, sm.order);
      int issued_q = 0, issued_k = 0, issued_v = 0;
      while (ti.valid) {
        const int zkv = ti.b * prm.H_kv + ti.h / (H / prm.H_kv);
        if (ti.first()) {
          if (ti.k >= 1 && !mbar_wait(&sm.q_empty, static_cast<uint32_t>(ti.k - 1) & 1u, abort_flag, err, wait_ns)) break;
          mbar_arrive_expect_tx(&sm.q_full, 2 * kTileBytes);
          const int zq = ti.b * H + ti.h;
          tma_load_3d(sm.q, &tmap_q, 0, ti.i0, zq, &sm.q_full);
          tma_load_3d(sm.q + kChunkBytes, &tmap_q, 64, ti.i0, zq, &sm.q_full);
          tma_load_3d(sm.dO, &tmap_do, 0, ti.i0, zq, &sm.q_full);
          tma_load_3d(sm.dO + kChunkBytes, &tmap_do, 64, ti.i0, zq, &sm.q_full);
          issued_q = ti.k + 1;
        }
        const int st = ti.g % kStages;
        const uint32_t ph = static_cast<uint32_t>(ti.g / kStages) & 1u;
        const int j0 = ti.j0();
        if (ti.g >= kStages && !mbar_wait(&sm.k_empty[st], ph ^ 1u, abort_flag, err, wait_ns)) break;
        mbar_arrive_expect_tx(&sm.k_full[st], kTileBytes);
        tma_load_3d(sm.k[st], &tmap_k, 0, j0, zkv, &sm.k_full[st]);
        tma_load_3d(sm.k[st] + kChunkBytes, &tmap_k, 64, j0, zkv, &sm.k_full[st]);
        issued_k = ti.g + 1;
        if (ti.g >= kStages && !mbar_wait(&sm.v_empty[st], ph ^ 1u, abort_flag, err, wait_ns)) break;
        mbar_arrive_expect_tx(&sm.v_full[st], kTileBytes);
        tma_load_3d(sm.v[st], &tmap_v, 0, j0, zkv, &sm.v_full[st]);
        tma_load_3d(sm.v[st] + kChunkBytes, &tmap_v, 64, j0, zkv, &sm.v_full[st]);
        issued_v = ti.g + 1;
        ti.next();
      }
      if (*abort_flag) {
        if (issued_q > 0) mbar_wait_drain(&sm.q_full, static_cast<uint32_t>(issued_q - 1) & 1u, kDrainNs);
        for (int gg = (issued_k > kStages ? issued_k - kStages : 0); gg < issued_k; ++gg)
          mbar_wait_drain(&sm.k_full[gg % kStages], static_cast<uint32_t>(gg / kStages) & 1u, kDrainNs);
        for (int gg = (issued_v > kStages ? issued_v - kStages : 0); gg < issued_v; ++gg)
          mbar_wait_drain(&sm.v_full[gg % kStages], static_cast<uint32_t>(gg / kStages) & 1u, kDrainNs);
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    // Per tile g: S(g) = Q K^T into the S buffer of g's parity, dP(g) = dO V^T; once dS(g) is written
    // over S(g): dQ += dS(g) K. S(g+1) is issued before waiting for dS(g), so it computes while the
    // elementwise warps work on tile g, and dP(g+1) right after dS(g), before dQ's MMAs, so the
    // elementwise warps wait for one MMA between tiles. S(g+2) reuses dS(g)'s buffer and follows
    // dQ(g)'s MMAs in issue order, so it overwrites dS only after dQ has read it.
    if (lane == 0) {
      constexpr uint32_t idesc_nt = idesc_bf16_f32(128, 128, 0);  // B K-major (S, dP)
      constexpr uint32_t idesc_nn = idesc_bf16_f32(128, 128, 1);  // B MN-major (dQ += dS K)
      const uint64_t q_desc = smem_desc_sw128(smem_u32(sm.q), 16, 1024);
      const uint64_t do_desc = smem_desc_sw128(smem_u32(sm.dO), 16, 1024);
      uint64_t k_desc[kStages], v_desc[kStages], kmn_desc[kStages];
      for (int i = 0; i < kStages; ++i) {
        k_desc[i] = smem_desc_sw128(smem_u32(sm.k[i]), 16, 1024);
        v_desc[i] = smem_desc_sw128(smem_u32(sm.v[i]), 16, 1024);
        kmn_desc[i] = smem_desc_sw128(smem_u32(sm.k[i]), kChunkBytes, 1024);
      }
      auto s_col = [&](int g) { return (g & 1) ? kColS1 : kColS; };
      // S(t) = Q K^T (waits for the item's Q and the tile's K)
      auto issue_s = [&](const TileIter<false, false>& t) -> bool {
        const int st = t.g % kStages;
        if (t.first() && !mbar_wait(&sm.q_full, static_cast<uint32_t>(t.k) & 1u, abort_flag, err, wait_ns)) return false;
        if (!mbar_wait(&sm.k_full[st], static_cast<uint32_t>(t.g / kStages) & 1u, abort_flag, err, wait_ns)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>(((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4);
          mma_ss(tmem + s_col(t.g), q_desc + off, (st ? k_desc[1] : k_desc[0]) + off, idesc_nt, kk > 0 ? 1u : 0u);
        }
        return true;
      };
      // dP(t) = dO V^T, then s_full (S(t) and dP(t) complete)
      auto issue_dp = [&](const TileIter<false, false>& t) -> bool {
        const int st = t.g % kStages;
        if (!mbar_wait(&sm.v_full[st], static_cast<uint32_t>(t.g / kStages) & 1u, abort_flag, err, wait_ns)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>(((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4);
          mma_ss(tmem + kColDP, do_desc + off, (st ? v_desc[1] : v_desc[0]) + off, idesc_nt, kk > 0 ? 1u : 0u);
        }
        mma_commit(&sm.s_full);
        mma_commit(&sm.v_empty[st]);
        if (t.last()) mma_commit(&sm.q_empty);  // the item's Q and dO are no longer read
        return true;
      };
      TileIter<false, false> cur, nxt;
      cur.start(&prm, sm.order);
      nxt.start(&prm, sm.order);
      if (nxt.valid) nxt.next();
      bool ok = !cur.valid || (issue_s(cur) && issue_dp(cur));
      while (ok && cur.valid) {
        const int st = cur.g % kStages;
        // the next tile's scores, unless they need the next item's Q (loaded once this item's last
        // scores are done)
        const bool s_early = nxt.valid && !nxt.first();
        if (s_early && !(ok = issue_s(nxt))) break;
        if (!(ok = mbar_wait(&sm.p_full, static_cast<uint32_t>(cur.g) & 1u, abort_flag, err, wait_ns))) break;
        tc_fence_after();
        auto issue_dq = [&]() {
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            mma_ts(tmem + kColAcc, tmem + s_col(cur.g) + 8u * kk,
                   (st ? kmn_desc[1] : kmn_desc[0]) + static_cast<uint64_t>((kk * 2048) >> 4), idesc_nn,
                   (!cur.first() || kk > 0) ? 1u : 0u);
          mma_commit(&sm.k_empty[st]);
        };
        if (s_early) {  // within an item: the next tile's dP first, which the elementwise warps wait for
          if (!(ok = issue_dp(nxt))) break;
          issue_dq();
        } else {        // the item's last tile: its dQ first, which the item's epilogue waits for
          issue_dq();
          mma_commit(&sm.g_done);  // once per item: the item's dQ is complete
          if (nxt.valid && !(ok = issue_s(nxt) && issue_dp(nxt))) break;
        }
        cur.next();
        if (nxt.valid) nxt.next();
      }
      mma_commit(&sm.drain);
      mbar_wait_drain(&sm.drain, 0, kDrainNs);
    }
  } else if (warp == kWarpMask) {
    // ------------------------------------------------------------ mask warp (as in the forward)
    TileIter<false, false> ti, nx;
    ti.start(&prm, sm.order);
    nx.start(&prm, sm.order);
    if (nx.valid) nx.next();
    auto load_masks = [&](const TileIter<false, false>& t, MaskT (&v)[4], MaskT& v128) {
      const MaskT* bm_h = bmask + static_cast<size_t>(t.h) * n;
      const int j0 = t.j0();
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = j0 + 4 * lane + e;
        v[e] = (j >= 0 && j < n) ? bm_h[j] : FULL;
      }
      const int j = j0 + kTile;
      v128 = (lane == 0 && j >= 0 && j < n) ? bm_h[j] : FULL;
    };
    MaskT xv[4] = {FULL, FULL, FULL, FULL}, x128 = FULL;
    if (ti.valid) load_masks(ti, xv, x128);
    int g_end = 0;
    bool ok = true;
    while (ti.valid) {
      const int st = ti.g % kMaskStages;
      MaskT nv[4] = {FULL, FULL, FULL, FULL}, n128 = FULL;
      if (nx.valid) load_masks(nx, nv, n128);
      if (ti.g >= kMaskStages) {
        ok = mbar_wait(&sm.m_empty[st], (static_cast<uint32_t>(ti.g / kMaskStages) & 1u) ^ 1u, abort_flag, err, wait_ns);
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
        ms.sub = 0;
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
    if (ok && !*abort_flag) {
      const int st = g_end % kMaskStages;
      ok = g_end < kMaskStages ||
           mbar_wait(&sm.m_empty[st], (static_cast<uint32_t>(g_end / kMaskStages) & 1u) ^ 1u, abort_flag, err, wait_ns);
      if (__all_sync(0xffffffffu, ok) && lane == 0) {
        sm.m[st].valid = 0;
        mbar_arrive(&sm.m_full[st]);
      }
    }
  } else {
    // ------------------------------------------------------------ elementwise: dS = P o (dP - D)
    // Warp w owns rows 32 (w % 4) + 16 (w / 4) .. + 15; threads t and t + 16 share row t % 16 and
    // split each pair of 16-key chunks (the 16x32bx2 TMEM access shape), as in the forward.
    const int quarter = warp & 3;
    const int hq = warp >> 2;
    const int kh = lane >> 4;
    const int r = quarter * 32 + hq * 16 + (lane & 15);
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32 + hq * 16) << 16;
    const uint32_t dp_base = tmem + lane_off + kColDP;
    const float sc = kLog2e / sqrtf(static_cast<float>(kD));
    const float log2s = log2f(static_cast<float>(s));
    const uint64_t sc2 = f2_pack(sc, sc);
    uint64_t nbias2 = 0, nD2 = 0;
    MaskT Y = 0, Z = 0;
    int bb = 0, hh = 0, i0 = 0;
    bool pend = false;  // an item's epilogue is pending (the item of bb, hh, i0)
    int items = 0;      // items whose epilogue is done
    for (int g = 0;; ++g) {
      const int st = g % kMaskStages;
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.m_full[st], static_cast<uint32_t>(g / kMaskStages) & 1u,
                                             abort_flag, err, wait_ns)))
        break;
      const MaskStage<MaskT>& ms = sm.m[st];
      const bool valid = ms.valid != 0;
      const int kind = ms.kind, first = ms.first, last = ms.last, tx = ms.x;
      // the mask-only work first, while the previous item's last dQ MMA runs
      MaskT lo = 0, hi = 0;
      if (valid && kind == 0) diag_scan<MaskT, true, !kCausal>(ms, quarter, r, s, &sm.cw[0][threadIdx.x], kElemWarps * 32, lo, hi);
      if (pend) {
        pend = false;
        // the previous item's dQ once its last MMA has completed (g_done completes once per item,
        // and the next completion needs this item's successor's dS, so one parity wait is exact):
        // dQ / sqrt(d)
        if (!__all_sync(0xffffffffu, mbar_wait(&sm.g_done, static_cast<uint32_t>(items) & 1u, abort_flag, err, wait_ns)))
          break;
        ++items;
        tc_fence_after();
        store_rows(tmem + lane_off + kColAcc, 1.0f / sqrtf(static_cast<float>(kD)),
                   dQ + (static_cast<size_t>(bb) * H + hh) * static_cast<size_t>(n) * kD, i0,
                   quarter * 32 + hq * 16 + ((lane & 15) & ~3), n, kh, lane);
        tc_fence_before();
      }
      if (!valid) break;
      if (first) {
        // P_ij = c_ij 2^(S_ij log2(e)/sqrt(d) - (L_i log2(e) + log2 s)); rows past n get L = D = 0
        const int BT = prm.B * prm.T;
        hh = (H <= kMaxSortedHeads) ? static_cast<int>(sm.order[tx / BT]) : tx / BT;
        bb = (tx % BT) / prm.T;
        i0 = ((tx % BT) % prm.T) * kTile;
        const int i = i0 + r;
        const size_t at = (static_cast<size_t>(bb) * H + hh) * n + i;
        const float L = i < n ? row_sum[at] : 0.0f;
        const float Dv = i < n ? delta[at] : 0.0f;
        const float nb = -(L * kLog2e + log2s);
        nbias2 = f2_pack(nb, nb);
        nD2 = f2_pack(-Dv, -Dv);
      }
      const int n_pairs = (kCausal && kind == 0) ? quarter + 1 : kTile / 32;
      const MaskT Zc = static_cast<MaskT>(Z | ms.bm[0]);
      const MaskT keep_lo = static_cast<MaskT>(FULL & ~(kind == 1 ? Y : lo));
      const MaskT keep_hi = static_cast<MaskT>(FULL & ~(kind == 2 ? Zc : hi));
      const MaskT* km_tile = kind == 1 ? ms.suf : (kind == 2 ? ms.pre : ms.dq[quarter]);
      uint32_t live = 0;
#pragma unroll
      for (int m = 0; m < kTile / 32; ++m) {
        bool lv = m < n_pairs;
        if (lv && !(kind == 0 && m == quarter)) {
          const bool below = kind == 1 || (kind == 0 && m < quarter);
          const MaskT kn = km_tile[below ? 32 * m + 31 : 32 * m];
          lv = static_cast<MaskT>((below ? keep_lo : keep_hi) & ~kn) != 0;
        }
        if (__any_sync(0xffffffffu, lv)) live |= 1u << m;
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full, static_cast<uint32_t>(g) & 1u, abort_flag, err, wait_ns)))
        break;
      tc_fence_after();
      const uint32_t s_base = tmem + lane_off + ((g & 1) ? kColS1 : kColS);  // S(g), then dS(g)
#pragma unroll 1
      for (int m = 0; m < kTile / 32; ++m) {
        uint32_t pk[8];
        if (live & (1u << m)) {
          uint32_t sv[16], dv[16];
          tmem_ld16x2_16<16>(s_base + 32u * m, sv);
          tmem_ld16x2_16<16>(dp_base + 32u * m, dv);
          tmem_wait_ld();
          regs_after_wait(sv);
          regs_after_wait(dv);
          const int ch = 2 * m + kh;
          // the chunk's counts as the float bits of 2^23 + c, from the diagonal scan's bytes or from
          // the masks, then one dS body for both (a smaller loop than two inlined bodies)
          uint32_t cf[16];
          if (kind == 0 && m == quarter) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const uint32_t c4 = sm.cw[4 * kh + u][threadIdx.x];
#pragma unroll
              for (int e = 0; e < 4; ++e) cf[4 * u + e] = __byte_perm(c4, 0x4B000000u, 0x7540u | e);
            }
          } else {
            const bool below = kind == 1 || (kind == 0 && m < quarter);
            const MaskT keep = below ? keep_lo : keep_hi;
            const MaskT* km = km_tile + 16 * ch;
#pragma unroll
            for (int g4 = 0; g4 < 4; ++g4) {
              MaskT kb4[4];
              load4(km + 4 * g4, kb4);
#pragma unroll
              for (int e = 0; e < 4; ++e)
                cf[4 * g4 + e] = 0x4B000000u | static_cast<uint32_t>(popc_m(static_cast<MaskT>(keep & ~kb4[e])));
            }
          }
          ds16_cf(sv, dv, cf, sc2, nbias2, nD2, pk);
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) pk[e] = 0u;
        }
        tmem_st16x2_8<8>(s_base + 16u * m, pk);
      }
      if (kind == 1) {
        Y = static_cast<MaskT>(Y | ms.bm[0] | ms.suf[0]);
      } else if (kind == 2) {
        Z = static_cast<MaskT>(Zc | ms.pre[kTile - 1]);
      } else {
        Y = static_cast<MaskT>(ms.bm[0] | ms.pre[r]);
        if (!kCausal) Z = ms.suf[r];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.m_empty[st]);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.p_full);
      if (last) pend = true;  // the item's epilogue runs at the top of the next iteration
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

// ================================================================ dK, dV

// A walked query tile as the elementwise warps need it: its masks, and per query row (column) of
// the tile -(L log2(e) + log2 s) and -D.
template <typename MaskT>
struct alignas(16) KvStage {
  MaskStage<MaskT> m;
  float nbias[kTile];
  float nD[kTile];
};

template <typename MaskT>
struct __align__(1024) KvSmem {
  uint8_t k[kTileBytes];
  uint8_t v[kTileBytes];
  uint8_t q[kStages][kTileBytes];
  uint8_t dO[kStages][kTileBytes];
  KvStage<MaskT> m[kMaskStages];
  uint32_t cw[8][kElemWarps * 32];
  uint64_t kv_full, kv_empty;
  uint64_t qd_full[kStages], qd_empty[kStages];
  uint64_t m_full[kMaskStages], m_empty[kMaskStages];
  uint64_t s_full, p_full, g_done;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

static_assert(sizeof(KvSmem<unsigned long long>) + 1024 <= 232448, "shared memory budget");

template <typename MaskT, bool kCausal>
__global__ void __launch_bounds__(kThreads, 1)
bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_do,
                   const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                   const __grid_constant__ BwdTcParams prm, const MaskT* __restrict__ bmask,
                   const float* __restrict__ row_sum, const float* __restrict__ delta,
                   __nv_bfloat16* __restrict__ dK, __nv_bfloat16* __restrict__ dV, uint32_t* __restrict__ err) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t smem_pad = (1024u - (static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw)) & 1023u)) & 1023u;
  auto& sm = *reinterpret_cast<KvSmem<MaskT>*>(smem_raw + smem_pad);
  volatile int* abort_flag = &sm.abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = prm.n, s = prm.s, H = prm.H;
  const uint64_t wait_ns = prm.wait_ns;
  const MaskT FULL = (s >= static_cast<int>(8 * sizeof(MaskT))) ? static_cast<MaskT>(~static_cast<MaskT>(0))
                                                              : static_cast<MaskT>((static_cast<MaskT>(1) << s) - 1);
  if (threadIdx.x == 0) {
    sm.abort_flag = 0;
    mbar_init(&sm.kv_full, 1);
    mbar_init(&sm.kv_empty, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sm.qd_full[i], 1);
      mbar_init(&sm.qd_empty[i], 1);
    }
    for (int i = 0; i < kMaskStages; ++i) {
      mbar_init(&sm.m_full[i], 1);
      mbar_init(&sm.m_empty[i], kElemWarps);
    }
    mbar_init(&sm.s_full, 1);
    mbar_init(&sm.p_full, kElemWarps);
    mbar_init(&sm.g_done, 1);
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
  constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 384;

  if (warp == kWarpTma) {
    // ------------------------------------------------------------ TMA: K and V per item, Q and dO per tile
    if (lane == 0) {
      tma_prefetch_desc(&tmap_q);
      tma_prefetch_desc(&tmap_do);
      tma_prefetch_desc(&tmap_k);
      tma_prefetch_desc(&tmap_v);
      KvIter ti;
      ti.start(&prm);
      int issued_kv = 0, issued_qd = 0;
      while (ti.valid) {
        if (ti.first()) {
          if (ti.k >= 1 && !mbar_wait(&sm.kv_empty, static_cast<uint32_t>(ti.k - 1) & 1u, abort_flag, err, wait_ns)) break;
          mbar_arrive_expect_tx(&sm.kv_full, 2 * kTileBytes);
          const int zkv = ti.b * prm.H_kv + ti.g;
          tma_load_3d(sm.k, &tmap_k, 0, ti.j0, zkv, &sm.kv_full);
          tma_load_3d(sm.k + kChunkBytes, &tmap_k, 64, ti.j0, zkv, &sm.kv_full);
          tma_load_3d(sm.v, &tmap_v, 0, ti.j0, zkv, &sm.kv_full);
          tma_load_3d(sm.v + kChunkBytes, &tmap_v, 64, ti.j0, zkv, &sm.kv_full);
          issued_kv = ti.k + 1;
        }
        const int st = ti.gt % kStages;
        const uint32_t ph = static_cast<uint32_t>(ti.gt / kStages) & 1u;
        if (ti.gt >= kStages && !mbar_wait(&sm.qd_empty[st], ph ^ 1u, abort_flag, err, wait_ns)) break;
        mbar_arrive_expect_tx(&sm.qd_full[st], 2 * kTileBytes);
        const int zq = ti.b * H + ti.h, i0 = ti.i0();
        tma_load_3d(sm.q[st], &tmap_q, 0, i0, zq, &sm.qd_full[st]);
        tma_load_3d(sm.q[st] + kChunkBytes, &tmap_q, 64, i0, zq, &sm.qd_full[st]);
        tma_load_3d(sm.dO[st], &tmap_do, 0, i0, zq, &sm.qd_full[st]);
        tma_load_3d(sm.dO[st] + kChunkBytes, &tmap_do, 64, i0, zq, &sm.qd_full[st]);
        issued_qd = ti.gt + 1;
        ti.next();
      }
      if (*abort_flag) {
        if (issued_kv > 0) mbar_wait_drain(&sm.kv_full, static_cast<uint32_t>(issued_kv - 1) & 1u, kDrainNs);
        for (int gg = (issued_qd > kStages ? issued_qd - kStages : 0); gg < issued_qd; ++gg)
          mbar_wait_drain(&sm.qd_full[gg % kStages], static_cast<uint32_t>(gg / kStages) & 1u, kDrainNs);
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    // Per walked tile: S^T = K Q^T, dP^T = V dO^T; once P^T and dS^T are written over them:
    // dV += P^T dO, dK += dS^T Q. The next tile's S^T and dP^T follow in issue order.
    if (lane == 0) {
      constexpr uint32_t idesc_nt = idesc_bf16_f32(128, 128, 0);
      constexpr uint32_t idesc_nn = idesc_bf16_f32(128, 128, 1);
      const uint64_t k_desc = smem_desc_sw128(smem_u32(sm.k), 16, 1024);
      const uint64_t v_desc = smem_desc_sw128(smem_u32(sm.v), 16, 1024);
      uint64_t q_desc[kStages], do_desc[kStages], qmn_desc[kStages], domn_desc[kStages];
      for (int i = 0; i < kStages; ++i) {
        q_desc[i] = smem_desc_sw128(smem_u32(sm.q[i]), 16, 1024);
        do_desc[i] = smem_desc_sw128(smem_u32(sm.dO[i]), 16, 1024);
        qmn_desc[i] = smem_desc_sw128(smem_u32(sm.q[i]), kChunkBytes, 1024);
        domn_desc[i] = smem_desc_sw128(smem_u32(sm.dO[i]), kChunkBytes, 1024);
      }
      KvIter ti;
      ti.start(&prm);
      bool ok = true;
      while (ok && ti.valid) {
        const int st = ti.gt % kStages;
        if (ti.first() && !(ok = mbar_wait(&sm.kv_full, static_cast<uint32_t>(ti.k) & 1u, abort_flag, err, wait_ns)))
          break;
        if (!(ok = mbar_wait(&sm.qd_full[st], static_cast<uint32_t>(ti.gt / kStages) & 1u, abort_flag, err, wait_ns)))
          break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>(((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4);
          mma_ss(tmem + kColS, k_desc + off, (st ? q_desc[1] : q_desc[0]) + off, idesc_nt, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>(((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4);
          mma_ss(tmem + kColDP, v_desc + off, (st ? do_desc[1] : do_desc[0]) + off, idesc_nt, kk > 0 ? 1u : 0u);
        }
        mma_commit(&sm.s_full);
        if (ti.last()) mma_commit(&sm.kv_empty);
        if (!(ok = mbar_wait(&sm.p_full, static_cast<uint32_t>(ti.gt) & 1u, abort_flag, err, wait_ns))) break;
        tc_fence_after();
        const uint32_t acc = (!ti.first()) ? 1u : 0u;
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          mma_ts(tmem + kColDV, tmem + kColS + 8u * kk,
                 (st ? domn_desc[1] : domn_desc[0]) + static_cast<uint64_t>((kk * 2048) >> 4), idesc_nn,
                 (acc || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          mma_ts(tmem + kColDK, tmem + kColDP + 8u * kk,
                 (st ? qmn_desc[1] : qmn_desc[0]) + static_cast<uint64_t>((kk * 2048) >> 4), idesc_nn,
                 (acc || kk > 0) ? 1u : 0u);
        mma_commit(&sm.g_done);
        mma_commit(&sm.qd_empty[st]);
        ti.next();
      }
      mma_commit(&sm.drain);
      mbar_wait_drain(&sm.drain, 0, kDrainNs);
    }
  } else if (warp == kWarpMask) {
    // ------------------------------------------------------------ mask warp: the walked tile's masks
    // (of the sub-item's query head) and its rows' -(L log2 e + log2 s), -D
    const float log2s = log2f(static_cast<float>(s));
    KvIter ti;
    ti.start(&prm);
    int g_end = 0;
    bool ok = true;
    while (ti.valid) {
      const int st = ti.gt % kMaskStages;
      MaskT xv[4], x128;
      {
        const MaskT* bm_h = bmask + static_cast<size_t>(ti.h) * n;
        const int j0 = ti.i0();
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = j0 + 4 * lane + e;
          xv[e] = (j >= 0 && j < n) ? bm_h[j] : FULL;
        }
        const int j = j0 + kTile;
        x128 = (lane == 0 && j >= 0 && j < n) ? bm_h[j] : FULL;
      }
      float nb[4], nd[4];
      {
        const size_t row0 = (static_cast<size_t>(ti.b) * H + ti.h) * n;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = ti.i0() + 4 * lane + e;
          nb[e] = i < n ? -(row_sum[row0 + i] * kLog2e + log2s) : -log2s;
          nd[e] = i < n ? -delta[row0 + i] : 0.0f;
        }
      }
      if (ti.gt >= kMaskStages) {
        ok = mbar_wait(&sm.m_empty[st], (static_cast<uint32_t>(ti.gt / kMaskStages) & 1u) ^ 1u, abort_flag, err, wait_ns);
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
      }
      KvStage<MaskT>& ks = sm.m[st];
      publish_masks<MaskT, !kCausal, true>(ks.m, xv, x128, ti.kind() == 0, lane);
      *reinterpret_cast<float4*>(ks.nbias + 4 * lane) = make_float4(nb[0], nb[1], nb[2], nb[3]);
      *reinterpret_cast<float4*>(ks.nD + 4 * lane) = make_float4(nd[0], nd[1], nd[2], nd[3]);
      if (lane == 0) {
        ks.m.valid = 1;
        ks.m.kind = ti.kind();
        ks.m.first = ti.first() ? 1 : 0;
        ks.m.last = ti.last() ? 1 : 0;
        ks.m.x = ti.x;
        ks.m.j0 = ti.i0();
        ks.m.sub = ti.sub;
        if (ti.it == 0 && ti.bad_window) atomicOr(err, PLSH_DEVERR_WINDOW);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.m_full[st]);
      g_end = ti.gt + 1;
      ti.next();
    }
    if (ok && !*abort_flag) {
      const int st = g_end % kMaskStages;
      ok = g_end < kMaskStages ||
           mbar_wait(&sm.m_empty[st], (static_cast<uint32_t>(g_end / kMaskStages) & 1u) ^ 1u, abort_flag, err, wait_ns);
      if (__all_sync(0xffffffffu, ok) && lane == 0) {
        sm.m[st].m.valid = 0;
        mbar_arrive(&sm.m_full[st]);
      }
    }
  } else {
    // ------------------------------------------------------------ elementwise: P^T and dS^T
    // Rows are the item's keys (TMEM lanes), columns the walked tile's query rows; warp and thread
    // layout as in the dQ kernel. The counts are symmetric in (i, j), so the forward's carries
    // apply with the roles of rows and keys exchanged; when causal only query rows at or after a
    // key count (the diagonal tile's columns before the key, and no tiles before the item's own).
    const int quarter = warp & 3;
    const int hq = warp >> 2;
    const int kh = lane >> 4;
    const int r = quarter * 32 + hq * 16 + (lane & 15);
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32 + hq * 16) << 16;
    const uint32_t s_base = tmem + lane_off + kColS, dp_base = tmem + lane_off + kColDP;
    const float sc = kLog2e / sqrtf(static_cast<float>(kD));
    const uint64_t sc2 = f2_pack(sc, sc);
    MaskT Y = 0, Z = 0;
    bool pend = false;  // an item's epilogue is pending (item pend_tx, last tile pend_g; g_done completes
                        // once per tile, and tile pend_g + 1's MMAs wait for these warps, so one
                        // parity wait is exact)
    int pend_g = 0, pend_tx = 0;
    for (int g = 0;; ++g) {
      const int st = g % kMaskStages;
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.m_full[st], static_cast<uint32_t>(g / kMaskStages) & 1u,
                                             abort_flag, err, wait_ns)))
        break;
      const KvStage<MaskT>& ks = sm.m[st];
      const MaskStage<MaskT>& ms = ks.m;
      const bool valid = ms.valid != 0;
      const int kind = ms.kind, last = ms.last, tx = ms.x;
      // the mask-only work first, while the previous item's last MMAs run
      MaskT lo = 0, hi = 0;
      if (valid && kind == 0) diag_scan<MaskT, !kCausal, true>(ms, quarter, r, s, &sm.cw[0][threadIdx.x], kElemWarps * 32, lo, hi);
      if (pend) {
        pend = false;
        // the previous item's dV and dK once its last MMAs have completed (dK / sqrt(d))
        if (!__all_sync(0xffffffffu, mbar_wait(&sm.g_done, static_cast<uint32_t>(pend_g) & 1u, abort_flag, err, wait_ns)))
          break;
        tc_fence_after();
        const int BT = prm.B * prm.T;
        const int gg = pend_tx / BT, bb = (pend_tx % BT) / prm.T, j0 = (pend_tx % prm.T) * kTile;
        const size_t plane = (static_cast<size_t>(bb) * prm.H_kv + gg) * static_cast<size_t>(n) * kD;
        const int quad_row = quarter * 32 + hq * 16 + ((lane & 15) & ~3);
        store_rows(tmem + lane_off + kColDV, 1.0f, dV + plane, j0, quad_row, n, kh, lane);
        store_rows(tmem + lane_off + kColDK, 1.0f / sqrtf(static_cast<float>(kD)), dK + plane, j0, quad_row, n, kh, lane);
        tc_fence_before();
      }
      if (!valid) break;
      const MaskT Zc = static_cast<MaskT>(Z | ms.bm[0]);
      const MaskT keep_lo = static_cast<MaskT>(FULL & ~(kind == 1 ? Y : lo));
      const MaskT keep_hi = static_cast<MaskT>(FULL & ~(kind == 2 ? Zc : hi));
      const MaskT* km_tile = kind == 1 ? ms.suf : (kind == 2 ? ms.pre : ms.dq[quarter]);
      uint32_t live = 0;
#pragma unroll
      for (int m = 0; m < kTile / 32; ++m) {
        bool lv = !(kCausal && kind == 0 && m < quarter);
        if (lv && !(kind == 0 && m == quarter)) {
          const bool below = kind == 1 || (kind == 0 && m < quarter);
          const MaskT kn = km_tile[below ? 32 * m + 31 : 32 * m];
          lv = static_cast<MaskT>((below ? keep_lo : keep_hi) & ~kn) != 0;
        }
        if (__any_sync(0xffffffffu, lv)) live |= 1u << m;
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full, static_cast<uint32_t>(g) & 1u, abort_flag, err, wait_ns)))
        break;
      tc_fence_after();
#pragma unroll 1
      for (int m = 0; m < kTile / 32; ++m) {
        uint32_t pp[8], pd[8];
        if (live & (1u << m)) {
          uint32_t sv[16], dv[16];
          tmem_ld16x2_16<16>(s_base + 32u * m, sv);
          tmem_ld16x2_16<16>(dp_base + 32u * m, dv);
          tmem_wait_ld();
          regs_after_wait(sv);
          regs_after_wait(dv);
          const int ch = 2 * m + kh;
          float w16[16];
          if (kind == 0 && m == quarter) {
            uint32_t c4[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) c4[u] = sm.cw[4 * kh + u][threadIdx.x];
            w16_counts(c4, w16);
          } else {
            const bool below = kind == 1 || (kind == 0 && m < quarter);
            w16_carry<MaskT>(km_tile + 16 * ch, below ? keep_lo : keep_hi, w16);
          }
          pds16_cols(sv, dv, w16, ks.nbias + 16 * ch, ks.nD + 16 * ch, sc2, pp, pd);
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) pp[e] = pd[e] = 0u;
        }
        tmem_st16x2_8<8>(s_base + 16u * m, pp);
        tmem_st16x2_8<8>(dp_base + 16u * m, pd);
      }
      if (kind == 1) {
        Y = static_cast<MaskT>(Y | ms.bm[0] | ms.suf[0]);
      } else if (kind == 2) {
        Z = static_cast<MaskT>(Zc | ms.pre[kTile - 1]);
      } else {
        Y = static_cast<MaskT>(ms.bm[0] | ms.pre[r]);
        Z = ms.suf[r];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.m_empty[st]);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.p_full);
      if (last) {  // the item's epilogue runs at the top of the next iteration
        pend = true;
        pend_g = g;
        pend_tx = tx;
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

template <typename MaskT, bool kCausal>
int launch_typed(const BwdTcArgs& a, cudaStream_t st) {
  CUtensorMap mq, mdo, mk, mv;
  if (int rc = make_map(&mq, a.Q, a.n, a.B * a.H)) return rc;
  if (int rc = make_map(&mdo, a.dO, a.n, a.B * a.H)) return rc;
  if (int rc = make_map(&mk, a.K, a.n, a.B * a.H_kv)) return rc;
  if (int rc = make_map(&mv, a.V, a.n, a.B * a.H_kv)) return rc;
  const int T = ceil_div(a.n, kTile);
  // dQ: the forward's item list and windows
  Params p{};
  p.B = a.B;
  p.H = a.H;
  p.H_kv = a.H_kv;
  p.n = a.n;
  p.s = a.s;
  p.causal = a.causal;
  p.T = T;
  p.items = a.B * a.H * T;
  p.spans = a.tile_spans;
  p.wait_ns = wait_limit_ns();
  auto kq = bwd_dq_tc_kernel<MaskT, kCausal>;
  const size_t smem_q = sizeof(DqSmem<MaskT>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem_q));
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(bwd_dq_tc_kernel)");
  const int grid_q = p.items < sm_count() ? p.items : sm_count();
  kq<<<grid_q, kThreads, smem_q, st>>>(mq, mdo, mk, mv, p, static_cast<const MaskT*>(a.bmask), a.row_sum, a.delta,
                                       static_cast<__nv_bfloat16*>(a.dQ), a.err);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "bwd_dq_tc_kernel launch");
  // dK, dV: one item per (KV head, batch, key tile), windows by symmetry
  BwdTcParams pk{a.B, a.H, a.H_kv, a.n, a.s, a.causal, T, a.B * a.H_kv * T, a.key_spans, wait_limit_ns()};
  auto kk = bwd_dkdv_tc_kernel<MaskT, kCausal>;
  const size_t smem_k = sizeof(KvSmem<MaskT>) + 1024;
  e = cudaFuncSetAttribute(kk, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem_k));
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(bwd_dkdv_tc_kernel)");
  const int grid_k = pk.items < sm_count() ? pk.items : sm_count();
  kk<<<grid_k, kThreads, smem_k, st>>>(mq, mdo, mk, mv, pk, static_cast<const MaskT*>(a.bmask), a.row_sum, a.delta,
                                       static_cast<__nv_bfloat16*>(a.dK), static_cast<__nv_bfloat16*>(a.dV), a.err);
  e = cudaGetLastError();
  return e == cudaSuccess ? PLSH_OK : cuda_fail(e, "bwd_dkdv_tc_kernel launch");
}

}  // namespace

int launch_bwd_tc(const BwdTcArgs& a, cudaStream_t st) {
  if (static_cast<long long>(a.B) * a.H * ceil_div(a.n, kTile) > 0x7fffffffLL)
    return fail(PLSH_ERR_RANGE, "plsh_attention_bwd_tc: too many tiles");
  if (int rc = launch_bwd_delta(a.O, a.dO, PLSH_BF16, a.d, static_cast<size_t>(a.B) * a.H * a.n, a.delta, st))
    return rc;
  if (a.causal)
    return a.s <= 32 ? launch_typed<uint32_t, true>(a, st) : launch_typed<unsigned long long, true>(a, st);
  return a.s <= 32 ? launch_typed<uint32_t, false>(a, st) : launch_typed<unsigned long long, false>(a, st);
}

}  // namespace plsh
