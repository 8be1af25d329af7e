// Decode: single query rows against the cached keys -- plsh_decode_fwd.
//
// For query row t of (batch b, head h) at position i = pos[t], the output is
// row i of T~ = D~^{-1} (exp(Q K^T / sqrt d) o M~) V (Positional LSH technical
// summary, Methodology 2 and 3), with the key range ending at i when causal:
//   O = sum_j c_ij e^{S_ij} V_j / sum_j c_ij e^{S_ij},  S_ij = q . K_j / sqrt d,
// c_ij = s - popcount(OR of the boundary masks over (min(i,j), max(i,j)]).
// Blocks are contiguous (Methodology 1, structure), so walking away from i
// the OR only grows and c_ij only falls: the walk stops at the first chunk
// of keys whose counts are all zero. Only the keys sharing a block with i in
// some hash are read: their K and V rows are the bytes the call must move, and
// the chain of dependent loads along the walk sets its latency.
//
// Each query row's walk is spread over G CTAs of 256 threads (G chosen so the
// grid covers the SMs about twelve times, at most 8; four CTAs fit on an SM,
// at 64 registers a thread). Keys are taken in chunks of 256
// on each side of i (i and below, then above when not causal); CTA g of a row
// takes chunks g, g + G, g + 2G, ... Its carry -- the OR of the masks between
// i and its chunk -- is OR-reduced from the masks of the chunks in between,
// and a CTA-wide OR-scan inside the chunk gives every key its count. Each warp
// scores its 32 keys (lane = key, q from shared memory), keeps a running
// maximum, sum and output row (lanes over dims), and the CTA writes the merge
// of its warps as a partial result (maximum, sum, unnormalised row) to caller
// scratch. The last of a row's G CTAs to finish (a ticket from a per-row
// counter in the same scratch) merges the G partials into O and row_sum and
// resets the counter.
#include <algorithm>
#include <cmath>

#include <cuda_bf16.h>

#include "plsh_internal.h"

namespace plsh {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

template <typename MaskT>
__device__ __forceinline__ int popc_mask(MaskT m) {
  if constexpr (sizeof(MaskT) == 8) return __popcll(static_cast<unsigned long long>(m));
  else return __popc(static_cast<unsigned>(m));
}

__device__ __forceinline__ float to_f(float x) { return x; }

// q . row for one key row (q in shared memory), 16-byte loads, all issued before the first FMA.
template <int D>
__device__ __forceinline__ float dot_row(const float* q, const float* row) {
  float acc = 0.0f;
#pragma unroll
  for (int e = 0; e < D; e += 4) {
    const float4 k4 = *reinterpret_cast<const float4*>(row + e);
    acc = fmaf(q[e], k4.x, fmaf(q[e + 1], k4.y, fmaf(q[e + 2], k4.z, fmaf(q[e + 3], k4.w, acc))));
  }
  return acc;
}
template <int D>
__device__ __forceinline__ float dot_row(const float* q, const __nv_bfloat16* row) {
  float acc = 0.0f;
#pragma unroll 1
  for (int h0 = 0; h0 < D; h0 += 64) {  // 64 dims (eight 16-byte loads) at a time
#pragma unroll
    for (int e = h0; e < h0 + 64; e += 8) {
      const uint4 u = *reinterpret_cast<const uint4*>(row + e);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float lo = __uint_as_float(w[k] << 16), hi = __uint_as_float(w[k] & 0xFFFF0000u);
        acc = fmaf(q[e + 2 * k], lo, fmaf(q[e + 2 * k + 1], hi, acc));
      }
    }
  }
  return acc;
}
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

// The lane's N consecutive values of a row (N = 2 or 4), one vector load.
template <int N>
__device__ __forceinline__ void load_n(const float* p, float* out) {
  if constexpr (N == 4) {
    const float4 x = *reinterpret_cast<const float4*>(p);
    out[0] = x.x; out[1] = x.y; out[2] = x.z; out[3] = x.w;
  } else {
    const float2 x = *reinterpret_cast<const float2*>(p);
    out[0] = x.x; out[1] = x.y;
  }
}
template <int N>
__device__ __forceinline__ void load_n(const __nv_bfloat16* p, float* out) {
  if constexpr (N == 4) {
    const uint2 x = *reinterpret_cast<const uint2*>(p);
    out[0] = __uint_as_float(x.x << 16); out[1] = __uint_as_float(x.x & 0xFFFF0000u);
    out[2] = __uint_as_float(x.y << 16); out[3] = __uint_as_float(x.y & 0xFFFF0000u);
  } else {
    const uint32_t x = *reinterpret_cast<const uint32_t*>(p);
    out[0] = __uint_as_float(x << 16); out[1] = __uint_as_float(x & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void from_f(float& y, float x) { y = x; }
__device__ __forceinline__ void from_f(__nv_bfloat16& y, float x) { y = __float2bfloat16_rn(x); }

template <typename T, int D, typename MaskT>
struct DecodeSmem {
  float q[D];
  MaskT wsum[kWarps];          // OR of each warp's masks
  float wm[kWarps], wl[kWarps];
  float wo[kWarps][D];
  int live;                    // some key of the chunk carries weight
};

// The mask the walk's key at offset kk from i contributes on `side` (0: i and below, 1: above), and
// that key. Below, key j needs the masks over (j, i], i.e. bm[j + 1 .. i] (none for j = i, which has
// count s); above, over (i, j], bm[i + 1 .. j]. Keys outside [0, n) contribute every hash.
template <typename MaskT>
__device__ __forceinline__ MaskT walk_mask(const MaskT* bm, int i, int n, int side, int kk, MaskT full, int& j,
                                           bool& in) {
  j = side == 0 ? i - kk : i + 1 + kk;
  in = j >= 0 && j < n;
  return !in ? full : side == 1 ? bm[j] : j == i ? static_cast<MaskT>(0) : bm[j + 1];
}

// OR of v over the CTA (every thread gets it).
template <typename MaskT>
__device__ __forceinline__ MaskT cta_or(MaskT v, MaskT* wsum, int lane, int warp) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v |= __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) wsum[warp] = v;
  __syncthreads();
  MaskT all = 0;
#pragma unroll
  for (int w2 = 0; w2 < kWarps; ++w2) all |= wsum[w2];
  __syncthreads();
  return all;
}

// OR of the walk masks at offsets [k0, k1) on `side`.
template <typename MaskT>
__device__ __forceinline__ MaskT walk_or(const MaskT* bm, int i, int n, int side, int k0, int k1, MaskT full,
                                         MaskT* wsum, int lane, int warp) {
  MaskT acc = 0;
#pragma unroll 8
  for (int kk = k0 + static_cast<int>(threadIdx.x); kk < k1; kk += kThreads) {
    int j;
    bool in;
    acc |= walk_mask(bm, i, n, side, kk, full, j, in);
  }
  return cta_or(acc, wsum, lane, warp);
}

// One of G CTAs of query row t of (b, h): the chunks g, g + G, g + 2G, ... of each side's walk. Its
// partial result -- running maximum, sum and unnormalised output row -- goes to part.
template <typename T, int D, typename MaskT>
__global__ void __launch_bounds__(kThreads, 4) decode_partial_kernel(
    const T* __restrict__ Q, const int32_t* __restrict__ pos, int m, const T* __restrict__ K,
    const T* __restrict__ V, int H, int H_kv, int n, int s, int causal, const MaskT* __restrict__ bmask, int G,
    float* __restrict__ part, unsigned* __restrict__ done, T* __restrict__ O, float* __restrict__ row_sum,
    uint32_t* __restrict__ err) {
  constexpr int DPL = D / 32;  // output dims per lane
  __shared__ DecodeSmem<T, D, MaskT> sm;
  const int t = blockIdx.x / G, g = blockIdx.x % G, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int i = pos[t];
  if (i < 0 || i >= n) {
    if (tid == 0 && g == 0) atomicOr(err, PLSH_DEVERR_POSITION);
    return;
  }
  const int kvh = h / (H / H_kv);
  const MaskT FULL = (s >= static_cast<int>(8 * sizeof(MaskT))) ? static_cast<MaskT>(~static_cast<MaskT>(0))
                                                              : static_cast<MaskT>((static_cast<MaskT>(1) << s) - 1);
  const MaskT* bm = bmask + static_cast<size_t>(h) * n;
  const size_t row = (static_cast<size_t>(b) * H + h) * m + t;
  const T* qrow = Q + row * D;
  for (int e = tid; e < D; e += kThreads) sm.q[e] = to_f(qrow[e]);
  const T* Kh = K + (static_cast<size_t>(b) * H_kv + kvh) * static_cast<size_t>(n) * D;
  const T* Vh = V + (static_cast<size_t>(b) * H_kv + kvh) * static_cast<size_t>(n) * D;
  const float scale = 1.0f / sqrtf(static_cast<float>(D));
  __syncthreads();

  float mw = -INFINITY, lw = 0.0f, ow[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) ow[e] = 0.0f;

  // Scores the warp's 32 keys (key j of this lane, weight c; c == 0 or j out of range: no key) and
  // folds them into the warp's running maximum, sum and output.
  auto fold = [&](int j, int c) {
    float sj = -INFINITY;
    if (c > 0) {
      sj = dot_row<D>(sm.q, Kh + static_cast<size_t>(j) * D) * scale;
    }
    float cmax = sj;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, o));
    if (cmax == -INFINITY) return;
    const float m_new = fmaxf(mw, cmax);
    const float corr = expf(mw - m_new);
    lw *= corr;
#pragma unroll
    for (int e = 0; e < DPL; ++e) ow[e] *= corr;
    mw = m_new;
    const float p = c > 0 ? static_cast<float>(c) * expf(sj - mw) : 0.0f;
    float psum = p;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o);
    lw += psum;
    // O += p_j V_j over the warp's keys, lanes over dims; 8 keys at a time, their loads issued together
#pragma unroll 1
    for (int k0 = 0; k0 < 32; k0 += 8) {
      float pk[8], vv[8][DPL];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        pk[u] = __shfl_sync(0xffffffffu, p, k0 + u);
        const int jk = __shfl_sync(0xffffffffu, j, k0 + u);
        if (pk[u] != 0.0f) {
          load_n<DPL>(Vh + static_cast<size_t>(jk) * D + lane * DPL, vv[u]);
        } else {
#pragma unroll
          for (int e = 0; e < DPL; ++e) vv[u][e] = 0.0f;
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int e = 0; e < DPL; ++e) ow[e] = fmaf(pk[u], vv[u][e], ow[e]);
    }
  };

  for (int side = 0; side < (causal ? 1 : 2); ++side) {
    // OR of the masks between i and the nearest key of chunk g
    MaskT carry = walk_or(bm, i, n, side, 0, g * kThreads, FULL, sm.wsum, lane, warp);
    for (int c = g; carry != FULL; c += G) {   // a carry holding every hash leaves no key any weight
      int j;
      bool in;
      const MaskT mine = walk_mask(bm, i, n, side, c * kThreads + tid, FULL, j, in);
      // inclusive OR-scan over the CTA in walking order
      MaskT v = mine;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const MaskT y = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v |= y;
      }
      if (lane == 31) sm.wsum[warp] = v;
      __syncthreads();
      MaskT before = carry;
      for (int w2 = 0; w2 < warp; ++w2) before |= sm.wsum[w2];
      MaskT all = carry;
      for (int w2 = 0; w2 < kWarps; ++w2) all |= sm.wsum[w2];
      const MaskT R = before | v;
      const int cnt = in ? s - popc_mask(R) : 0;
      if (tid == 0) sm.live = 0;
      __syncthreads();
      if (cnt > 0) sm.live = 1;
      __syncthreads();
      const bool live = sm.live != 0;
      __syncthreads();
      if (!live) break;   // the OR only grows along the walk: no later key has weight
      fold(j, cnt);
      // through chunk c, then the chunks the other CTAs of the row take before chunk c + G
      carry = all | walk_or(bm, i, n, side, (c + 1) * kThreads, (c + G) * kThreads, FULL, sm.wsum, lane, warp);
    }
  }

  // merge the warps into the CTA's partial result
  if (lane == 0) {
    sm.wm[warp] = mw;
    sm.wl[warp] = lw;
  }
#pragma unroll
  for (int e = 0; e < DPL; ++e) sm.wo[warp][lane * DPL + e] = ow[e];
  __syncthreads();
  if (warp == 0) {
    float mt = -INFINITY;
    for (int w2 = 0; w2 < kWarps; ++w2) mt = fmaxf(mt, sm.wm[w2]);
    float lt = 0.0f, ot[DPL];
#pragma unroll
    for (int e = 0; e < DPL; ++e) ot[e] = 0.0f;
    for (int w2 = 0; w2 < kWarps; ++w2) {
      if (sm.wm[w2] == -INFINITY) continue;
      const float f = expf(sm.wm[w2] - mt);
      lt += sm.wl[w2] * f;
#pragma unroll
      for (int e = 0; e < DPL; ++e) ot[e] += sm.wo[w2][lane * DPL + e] * f;
    }
    float* pr = part + (row * G + g) * (D + 2);
#pragma unroll
    for (int e = 0; e < DPL; ++e) pr[2 + lane * DPL + e] = ot[e];
    if (lane == 0) {
      pr[0] = mt;
      pr[1] = lt;
    }
    // the row's last CTA to finish merges the G partial results (the others' writes are visible to it
    // once its ticket shows they have all been published) and leaves the row's counter at zero again
    __threadfence();
    __syncwarp();
    unsigned ticket = 0;
    if (lane == 0) ticket = atomicAdd(&done[row], 1u);
    ticket = __shfl_sync(0xffffffffu, ticket, 0);
    if (ticket == static_cast<unsigned>(G - 1)) {
      __threadfence();
      const float* p0 = part + row * G * (D + 2);
      float M = -INFINITY;
      for (int g2 = 0; g2 < G; ++g2) M = fmaxf(M, __ldcg(p0 + g2 * (D + 2)));
      float L = 0.0f, acc[DPL];
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[e] = 0.0f;
      for (int g2 = 0; g2 < G; ++g2) {
        const float* q2 = p0 + g2 * (D + 2);
        const float m2 = __ldcg(q2);
        if (m2 == -INFINITY) continue;
        const float f = expf(m2 - M);
        L += __ldcg(q2 + 1) * f;
#pragma unroll
        for (int e = 0; e < DPL; ++e) acc[e] += __ldcg(q2 + 2 + lane * DPL + e) * f;
      }
      const float inv = 1.0f / L;
      T* orow = O + row * D;
#pragma unroll
      for (int e = 0; e < DPL; ++e) from_f(orow[lane * DPL + e], acc[e] * inv);
      if (lane == 0) {
        row_sum[row] = logf(L) + M - logf(static_cast<float>(s));
        done[row] = 0u;
      }
    }
  }
}

template <typename T, int D, typename MaskT>
int launch_decode_typed(const DecodeArgs& a, int G, cudaStream_t st) {
  const size_t rows = static_cast<size_t>(a.B) * a.H * a.m;
  unsigned* done = reinterpret_cast<unsigned*>(a.part + rows * kDecodeMaxSplit * (a.d + 2));
  decode_partial_kernel<T, D, MaskT><<<dim3(a.m * G, a.H, a.B), kThreads, 0, st>>>(
      static_cast<const T*>(a.Q), a.pos, a.m, static_cast<const T*>(a.K), static_cast<const T*>(a.V), a.H, a.H_kv,
      a.n, a.s, a.causal, static_cast<const MaskT*>(a.bmask), G, a.part, done, static_cast<T*>(a.O), a.row_sum,
      a.err);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? PLSH_OK : cuda_fail(e, "decode_partial_kernel launch");
}

template <typename T, int D>
int launch_decode_mask(const DecodeArgs& a, int G, cudaStream_t st) {
  return a.s <= 32 ? launch_decode_typed<T, D, uint32_t>(a, G, st)
                   : launch_decode_typed<T, D, unsigned long long>(a, G, st);
}

}  // namespace

int launch_decode(const DecodeArgs& a, cudaStream_t st) {
  // CTAs per row: enough for about twelve CTAs per SM over all rows (a row's walk can be long, and
  // a few long rows would otherwise set the time of the whole grid), at most kDecodeMaxSplit
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    sms = 148;
  const long long rows = static_cast<long long>(a.B) * a.H * a.m;
  const int G = static_cast<int>(std::min<long long>(kDecodeMaxSplit, std::max<long long>(1, (12LL * sms + rows - 1) / rows)));
  if (a.dtype == PLSH_F32)
    return a.d == 64 ? launch_decode_mask<float, 64>(a, G, st) : launch_decode_mask<float, 128>(a, G, st);
  return a.d == 64 ? launch_decode_mask<__nv_bfloat16, 64>(a, G, st) : launch_decode_mask<__nv_bfloat16, 128>(a, G, st);
}

}  // namespace plsh
