// Backward pass of T~: dQ, dK, dV with the (delta, u) table held fixed -- plsh_attention_bwd.
//
// T~ = P V with P_ij = c_ij e^{S_ij} / sum_l c_il e^{S_il} (Positional LSH technical
// summary, Methodology 2 and 3; the pages train and fine-tune models with this
// attention, Results, experimental validation). With the forward's row_sum
// L_i = ln( sum_j (c_ij / s) e^{S_ij} ) the weights are recomputed exactly:
//   P_ij = (c_ij / s) e^{S_ij - L_i},
// and by the chain rule
//   dV = P^T dO,  dP = dO V^T,  D_i = dO_i . O_i,  dS = P o (dP - D),
//   dQ = dS K / sqrt d,  dK = dS^T Q / sqrt d.
// c_ij counts the hashes whose bin ids agree for i and j (ids [H][s][n]).
// Blocks are contiguous (Methodology 1, structure), so the keys that share a
// block with any row of [r0, r1] form one range: from the first position of
// r0's block to the last position of r1's block, the widest over the hashes,
// found by binary search in the non-decreasing ids. By symmetry of c_ij the
// same range holds the query rows that reach a key tile.
//
// Three kernels, fp32 arithmetic on CUDA cores for both dtypes:
//   bwd_delta_kernel  D_i = dO_i . O_i                       (one warp per row)
//   bwd_dq_kernel     one CTA per 64-row query tile: walks its key range in
//                     chunks of 64, recomputes S and dP, forms dS, dQ += dS K
//   bwd_dkdv_kernel   one CTA per 64-key tile of a KV head: for every query head
//                     of its group walks the query range in chunks of 64,
//                     dV += P^T dO, dK += dS^T Q; each dK, dV row is written once
//                     (no atomics; the result does not depend on scheduling).
#include <climits>
#include <cmath>

#include <cuda_bf16.h>

#include "plsh_internal.h"

namespace plsh {
namespace {

constexpr int kT = 64;          // rows per query tile and keys per key tile
constexpr int kThreads = 256;   // 16 x 16 threads; each owns 4 x 4 (row, key) pairs
constexpr int kSP = kT + 4;     // pitch of the 64 x 64 score tiles (16-byte rows, spread over the banks)
template <int D>
__host__ __device__ constexpr int pitch() { return D + 4; }   // pitch of the 64 x D row tiles (16-byte rows)

__device__ __forceinline__ float4 lds4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float comp(const float4& v, int u) {
  return u == 0 ? v.x : (u == 1 ? v.y : (u == 2 ? v.z : v.w));
}

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 ld4(const __nv_bfloat16* p) {
  const uint2 raw = *reinterpret_cast<const uint2*>(p);
  return make_float4(__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xFFFF0000u),
                     __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xFFFF0000u));
}
__device__ __forceinline__ void st1(float* p, float x) { *p = x; }
__device__ __forceinline__ void st1(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

// rows [r0, r0 + 64) of a [n][D] matrix into fp32 shared memory of pitch D + 4 (zeros past `last`)
template <typename T, int D>
__device__ __forceinline__ void load_rows(float* dst, const T* src, int r0, int last) {
  constexpr int F4 = D / 4;
  for (int x = threadIdx.x; x < kT * F4; x += kThreads) {
    const int r = x / F4, c = (x % F4) * 4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r0 + r <= last) v = ld4(src + static_cast<size_t>(r0 + r) * D + c);
    *reinterpret_cast<float4*>(dst + r * pitch<D>() + c) = v;
  }
}

// ids of hashes 0..s-1 at positions [p0, p0 + 64) into idt[k][64] (`none` past `last`)
__device__ __forceinline__ void load_ids(int* idt, const int32_t* ids_h, int n, int s, int p0, int last,
                                         int none) {
  for (int x = threadIdx.x; x < s * kT; x += kThreads) {
    const int k = x / kT, c = x % kT;
    idt[x] = (p0 + c <= last) ? ids_h[static_cast<size_t>(k) * n + p0 + c] : none;
  }
}

// The range [lo, hi] of positions sharing a block with some position of [a, b] in some hash of
// ids_h; written to range[0..1] by threads 0..s-1 (range must hold {INT_MAX, INT_MIN} before).
__device__ __forceinline__ void block_range(int* range, const int32_t* ids_h, int n, int s, int a, int b) {
  const int k = threadIdx.x;
  if (k >= s) return;
  const int32_t* row = ids_h + static_cast<size_t>(k) * n;
  const int ia = row[a], ib = row[b];
  int lo = 0, hi = a;             // first p in [0, a] with row[p] == ia (row is non-decreasing)
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (row[mid] < ia) lo = mid + 1; else hi = mid;
  }
  const int first = lo;
  lo = b; hi = n - 1;             // last p in [b, n) with row[p] == ib
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (row[mid] > ib) hi = mid - 1; else lo = mid;
  }
  atomicMin(&range[0], first);
  atomicMax(&range[1], lo);
}

// S = q k^T and dP = dO v^T for the thread's 4 x 4 pairs (rows ty + 16a, keys tx + 16b), four
// dims per step through 16-byte shared loads
template <int D>
__device__ __forceinline__ void scores(const float* qs, const float* dos, const float* ks, const float* vs,
                                       int ty, int tx, float (&sacc)[4][4], float (&pacc)[4][4]) {
  constexpr int P = pitch<D>();
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) sacc[a][b] = pacc[a][b] = 0.0f;
#pragma unroll 2
  for (int e = 0; e < D; e += 4) {
    float4 qa[4], oa[4], kb[4], vb[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      qa[a] = lds4(qs + (ty + 16 * a) * P + e);
      oa[a] = lds4(dos + (ty + 16 * a) * P + e);
    }
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      kb[b] = lds4(ks + (tx + 16 * b) * P + e);
      vb[b] = lds4(vs + (tx + 16 * b) * P + e);
    }
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        sacc[a][b] = fmaf(qa[a].x, kb[b].x, fmaf(qa[a].y, kb[b].y, fmaf(qa[a].z, kb[b].z, fmaf(qa[a].w, kb[b].w,
                          sacc[a][b]))));
        pacc[a][b] = fmaf(oa[a].x, vb[b].x, fmaf(oa[a].y, vb[b].y, fmaf(oa[a].z, vb[b].z, fmaf(oa[a].w, vb[b].w,
                          pacc[a][b]))));
      }
  }
}

// c_ij for the thread's pairs: hashes whose ids agree (row ids in idq, key ids in idk)
__device__ __forceinline__ void counts(const int* idq, const int* idk, int s, int ty, int tx, int (&c)[4][4]) {
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) c[a][b] = 0;
  for (int k = 0; k < s; ++k) {
    int iq[4], ik[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) iq[a] = idq[k * kT + ty + 16 * a];
#pragma unroll
    for (int b = 0; b < 4; ++b) ik[b] = idk[k * kT + tx + 16 * b];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) c[a][b] += (iq[a] == ik[b]);
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) bwd_delta_kernel(const T* __restrict__ O, const T* __restrict__ dO,
                                                             float* __restrict__ delta, size_t rows) {
  const size_t r = static_cast<size_t>(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  float acc = 0.0f;
  for (int e = lane * 4; e < D; e += 128) {
    const float4 o = ld4(O + r * D + e), g = ld4(dO + r * D + e);
    acc = fmaf(o.x, g.x, fmaf(o.y, g.y, fmaf(o.z, g.z, fmaf(o.w, g.w, acc))));
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) delta[r] = acc;
}

struct BwdParams {
  int B, H, H_kv, n, s, causal;
};

template <int D>
__host__ __device__ constexpr size_t dq_smem_floats() { return 4 * kT * pitch<D>() + kT * kSP + 2 * kT; }
template <int D>
__host__ __device__ constexpr size_t dkdv_smem_floats() { return 4 * kT * pitch<D>() + 2 * kT * kSP + 2 * kT; }

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) bwd_dq_kernel(const T* __restrict__ Q, const T* __restrict__ K,
                                                          const T* __restrict__ V, const T* __restrict__ dO,
                                                          const float* __restrict__ row_sum,
                                                          const float* __restrict__ delta,
                                                          const int32_t* __restrict__ ids, BwdParams p,
                                                          T* __restrict__ dQ) {
  constexpr int P = pitch<D>();
  constexpr int NB = D / 16;   // output dims per thread: tx * NB .. tx * NB + NB - 1
  extern __shared__ __align__(16) float smf[];
  float* qs = smf;
  float* dos = qs + kT * P;
  float* ks = dos + kT * P;
  float* vs = ks + kT * P;
  float* ds = vs + kT * P;
  float* Ls = ds + kT * kSP;
  float* Ds = Ls + kT;
  int* idq = reinterpret_cast<int*>(Ds + kT);
  int* idk = idq + p.s * kT;
  int* range = idk + p.s * kT;

  const int n = p.n, s = p.s;
  const int r0 = blockIdx.x * kT, h = blockIdx.y, b = blockIdx.z;
  const int r1 = min(n - 1, r0 + kT - 1);
  const int kvh = h / (p.H / p.H_kv);
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const size_t bh = static_cast<size_t>(b) * p.H + h;
  const size_t bg = static_cast<size_t>(b) * p.H_kv + kvh;
  const int32_t* ids_h = ids + static_cast<size_t>(h) * s * n;
  const float scale = 1.0f / sqrtf(static_cast<float>(D));
  const float inv_s = 1.0f / static_cast<float>(s);

  if (tid == 0) { range[0] = INT_MAX; range[1] = INT_MIN; }
  load_rows<T, D>(qs, Q + bh * n * D, r0, r1);
  load_rows<T, D>(dos, dO + bh * n * D, r0, r1);
  load_ids(idq, ids_h, n, s, r0, r1, -1);
  if (tid < kT) {
    const bool in = r0 + tid <= r1;
    Ls[tid] = in ? row_sum[bh * n + r0 + tid] : 0.0f;
    Ds[tid] = in ? delta[bh * n + r0 + tid] : 0.0f;
  }
  __syncthreads();
  block_range(range, ids_h, n, s, r0, r1);
  __syncthreads();
  const int lo = range[0];
  const int hi = p.causal ? min(range[1], r1) : range[1];

  float acc[4][NB];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < NB; ++c) acc[a][c] = 0.0f;

  for (int c0 = lo; c0 <= hi; c0 += kT) {
    __syncthreads();   // the previous chunk's readers are done with ks, vs, idk and ds
    load_rows<T, D>(ks, K + bg * n * D, c0, hi);
    load_rows<T, D>(vs, V + bg * n * D, c0, hi);
    load_ids(idk, ids_h, n, s, c0, hi, -2);
    __syncthreads();
    float sacc[4][4], pacc[4][4];
    int cnt[4][4];
    scores<D>(qs, dos, ks, vs, ty, tx, sacc, pacc);
    counts(idq, idk, s, ty, tx, cnt);
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int i = r0 + ty + 16 * a;
#pragma unroll
      for (int bb = 0; bb < 4; ++bb) {
        const int j = c0 + tx + 16 * bb;
        float dsv = 0.0f;
        if (cnt[a][bb] > 0 && !(p.causal && j > i)) {
          const float pij = static_cast<float>(cnt[a][bb]) * inv_s * expf(sacc[a][bb] * scale - Ls[ty + 16 * a]);
          dsv = pij * (pacc[a][bb] - Ds[ty + 16 * a]);
        }
        ds[(ty + 16 * a) * kSP + tx + 16 * bb] = dsv;
      }
    }
    __syncthreads();
#pragma unroll 1
    for (int j = 0; j < kT; j += 4) {
      float4 dv[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) dv[a] = lds4(ds + (ty + 16 * a) * kSP + j);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        float4 kv[NB / 4];
#pragma unroll
        for (int c4 = 0; c4 < NB / 4; ++c4) kv[c4] = lds4(ks + (j + u) * P + tx * NB + 4 * c4);
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          const float w = comp(dv[a], u);
#pragma unroll
          for (int c4 = 0; c4 < NB / 4; ++c4) {
            acc[a][4 * c4] = fmaf(w, kv[c4].x, acc[a][4 * c4]);
            acc[a][4 * c4 + 1] = fmaf(w, kv[c4].y, acc[a][4 * c4 + 1]);
            acc[a][4 * c4 + 2] = fmaf(w, kv[c4].z, acc[a][4 * c4 + 2]);
            acc[a][4 * c4 + 3] = fmaf(w, kv[c4].w, acc[a][4 * c4 + 3]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int i = r0 + ty + 16 * a;
    if (i > r1) continue;
    T* out = dQ + (bh * n + i) * D + tx * NB;
#pragma unroll
    for (int c = 0; c < NB; ++c) st1(out + c, acc[a][c] * scale);
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) bwd_dkdv_kernel(const T* __restrict__ Q, const T* __restrict__ K,
                                                            const T* __restrict__ V, const T* __restrict__ dO,
                                                            const float* __restrict__ row_sum,
                                                            const float* __restrict__ delta,
                                                            const int32_t* __restrict__ ids, BwdParams p,
                                                            T* __restrict__ dK, T* __restrict__ dV) {
  constexpr int P = pitch<D>();
  constexpr int NB = D / 16;   // output dims per thread: tx * NB .. tx * NB + NB - 1
  extern __shared__ __align__(16) float smf[];
  float* ks = smf;
  float* vs = ks + kT * P;
  float* qs = vs + kT * P;
  float* dos = qs + kT * P;
  float* ps = dos + kT * P;
  float* dss = ps + kT * kSP;
  float* Ls = dss + kT * kSP;
  float* Ds = Ls + kT;
  int* idk = reinterpret_cast<int*>(Ds + kT);
  int* idq = idk + p.s * kT;
  int* range = idq + p.s * kT;

  const int n = p.n, s = p.s;
  const int j0 = blockIdx.x * kT, g = blockIdx.y, b = blockIdx.z;
  const int j1 = min(n - 1, j0 + kT - 1);
  const int group = p.H / p.H_kv;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const size_t bg = static_cast<size_t>(b) * p.H_kv + g;
  const float scale = 1.0f / sqrtf(static_cast<float>(D));
  const float inv_s = 1.0f / static_cast<float>(s);

  load_rows<T, D>(ks, K + bg * n * D, j0, j1);
  load_rows<T, D>(vs, V + bg * n * D, j0, j1);

  float accK[4][NB], accV[4][NB];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < NB; ++c) accK[a][c] = accV[a][c] = 0.0f;

  for (int hq = 0; hq < group; ++hq) {
    const int h = g * group + hq;
    const size_t bh = static_cast<size_t>(b) * p.H + h;
    const int32_t* ids_h = ids + static_cast<size_t>(h) * s * n;
    __syncthreads();   // the previous head's readers are done with idk and range
    if (tid == 0) { range[0] = INT_MAX; range[1] = INT_MIN; }
    load_ids(idk, ids_h, n, s, j0, j1, -2);
    __syncthreads();
    block_range(range, ids_h, n, s, j0, j1);
    __syncthreads();
    const int lo = p.causal ? max(range[0], j0) : range[0];
    const int hi = range[1];
    for (int c0 = lo; c0 <= hi; c0 += kT) {
      __syncthreads();   // the previous chunk's readers are done with qs, dos, idq, ps and dss
      load_rows<T, D>(qs, Q + bh * n * D, c0, hi);
      load_rows<T, D>(dos, dO + bh * n * D, c0, hi);
      load_ids(idq, ids_h, n, s, c0, hi, -1);
      if (tid < kT) {
        const bool in = c0 + tid <= hi;
        Ls[tid] = in ? row_sum[bh * n + c0 + tid] : 0.0f;
        Ds[tid] = in ? delta[bh * n + c0 + tid] : 0.0f;
      }
      __syncthreads();
      float sacc[4][4], pacc[4][4];
      int cnt[4][4];
      scores<D>(qs, dos, ks, vs, ty, tx, sacc, pacc);   // rows = query rows of the chunk, keys = the tile
      counts(idq, idk, s, ty, tx, cnt);
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const int i = c0 + ty + 16 * a;
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) {
          const int j = j0 + tx + 16 * bb;
          float pij = 0.0f, dsv = 0.0f;
          if (cnt[a][bb] > 0 && !(p.causal && j > i)) {
            pij = static_cast<float>(cnt[a][bb]) * inv_s * expf(sacc[a][bb] * scale - Ls[ty + 16 * a]);
            dsv = pij * (pacc[a][bb] - Ds[ty + 16 * a]);
          }
          // transposed, [key][row], so that a key's 4 consecutive rows are one 16-byte load
          ps[(tx + 16 * bb) * kSP + ty + 16 * a] = pij;
          dss[(tx + 16 * bb) * kSP + ty + 16 * a] = dsv;
        }
      }
      __syncthreads();
      // keys ty + 16a of the tile, dims tx * NB ..: four query rows per step
#pragma unroll 1
      for (int i = 0; i < kT; i += 4) {
        float4 pv[4], dv[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          pv[a] = lds4(ps + (ty + 16 * a) * kSP + i);
          dv[a] = lds4(dss + (ty + 16 * a) * kSP + i);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float4 ov[NB / 4], qv[NB / 4];
#pragma unroll
          for (int c4 = 0; c4 < NB / 4; ++c4) {
            ov[c4] = lds4(dos + (i + u) * P + tx * NB + 4 * c4);
            qv[c4] = lds4(qs + (i + u) * P + tx * NB + 4 * c4);
          }
#pragma unroll
          for (int a = 0; a < 4; ++a) {
            const float wp = comp(pv[a], u), wd = comp(dv[a], u);
#pragma unroll
            for (int c4 = 0; c4 < NB / 4; ++c4) {
              accV[a][4 * c4] = fmaf(wp, ov[c4].x, accV[a][4 * c4]);
              accV[a][4 * c4 + 1] = fmaf(wp, ov[c4].y, accV[a][4 * c4 + 1]);
              accV[a][4 * c4 + 2] = fmaf(wp, ov[c4].z, accV[a][4 * c4 + 2]);
              accV[a][4 * c4 + 3] = fmaf(wp, ov[c4].w, accV[a][4 * c4 + 3]);
              accK[a][4 * c4] = fmaf(wd, qv[c4].x, accK[a][4 * c4]);
              accK[a][4 * c4 + 1] = fmaf(wd, qv[c4].y, accK[a][4 * c4 + 1]);
              accK[a][4 * c4 + 2] = fmaf(wd, qv[c4].z, accK[a][4 * c4 + 2]);
              accK[a][4 * c4 + 3] = fmaf(wd, qv[c4].w, accK[a][4 * c4 + 3]);
            }
          }
        }
      }
    }
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int j = j0 + ty + 16 * a;
    if (j > j1) continue;
    T* ok = dK + (bg * n + j) * D + tx * NB;
    T* ov = dV + (bg * n + j) * D + tx * NB;
#pragma unroll
    for (int c = 0; c < NB; ++c) {
      st1(ok + c, accK[a][c] * scale);
      st1(ov + c, accV[a][c]);
    }
  }
}

template <typename T, int D>
int launch_bwd_typed(const BwdArgs& a, cudaStream_t st) {
  const size_t rows = static_cast<size_t>(a.B) * a.H * a.n;
  const unsigned delta_blocks = static_cast<unsigned>((rows + kThreads / 32 - 1) / (kThreads / 32));
  bwd_delta_kernel<T, D><<<delta_blocks, kThreads, 0, st>>>(static_cast<const T*>(a.O), static_cast<const T*>(a.dO),
                                                            a.delta, rows);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "bwd_delta_kernel launch");

  const BwdParams p{a.B, a.H, a.H_kv, a.n, a.s, a.causal};
  const size_t id_bytes = 2 * sizeof(int) * static_cast<size_t>(a.s) * kT + 2 * sizeof(int);
  const size_t dq_bytes = dq_smem_floats<D>() * sizeof(float) + id_bytes;
  const size_t dkdv_bytes = dkdv_smem_floats<D>() * sizeof(float) + id_bytes;
  e = cudaFuncSetAttribute(bwd_dq_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(dq_bytes));
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(bwd_dq_kernel)");
  e = cudaFuncSetAttribute(bwd_dkdv_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(dkdv_bytes));
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(bwd_dkdv_kernel)");

  const unsigned tiles = static_cast<unsigned>((a.n + kT - 1) / kT);
  bwd_dkdv_kernel<T, D><<<dim3(tiles, a.H_kv, a.B), kThreads, dkdv_bytes, st>>>(
      static_cast<const T*>(a.Q), static_cast<const T*>(a.K), static_cast<const T*>(a.V),
      static_cast<const T*>(a.dO), a.row_sum, a.delta, a.ids, p, static_cast<T*>(a.dK), static_cast<T*>(a.dV));
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "bwd_dkdv_kernel launch");
  bwd_dq_kernel<T, D><<<dim3(tiles, a.H, a.B), kThreads, dq_bytes, st>>>(
      static_cast<const T*>(a.Q), static_cast<const T*>(a.K), static_cast<const T*>(a.V),
      static_cast<const T*>(a.dO), a.row_sum, a.delta, a.ids, p, static_cast<T*>(a.dQ));
  e = cudaGetLastError();
  return e == cudaSuccess ? PLSH_OK : cuda_fail(e, "bwd_dq_kernel launch");
}

}  // namespace

int launch_bwd_delta(const void* O, const void* dO, int dtype, int d, size_t rows, float* delta, cudaStream_t st) {
  const unsigned blocks = static_cast<unsigned>((rows + kThreads / 32 - 1) / (kThreads / 32));
  if (dtype == PLSH_F32) {
    if (d == 64)
      bwd_delta_kernel<float, 64><<<blocks, kThreads, 0, st>>>(static_cast<const float*>(O), static_cast<const float*>(dO), delta, rows);
    else
      bwd_delta_kernel<float, 128><<<blocks, kThreads, 0, st>>>(static_cast<const float*>(O), static_cast<const float*>(dO), delta, rows);
  } else {
    using bf = __nv_bfloat16;
    if (d == 64)
      bwd_delta_kernel<bf, 64><<<blocks, kThreads, 0, st>>>(static_cast<const bf*>(O), static_cast<const bf*>(dO), delta, rows);
    else
      bwd_delta_kernel<bf, 128><<<blocks, kThreads, 0, st>>>(static_cast<const bf*>(O), static_cast<const bf*>(dO), delta, rows);
  }
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? PLSH_OK : cuda_fail(e, "bwd_delta_kernel launch");
}

int launch_bwd(const BwdArgs& a, cudaStream_t st) {
  if (a.dtype == PLSH_F32) return a.d == 64 ? launch_bwd_typed<float, 64>(a, st) : launch_bwd_typed<float, 128>(a, st);
  return a.d == 64 ? launch_bwd_typed<__nv_bfloat16, 64>(a, st) : launch_bwd_typed<__nv_bfloat16, 128>(a, st);
}

}  // namespace plsh
