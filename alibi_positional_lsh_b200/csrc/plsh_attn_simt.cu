// K3f: fused banded Positional-LSH attention on CUDA cores (fp32 arithmetic).
//
// Serves dtype PLSH_F32 (fp32 in/out; the tensor cores' TF32 path would not
// meet a 1e-5 output tolerance) and bf16 inputs whose head dim has no
// tensor-core kernel. One CTA owns one 128-row query tile of one
// (batch, head); D/32 threads share a row, each holding 32 of its dims.
//
// The weight of key j for query i is the number of hashes putting both in
// one bin (Positional LSH technical summary, Methodology 2: M~ = (1/s) sum of
// the s masks; the 1/s cancels in O). Blocks are contiguous (Methodology 1,
// structure), so with bmask bit k marking where hash k opens a block,
//     c_ij = s - popcount(OR of bmask over (min(i,j), max(i,j)]).
// Key tiles are visited diagonal first, then downward, then upward (non-
// causal), which lets each row carry the OR of the tiles already passed:
//   below the diagonal:  R(j) = SUF[c] | Y,   Y = OR bmask over [j0+128, i]
//   above the diagonal:  R(j) = Z | PRE[c],   Z = OR bmask over (i, j0]
// with SUF[c] = OR over (j0+c, j0+127] and PRE[c] = OR over (j0, j0+c] of the
// tile. Inside the diagonal tile each row scans outward from itself.
#include <cmath>

#include <cuda_bf16.h>

#include "plsh_internal.h"

namespace plsh {
namespace {

constexpr int kTile = PLSH_TILE;
constexpr int kDiagStride = 132;  // bytes per row of the diagonal weight table (bank spread)

template <typename MaskT>
__device__ __forceinline__ int popc_mask(MaskT m) {
  if constexpr (sizeof(MaskT) == 8) return __popcll(static_cast<unsigned long long>(m));
  else return __popc(static_cast<unsigned>(m));
}

__device__ __forceinline__ float4 load4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
  const uint2 raw = *reinterpret_cast<const uint2*>(p);
  const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
  const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
  const float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
  return make_float4(fa.x, fa.y, fb.x, fb.y);
}
__device__ __forceinline__ void store4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
__device__ __forceinline__ void store4(__nv_bfloat16* p, float4 v) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
  uint2 raw;
  raw.x = *reinterpret_cast<uint32_t*>(&a);
  raw.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = raw;
}

template <int D, typename MaskT>
struct SimtSmem {
  float k[kTile * D];
  float v[kTile * D];
  MaskT bm[kTile + 8];   // bm[c] = bmask[j0 + c], c = 0..128 (FULL past n)
  MaskT suf[kTile];
  MaskT pre[kTile];
  MaskT ycarry[kTile];   // per-row carries produced by the diagonal tile
  MaskT zcarry[kTile];
  unsigned char wdiag[kTile * kDiagStride];
};

template <typename T, int D, typename MaskT>
__global__ void __launch_bounds__(kTile * (D / 32))
attn_simt_kernel(const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V, int H,
                 int H_kv, int n, int s, int causal, const double* __restrict__ sigma,
                 const double* __restrict__ table, const int32_t* __restrict__ spans,
                 const MaskT* __restrict__ bmask, T* __restrict__ O, float* __restrict__ row_sum,
                 uint32_t* __restrict__ err, int varlen, int alibi, double log_inv_eps) {
  constexpr int TPR = D / 32;            // threads per query row
  constexpr int NT = kTile * TPR;
  constexpr int F4 = D / 4;              // float4 per row
  extern __shared__ __align__(16) unsigned char smem_raw[];
  auto& sm = *reinterpret_cast<SimtSmem<D, MaskT>*>(smem_raw);

  const int T_tiles = (n + kTile - 1) / kTile;
  const int t = blockIdx.x;
  const int h = H - 1 - static_cast<int>(blockIdx.y);   // longest windows (largest sigma) first
  const int b = blockIdx.z;
  const int tid = threadIdx.x;
  const int r = tid / TPR, part = tid % TPR;
  const int i0 = t * kTile, i = i0 + r;
  const bool row_ok = i < n;
  const int kvh = h / (H / H_kv);
  const MaskT FULL = (s >= static_cast<int>(8 * sizeof(MaskT))) ? static_cast<MaskT>(~static_cast<MaskT>(0))
                                                              : static_cast<MaskT>((static_cast<MaskT>(1) << s) - 1);
  uint32_t flags = 0;
  if (tid == 0 && t == 0 && b == 0) {
    if (sigma && !(isfinite(sigma[h]) && sigma[h] > 0.0)) flags |= PLSH_DEVERR_SIGMA;
    if (table)
      for (int k = 0; k < s; ++k) {
        const double dl = table[(static_cast<size_t>(h) * s + k) * 2];
        if (!(isfinite(dl) && dl > 0.0)) flags |= PLSH_DEVERR_TABLE;
      }
  }

  // this thread's 32 dims of q: float4 indices f = part + TPR * m, m = 0..7
  const size_t q_row = ((static_cast<size_t>(b) * H + h) * n + (row_ok ? i : 0)) * D;
  float q[32];
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    const float4 x = load4(Q + q_row + 4 * (part + TPR * m));
    q[4 * m] = x.x; q[4 * m + 1] = x.y; q[4 * m + 2] = x.z; q[4 * m + 3] = x.w;
  }
  const float scale = 1.0f / sqrtf(static_cast<float>(D));
  float m_run = -INFINITY, l_run = 0.0f;
  float acc[32];
#pragma unroll
  for (int e = 0; e < 32; ++e) acc[e] = 0.0f;
  MaskT Y = 0, Z = 0;

  const size_t kv_base = (static_cast<size_t>(b) * H_kv + kvh) * static_cast<size_t>(n) * D;
  const MaskT* bm_h = alibi ? nullptr : bmask + static_cast<size_t>(h) * n;
  // K3: one pass over the union window with weights c_ij (sw = s). K4 (varlen): one pass per hash k
  // over that hash's window with the hash-k masks alone, so each weight is hash k's 0/1 block
  // indicator (sw = 1); the passes share the running maximum, sum and accumulator.
  const int n_pass = varlen ? s : 1;
  const int sw = varlen ? 1 : s;
  // exact banded ALiBi: weight exp(-|i - j| / sigma_h) over |i - j| <= ceil(sigma_h ln(1/eps))
  const float inv_sigma = alibi ? static_cast<float>(1.0 / sigma[h]) : 0.0f;
  const int last_row = min(n, i0 + kTile) - 1;
  for (int pass = 0; pass < n_pass; ++pass) {
    const MaskT bits = varlen ? static_cast<MaskT>(static_cast<MaskT>(1) << pass) : FULL;
    const size_t span_at = varlen ? ((static_cast<size_t>(h) * s + pass) * T_tiles + t) * 2
                                  : (static_cast<size_t>(h) * T_tiles + t) * 2;
    int lo, hi;
    if (alibi) {
      const double wr = ceil(sigma[h] * log_inv_eps);
      const int reach = (wr >= static_cast<double>(n) || !(wr >= 0.0)) ? n : static_cast<int>(wr);
      lo = max(0, i0 - reach);
      hi = causal ? last_row : min(n - 1, last_row + reach);
    } else {
      lo = spans[span_at];
      hi = spans[span_at + 1];
    }
    if (lo < 0 || lo > i0 || hi >= n || hi < last_row) {
      flags |= PLSH_DEVERR_WINDOW;
      lo = max(0, min(lo, i0));
      hi = min(n - 1, max(hi, last_row));
    }
    const int n_below = (i0 - lo + kTile - 1) / kTile;
    const int n_above = causal ? 0 : (hi - i0) / kTile;
    const int total = 1 + n_below + n_above;
    for (int it = 0; it < total; ++it) {
      const int kind = it == 0 ? 0 : (it <= n_below ? 1 : 2);   // 0 diagonal, 1 below, 2 above
      const int j0 = kind == 0 ? i0 : (kind == 1 ? i0 - kTile * it : i0 + kTile * (it - n_below));
      __syncthreads();
      for (int idx = tid; idx < kTile * F4; idx += NT) {
        const int row = idx / F4, c4 = idx % F4;
        const int j = j0 + row;
        float4 kx = make_float4(0.f, 0.f, 0.f, 0.f), vx = kx;
        if (j >= 0 && j < n) {
          kx = load4(K + kv_base + static_cast<size_t>(j) * D + 4 * c4);
          vx = load4(V + kv_base + static_cast<size_t>(j) * D + 4 * c4);
        }
        store4(&sm.k[row * D + 4 * c4], kx);
        store4(&sm.v[row * D + 4 * c4], vx);
      }
      for (int c = tid; c <= kTile; c += NT) {
        const int j = j0 + c;
        sm.bm[c] = alibi ? static_cast<MaskT>(0) : static_cast<MaskT>(((j >= 0 && j < n) ? bm_h[j] : FULL) & bits);
      }
      __syncthreads();
      if (tid < kTile) {
        MaskT a = 0, z = 0;
        for (int q2 = tid + 1; q2 < kTile; ++q2) a |= sm.bm[q2];
        for (int q2 = 1; q2 <= tid; ++q2) z |= sm.bm[q2];
        sm.suf[tid] = a;
        sm.pre[tid] = z;
      }
      if (kind == 0 && part == 0) {
        unsigned char* wr = sm.wdiag + r * kDiagStride;
        wr[r] = static_cast<unsigned char>(sw);
        MaskT R = 0;
        for (int c = r - 1; c >= 0; --c) {
          R |= sm.bm[c + 1];
          wr[c] = static_cast<unsigned char>(sw - popc_mask(R));
        }
        sm.ycarry[r] = R | sm.bm[0];       // OR over [i0, i]
        R = 0;
        for (int c = r + 1; c < kTile; ++c) {
          R |= sm.bm[c];
          wr[c] = static_cast<unsigned char>(sw - popc_mask(R));
        }
        sm.zcarry[r] = R;                  // OR over (i, i0 + 127]
      }
      __syncthreads();
      if (kind == 2) Z |= sm.bm[0];          // now OR over (i, j0]

  #pragma unroll 1
      for (int chunk = 0; chunk < kTile / 32; ++chunk) {
        float sv[32];
        int wv[32];
  #pragma unroll
        for (int cc = 0; cc < 32; ++cc) {
          const int c = chunk * 32 + cc;
          int w;
          if (alibi) w = (causal && j0 + c > i) || j0 + c >= n ? 0 : 1;
          else if (kind == 0) w = (causal && c > r) ? 0 : sm.wdiag[r * kDiagStride + c];
          else if (kind == 1) w = sw - popc_mask(static_cast<MaskT>(sm.suf[c] | Y));
          else w = sw - popc_mask(static_cast<MaskT>(Z | sm.pre[c]));
          float dot = 0.0f;
  #pragma unroll
          for (int m = 0; m < 8; ++m) {
            const float4 kx = *reinterpret_cast<const float4*>(&sm.k[c * D + 4 * (part + TPR * m)]);
            dot = fmaf(q[4 * m], kx.x, dot);
            dot = fmaf(q[4 * m + 1], kx.y, dot);
            dot = fmaf(q[4 * m + 2], kx.z, dot);
            dot = fmaf(q[4 * m + 3], kx.w, dot);
          }
  #pragma unroll
          for (int o = TPR / 2; o >= 1; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
          sv[cc] = w > 0 ? dot * scale - (alibi ? fabsf(static_cast<float>(i - (j0 + c))) * inv_sigma : 0.0f)
                         : -INFINITY;
          wv[cc] = w;
        }
        float cmax = -INFINITY;
  #pragma unroll
        for (int cc = 0; cc < 32; ++cc) cmax = fmaxf(cmax, sv[cc]);
        if (cmax == -INFINITY) continue;
        const float m_new = fmaxf(m_run, cmax);
        const float corr = expf(m_run - m_new);   // 0 when m_run = -inf
        l_run *= corr;
  #pragma unroll
        for (int e = 0; e < 32; ++e) acc[e] *= corr;
        m_run = m_new;
  #pragma unroll
        for (int cc = 0; cc < 32; ++cc) {
          if (wv[cc] <= 0) continue;
          const int c = chunk * 32 + cc;
          const float p = static_cast<float>(wv[cc]) * expf(sv[cc] - m_run);
          l_run += p;
  #pragma unroll
          for (int m = 0; m < 8; ++m) {
            const float4 vx = *reinterpret_cast<const float4*>(&sm.v[c * D + 4 * (part + TPR * m)]);
            acc[4 * m] = fmaf(p, vx.x, acc[4 * m]);
            acc[4 * m + 1] = fmaf(p, vx.y, acc[4 * m + 1]);
            acc[4 * m + 2] = fmaf(p, vx.z, acc[4 * m + 2]);
            acc[4 * m + 3] = fmaf(p, vx.w, acc[4 * m + 3]);
          }
        }
      }
      if (kind == 0) {
        Y = sm.ycarry[r];
        Z = sm.zcarry[r];
      } else if (kind == 1) {
        Y |= static_cast<MaskT>(sm.bm[0] | sm.suf[0]);   // tile fully passed: OR over [j0, i]
      } else {
        Z |= sm.pre[kTile - 1];                           // OR over (i, j0 + 127]
      }
    }
  }

  if (row_ok) {
    const float inv = 1.0f / l_run;
    const size_t o_row = ((static_cast<size_t>(b) * H + h) * n + i) * D;
#pragma unroll
    for (int m = 0; m < 8; ++m)
      store4(O + o_row + 4 * (part + TPR * m),
             make_float4(acc[4 * m] * inv, acc[4 * m + 1] * inv, acc[4 * m + 2] * inv, acc[4 * m + 3] * inv));
    if (part == 0)
      row_sum[(static_cast<size_t>(b) * H + h) * n + i] = logf(l_run) + m_run - (alibi ? 0.0f : logf(static_cast<float>(s)));
  }
  if (flags) atomicOr(err, flags);
}

template <typename T, int D, typename MaskT>
int launch_simt_typed(const AttnArgs& a, cudaStream_t st) {
  auto kern = attn_simt_kernel<T, D, MaskT>;
  const size_t smem = sizeof(SimtSmem<D, MaskT>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(attn_simt_kernel)");
  dim3 grid(ceil_div(a.n, kTile), a.H, a.B);
  kern<<<grid, kTile * (D / 32), smem, st>>>(
      static_cast<const T*>(a.Q), static_cast<const T*>(a.K), static_cast<const T*>(a.V), a.H, a.H_kv, a.n, a.s,
      a.causal, a.sigma, a.table, a.spans, static_cast<const MaskT*>(a.bmask), static_cast<T*>(a.O), a.row_sum,
      a.err, a.varlen, a.alibi, a.log_inv_eps);
  e = cudaGetLastError();
  return e == cudaSuccess ? PLSH_OK : cuda_fail(e, "attn_simt_kernel launch");
}

template <typename T, int D>
int launch_simt_mask(const AttnArgs& a, cudaStream_t st) {
  return a.s <= 32 ? launch_simt_typed<T, D, uint32_t>(a, st)
                   : launch_simt_typed<T, D, unsigned long long>(a, st);
}

}  // namespace

int launch_attention_simt(const AttnArgs& a, cudaStream_t st) {
  if (a.dtype == PLSH_F32)
    return a.d == 64 ? launch_simt_mask<float, 64>(a, st) : launch_simt_mask<float, 128>(a, st);
  return a.d == 64 ? launch_simt_mask<__nv_bfloat16, 64>(a, st) : launch_simt_mask<__nv_bfloat16, 128>(a, st);
}

}  // namespace plsh
