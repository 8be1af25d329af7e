// Internal declarations shared by the libplsh translation units.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "plsh.h"

namespace plsh {

// Records a message for plsh_last_error() and returns `code`.
int fail(int code, const char* fmt, ...);
// Maps a CUDA error to PLSH_ERR_CUDA with the call site in the message.
int cuda_fail(cudaError_t e, const char* what);

inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Process-wide settings of the fused attention kernel's bounded waits (plsh_set_wait_limit_ns,
// plsh_test_withhold_mma), read at each launch.
constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;
uint64_t wait_limit_ns();
bool withhold_mma();

// Kernel launchers (each returns PLSH_OK or an error code; arguments are
// already validated by the entry point).
int launch_sample_bins(const double* table, int H, int s, int n, int32_t* ids, uint32_t* err,
                       cudaStream_t st);
int launch_window(const int32_t* ids, int H, int s, int n, int causal, int32_t* bmax,
                  int32_t* spans, void* bmask, uint32_t* err, cudaStream_t st);
int launch_window_from_table(const double* table, int H, int s, int n, int causal, int32_t* bmax,
                             int32_t* spans, void* bmask, uint32_t* err, cudaStream_t st);

struct AttnArgs {
  const void* Q; const void* K; const void* V;
  int dtype, B, H, H_kv, n, d, s, causal;
  const double* sigma; const double* table;
  const int32_t* spans; const void* bmask;
  void* O; float* row_sum; uint32_t* err;
  // 0: K3 (spans = [H][T][2] union windows, weights c_ij). 1: K4, the per-sample comparator
  // (spans = [H][s][T][2] per-hash windows; each sample's block indicator, summed over samples).
  int varlen;
  // 1: exact banded ALiBi instead of Positional LSH (spans, bmask, table unused): weights
  // exp(-|i - j| / sigma_h) over |i - j| <= ceil(sigma_h ln(1/eps)), with log_inv_eps = ln(1/eps)
  int alibi;
  double log_inv_eps;
};
// Decode: query rows Q [B][H][m][d] at positions pos [m] against K, V [B][H_kv][n][d].
// part: caller scratch (decode_scratch_bytes): B*H*m*kDecodeMaxSplit*(d+2) floats for the partial
// results of a row's work units, the call's work list, then one unsigned counter per row (zero before
// the first call; every completed call leaves them zero).
constexpr int kDecodeMaxSplit = 8;
struct DecodeArgs {
  const void* Q; const int32_t* pos; int m;
  const void* K; const void* V;
  int dtype, B, H, H_kv, n, d, s, causal;
  const void* bmask;
  void* O; float* row_sum; uint32_t* err;
  float* part;
};
int launch_decode(const DecodeArgs& a, cudaStream_t st);
// Bytes of decode scratch for `rows` query rows of width d (partial results, per-row walk data,
// one counter per row at the end).
size_t decode_scratch_bytes(long long rows, int d);
// Backward: dQ, dK, dV of T~ (Q, O, dO, dQ [B][H][n][d]; K, V, dK, dV [B][H_kv][n][d]).
struct BwdArgs {
  const void* Q; const void* K; const void* V; const void* O; const void* dO;
  const float* row_sum; const int32_t* ids;
  int dtype, B, H, H_kv, n, d, s, causal;
  float* delta;
  void* dQ; void* dK; void* dV;
};
int launch_bwd(const BwdArgs& a, cudaStream_t st);
// D_i = dO_i . O_i for `rows` rows of d elements (the backward's row dots).
int launch_bwd_delta(const void* O, const void* dO, int dtype, int d, size_t rows, float* delta, cudaStream_t st);
// Tensor-core backward (bf16, d = 128): masks and windows instead of ids. tile_spans are the forward's
// windows (plsh_window with the same causal flag), key_spans the non-causal ones (the query rows that
// reach each key tile, by the symmetry of c_ij).
struct BwdTcArgs {
  const void* Q; const void* K; const void* V; const void* O; const void* dO;
  const float* row_sum; const void* bmask; const int32_t* tile_spans; const int32_t* key_spans;
  int B, H, H_kv, n, d, s, causal;
  float* delta;
  void* dQ; void* dK; void* dV;
  uint32_t* err;
};
int launch_bwd_tc(const BwdTcArgs& a, cudaStream_t st);
int launch_varlen_spans(const int32_t* ids, int H, int s, int n, int causal, int32_t* spans, cudaStream_t st);
int launch_attention_simt(const AttnArgs& a, cudaStream_t st);
int launch_attention_tc(const AttnArgs& a, cudaStream_t st);

}  // namespace plsh
