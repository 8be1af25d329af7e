// Entry points of libplsh (declared in include/plsh.h): argument checks,
// then the launch. Every check that can be made on the host is made here,
// before anything is enqueued.
#include <cmath>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "plsh_internal.h"

namespace plsh {

namespace {
thread_local char g_last_error[512] = "";
}

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(PLSH_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_sizes(const char* fn, int H, int s, int n) {
  if (H < 1 || n < 1) return fail(PLSH_ERR_INVALID_ARG, "%s: need H >= 1 and n >= 1 (H=%d n=%d)", fn, H, n);
  if (s < 1 || s > PLSH_MAX_S)
    return fail(PLSH_ERR_INVALID_ARG, "%s: need 1 <= s <= %d (s=%d)", fn, PLSH_MAX_S, s);
  if (H > 65535) return fail(PLSH_ERR_RANGE, "%s: H=%d exceeds 65535", fn, H);
  if (n > (1 << 30)) return fail(PLSH_ERR_RANGE, "%s: n=%d exceeds 2^30", fn, n);
  return PLSH_OK;
}

}  // namespace
}  // namespace plsh

using plsh::fail;

extern "C" const char* plsh_last_error(void) { return plsh::g_last_error; }

extern "C" int plsh_version(void) { return 100; }

// ---------------------------------------------------------------- bounded waits (failure detection)

namespace plsh {
namespace {
std::atomic<uint64_t> g_wait_limit_ns{0};  // 0: the kernel's default
std::atomic<int> g_withhold_mma{0};
}  // namespace

uint64_t wait_limit_ns() {
  const uint64_t v = g_wait_limit_ns.load(std::memory_order_relaxed);
  return v ? v : plsh::kDefaultWaitLimitNs;
}
bool withhold_mma() { return g_withhold_mma.load(std::memory_order_relaxed) != 0; }
}  // namespace plsh

extern "C" int plsh_set_wait_limit_ns(uint64_t limit_ns) {
  if (limit_ns > PLSH_MAX_WAIT_LIMIT_NS)
    return fail(PLSH_ERR_RANGE, "plsh_set_wait_limit_ns: %llu ns exceeds the maximum %llu ns",
                static_cast<unsigned long long>(limit_ns), static_cast<unsigned long long>(PLSH_MAX_WAIT_LIMIT_NS));
  plsh::g_wait_limit_ns.store(limit_ns, std::memory_order_relaxed);
  return PLSH_OK;
}

extern "C" int plsh_test_withhold_mma(int on) {
  plsh::g_withhold_mma.store(on ? 1 : 0, std::memory_order_relaxed);
  return PLSH_OK;
}

extern "C" int plsh_sample_bins(const double* table_dev, int H, int s, int n, int32_t* ids_dev,
                                uint32_t* err_dev, void* stream) {
  if (int rc = plsh::check_sizes("plsh_sample_bins", H, s, n)) return rc;
  if (!table_dev || !ids_dev || !err_dev) return fail(PLSH_ERR_INVALID_ARG, "plsh_sample_bins: null pointer");
  return plsh::launch_sample_bins(table_dev, H, s, n, ids_dev, err_dev, static_cast<cudaStream_t>(stream));
}

extern "C" int plsh_window(const int32_t* ids_dev, int H, int s, int n, int causal, int32_t* bmax_dev,
                           int32_t* tile_span_dev, void* bmask_dev, uint32_t* err_dev, void* stream) {
  if (int rc = plsh::check_sizes("plsh_window", H, s, n)) return rc;
  if (!ids_dev || !bmax_dev || !tile_span_dev || !bmask_dev || !err_dev)
    return fail(PLSH_ERR_INVALID_ARG, "plsh_window: null pointer");
  if (causal != 0 && causal != 1) return fail(PLSH_ERR_INVALID_ARG, "plsh_window: causal must be 0 or 1");
  return plsh::launch_window(ids_dev, H, s, n, causal, bmax_dev, tile_span_dev, bmask_dev, err_dev,
                             static_cast<cudaStream_t>(stream));
}

extern "C" int plsh_window_from_table(const double* table_dev, int H, int s, int n, int causal, int32_t* bmax_dev,
                                      int32_t* tile_span_dev, void* bmask_dev, uint32_t* err_dev, void* stream) {
  if (int rc = plsh::check_sizes("plsh_window_from_table", H, s, n)) return rc;
  if (!table_dev || !bmax_dev || !tile_span_dev || !bmask_dev || !err_dev)
    return fail(PLSH_ERR_INVALID_ARG, "plsh_window_from_table: null pointer");
  if (causal != 0 && causal != 1)
    return fail(PLSH_ERR_INVALID_ARG, "plsh_window_from_table: causal must be 0 or 1");
  return plsh::launch_window_from_table(table_dev, H, s, n, causal, bmax_dev, tile_span_dev, bmask_dev, err_dev,
                                        static_cast<cudaStream_t>(stream));
}

namespace plsh {
namespace {

// Checks shared by the two attention entry points.
int check_attention(const char* fn, const void* Q, const void* K, const void* V, int dtype, int B, int H,
                    int H_kv, int n, int d, int s, int causal, const void* bmask_dev, const void* O,
                    const float* row_sum, const uint32_t* err_dev) {
  if (int rc = check_sizes(fn, H, s, n)) return rc;
  if (B < 1 || B > 65535) return fail(PLSH_ERR_INVALID_ARG, "%s: need 1 <= B <= 65535 (B=%d)", fn, B);
  if (H_kv < 1 || H % H_kv != 0)
    return fail(PLSH_ERR_INVALID_ARG, "%s: H_kv must divide H (H=%d H_kv=%d)", fn, H, H_kv);
  if (causal != 0 && causal != 1) return fail(PLSH_ERR_INVALID_ARG, "%s: causal must be 0 or 1", fn);
  if (dtype != PLSH_BF16 && dtype != PLSH_F32) return fail(PLSH_ERR_UNSUPPORTED, "%s: dtype %d", fn, dtype);
  if (d != 64 && d != 128) return fail(PLSH_ERR_UNSUPPORTED, "%s: head dim %d (64 or 128 supported)", fn, d);
  if (!Q || !K || !V || !O || !row_sum || !bmask_dev || !err_dev)
    return fail(PLSH_ERR_INVALID_ARG, "%s: null pointer", fn);
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
    return fail(PLSH_ERR_INVALID_ARG, "%s: Q, K, V and O must be 16-byte aligned", fn);
  return PLSH_OK;
}

int launch_attention(const AttnArgs& a, cudaStream_t st) {
  if (a.dtype == PLSH_BF16 && a.d == 128) return launch_attention_tc(a, st);
  return launch_attention_simt(a, st);
}

}  // namespace
}  // namespace plsh

extern "C" int plsh_attention_fwd(const void* Q, const void* K, const void* V, int dtype, int B, int H,
                                  int H_kv, int n, int d, const double* sigma_dev, int s,
                                  const double* table_dev, const int32_t* tile_span_dev,
                                  const void* bmask_dev, int causal, void* O, float* row_sum,
                                  uint32_t* err_dev, void* stream) {
  const char* fn = "plsh_attention_fwd";
  if (int rc = plsh::check_attention(fn, Q, K, V, dtype, B, H, H_kv, n, d, s, causal, bmask_dev, O, row_sum,
                                     err_dev))
    return rc;
  if (!tile_span_dev) return fail(PLSH_ERR_INVALID_ARG, "%s: null pointer", fn);
  plsh::AttnArgs a{Q, K, V, dtype, B, H, H_kv, n, d, s, causal, sigma_dev, table_dev,
                   tile_span_dev, bmask_dev, O, row_sum, err_dev, 0};
  return plsh::launch_attention(a, static_cast<cudaStream_t>(stream));
}

extern "C" size_t plsh_varlen_scratch_bytes(int H, int s, int n) {
  if (H < 1 || s < 1 || n < 1) return 0;
  return static_cast<size_t>(H) * static_cast<size_t>(s) * static_cast<size_t>(plsh::ceil_div(n, PLSH_TILE)) * 2 *
         sizeof(int32_t);
}

extern "C" int plsh_varlen_spans(const int32_t* ids_dev, int H, int s, int n, int causal, int32_t* spans_dev,
                                 void* stream) {
  const char* fn = "plsh_varlen_spans";
  if (int rc = plsh::check_sizes(fn, H, s, n)) return rc;
  if (causal != 0 && causal != 1) return fail(PLSH_ERR_INVALID_ARG, "%s: causal must be 0 or 1", fn);
  if (!ids_dev || !spans_dev) return fail(PLSH_ERR_INVALID_ARG, "%s: null pointer", fn);
  return plsh::launch_varlen_spans(ids_dev, H, s, n, causal, spans_dev, static_cast<cudaStream_t>(stream));
}

extern "C" int plsh_attention_varlen_fwd(const void* Q, const void* K, const void* V, int dtype, int B, int H,
                                         int H_kv, int n, int d, const double* sigma_dev, int s,
                                         const double* table_dev, const int32_t* ids_dev, const void* bmask_dev,
                                         int causal, void* scratch_dev, size_t scratch_bytes, void* O,
                                         float* row_sum, uint32_t* err_dev, void* stream) {
  const char* fn = "plsh_attention_varlen_fwd";
  if (int rc = plsh::check_attention(fn, Q, K, V, dtype, B, H, H_kv, n, d, s, causal, bmask_dev, O, row_sum,
                                     err_dev))
    return rc;
  if (!ids_dev || !scratch_dev) return fail(PLSH_ERR_INVALID_ARG, "%s: null pointer", fn);
  if (!plsh::aligned16(scratch_dev)) return fail(PLSH_ERR_INVALID_ARG, "%s: scratch must be 16-byte aligned", fn);
  const size_t need = plsh_varlen_scratch_bytes(H, s, n);
  if (scratch_bytes < need)
    return fail(PLSH_ERR_INVALID_ARG, "%s: scratch holds %zu bytes, %zu needed", fn, scratch_bytes, need);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* spans = static_cast<int32_t*>(scratch_dev);
  if (int rc = plsh::launch_varlen_spans(ids_dev, H, s, n, causal, spans, st)) return rc;
  plsh::AttnArgs a{Q, K, V, dtype, B, H, H_kv, n, d, s, causal, sigma_dev, table_dev,
                   spans, bmask_dev, O, row_sum, err_dev, 1};
  return plsh::launch_attention(a, st);
}

// ---------------------------------------------------------------- comparator without caller scratch
//
// plsh_attention_varlen_fwd_static: the per-sample comparator for callers that cannot hand the
// library any device memory of their own for scratch. Such a caller has only its inputs and
// outputs: it may run where the device allocator must not be entered (a hook inside the
// caller's own memory management) or where every device allocation is budgeted up front. The
// per-hash windows then live in a fixed file-scope device buffer of this library.
namespace plsh {
namespace {

// Per-hash windows of the comparator: [H][s][ceil(n/128)][2] int32, fully written by the window
// kernel before the attention kernel reads it, so nothing in it needs to start at zero.
static __device__ __align__(256) int32_t g_varlen_static_scratch[PLSH_VARLEN_STATIC_SCRATCH_BYTES / sizeof(int32_t)];

// The buffer's device address in the current context. Looked up on every call rather than
// cached: the lookup allocates nothing, and a cached address would outlive a reset or re-created
// context, after which the module (and the buffer) may sit elsewhere.
int static_scratch_ptr(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_varlen_static_scratch);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(g_varlen_static_scratch)");
  *out = p;
  return PLSH_OK;
}

}  // namespace
}  // namespace plsh

extern "C" int plsh_attention_varlen_fwd_static(const void* Q, const void* K, const void* V, int dtype, int B,
                                                int H, int H_kv, int n, int d, const double* sigma_dev, int s,
                                                const double* table_dev, const int32_t* ids_dev,
                                                const void* bmask_dev, int causal, void* O, float* row_sum,
                                                uint32_t* err_dev, void* stream) {
  const char* fn = "plsh_attention_varlen_fwd_static";
  if (int rc = plsh::check_attention(fn, Q, K, V, dtype, B, H, H_kv, n, d, s, causal, bmask_dev, O, row_sum,
                                     err_dev))
    return rc;
  if (!ids_dev) return fail(PLSH_ERR_INVALID_ARG, "%s: null pointer", fn);
  const size_t need = plsh_varlen_scratch_bytes(H, s, n);
  if (need > PLSH_VARLEN_STATIC_SCRATCH_BYTES)
    return fail(PLSH_ERR_RANGE,
                "%s: the per-hash windows need %zu bytes (8 * H * s * ceil(n/128)), more than the %zu-byte "
                "static buffer; use plsh_attention_varlen_fwd with caller scratch",
                fn, need, static_cast<size_t>(PLSH_VARLEN_STATIC_SCRATCH_BYTES));
  void* scratch = nullptr;
  if (int rc = plsh::static_scratch_ptr(&scratch)) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* spans = static_cast<int32_t*>(scratch);
  if (int rc = plsh::launch_varlen_spans(ids_dev, H, s, n, causal, spans, st)) return rc;
  plsh::AttnArgs a{Q, K, V, dtype, B, H, H_kv, n, d, s, causal, sigma_dev, table_dev,
                   spans, bmask_dev, O, row_sum, err_dev, 1};
  return plsh::launch_attention(a, st);
}

// ---------------------------------------------------------------- exact banded ALiBi (the competitor)

extern "C" int plsh_alibi_banded_fwd(const void* Q, const void* K, const void* V, int dtype, int B, int H, int H_kv,
                                     int n, int d, const double* sigma_dev, double eps, int causal, void* O,
                                     float* row_sum, uint32_t* err_dev, void* stream) {
  const char* fn = "plsh_alibi_banded_fwd";
  if (H < 1 || n < 1) return fail(PLSH_ERR_INVALID_ARG, "%s: need H >= 1 and n >= 1 (H=%d n=%d)", fn, H, n);
  if (H > 65535) return fail(PLSH_ERR_RANGE, "%s: H=%d exceeds 65535", fn, H);
  if (n > (1 << 30)) return fail(PLSH_ERR_RANGE, "%s: n=%d exceeds 2^30", fn, n);
  if (B < 1 || B > 65535) return fail(PLSH_ERR_INVALID_ARG, "%s: need 1 <= B <= 65535 (B=%d)", fn, B);
  if (H_kv < 1 || H % H_kv != 0)
    return fail(PLSH_ERR_INVALID_ARG, "%s: H_kv must divide H (H=%d H_kv=%d)", fn, H, H_kv);
  if (causal != 0 && causal != 1) return fail(PLSH_ERR_INVALID_ARG, "%s: causal must be 0 or 1", fn);
  if (dtype != PLSH_BF16 && dtype != PLSH_F32) return fail(PLSH_ERR_UNSUPPORTED, "%s: dtype %d", fn, dtype);
  if (d != 64 && d != 128) return fail(PLSH_ERR_UNSUPPORTED, "%s: head dim %d (64 or 128 supported)", fn, d);
  if (!(eps > 0.0 && eps < 1.0)) return fail(PLSH_ERR_INVALID_ARG, "%s: need 0 < eps < 1 (eps=%g)", fn, eps);
  if (!Q || !K || !V || !O || !row_sum || !sigma_dev || !err_dev)
    return fail(PLSH_ERR_INVALID_ARG, "%s: null pointer", fn);
  if (!plsh::aligned16(Q) || !plsh::aligned16(K) || !plsh::aligned16(V) || !plsh::aligned16(O))
    return fail(PLSH_ERR_INVALID_ARG, "%s: Q, K, V and O must be 16-byte aligned", fn);
  if (static_cast<long long>(B) * H * plsh::ceil_div(n, PLSH_TILE) > 0x7fffffffLL)
    return fail(PLSH_ERR_RANGE, "%s: too many query tiles", fn);
  plsh::AttnArgs a{Q, K, V, dtype, B, H, H_kv, n, d, 1, causal, sigma_dev, nullptr,
                   nullptr, nullptr, O, row_sum, err_dev, 0, 1, -std::log(eps)};
  return plsh::launch_attention(a, static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------- decode

extern "C" size_t plsh_decode_scratch_bytes(int B, int H, int m, int d) {
  if (B < 1 || H < 1 || m < 1 || d < 1) return 0;
  return plsh::decode_scratch_bytes(static_cast<long long>(B) * H * m, d);
}

extern "C" int plsh_decode_fwd(const void* Q, const int32_t* pos_dev, int m, const void* K, const void* V, int dtype,
                               int B, int H, int H_kv, int n, int d, int s, const void* bmask_dev, int causal,
                               void* scratch_dev, size_t scratch_bytes, void* O, float* row_sum, uint32_t* err_dev,
                               void* stream) {
  const char* fn = "plsh_decode_fwd";
  if (int rc = plsh::check_attention(fn, Q, K, V, dtype, B, H, H_kv, n, d, s, causal, bmask_dev, O, row_sum,
                                     err_dev))
    return rc;
  if (m < 1) return fail(PLSH_ERR_INVALID_ARG, "%s: need m >= 1 (m=%d)", fn, m);
  if (!pos_dev || !scratch_dev) return fail(PLSH_ERR_INVALID_ARG, "%s: null pointer", fn);
  if (static_cast<size_t>(m) * plsh::kDecodeMaxSplit > (size_t{1} << 31) - 1)
    return fail(PLSH_ERR_RANGE, "%s: m=%d too large", fn, m);
  const size_t need = plsh_decode_scratch_bytes(B, H, m, d);
  if (scratch_bytes < need)
    return fail(PLSH_ERR_INVALID_ARG, "%s: scratch holds %zu bytes, %zu needed", fn, scratch_bytes, need);
  plsh::DecodeArgs a{Q, pos_dev, m, K, V, dtype, B, H, H_kv, n, d, s, causal, bmask_dev, O, row_sum, err_dev,
                     static_cast<float*>(scratch_dev)};
  return plsh::launch_decode(a, static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------- backward

extern "C" int plsh_attention_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                                  const float* row_sum, int dtype, int B, int H, int H_kv, int n, int d, int s,
                                  const int32_t* ids_dev, int causal, float* delta_dev, void* dQ, void* dK,
                                  void* dV, uint32_t* err_dev, void* stream) {
  const char* fn = "plsh_attention_bwd";
  if (int rc = plsh::check_sizes(fn, H, s, n)) return rc;
  if (B < 1 || B > 65535) return fail(PLSH_ERR_INVALID_ARG, "%s: need 1 <= B <= 65535 (B=%d)", fn, B);
  if (H_kv < 1 || H % H_kv != 0)
    return fail(PLSH_ERR_INVALID_ARG, "%s: H_kv must divide H (H=%d H_kv=%d)", fn, H, H_kv);
  if (causal != 0 && causal != 1) return fail(PLSH_ERR_INVALID_ARG, "%s: causal must be 0 or 1", fn);
  if (dtype != PLSH_BF16 && dtype != PLSH_F32) return fail(PLSH_ERR_UNSUPPORTED, "%s: dtype %d", fn, dtype);
  if (d != 64 && d != 128) return fail(PLSH_ERR_UNSUPPORTED, "%s: head dim %d (64 or 128 supported)", fn, d);
  if (!Q || !K || !V || !O || !dO || !row_sum || !ids_dev || !delta_dev || !dQ || !dK || !dV || !err_dev)
    return fail(PLSH_ERR_INVALID_ARG, "%s: null pointer", fn);
  if (!plsh::aligned16(Q) || !plsh::aligned16(K) || !plsh::aligned16(V) || !plsh::aligned16(O) ||
      !plsh::aligned16(dO))
    return fail(PLSH_ERR_INVALID_ARG, "%s: Q, K, V, O and dO must be 16-byte aligned", fn);
  if (static_cast<size_t>(B) * H * n > (size_t{1} << 31))
    return fail(PLSH_ERR_RANGE, "%s: B*H*n exceeds 2^31", fn);
  plsh::BwdArgs a{Q, K, V, O, dO, row_sum, ids_dev, dtype, B, H, H_kv, n, d, s, causal, delta_dev, dQ, dK, dV};
  return plsh::launch_bwd(a, static_cast<cudaStream_t>(stream));
}

extern "C" int plsh_attention_bwd_tc(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                                     const float* row_sum, int B, int H, int H_kv, int n, int d, int s,
                                     const void* bmask_dev, const int32_t* tile_span_dev,
                                     const int32_t* key_span_dev, int causal, float* delta_dev, void* dQ, void* dK,
                                     void* dV, uint32_t* err_dev, void* stream) {
  const char* fn = "plsh_attention_bwd_tc";
  if (int rc = plsh::check_sizes(fn, H, s, n)) return rc;
  if (B < 1 || B > 65535) return fail(PLSH_ERR_INVALID_ARG, "%s: need 1 <= B <= 65535 (B=%d)", fn, B);
  if (H_kv < 1 || H % H_kv != 0)
    return fail(PLSH_ERR_INVALID_ARG, "%s: H_kv must divide H (H=%d H_kv=%d)", fn, H, H_kv);
  if (causal != 0 && causal != 1) return fail(PLSH_ERR_INVALID_ARG, "%s: causal must be 0 or 1", fn);
  if (d != 128) return fail(PLSH_ERR_UNSUPPORTED, "%s: head dim %d (the tensor-core backward needs 128)", fn, d);
  if (!Q || !K || !V || !O || !dO || !row_sum || !bmask_dev || !tile_span_dev || !key_span_dev || !delta_dev || !dQ ||
      !dK || !dV || !err_dev)
    return fail(PLSH_ERR_INVALID_ARG, "%s: null pointer", fn);
  if (!plsh::aligned16(Q) || !plsh::aligned16(K) || !plsh::aligned16(V) || !plsh::aligned16(O) ||
      !plsh::aligned16(dO) || !plsh::aligned16(dQ) || !plsh::aligned16(dK) || !plsh::aligned16(dV))
    return fail(PLSH_ERR_INVALID_ARG, "%s: Q, K, V, O, dO, dQ, dK and dV must be 16-byte aligned", fn);
  if (static_cast<size_t>(B) * H * n > (size_t{1} << 31))
    return fail(PLSH_ERR_RANGE, "%s: B*H*n exceeds 2^31", fn);
  plsh::BwdTcArgs a{Q, K, V, O, dO, row_sum, bmask_dev, tile_span_dev, key_span_dev, B, H, H_kv, n, d, s, causal,
                    delta_dev, dQ, dK, dV, err_dev};
  return plsh::launch_bwd_tc(a, static_cast<cudaStream_t>(stream));
}
