/*
 * plsh.h -- C ABI of libplsh: Positional-LSH approximate ALiBi attention on
 * NVIDIA B200 (sm_100a).
 *
 * Method: "Positional LSH: Binary Block Matrix Approximation for Attention
 * with Linear Biases" (Wolfson & Wagner, arXiv 2605.09472), as summarised by
 * the gist.science explainer pages (nl/zh/ja). ALiBi's bias matrix
 * L*_ij = e^{-|i-j|/sigma} is the expectation of the binary block masks M(h)
 * of random binnings of the token positions (technical summary, Methodology
 * 1, "mechanism" and "expectation"); the mean M~ of s such masks approximates
 * it (Methodology 2, Theorem 2.1), and attention weighted by M~ approximates
 * ALiBi attention (Methodology 3, Theorem 2.2; Results, convergence of
 * ||T* - T~||). This library computes
 *
 *     T~ = D~^{-1} (exp(Q K^T / sqrt d) o M~) V,   M~ = (1/s) sum_k M(h_k),
 *
 * optionally with the causal mask j <= i, for grouped-query attention.
 *
 * Conventions for every entry point:
 *   - Returns PLSH_OK (0) or a PLSH_ERR_* code; on error nothing was
 *     launched and plsh_last_error() (thread-local) says why.
 *   - "_dev" pointers are device memory owned by the caller; "_host"
 *     pointers are host memory owned by the caller. The library allocates
 *     no device memory and keeps no state between calls except the
 *     thread-local error string and a cached driver entry point.
 *   - Device work is enqueued on `stream` (a cudaStream_t passed as void*,
 *     NULL = legacy default stream) and is asynchronous: no entry point
 *     synchronises the device.
 *   - err_dev is a caller-zeroed device uint32 word. Kernels OR PLSH_DEVERR_*
 *     bits into it when they meet bad data that only the device can see
 *     (a bin id overflowing int32, a window outside [0, n), a bounded wait
 *     that gave up). Read it after the stream has finished. A kernel that
 *     sets a bit still ends normally; its outputs are then unspecified.
 *   - Positions are 0-based. Tensors are dense row-major (C order).
 */
#ifndef PLSH_H_
#define PLSH_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PLSH_API __attribute__((visibility("default")))
#else
#define PLSH_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
#define PLSH_OK               0
#define PLSH_ERR_INVALID_ARG  1  /* a null pointer, a negative size, s out of range, H % H_kv != 0 */
#define PLSH_ERR_UNSUPPORTED  2  /* head dim / dtype combination without a kernel */
#define PLSH_ERR_RANGE        3  /* a size whose index arithmetic would overflow */
#define PLSH_ERR_CUDA         4  /* a CUDA runtime or driver call failed */

/* Bits a kernel ORs into *err_dev. */
#define PLSH_DEVERR_RANGE    1u  /* a relative bin id did not fit in int32 */
#define PLSH_DEVERR_TABLE    2u  /* a table entry with delta not finite and > 0, or u not finite */
#define PLSH_DEVERR_WINDOW   4u  /* a tile window outside [0, n) or not covering the tile's own rows */
#define PLSH_DEVERR_TIMEOUT  8u  /* a bounded wait on a barrier gave up (the kernel returned early) */
#define PLSH_DEVERR_SIGMA   16u  /* a per-head sigma not finite and > 0 */
#define PLSH_DEVERR_POSITION 32u /* a decode query position outside [0, n) */

#define PLSH_TILE   128   /* query/key tile height of the windows */
#define PLSH_MAX_S  64    /* most hashes per head (one bit each in a 64-bit boundary mask) */

/* dtype codes for Q, K, V and O. */
#define PLSH_BF16 0
#define PLSH_F32  1

/* Thread-local description of the last error returned on this thread. */
PLSH_API const char* plsh_last_error(void);

/* ABI version (major * 100 + minor). */
PLSH_API int plsh_version(void);

/*
 * Failure detection of the fused attention kernel. The pages have no
 * counterpart: these govern how the kernel gives up, not what it computes.
 *
 * Every wait of the tensor-core attention kernel (plsh_attention_fwd,
 * plsh_attention_varlen_fwd[_static], plsh_alibi_banded_fwd with bf16,
 * d = 128), of the tensor-core backward (plsh_attention_bwd_tc) and of the
 * decode kernels (plsh_decode_fwd) on one of its roles is bounded in
 * wall-clock time. A wait that runs out sets PLSH_DEVERR_TIMEOUT in err_dev;
 * every role then leaves its loop, copies and tensor-core operations already
 * in flight are drained (with a separate limit of 0.1 s), Tensor Memory is
 * freed and the kernel returns, so the context stays usable. The outputs of
 * such a launch are unspecified.
 *
 * plsh_set_wait_limit_ns -- the limit for launches made after the call, in
 *   every host thread. 0 restores the default (2 s); above
 *   PLSH_MAX_WAIT_LIMIT_NS (60 s) returns PLSH_ERR_RANGE and changes nothing.
 *
 * plsh_test_withhold_mma -- test hook: while `on` is nonzero, the attention
 *   kernel's tensor-core issuer issues nothing, so every wait for a tile of
 *   scores runs out after the wait limit, and the decode kernel's producer
 *   issues no copies, so every wait for a segment runs out. For testing the
 *   failure path only (pair it with a short limit); off by default.
 */
#define PLSH_MAX_WAIT_LIMIT_NS 60000000000ull
PLSH_API int plsh_set_wait_limit_ns(uint64_t limit_ns);
PLSH_API int plsh_test_withhold_mma(int on);

/*
 * plsh_draw_table -- the (delta, u) table of s random binnings per head, on
 * the host.
 *
 * Cites: Methodology 1 (random binning of the integer positions, after
 * Rahimi & Recht's Random Binning Features for the Laplace kernel) and
 * Methodology 2 (s i.i.d. hashes; the Gamma law behind the binning).
 * For head h and hash k: delta = -sigma_h (ln U1 + ln U2) ~ Gamma(shape 2,
 * scale sigma_h) and u = U3 * delta ~ U[0, delta), with U1, U2 in (0,1) and
 * U3 in [0,1) taken from SplitMix64(seed) outputs ((h << 16) | k) * 3 + 0,1,2
 * (U_open = ((z >> 12) + 1/2) 2^-52, U3 = (z >> 11) 2^-53). A table with s
 * hashes is a prefix of one with more.
 *
 *   seed        64-bit seed.
 *   H           heads, >= 1.
 *   s           hashes per head, 1..PLSH_MAX_S.
 *   sigma_host  [H] doubles, each finite and > 0 (else PLSH_ERR_INVALID_ARG).
 *   table_host  [H][s][2] doubles written as (delta, u).
 * Pure host code; needs no GPU.
 */
PLSH_API int plsh_draw_table(uint64_t seed, int H, int s, const double* sigma_host, double* table_host);

/*
 * plsh_draw_table_heads -- rows h0 .. h0 + H - 1 of the table plsh_draw_table
 * would draw for a larger head count: row h comes from the counters of head
 * h0 + h, so the slices that the ranks of a head partition draw concatenate,
 * bit for bit, to the whole table. (The pages shard nothing; this only lets a
 * problem be split over devices by heads.)
 *
 *   h0          first global head, >= 0, with h0 + H <= PLSH_MAX_HEADS.
 *   H, s, sigma_host, table_host   as plsh_draw_table, for the H heads of the
 *               slice (sigma_host[h] belongs to global head h0 + h).
 * Pure host code; needs no GPU.
 */
#define PLSH_MAX_HEADS 65536
PLSH_API int plsh_draw_table_heads(uint64_t seed, int h0, int H, int s, const double* sigma_host,
                                   double* table_host);

/*
 * plsh_sample_bins (K1) -- bin ids of every (head, hash, position).
 *
 * Cites: Methodology 1, mechanism (h splits the positions into contiguous
 * bins). id_{h,k}(i) = floor((i + u)/delta) - floor(u/delta) with IEEE
 * float64 add and divide, round to nearest, so ids are bit-exact with any
 * IEEE float64 evaluation of the same formula.
 *
 *   table_dev  [H][s][2] doubles (delta, u).
 *   H, s, n    heads, hashes (1..PLSH_MAX_S), positions (>= 1).
 *   ids_dev    [H][s][n] int32 out.
 *   err_dev    device error word (PLSH_DEVERR_RANGE, PLSH_DEVERR_TABLE).
 */
PLSH_API int plsh_sample_bins(const double* table_dev, int H, int s, int n, int32_t* ids_dev,
                     uint32_t* err_dev, void* stream);

/*
 * plsh_window (K2) -- b_max, per-tile key windows and boundary masks.
 *
 * Cites: Methodology 1, structure (blocks are contiguous and do not
 * overlap) and Methodology 2, block-size control (b_max ~ sigma log log n).
 *
 *   ids_dev        [H][s][n] int32 from plsh_sample_bins.
 *   causal         0 or 1.
 *   bmax_dev       [H] int32 out: longest run of equal ids over the s hashes.
 *   tile_span_dev  [H][ceil(n/128)][2] int32 out: for query rows
 *                  [128t, min(n,128t+128)), the inclusive key range [lo, hi]
 *                  holding every key with a nonzero M~ weight for some row of
 *                  the tile (and key <= row when causal).
 *   bmask_dev      [H][n] boundary masks out: bit k of entry p is set iff
 *                  hash k starts a block at p (entry 0 has all s bits).
 *                  uint32 entries when s <= 32, uint64 entries when s > 32.
 *   err_dev        device error word.
 */
PLSH_API int plsh_window(const int32_t* ids_dev, int H, int s, int n, int causal, int32_t* bmax_dev,
                int32_t* tile_span_dev, void* bmask_dev, uint32_t* err_dev, void* stream);

/*
 * plsh_window_from_table (K1 + K2 fused) -- plsh_window's outputs straight
 * from the (delta, u) table, without the [H][s][n] bin ids.
 *
 * Cites: Methodology 1 (mechanism: bin(i) = floor((i + u)/delta); structure:
 * contiguous blocks) and Methodology 2 (block-size control). Every id the
 * window reduction needs is evaluated where it is needed, with the same
 * IEEE float64 steps as plsh_sample_bins, so bmax_dev, tile_span_dev and
 * bmask_dev equal those of plsh_sample_bins followed by plsh_window, bit for
 * bit, and err_dev receives the same PLSH_DEVERR_TABLE / PLSH_DEVERR_RANGE
 * bits. Call plsh_sample_bins as well when the ids themselves are needed
 * (plsh_attention_varlen_fwd, plsh_attention_bwd).
 *
 *   table_dev  [H][s][2] float64 (delta, u), as given to plsh_sample_bins.
 *   Other arguments as plsh_window.
 */
PLSH_API int plsh_window_from_table(const double* table_dev, int H, int s, int n, int causal, int32_t* bmax_dev,
                                    int32_t* tile_span_dev, void* bmask_dev, uint32_t* err_dev, void* stream);

/*
 * plsh_attention_fwd (K3) -- the fused banded Positional-LSH attention.
 *
 * Cites: Methodology 2 (M~ = (1/s) sum_k M(h_k)), Methodology 3 (ALiBi
 * attention reduced to attention restricted to short random blocks) and the
 * Results' convergence bullet (T~ as the approximation of T*). Per query
 * head h with KV head h / (H/H_kv):
 *   O_i       = sum_j c_ij e^{S_ij} V_j / sum_j c_ij e^{S_ij},  S = Q K^T / sqrt d,
 *   row_sum_i = ln( sum_j (c_ij / s) e^{S_ij} )   (natural log, float32),
 * with c_ij = number of hashes putting i and j in one bin, restricted to
 * j <= i when causal. c_ij is read from the boundary masks:
 * c_ij = s - popcount(OR of bmask over (min(i,j), max(i,j)]).
 *
 *   Q              [B][H][n][d]; K, V [B][H_kv][n][d]; O like Q.
 *   dtype          PLSH_BF16 (bf16 in and out, fp32 accumulation, tcgen05
 *                  tensor cores when d == 128) or PLSH_F32 (fp32 in and out,
 *                  fp32 CUDA-core arithmetic).
 *   d              64 or 128. bf16 with d == 64 is served by the CUDA-core
 *                  kernel on purpose: the bf16 inputs are widened to fp32 and
 *                  the result is rounded to bf16 once, so it meets the bf16
 *                  tolerance with room to spare, but it runs at CUDA-core
 *                  speed (the tensor-core kernel is built for d == 128).
 *   sigma_dev      [H] doubles, the ALiBi length scales the table was drawn
 *                  for; checked finite and > 0 (PLSH_DEVERR_SIGMA). May be NULL.
 *   s              hashes per head, as given to plsh_window.
 *   table_dev      [H][s][2] the table the masks were built from; its pitches
 *                  are checked (PLSH_DEVERR_TABLE). May be NULL.
 *   tile_span_dev, bmask_dev   from plsh_window with the same causal flag.
 *   row_sum        [B][H][n] float32 out.
 * Every pointer must be 16-byte aligned.
 * Range of the scores (bf16, d == 128): the tensor-core kernel scales each
 * row's exponentials by a running maximum of S taken over every key of the
 * 32-key chunk pairs it evaluates, weighted or not. If a row's weighted scores
 * all lie more than about 87 (natural log) below a zero-weight score in those
 * pairs, its weighted terms underflow: O is NaN and row_sum -inf for that row.
 * Scores of ordinary attention are far from this (it took Q x 32 on unit
 * normal inputs to reach it).
 */
PLSH_API int plsh_attention_fwd(const void* Q, const void* K, const void* V, int dtype, int B, int H,
                       int H_kv, int n, int d, const double* sigma_dev, int s,
                       const double* table_dev, const int32_t* tile_span_dev,
                       const void* bmask_dev, int causal, void* O, float* row_sum,
                       uint32_t* err_dev, void* stream);

/*
 * plsh_varlen_scratch_bytes -- bytes of scratch plsh_attention_varlen_fwd
 * needs: 8 * H * s * ceil(n/128) (one int32 pair per head, hash and query
 * tile). Returns 0 for a non-positive size.
 */
PLSH_API size_t plsh_varlen_scratch_bytes(int H, int s, int n);

/*
 * plsh_varlen_spans (K4 set-up) -- the key window of every query tile in
 * each single hash's blocks.
 *
 * Cites: Methodology 3 (Theorem 2.2's construction: attention restricted,
 * per sample, to that sample's blocks) and Methodology 1, structure (blocks
 * are contiguous). For head h, hash k and query rows [128t, min(n,128t+128)):
 * lo = the first position of the hash-k block holding row 128t, hi = the last
 * position of the hash-k block holding the tile's last row, or that row
 * itself when causal.
 *
 *   ids_dev    [H][s][n] int32 from plsh_sample_bins (non-decreasing in n).
 *   spans_dev  [H][s][ceil(n/128)][2] int32 out, (lo, hi) inclusive.
 */
PLSH_API int plsh_varlen_spans(const int32_t* ids_dev, int H, int s, int n, int causal, int32_t* spans_dev,
                               void* stream);

/*
 * plsh_attention_varlen_fwd (K4) -- the per-sample comparator: the same
 * T~ and row_sum as plsh_attention_fwd, computed the way Theorem 2.2 builds
 * it (Methodology 3): for each hash k separately, every query row attends
 * only to the keys of its own hash-k block (the block-diagonal mask M(h_k)),
 * and the s block-diagonal attentions are summed, numerator and denominator,
 * before the division:
 *   O_i = sum_k sum_j M_k[i,j] e^{S_ij} V_j / sum_k sum_j M_k[i,j] e^{S_ij}.
 * Each query tile visits the key tiles of every hash's window, so the
 * tensor work grows with the sum of the s windows instead of their union.
 *
 *   Arguments as plsh_attention_fwd, with
 *   ids_dev        [H][s][n] int32 from plsh_sample_bins.
 *   bmask_dev      [H][n] from plsh_window (bit k gives hash k's blocks).
 *   scratch_dev    caller-owned device memory of at least
 *                  plsh_varlen_scratch_bytes(H, s, n) bytes, 16-byte
 *                  aligned; it receives the per-hash windows
 *                  (plsh_varlen_spans) and is read by the attention kernel
 *                  on the same stream. Nothing in it needs clearing.
 *   scratch_bytes  its size; smaller than needed is PLSH_ERR_INVALID_ARG.
 */
PLSH_API int plsh_attention_varlen_fwd(const void* Q, const void* K, const void* V, int dtype, int B, int H,
                                       int H_kv, int n, int d, const double* sigma_dev, int s,
                                       const double* table_dev, const int32_t* ids_dev, const void* bmask_dev,
                                       int causal, void* scratch_dev, size_t scratch_bytes, void* O,
                                       float* row_sum, uint32_t* err_dev, void* stream);

/* Size of the library's own buffer behind plsh_attention_varlen_fwd_static. */
#define PLSH_VARLEN_STATIC_SCRATCH_BYTES (4u << 20)

/*
 * plsh_attention_varlen_fwd_static -- plsh_attention_varlen_fwd without
 * caller scratch. The paper has no counterpart: this is a calling
 * convention, not part of the method.
 *
 * It is for callers that cannot give the library device memory of their
 * own: code that may not enter the device allocator at the point of the
 * call (a hook running inside the caller's own memory management), or that
 * budgets every device allocation up front. The per-hash windows go to a
 * fixed buffer inside the library instead: a file-scope __device__ array of
 * PLSH_VARLEN_STATIC_SCRATCH_BYTES (4 MiB) per device. Nothing in it needs to
 * start at zero, and the library allocates nothing.
 *
 *   Arguments and results as plsh_attention_varlen_fwd, without scratch_dev
 *   and scratch_bytes.
 *   Limit: 8 * H * s * ceil(n/128) <= PLSH_VARLEN_STATIC_SCRATCH_BYTES, else
 *   PLSH_ERR_RANGE with nothing launched (H=16, s=20 fits up to n = 209,664).
 *   Every call looks the buffer's address up in the current context
 *   (cudaGetSymbolAddress, which allocates nothing), so a reset or re-created
 *   context never leaves a stale address behind; the first call in a context
 *   also loads the library's module there, so make it before any stream
 *   capture. Calls that overlap on one device
 *   (on different streams, or from different host threads without ordering)
 *   share the buffer and race: order them, or use plsh_attention_varlen_fwd.
 */
PLSH_API int plsh_attention_varlen_fwd_static(const void* Q, const void* K, const void* V, int dtype, int B,
                                              int H, int H_kv, int n, int d, const double* sigma_dev, int s,
                                              const double* table_dev, const int32_t* ids_dev,
                                              const void* bmask_dev, int causal, void* O, float* row_sum,
                                              uint32_t* err_dev, void* stream);

/*
 * plsh_alibi_banded_fwd -- exact ALiBi attention, the computation Positional
 * LSH approximates (technical summary, Methodology 1: L*_ij = e^{-|i-j|/sigma}
 * as the ALiBi bias matrix; Results: the approximation error ||T* - T~||),
 * restricted to a band: per query head h with KV head h / (H/H_kv),
 *   O_i       = sum_j w_ij e^{S_ij} V_j / sum_j w_ij e^{S_ij},  S = Q K^T / sqrt d,
 *   row_sum_i = ln( sum_j w_ij e^{S_ij} ),   w_ij = e^{-|i-j| / sigma_h},
 * over every key in the 128-key tiles that cover |i - j| <= ceil(sigma_h ln(1/eps))
 * (and j <= i when causal). Keys outside that band weigh less than eps each
 * relative to the diagonal and are left out. No table, ids or masks are used.
 *
 *   Arguments as plsh_attention_fwd, plus
 *   sigma_dev  [H] doubles, the ALiBi length scales (1 / slope); required.
 *   eps        the band's cut-off, 0 < eps < 1.
 * Every pointer must be 16-byte aligned.
 */
PLSH_API int plsh_alibi_banded_fwd(const void* Q, const void* K, const void* V, int dtype, int B, int H, int H_kv,
                                   int n, int d, const double* sigma_dev, double eps, int causal, void* O,
                                   float* row_sum, uint32_t* err_dev, void* stream);

/*
 * plsh_decode_fwd -- single query rows against cached keys and values: row i
 * of the same T~ as plsh_attention_fwd, for a handful of rows at a time
 * (autoregressive decoding, where the new token at position i attends to
 * the cached keys 0..i).
 *
 * Cites: Methodology 2 (M~ = (1/s) sum_k M(h_k)), Methodology 3 (attention
 * restricted to short random blocks) and Methodology 1, structure (blocks
 * are contiguous, so c_ij only falls as j moves away from i and the key walk
 * can stop at the first stretch where it is 0 for every key). For query row
 * t of (b, h) at position i = pos[t], with KV head h / (H/H_kv):
 *   O[b][h][t]       = sum_j c_ij e^{S_ij} V_j / sum_j c_ij e^{S_ij},
 *   row_sum[b][h][t] = ln( sum_j (c_ij / s) e^{S_ij} ),
 *   S_ij = Q[b][h][t] . K[b][h_kv][j] / sqrt d,
 * c_ij = s - popcount(OR of bmask over (min(i,j), max(i,j)]), over j <= i
 * when causal, every j in [0, n) otherwise.
 *
 *   Q          [B][H][m][d] query rows; O like Q (out).
 *   pos_dev    [m] int32 device positions, each in [0, n); a position
 *              outside sets PLSH_DEVERR_POSITION and leaves that row's
 *              O and row_sum unwritten. Positions may repeat.
 *   m          rows per (b, h), >= 1.
 *   K, V       [B][H_kv][n][d] the cache, n positions.
 *   dtype, d, s, causal, bmask_dev, err_dev   as plsh_attention_fwd; the
 *              masks are plsh_window's for this n (with causal, only the
 *              entries at positions <= max(pos) are read).
 *   scratch_dev    device scratch: the partial results of the work units
 *                  that share a row's walk (up to 8 per row), the row's
 *                  walk data, then one counter per row. Zero the whole
 *                  buffer once before its first use (for example with
 *                  cudaMemsetAsync). Every call that runs to completion
 *                  leaves the counters at zero again; after a call that did
 *                  not (a CUDA error, or PLSH_DEVERR_TIMEOUT), zero it again.
 *                  scratch_bytes is its size, at least
 *                  plsh_decode_scratch_bytes(B, H, m, d), else
 *                  PLSH_ERR_INVALID_ARG.
 *   row_sum    [B][H][m] float32 out.
 * Q, K, V and O must be 16-byte aligned.
 */
PLSH_API int plsh_decode_fwd(const void* Q, const int32_t* pos_dev, int m, const void* K, const void* V, int dtype,
                             int B, int H, int H_kv, int n, int d, int s, const void* bmask_dev, int causal,
                             void* scratch_dev, size_t scratch_bytes, void* O, float* row_sum, uint32_t* err_dev,
                             void* stream);

/*
 * plsh_decode_scratch_bytes -- bytes of scratch plsh_decode_fwd needs:
 * B * H * m * (32 * (d + 2) + 260) + 16: the partial results of up to 8
 * work units per row, the call's work list (up to 8 units of 32 bytes per
 * row, and its counter), then one 4-byte counter per row (the buffer's last
 * B * H * m words). Returns 0 for a non-positive size.
 */
PLSH_API size_t plsh_decode_scratch_bytes(int B, int H, int m, int d);

/*
 * plsh_attention_bwd -- gradients of T~ for training: dQ, dK, dV of
 * <dO, O> with the (delta, u) table, and so the bins, held fixed.
 *
 * Cites: Methodology 2 and 3 (T~ = P V with row weights P_ij = M~_ij e^{S_ij}
 * / sum_l M~_il e^{S_il}) and the Results' experimental validation (models
 * trained from scratch and fine-tuned with Positional LSH in the attention,
 * which needs these gradients). With the forward's row_sum L_i,
 * P_ij = (c_ij / s) e^{S_ij - L_i} is recomputed, and
 *   dV = P^T dO,  D_i = dO_i . O_i,  dS = P o (dO V^T - D),
 *   dQ = dS K / sqrt d,  dK = dS^T Q / sqrt d,
 * restricted to j <= i when causal. For grouped-query attention dK and dV of
 * KV head g sum the query heads h with h / (H/H_kv) == g.
 *
 *   Q, O, dO       [B][H][n][d]; O and row_sum are plsh_attention_fwd's
 *                  outputs for the same inputs, table and causal flag.
 *   K, V           [B][H_kv][n][d].
 *   row_sum        [B][H][n] float32, the forward's.
 *   dtype, d, s    as plsh_attention_fwd (both dtypes compute in fp32 on
 *                  CUDA cores).
 *   ids_dev        [H][s][n] int32 bin ids from plsh_sample_bins (the
 *                  key and query ranges of every tile come from them; no
 *                  masks or windows are needed).
 *   delta_dev      [B][H][n] float32 scratch (written: D_i).
 *   dQ             [B][H][n][d] out; dK, dV [B][H_kv][n][d] out, each row
 *                  written once (no accumulation into the caller's buffers).
 *   err_dev        device error word (no bit is set today).
 * Q, K, V, O and dO must be 16-byte aligned.
 */
PLSH_API int plsh_attention_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                                const float* row_sum, int dtype, int B, int H, int H_kv, int n, int d, int s,
                                const int32_t* ids_dev, int causal, float* delta_dev, void* dQ, void* dK,
                                void* dV, uint32_t* err_dev, void* stream);

/*
 * plsh_attention_bwd_tc -- the same gradients on the tcgen05 tensor cores,
 * for bf16 inputs with d = 128 (else PLSH_ERR_UNSUPPORTED; use
 * plsh_attention_bwd).
 *
 * Cites: as plsh_attention_bwd. The counts c_ij come from the boundary masks
 * as in plsh_attention_fwd (Methodology 1, structure: contiguous blocks).
 * S, dP and the gradient products run as bf16 MMAs with fp32 accumulation;
 * P and dS are rounded to bf16 for the products, so the gradients meet a
 * bf16 tolerance (they are not the fp32 path's results bit for bit).
 *
 *   Q, K, V, O, dO, row_sum, B, H, H_kv, n, s, causal   as plsh_attention_bwd
 *                  (bf16 tensors).
 *   bmask_dev      [H][n] boundary masks from plsh_window (or
 *                  plsh_window_from_table) for this table.
 *   tile_span_dev  [H][ceil(n/128)][2] windows from plsh_window with the same
 *                  causal flag (the key range each 128-row query tile reaches).
 *   key_span_dev   [H][ceil(n/128)][2] windows from plsh_window with
 *                  causal = 0: by the symmetry of c_ij, the query rows that
 *                  reach each 128-key tile (equal to tile_span_dev when
 *                  causal = 0).
 *   delta_dev      [B][H][n] float32 scratch (written: D_i).
 *   dQ             [B][H][n][128] out; dK, dV [B][H_kv][n][128] out, each row
 *                  written once.
 *   err_dev        device error word: PLSH_DEVERR_WINDOW for a window that
 *                  does not cover its tile, PLSH_DEVERR_TIMEOUT as for
 *                  plsh_attention_fwd (same wait limit).
 * Every pointer to a tensor must be 16-byte aligned.
 */
PLSH_API int plsh_attention_bwd_tc(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                                   const float* row_sum, int B, int H, int H_kv, int n, int d, int s,
                                   const void* bmask_dev, const int32_t* tile_span_dev,
                                   const int32_t* key_span_dev, int causal, float* delta_dev, void* dQ, void* dK,
                                   void* dV, uint32_t* err_dev, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PLSH_H_ */
