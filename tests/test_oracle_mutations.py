"""Plant plausible mistakes in the CPU oracle and check that its pins catch them.

Each case replaces one oracle function with a subtly wrong copy (a dropped
term, a wrong sign or index, a transposed operand, a wrong law) and runs the
pins that should notice. A mutation no pin catches would mean the oracle is
not really pinned there. Everything runs on the CPU.
"""
import math

import numpy as np
import pytest

import oracle.plsh_oracle as O
from tests import oracle_pins as P

_orig = {name: getattr(O, name) for name in dir(O) if not name.startswith("__")}


def _draw_table_shape1(seed, sigma, s):
    # wrong law: Exp(sigma) pitch (Gamma shape 1) from the same generator
    t = np.empty((len(sigma), s, 2))
    for h in range(len(sigma)):
        for k in range(s):
            base = ((h << O.COUNTER_HEAD_SHIFT) | k) * 3
            u1 = O.uniform_open(O.splitmix64(seed, base))
            u3 = O.uniform_closed_open(O.splitmix64(seed, base + 2))
            delta = -float(sigma[h]) * math.log(u1)
            t[h, k] = (delta, u3 * delta)
    return t


def _draw_table_scale_rate(seed, sigma, s):
    # wrong parameter: Gamma(2) with rate sigma instead of scale sigma
    sig = np.asarray(sigma, dtype=float)
    t = _orig["draw_table"](seed, list(1.0 / sig), s)
    return t


def _bins_ceil(delta, u, n):
    i = np.arange(n, dtype=np.float64)
    d = np.asarray(delta, dtype=np.float64)[..., None]
    sh = np.asarray(u, dtype=np.float64)[..., None]
    return np.ceil((i + sh) / d).astype(np.int64)


def _bins_minus_u(delta, u, n):
    i = np.arange(n, dtype=np.float64)
    d = np.asarray(delta, dtype=np.float64)[..., None]
    sh = np.asarray(u, dtype=np.float64)[..., None]
    return np.floor((i - sh) / d).astype(np.int64)


def _boundary_bits_shifted(ids_hs):
    b = _orig["boundary_bits"](ids_hs)
    out = np.zeros_like(b)
    out[:-1] = b[1:]          # bit placed one position early
    out[0] |= b[0]
    return out


def _approx_transposed(q, k, v, ids_hs, causal, rows=None):
    n, d = k.shape
    r = np.arange(q.shape[0]) if rows is None else np.asarray(rows)
    S = (k[r] @ q.T) / math.sqrt(d)        # roles of Q and K swapped
    W = O.counts_rows(ids_hs, r).astype(float) / ids_hs.shape[0]
    if causal:
        W[np.arange(n)[None, :] > r[:, None]] = 0.0
    return O._weighted_softmax(S, W, v)


def _approx_no_inv_s(q, k, v, ids_hs, causal, rows=None):
    n, d = k.shape
    r = np.arange(q.shape[0]) if rows is None else np.asarray(rows)
    S = (q[r] @ k.T) / math.sqrt(d)
    W = O.counts_rows(ids_hs, r).astype(float)    # 1/s of M~ dropped
    if causal:
        W[np.arange(n)[None, :] > r[:, None]] = 0.0
    return O._weighted_softmax(S, W, v)


def _approx_mean_of_softmaxes(q, k, v, ids_hs, causal, rows=None):
    # average of s per-hash softmaxes instead of one joint normalisation
    outs, rs = [], []
    for kk in range(ids_hs.shape[0]):
        o, rr = _orig["approx_attention"](q, k, v, ids_hs[kk:kk + 1], causal, rows)
        outs.append(o)
        rs.append(rr)
    return np.mean(outs, axis=0), np.mean(rs, axis=0)


def _approx_strict_causal(q, k, v, ids_hs, causal, rows=None):
    n, d = k.shape
    r = np.arange(q.shape[0]) if rows is None else np.asarray(rows)
    S = (q[r] @ k.T) / math.sqrt(d)
    W = O.counts_rows(ids_hs, r).astype(float) / ids_hs.shape[0]
    if causal:
        W[np.arange(n)[None, :] >= r[:, None]] = 0.0   # j < i instead of j <= i
        W[:, 0] += 1e-300 * (W.sum(1) == 0)            # keep row 0 finite
    return O._weighted_softmax(S, W, v)


def _approx_no_sqrt_d(q, k, v, ids_hs, causal, rows=None):
    n, d = k.shape
    r = np.arange(q.shape[0]) if rows is None else np.asarray(rows)
    S = q[r] @ k.T                                     # 1/sqrt(d) dropped
    W = O.counts_rows(ids_hs, r).astype(float) / ids_hs.shape[0]
    if causal:
        W[np.arange(n)[None, :] > r[:, None]] = 0.0
    return O._weighted_softmax(S, W, v)


def _alibi_times_sigma(n, sigma, rows=None):
    r = np.arange(n) if rows is None else np.asarray(rows)
    return np.exp(-np.abs(r[:, None] - np.arange(n)[None, :]) * sigma)


def _forward_wrong_gqa(Q, K, V, table, causal, rows=None):
    B, H, n, d = Q.shape
    Hkv = K.shape[1]
    ids = O.bin_ids(table, n)
    nr = n if rows is None else len(rows)
    out = np.empty((B, H, nr, d))
    R = np.empty((B, H, nr))
    for b in range(B):
        for h in range(H):
            out[b, h], R[b, h] = O.approx_attention(Q[b, h], K[b, h % Hkv], V[b, h % Hkv],
                                                    ids[h], causal, rows)
    return out, R


def _spans_ignore_causal(ids_hs, causal, tile=O.TILE):
    return _orig["tile_spans"](ids_hs, False, tile)


def _varlen_union_window(ids_hs, causal, tile=O.TILE, tiles=None):
    # wrong reading: every hash takes the union window of all hashes (the K3 window)
    one = _orig["tile_spans"](ids_hs, causal, tile)
    return np.repeat(one[None], ids_hs.shape[0], axis=0)


def _varlen_shared_row(ids_hs, causal, tile=O.TILE, tiles=None):
    # wrong index: the window of the tile's first row only (misses the last row's block)
    s, n = ids_hs.shape
    out = _orig["varlen_spans"](ids_hs, causal, tile, tiles)
    for k in range(s):
        for t in range(out.shape[1]):
            i = t * tile
            same = np.nonzero(ids_hs[k] == ids_hs[k][i])[0]
            out[k, t] = (same.min(), i if causal else same.max())
    return out


def _bmax_interior_only(ids_hs):
    return int(max(O.block_lengths(ids_hs[k])[1:-1].max(initial=1) for k in range(ids_hs.shape[0])))


def _grad_no_row_term(q, k, v, do, ids_hs, causal):
    # drops D_i from dS = P o (dP - D)
    n, d = k.shape
    S = (q @ k.T) / math.sqrt(d)
    W = O.match_counts(ids_hs).astype(np.float64)
    if causal:
        W = np.tril(W)
    A = np.where(W > 0, np.exp(S - S.max(axis=1, keepdims=True)), 0.0) * W
    P_ = A / A.sum(axis=1, keepdims=True)
    dS = P_ * (do @ v.T)
    return dS @ k / math.sqrt(d), dS.T @ q / math.sqrt(d), P_.T @ do


def _grad_dk_unscaled(q, k, v, do, ids_hs, causal):
    dq, dk, dv = _ORIG_GRAD(q, k, v, do, ids_hs, causal)
    return dq, dk * math.sqrt(k.shape[1]), dv


def _backward_wrong_gqa(Q, K, V, dO, table, causal):
    # query head h reads KV head h % H_kv instead of h // (H / H_kv)
    B, H, n, d = Q.shape
    H_kv = K.shape[1]
    ids = O.bin_ids(table, n)
    dQ, dK, dV = np.zeros(Q.shape), np.zeros(K.shape), np.zeros(V.shape)
    for b in range(B):
        for h in range(H):
            g = h % H_kv
            dq, dk, dv = O.approx_attention_grad(Q[b, h], K[b, g], V[b, g], dO[b, h], ids[h], causal)
            dQ[b, h] = dq
            dK[b, g] += dk
            dV[b, g] += dv
    return dQ, dK, dV


_ORIG_GRAD = O.approx_attention_grad
_ORIG_SAMPLED = O.approx_attention_grad_sampled


def _forward_exact_wrong_gqa(Q, K, V, sigma, causal, rows=None):
    B, H, n, d = Q.shape
    Hkv = K.shape[1]
    nr = n if rows is None else len(rows)
    out = np.empty((B, H, nr, d))
    for b in range(B):
        for h in range(H):
            out[b, h], _ = O.exact_attention(Q[b, h], K[b, h % Hkv], V[b, h % Hkv], float(sigma[h]), causal, rows)
    return out


def _forward_exact_sigma_of_kv_head(Q, K, V, sigma, causal, rows=None):
    # the length scale of the KV head instead of the query head's own
    B, H, n, d = Q.shape
    group = H // K.shape[1]
    nr = n if rows is None else len(rows)
    out = np.empty((B, H, nr, d))
    for b in range(B):
        for h in range(H):
            out[b, h], _ = O.exact_attention(Q[b, h], K[b, h // group], V[b, h // group],
                                             float(sigma[(h // group) * group]), causal, rows)
    return out


def _sampled_reach_ignores_causal(q, k, v, do, ids_hs, causal, rows, keys, chunk=256):
    # collects dK, dV from the non-causal rows' P (rows above the key are skipped, but P is not causal)
    dq, _, _ = _ORIG_SAMPLED(q, k, v, do, ids_hs, causal, rows, keys, chunk)
    _, dk, dv = _ORIG_SAMPLED(q, k, v, do, ids_hs, False, rows, keys, chunk)
    return dq, dk, dv

MUTATIONS = [
    ("draw_table", _draw_table_shape1, [P.check_table_moments, P.check_table_laws]),
    ("draw_table", _draw_table_scale_rate, [P.check_table_moments]),
    ("bins", _bins_ceil, [P.check_bins_worked]),
    ("bins", _bins_minus_u, [P.check_bins_worked]),
    ("boundary_bits", _boundary_bits_shifted, [P.check_bins_worked, P.check_boundary_identity]),
    ("approx_attention", _approx_transposed, [P.check_tiny_attention]),
    ("approx_attention", _approx_no_inv_s, [P.check_tiny_attention]),
    ("approx_attention", _approx_mean_of_softmaxes, [P.check_tiny_attention]),
    ("approx_attention", _approx_strict_causal, [P.check_tiny_attention]),
    ("approx_attention", _approx_no_sqrt_d, [P.check_one_bin_dense]),
    ("alibi_matrix", _alibi_times_sigma, [P.check_tiny_attention, P.check_exact_alibi_sdpa]),
    ("forward", _forward_wrong_gqa, [P.check_rows_and_gqa]),
    ("forward_exact", _forward_exact_wrong_gqa, [P.check_forward_exact_gqa]),
    ("forward_exact", _forward_exact_sigma_of_kv_head, [P.check_forward_exact_gqa]),
    ("tile_spans", _spans_ignore_causal, [P.check_bins_worked]),
    ("bmax", _bmax_interior_only, [P.check_bins_worked]),
    ("varlen_spans", _varlen_union_window, [P.check_bins_worked, P.check_varlen_spans_from_blocks]),
    ("varlen_spans", _varlen_shared_row, [P.check_bins_worked, P.check_varlen_spans_from_blocks]),
    ("approx_attention_grad", _grad_no_row_term, [P.check_grad_autograd, P.check_grad_finite_differences]),
    ("approx_attention_grad", _grad_dk_unscaled, [P.check_grad_autograd, P.check_grad_finite_differences]),
    ("backward", _backward_wrong_gqa, [P.check_backward_gqa]),
    ("approx_attention_grad_sampled", _sampled_reach_ignores_causal, [P.check_grad_sampled_equals_full]),
]


@pytest.mark.parametrize("name,bad,checks", MUTATIONS,
                         ids=[f"{m[0]}:{m[1].__name__}" for m in MUTATIONS])
def test_planted_mistake_is_caught(monkeypatch, name, bad, checks):
    monkeypatch.setattr(O, name, bad)
    for check in checks:
        with pytest.raises(AssertionError):
            check(O)


def test_unmutated_oracle_passes_the_same_checks():
    for _, _, checks in MUTATIONS:
        for check in checks:
            check(O)
