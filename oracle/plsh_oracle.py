"""Plain float64 CPU oracle for Positional-LSH approximate ALiBi attention.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py): imported by tests/, the
smoke check and bench.py's CPU-baseline leg, never by the library.

Page citations use the technical summary of the gist.science explainer pages
for arXiv 2605.09472 ("Positional LSH: Binary Block Matrix Approximation for
Attention with Linear Biases"):
  [nl M1]  gist.science/nl/paper/2605.09472, Methodologie, 1. Theoretisch Kader: Positionele LSH
  [nl M2]  same page, 2. Structurele Benadering (Stelling 2.1)
  [nl M3]  same page, 3. Algorithmische Reductie (Stelling 2.2)
  [nl R]   same page, Belangrijkste Resultaten (Theoretische Bevindingen / Experimentele Validatie)
  [zh M1..M3], [ja M1..M3]: the same sections of the zh and ja pages, which
  agree with the nl page statement for statement.

Readings taken where the pages are silent:
  * The hash is the Random Binning Features construction of Rahimi & Recht
    for the Laplace kernel, applied to integer positions [nl M1]: pitch
    delta ~ Gamma(shape 2, scale sigma) (the Gamma law the proof leans on,
    [nl M2] "tools"), shift u ~ U[0, delta), bin(i) = floor((i + u)/delta).
    Gamma(2, sigma) is the pitch law whose binning reproduces e^{-|i-j|/sigma}
    exactly: P(same bin | delta) = max(0, 1 - |i-j|/delta).
  * Positions are 0-based; one (delta, u) table per query head, shared by
    every batch element.
  * ALiBi's additive logit bias -|i-j|/sigma is the Hadamard weight
    L*_ij = e^{-|i-j|/sigma} on exp(QK^T/sqrt d) [nl M1].
  * T~ = D~^{-1} (exp(QK^T/sqrt d) o M~) V with D~ the row sums of the same
    weighted matrix (one joint normalisation, not an average of s softmaxes);
    the causal mask j <= i multiplies on top.
  * row_sum_i = ln( sum_j M~_ij e^{S_ij} ) including the 1/s of M~.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "splitmix64", "uniform_open", "uniform_closed_open", "draw_table",
    "bins", "bin_ids", "hash_mask", "match_counts", "mean_mask", "counts_rows",
    "boundary_bits", "block_lengths", "bmax", "tile_spans", "varlen_spans", "alibi_matrix",
    "approx_attention", "exact_attention", "forward", "forward_exact",
    "approx_attention_grad", "approx_attention_grad_sampled", "backward",
    "COUNTER_HEAD_SHIFT", "TILE",
]

MASK64 = (1 << 64) - 1
SPLITMIX_GAMMA = 0x9E3779B97F4A7C15
# Counter layout of the table draw: the three uniforms of (head h, hash k)
# are outputs ((h << 16) | k) * 3 + {0, 1, 2} of one SplitMix64 stream, so a
# table with s hashes is a prefix of the table with more hashes.
COUNTER_HEAD_SHIFT = 16
# Query/key tile height of the windows the GPU path iterates over.
TILE = 128


# ---------------------------------------------------------------------------
# Counter-based generator and the (delta, u) table
# ---------------------------------------------------------------------------

def splitmix64(seed: int, index):
    """Output number `index` (0-based) of SplitMix64 seeded with `seed`.

    SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
    generators", OOPSLA 2014): the state advances by the golden gamma
    0x9E3779B97F4A7C15 and each state is finalised by xor-shift 30, multiply
    by 0xBF58476D1CE4E5B9, xor-shift 27, multiply by 0x94D049BB133111EB,
    xor-shift 31. The state after index+1 steps is seed + (index+1)*gamma, so
    every output is a pure function of (seed, index). `index` may be an int
    (returns an int) or an integer array (returns uint64, wrapping mod 2^64).
    Pinned by: the published test vectors in tests/golden/splitmix64.json.
    """
    if isinstance(index, (int, np.integer)):
        z = (seed + (int(index) + 1) * SPLITMIX_GAMMA) & MASK64
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
        return z ^ (z >> 31)
    idx = np.asarray(index, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(seed & MASK64) + (idx + np.uint64(1)) * np.uint64(SPLITMIX_GAMMA)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
        return z ^ (z >> np.uint64(31))


def uniform_open(z):
    """A double in the open interval (0, 1): ((z >> 12) + 1/2) * 2^-52 (exact)."""
    if isinstance(z, (int, np.integer)) and not isinstance(z, np.ndarray):
        return (float(int(z) >> 12) + 0.5) * 2.0 ** -52
    return ((np.asarray(z, np.uint64) >> np.uint64(12)).astype(np.float64) + 0.5) * 2.0 ** -52


def uniform_closed_open(z):
    """A double in [0, 1): (z >> 11) * 2^-53 (exact)."""
    if isinstance(z, (int, np.integer)) and not isinstance(z, np.ndarray):
        return float(int(z) >> 11) * 2.0 ** -53
    return (np.asarray(z, np.uint64) >> np.uint64(11)).astype(np.float64) * 2.0 ** -53


def draw_table(seed: int, sigma: Sequence[float], s: int) -> np.ndarray:
    """The (delta, u) table, float64 [H][s][2], of s random binnings per head.

    [nl M1]: the hash is Rahimi-Recht Random Binning for the Laplace kernel on
    integer positions; [nl M2]: the s hashes are i.i.d. Pitch
    delta = -sigma_h (ln U1 + ln U2) is Gamma(shape 2, scale sigma_h) (a sum
    of two Exp(1) variables, scaled), shift u = U3 * delta is U[0, delta).
    U1, U2, U3 are SplitMix64 outputs ((h << 16) | k) * 3 + {0, 1, 2}; the
    logarithm is the C library's (math.log), element by element.
    Pinned by: KS tests against the Gamma(2, sigma) and uniform laws, and the
    first two moments (tests/oracle_pins.py: check_table_laws, check_table_moments).
    """
    if s < 1 or s > (1 << COUNTER_HEAD_SHIFT):
        raise ValueError("s out of range")
    sig = np.asarray(sigma, dtype=np.float64)
    H = sig.shape[0]
    hk = (np.arange(H, dtype=np.uint64)[:, None] << np.uint64(COUNTER_HEAD_SHIFT)) | \
        np.arange(s, dtype=np.uint64)[None, :]
    base = hk * np.uint64(3)
    u1 = uniform_open(splitmix64(seed, base))
    u2 = uniform_open(splitmix64(seed, base + np.uint64(1)))
    u3 = uniform_closed_open(splitmix64(seed, base + np.uint64(2)))
    log = math.log
    table = np.empty((H, s, 2), dtype=np.float64)
    for h in range(H):
        neg_sigma = -float(sig[h])
        for k in range(s):
            delta = neg_sigma * (log(float(u1[h, k])) + log(float(u2[h, k])))
            table[h, k, 0] = delta
            table[h, k, 1] = float(u3[h, k]) * delta
    return table


# ---------------------------------------------------------------------------
# Binning, masks, M~
# ---------------------------------------------------------------------------

def bins(delta, u, n: int) -> np.ndarray:
    """bin(i) = floor((i + u) / delta), i = 0..n-1, in IEEE float64, as int64.

    [nl M1] mechanism: h partitions the indices into contiguous bins.
    delta and u may be arrays of equal shape [...]; the result is then [..., n].
    Pinned by: the worked examples in tests/golden/bins_worked.json and the
    contiguity / block-length invariants.
    """
    i = np.arange(n, dtype=np.float64)
    d = np.asarray(delta, dtype=np.float64)[..., None]
    sh = np.asarray(u, dtype=np.float64)[..., None]
    return np.floor((i + sh) / d).astype(np.int64)


def bin_ids(table: np.ndarray, n: int) -> np.ndarray:
    """Bin ids of every (head, hash, position), int64 [H][s][n], relative to bin(0).

    id_{h,k}(i) = floor((i+u)/delta) - floor(u/delta). Shifting all ids of one
    hash by the same integer leaves M(h) unchanged.
    """
    H, s, _ = table.shape
    out = np.empty((H, s, n), dtype=np.int64)
    for h in range(H):
        for k in range(s):
            b = bins(table[h, k, 0], table[h, k, 1], n)
            out[h, k] = b - b[0]
    return out


def hash_mask(ids_k: np.ndarray) -> np.ndarray:
    """M(h)_ij = 1 iff i and j fall in the same bin, float64 [n][n] ([nl M1])."""
    return (ids_k[:, None] == ids_k[None, :]).astype(np.float64)


def match_counts(ids_hs: np.ndarray) -> np.ndarray:
    """c_ij = sum_k M(h_k)_ij, int64 [n][n], for one head's s hashes."""
    s, n = ids_hs.shape
    c = np.zeros((n, n), dtype=np.int64)
    for k in range(s):
        c += (ids_hs[k][:, None] == ids_hs[k][None, :])
    return c


def mean_mask(ids_hs: np.ndarray) -> np.ndarray:
    """M~ = (1/s) sum_k M(h_k) ([nl M2], Theorem 2.1's empirical mean)."""
    return match_counts(ids_hs).astype(np.float64) / ids_hs.shape[0]


def counts_rows(ids_hs: np.ndarray, rows: Sequence[int]) -> np.ndarray:
    """Rows `rows` of the match-count matrix c, int64 [len(rows)][n]."""
    rows = np.asarray(rows, dtype=np.int64)
    s, n = ids_hs.shape
    c = np.zeros((len(rows), n), dtype=np.int64)
    for k in range(s):
        c += (ids_hs[k][rows][:, None] == ids_hs[k][None, :])
    return c


def boundary_bits(ids_hs: np.ndarray) -> np.ndarray:
    """Bm(p) = sum_k 2^k [id_k(p) != id_k(p-1)] for p >= 1, Bm(0) = 2^s - 1; uint64 [n].

    Bit k is set where hash k opens a new block. Because blocks are contiguous
    ([nl M1] structure), c_ij = s - popcount(OR_{min(i,j) < p <= max(i,j)} Bm(p)).
    Pinned by: that identity against match_counts (tests/oracle_pins.py:
    check_boundary_identity) and hand-worked bits (check_bins_worked).
    """
    s, n = ids_hs.shape
    bits = np.zeros(n, dtype=np.uint64)
    for k in range(s):
        change = (ids_hs[k, 1:] != ids_hs[k, :-1]).astype(np.uint64)
        bits[1:] |= change << np.uint64(k)
    bits[0] = np.uint64((1 << s) - 1)
    return bits


def block_lengths(ids_k: np.ndarray) -> np.ndarray:
    """Lengths of the consecutive runs of equal ids of one hash, in position order."""
    n = ids_k.shape[0]
    starts = np.concatenate(([0], np.nonzero(ids_k[1:] != ids_k[:-1])[0] + 1))
    ends = np.concatenate((starts[1:], [n]))
    return ends - starts


def bmax(ids_hs: np.ndarray) -> int:
    """b_max: the largest block over all s hashes of one head ([nl M2] block-size control)."""
    return int(max(block_lengths(ids_hs[k]).max() for k in range(ids_hs.shape[0])))


def tile_spans(ids_hs: np.ndarray, causal: bool, tile: int = TILE) -> np.ndarray:
    """Key window of every query tile, int64 [ceil(n/tile)][2] = (lo, hi) inclusive.

    For query rows [t*tile, min(n, (t+1)*tile)), [lo, hi] is the smallest key
    range holding every j with c_ij > 0 for some row i of the tile (and
    j <= i when causal). Brute force over the count rows.
    """
    s, n = ids_hs.shape
    T = (n + tile - 1) // tile
    out = np.empty((T, 2), dtype=np.int64)
    cols = np.arange(n)
    for t in range(T):
        rows = np.arange(t * tile, min(n, (t + 1) * tile))
        c = counts_rows(ids_hs, rows)
        if causal:
            c[cols[None, :] > rows[:, None]] = 0
        nz = np.nonzero(c.sum(axis=0))[0]
        out[t] = (nz.min(), nz.max())
    return out


def varlen_spans(ids_hs: np.ndarray, causal: bool, tile: int = TILE,
                 tiles: Optional[Sequence[int]] = None) -> np.ndarray:
    """Per-hash key windows of the per-sample comparator, int64 [s][T][2] = (lo, hi).

    [nl M3]: Theorem 2.2's construction attends, for each sample k, only
    inside that sample's blocks. For hash k and query rows
    [t*tile, min(n, (t+1)*tile)), [lo, hi] is the smallest key range holding
    every j in the same hash-k bin as some row i of the tile (and j <= i when
    causal). Brute force over the rows' bin-equality rows; `tiles` limits the
    work to those tile indices (the others stay -1).
    """
    s, n = ids_hs.shape
    T = (n + tile - 1) // tile
    out = np.full((s, T, 2), -1, dtype=np.int64)
    cols = np.arange(n)
    for k in range(s):
        for t in (range(T) if tiles is None else tiles):
            rows = np.arange(t * tile, min(n, (t + 1) * tile))
            same = ids_hs[k][rows][:, None] == ids_hs[k][None, :]
            if causal:
                same &= cols[None, :] <= rows[:, None]
            nz = np.nonzero(same.any(axis=0))[0]
            out[k, t] = (nz.min(), nz.max())
    return out


# ---------------------------------------------------------------------------
# Attention
# ---------------------------------------------------------------------------

def alibi_matrix(n: int, sigma: float, rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """L*_ij = exp(-|i-j| / sigma) ([nl M1]); rows `rows` only if given."""
    r = np.arange(n) if rows is None else np.asarray(rows)
    return np.exp(-np.abs(r[:, None] - np.arange(n)[None, :]) / sigma)


def _weighted_softmax(S: np.ndarray, W: np.ndarray, v: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """O = (exp(S) o W) V / ((exp(S) o W) 1) and ln((exp(S) o W) 1), per row.

    The row maximum is taken over entries with W > 0; it cancels in O and is
    added back in the log row sum.
    """
    valid = W > 0
    m = np.where(valid, S, -np.inf).max(axis=1)
    A = np.exp(np.where(valid, S - m[:, None], -np.inf))
    P = A * W
    D = P.sum(axis=1)
    O = (P @ v) / D[:, None]
    return O, np.log(D) + m


def approx_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, ids_hs: np.ndarray,
                     causal: bool, rows: Optional[Sequence[int]] = None
                     ) -> Tuple[np.ndarray, np.ndarray]:
    """T~ and row_sum for one query head (float64).

    T~ = D~^{-1} (exp(QK^T/sqrt d) o M~) V, M~ = (1/s) sum_k M(h_k)
    ([nl M2], [nl M3], [nl R] convergence bullet's T~). q: [n][d] (all query
    rows; `rows` selects which are computed), k, v: [n][d]. Returns
    (O [rows][d], row_sum [rows]) with row_sum_i = ln(sum_j M~_ij e^{S_ij}).
    """
    n, d = k.shape
    r = np.arange(q.shape[0]) if rows is None else np.asarray(rows, dtype=np.int64)
    S = (q[r] @ k.T) / math.sqrt(d)
    W = counts_rows(ids_hs, r).astype(np.float64) / ids_hs.shape[0]
    if causal:
        W[np.arange(n)[None, :] > r[:, None]] = 0.0
    return _weighted_softmax(S, W, v)


def exact_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, sigma: float, causal: bool,
                    rows: Optional[Sequence[int]] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Exact ALiBi attention T* = D*^{-1} (exp(QK^T/sqrt d) o L*) V for one head ([nl M1], [nl R])."""
    n, d = k.shape
    r = np.arange(q.shape[0]) if rows is None else np.asarray(rows, dtype=np.int64)
    S = (q[r] @ k.T) / math.sqrt(d)
    W = alibi_matrix(n, sigma, r)
    if causal:
        W[np.arange(n)[None, :] > r[:, None]] = 0.0
    return _weighted_softmax(S, W, v)


def forward(Q: np.ndarray, K: np.ndarray, V: np.ndarray, table: np.ndarray, causal: bool,
            rows: Optional[Sequence[int]] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Multi-head T~: Q [B][H][n][d], K, V [B][H_kv][n][d] (float64), table [H][s][2].

    Grouped-query attention: query head h reads KV head h // (H / H_kv).
    Returns O [B][H][rows][d] and row_sum [B][H][rows].
    """
    B, H, n, d = Q.shape
    group = H // K.shape[1]
    ids = bin_ids(table, n)
    nr = n if rows is None else len(rows)
    O = np.empty((B, H, nr, d))
    R = np.empty((B, H, nr))
    for b in range(B):
        for h in range(H):
            O[b, h], R[b, h] = approx_attention(Q[b, h], K[b, h // group], V[b, h // group],
                                                ids[h], causal, rows)
    return O, R


def forward_exact(Q: np.ndarray, K: np.ndarray, V: np.ndarray, sigma: Sequence[float],
                  causal: bool, rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """Multi-head exact ALiBi T*, same layout as forward() ([nl M1], [nl R]).

    Query head h reads KV head h // (H / H_kv) and uses its own sigma_h.
    Pinned by: torch SDPA's grouped-query attention with the additive bias
    -|i-j|/sigma_h, and sampled rows against all rows (tests/oracle_pins.py:
    check_forward_exact_gqa).
    """
    B, H, n, d = Q.shape
    group = H // K.shape[1]
    nr = n if rows is None else len(rows)
    O = np.empty((B, H, nr, d))
    for b in range(B):
        for h in range(H):
            O[b, h], _ = exact_attention(Q[b, h], K[b, h // group], V[b, h // group],
                                         float(sigma[h]), causal, rows)
    return O


# ---------------------------------------------------------------------------
# Gradients of T~ (training with Positional LSH in place of ALiBi)
# ---------------------------------------------------------------------------

def approx_attention_grad(q: np.ndarray, k: np.ndarray, v: np.ndarray, do: np.ndarray, ids_hs: np.ndarray,
                          causal: bool) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """dQ, dK, dV of <dO, T~> for one query head (float64), the table held fixed.

    The pages train and fine-tune models with Positional LSH in the attention
    ([nl R], experimental validation: Qwen3 from scratch, Mistral-7B
    fine-tuning), which needs these gradients; they follow from T~ by the
    chain rule. With P_ij = M~_ij e^{S_ij} / sum_l M~_il e^{S_il} (the row
    weights of T~ = P V, [nl M2], [nl M3]) and S = q k^T / sqrt d:
        dV = P^T dO,  dP = dO V^T,  D_i = sum_j P_ij dP_ij (= dO_i . T~_i),
        dS = P o (dP - D 1^T),  dQ = dS K / sqrt d,  dK = dS^T Q / sqrt d.
    The M~ weights only scale P; entries with M~_ij = 0 (and j > i when
    causal) carry no gradient.
    """
    n, d = k.shape
    S = (q @ k.T) / math.sqrt(d)
    W = match_counts(ids_hs).astype(np.float64) / ids_hs.shape[0]
    if causal:
        W[np.arange(n)[None, :] > np.arange(n)[:, None]] = 0.0
    valid = W > 0
    m = np.where(valid, S, -np.inf).max(axis=1)
    A = np.where(valid, np.exp(np.where(valid, S - m[:, None], 0.0)), 0.0) * W
    P = A / A.sum(axis=1)[:, None]
    O = P @ v
    dV = P.T @ do
    dP = do @ v.T
    Dv = (do * O).sum(axis=1)
    dS = P * (dP - Dv[:, None])
    dQ = dS @ k / math.sqrt(d)
    dK = dS.T @ q / math.sqrt(d)
    return dQ, dK, dV


def approx_attention_grad_sampled(q: np.ndarray, k: np.ndarray, v: np.ndarray, do: np.ndarray,
                                  ids_hs: np.ndarray, causal: bool, rows: Sequence[int], keys: Sequence[int],
                                  chunk: int = 256) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """dQ on `rows` and dK, dV on `keys` of approx_attention_grad, for long sequences (float64).

    The same formulas, evaluated only where they are needed: a query row's
    dQ needs its own row of P and dS; a key's dK and dV collect P_ij and
    dS_ij over the rows i that give it weight (c_ij > 0, and i >= j when
    causal), and each of those rows needs its whole row of P (for D_i).
    Rows are processed `chunk` at a time, each over the keys its rows weight.
    """
    n, d = k.shape
    sq = math.sqrt(d)
    s = ids_hs.shape[0]

    def rows_pass(r):
        W = counts_rows(ids_hs, r).astype(np.float64) / s
        if causal:
            W[np.arange(n)[None, :] > r[:, None]] = 0.0
        cols = np.nonzero((W > 0).any(axis=0))[0]
        Wc = W[:, cols]
        S = (q[r] @ k[cols].T) / sq
        valid = Wc > 0
        m = np.where(valid, S, -np.inf).max(axis=1)
        A = np.where(valid, np.exp(np.where(valid, S - m[:, None], 0.0)), 0.0) * Wc
        P = A / A.sum(axis=1)[:, None]
        Dv = (do[r] * (P @ v[cols])).sum(axis=1)
        dS = P * (do[r] @ v[cols].T - Dv[:, None])
        return cols, P, dS

    rows = np.asarray(rows, dtype=np.int64)
    keys = np.asarray(keys, dtype=np.int64)
    dQ = np.zeros((0, d))
    if len(rows):
        cols, _, dS = rows_pass(rows)
        dQ = dS @ k[cols] / sq
    # rows reaching the keys: c_ij = c_ji, so they are the positions the keys weight
    reach = (counts_rows(ids_hs, keys) > 0)
    if causal:
        reach &= np.arange(n)[None, :] >= keys[:, None]
    R = np.nonzero(reach.any(axis=0))[0]
    dK = np.zeros((len(keys), d))
    dV = np.zeros((len(keys), d))
    for c0 in range(0, len(R), chunk):
        r = R[c0:c0 + chunk]
        cols, P, dS = rows_pass(r)
        at = np.searchsorted(cols, keys)
        hit = (at < len(cols)) & (cols[np.minimum(at, len(cols) - 1)] == keys)
        for t in np.nonzero(hit)[0]:
            dK[t] += dS[:, at[t]] @ q[r] / sq
            dV[t] += P[:, at[t]] @ do[r]
    return dQ, dK, dV


def backward(Q: np.ndarray, K: np.ndarray, V: np.ndarray, dO: np.ndarray, table: np.ndarray,
             causal: bool) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Multi-head gradients, layout as forward(): dQ like Q, dK and dV like K.

    Grouped-query attention: KV head g collects the gradients of every query
    head h with h // (H / H_kv) == g.
    """
    B, H, n, d = Q.shape
    H_kv = K.shape[1]
    group = H // H_kv
    ids = bin_ids(table, n)
    dQ = np.zeros_like(Q, dtype=np.float64)
    dK = np.zeros(K.shape, dtype=np.float64)
    dV = np.zeros(V.shape, dtype=np.float64)
    for b in range(B):
        for h in range(H):
            g = h // group
            dq, dk, dv = approx_attention_grad(Q[b, h], K[b, g], V[b, g], dO[b, h], ids[h], causal)
            dQ[b, h] = dq
            dK[b, g] += dk
            dV[b, g] += dv
    return dQ, dK, dV
