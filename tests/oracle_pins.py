"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each check_* takes the oracle module (or a copy with one function replaced)
and raises AssertionError when the oracle disagrees with its pin. The
regular tests call them on the oracle; tests/test_oracle_mutations.py plants
a plausible mistake in the oracle and checks that some pin catches it.

Pins used (none of them re-types the oracle's own formula):
  * published SplitMix64 test vectors (golden file);
  * hand-worked bins, boundary bits, counts, b_max, windows and per-hash
    windows (golden file); per-hash windows against block starts / ends;
  * a hand-worked 3-token T~ / T* example with exact fractions (golden file);
  * the Gamma(2, sigma) and U[0,1) laws of the table (KS tests, moments);
  * the exact identity E_h[M(h)] = L* (Monte Carlo, 10^6 draws);
  * the O(1/sqrt s) decay of ||L* - M~|| (log-log slope);
  * the law of b_max (max of s Gamma(2) pitches, rounded) and its
    sigma*log log n growth;
  * special cases that reduce to textbook routines: s=1 is softmax inside
    each bin (a plain loop), one bin is dense softmax attention and
    singleton bins give O = V (torch scaled_dot_product_attention, fp64);
  * exact ALiBi as additive-bias softmax (torch SDPA with a float mask);
  * the convergence ||T* - T~|| -> 0 as s grows.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch
from scipy import stats

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- generator

def check_splitmix64_vectors(orc):
    g = _golden("splitmix64.json")
    got = [orc.splitmix64(g["seed"], i) for i in range(len(g["outputs"]))]
    assert got == [int(x) for x in g["outputs"]], got
    arr = orc.splitmix64(g["seed"], np.arange(len(g["outputs"])))
    assert [int(x) for x in arr] == [int(x) for x in g["outputs"]]


# ---------------------------------------------------------------- table law

def check_table_moments(orc, sigma=3.0, heads=20, s=5000, seed=11):
    """10^5 pitches: mean 2*sigma and variance 2*sigma^2 within 4 standard errors."""
    t = orc.draw_table(seed, [sigma] * heads, s)
    d = t[..., 0].ravel()
    N = d.size
    mean_se = math.sqrt(2.0 * sigma ** 2 / N)
    assert abs(d.mean() - 2 * sigma) <= 4 * mean_se, (d.mean(), 2 * sigma, mean_se)
    # Gamma(2, theta): variance 2 theta^2, fourth central moment 24 theta^4,
    # so the sample variance has standard error sqrt((24 - 4)/N) theta^2.
    var_se = math.sqrt(20.0 / N) * sigma ** 2
    assert abs(d.var() - 2 * sigma ** 2) <= 4 * var_se, (d.var(), 2 * sigma ** 2, var_se)
    assert np.all(d > 0)


def check_table_laws(orc, sigma=5.0, heads=10, s=2000, seed=12):
    """KS: delta ~ Gamma(shape 2, scale sigma); u/delta ~ U[0,1); hashes of one head independent."""
    t = orc.draw_table(seed, [sigma] * heads, s)
    d = t[..., 0].ravel()
    u = t[..., 1].ravel()
    p_gamma = stats.kstest(d, stats.gamma(a=2.0, scale=sigma).cdf).pvalue
    assert p_gamma >= 1e-3, p_gamma
    frac = u / d
    assert np.all((frac >= 0) & (frac <= 1))
    p_unif = stats.kstest(frac, "uniform").pvalue
    assert p_unif >= 1e-3, p_unif
    # neighbouring hashes uncorrelated
    r = np.corrcoef(t[:, :-1, 0].ravel(), t[:, 1:, 0].ravel())[0, 1]
    assert abs(r) < 4.0 / math.sqrt(d.size), r


def check_table_prefix(orc):
    """A table with fewer hashes is a prefix of one with more (counter layout)."""
    a = orc.draw_table(5, [2.0, 8.0, 32.0], 10)
    b = orc.draw_table(5, [2.0, 8.0, 32.0], 40)
    assert np.array_equal(a, b[:, :10])
    c = orc.draw_table(6, [2.0, 8.0, 32.0], 10)
    assert not np.array_equal(a, c)


# ---------------------------------------------------------------- bins / masks

def check_bins_worked(orc):
    g = _golden("bins_worked.json")
    for ex in g["examples"]:
        b = orc.bins(ex["delta"], ex["u"], ex["n"])
        assert b.tolist() == ex["bins"], (ex, b)
        assert orc.block_lengths(b).tolist() == ex["block_lengths"]
        # b_max counts edge blocks too (a single bin is one edge block)
        assert orc.bmax(b[None, :]) == max(ex["block_lengths"])
    hh = g["two_hash_head"]
    table = np.array([[[2.5, 0.7], [4.0, 0.0]]])
    ids = orc.bin_ids(table, 10)[0]
    assert ids.tolist() == hh["ids"]
    assert orc.boundary_bits(ids).tolist() == hh["boundary_bits"]
    assert orc.bmax(ids) == hh["bmax"]
    c = orc.match_counts(ids)
    for i, j, v in hh["counts_entries"]:
        assert c[i, j] == v and c[j, i] == v, (i, j, c[i, j], v)
    assert orc.tile_spans(ids, False, hh["tile"]).tolist() == hh["spans_noncausal"]
    assert orc.tile_spans(ids, True, hh["tile"]).tolist() == hh["spans_causal"]
    assert orc.varlen_spans(ids, False, hh["tile"]).tolist() == hh["varlen_spans_noncausal"]
    assert orc.varlen_spans(ids, True, hh["tile"]).tolist() == hh["varlen_spans_causal"]


def _tables_for_invariants(orc):
    return [orc.draw_table(21, [0.7, 1.0, 3.0, 17.0, 150.0], 12),
            orc.draw_table(22, [2.0 ** (h / 2) for h in range(1, 9)], 20)]


def check_contiguous_blocks(orc, n=700):
    """Every M(h) is block diagonal with contiguous, non-overlapping blocks and unit diagonal."""
    for table in _tables_for_invariants(orc):
        ids = orc.bin_ids(table, n)
        for h in range(ids.shape[0]):
            for k in range(ids.shape[1]):
                M = orc.hash_mask(ids[h, k])
                assert np.all(np.diag(M) == 1.0)
                assert np.array_equal(M, M.T)
                # rebuild the block-diagonal matrix from the run lengths
                L = orc.block_lengths(ids[h, k])
                assert L.sum() == n and np.all(L >= 1)
                R = np.zeros((n, n))
                p = 0
                for ln in L:
                    R[p:p + ln, p:p + ln] = 1.0
                    p += ln
                assert np.array_equal(M, R)


def check_block_lengths(orc, n=3000):
    """Interior blocks of a hash with pitch delta hold floor(delta) or ceil(delta) positions."""
    for table in _tables_for_invariants(orc):
        ids = orc.bin_ids(table, n)
        for h in range(ids.shape[0]):
            for k in range(ids.shape[1]):
                delta = table[h, k, 0]
                L = orc.block_lengths(ids[h, k])
                inner = L[1:-1]
                if delta >= 1.0:
                    ok = (inner == math.floor(delta)) | (inner == math.ceil(delta))
                else:
                    ok = inner == 1
                assert np.all(ok), (delta, np.unique(inner))
                assert L[0] <= math.ceil(delta) and L[-1] <= math.ceil(delta)


def check_boundary_identity(orc, n=300):
    """c_ij = s - popcount(OR of Bm over (min(i,j), max(i,j)]) for every pair."""
    table = orc.draw_table(23, [1.5, 6.0, 40.0], 13)
    ids = orc.bin_ids(table, n)
    for h in range(ids.shape[0]):
        c = orc.match_counts(ids[h])
        bm = orc.boundary_bits(ids[h]).astype(object)
        s = ids.shape[1]
        for i in range(n):
            acc = 0
            assert c[i, i] == s
            for j in range(i + 1, n):
                acc |= int(bm[j])
                want = s - bin(acc).count("1")
                assert c[i, j] == want and c[j, i] == want, (h, i, j)


def check_varlen_spans_from_blocks(orc, n=900, tile=128):
    """Per-hash windows equal (start of the first row's block, end of the last row's block).

    Blocks are contiguous (Methodology 1, structure), so the keys sharing a hash-k block with
    some row of a tile run from the first row's block start to the last row's block end; when
    causal the end is the last row. Block starts and ends come from the run lengths here.
    """
    for table in _tables_for_invariants(orc):
        ids = orc.bin_ids(table, n)
        for h in range(ids.shape[0]):
            for causal in (False, True):
                got = orc.varlen_spans(ids[h], causal, tile)
                for k in range(ids.shape[1]):
                    L = orc.block_lengths(ids[h, k])
                    ends = np.cumsum(L) - 1
                    starts = ends - L + 1
                    blk = np.repeat(np.arange(len(L)), L)     # block index of every position
                    for t in range(got.shape[1]):
                        first, last = t * tile, min(n, (t + 1) * tile) - 1
                        want = (starts[blk[first]], last if causal else ends[blk[last]])
                        assert tuple(got[k, t]) == want, (h, k, t, causal, got[k, t], want)


def check_expectation_identity(orc, n=64, draws=1_000_000, sigmas=(1.0, 4.0, 16.0)):
    """Monte Carlo: E_h[M(h)]_{i,i+D} = exp(-D/sigma) within 4 standard errors ([nl M1] expectation bullet)."""
    for si, sigma in enumerate(sigmas):
        heads = 1000
        s = draws // heads
        table = orc.draw_table(100 + si, [sigma] * heads, s)
        ids = orc.bins(table[..., 0].ravel(), table[..., 1].ravel(), n)  # [draws][n]
        for D in range(1, n):
            per = (ids[:, D:] == ids[:, :-D]).mean(axis=1)
            mean = per.mean()
            se = per.std(ddof=1) / math.sqrt(per.size)
            want = math.exp(-D / sigma)
            tol = 4 * se if se > 0 else 1e-12
            # when the true value is below ~1/draws the sample may be all zeros
            assert abs(mean - want) <= max(tol, 5.0 / per.size), (sigma, D, mean, want, se)


def check_thm21_rate(orc, n=512, sigma=16.0, s_list=(4, 16, 64, 256), tables=12):
    """||L* - M~||_max and ||L* - M~||_2 fall like 1/sqrt(s) ([nl M2]; [nl R] O(1/sqrt s))."""
    L = orc.alibi_matrix(n, sigma)
    med_max, med_spec = [], []
    for s in s_list:
        e_max, e_spec = [], []
        for t in range(tables):
            table = orc.draw_table(1000 + t, [sigma], s)
            Mt = orc.mean_mask(orc.bin_ids(table, n)[0])
            E = L - Mt
            e_max.append(np.abs(E).max())
            e_spec.append(np.abs(np.linalg.eigvalsh(E)).max())
        med_max.append(np.median(e_max))
        med_spec.append(np.median(e_spec))
    x = np.log(np.asarray(s_list, dtype=float))
    for med in (med_max, med_spec):
        slope = np.polyfit(x, np.log(med), 1)[0]
        assert -0.6 <= slope <= -0.4, (slope, med)
        assert all(a > b for a, b in zip(med, med[1:])), med


def check_bmax_law(orc, sigma=10.0, s=16, tables=2000, n=4096):
    """b_max = largest block; its pitch max follows F(x)^s, F(x) = 1-(1+x/sigma)e^{-x/sigma}."""
    table = orc.draw_table(77, [sigma] * tables, s)
    dmax = table[..., 0].max(axis=1)
    F = lambda x: (1.0 - (1.0 + x / sigma) * np.exp(-x / sigma)) ** s  # noqa: E731
    p = stats.kstest(dmax, F).pvalue
    assert p >= 1e-3, p
    ids = orc.bin_ids(table[:200], n)
    for h in range(200):
        bm = orc.bmax(ids[h])
        assert math.floor(dmax[h]) <= bm <= math.ceil(dmax[h]), (bm, dmax[h])


def check_bmax_loglog(orc, sigma=4.0, tables=1000):
    """b_max / sigma grows like log log n when s = ceil(2 ln n) ([nl M2] block-size bullet).

    b_max of a hash is its pitch rounded (checked on binned ids of a subset);
    the mean pitch maximum over s hashes grows with slope about
    1 + 1/ln s ~ 1.3 in ln ln n (Gumbel limit of the Gamma(2) maximum).
    """
    ns = [2 ** e for e in range(10, 18)]
    mean = []
    for n in ns:
        s = int(math.ceil(2 * math.log(n)))
        table = orc.draw_table(500 + n, [sigma] * tables, s)
        dmax = table[..., 0].max(axis=1)
        sub = orc.bin_ids(table[:20], min(n, 4096))
        for h in range(20):
            assert orc.bmax(sub[h]) <= math.ceil(dmax[h])
        mean.append(dmax.mean() / sigma)
    lln = np.log(np.log(np.asarray(ns, dtype=float)))
    slope = np.polyfit(lln, mean, 1)[0]
    assert 0.8 <= slope <= 1.8, (slope, mean)
    assert mean[-1] > mean[0], mean


# ---------------------------------------------------------------- attention

def check_tiny_attention(orc):
    g = _golden("tiny_attention.json")
    st = g["setup"]
    table = np.array([st["table"]])
    ids = orc.bin_ids(table, st["n"])[0]
    assert orc.match_counts(ids).tolist() == g["counts"]
    q = np.array(st["q"])[:, None]
    k = np.array(st["k"])[:, None]
    v = np.array(st["v"])[:, None]
    for causal, key in ((False, "noncausal"), (True, "causal")):
        O, R = orc.approx_attention(q, k, v, ids, causal)
        np.testing.assert_allclose(O[:, 0], g[key]["O"], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(R, g[key]["row_sum"], rtol=1e-12, atol=1e-12)
    sigma = 1.0 / math.log(2.0)
    for causal, key in ((False, "exact_noncausal"), (True, "exact_causal")):
        O, _ = orc.exact_attention(q, k, v, sigma, causal)
        np.testing.assert_allclose(O[:, 0], g[key]["O"], rtol=1e-12, atol=1e-12)


def _rand_qkv(n, d, seed):
    r = np.random.default_rng(seed)
    return r.standard_normal((n, d)), r.standard_normal((n, d)), r.standard_normal((n, d))


def _sdpa(q, k, v, mask=None, causal=False):
    tq, tk, tv = (torch.from_numpy(x)[None, None] for x in (q, k, v))
    m = None if mask is None else torch.from_numpy(mask)[None, None]
    return torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=m, is_causal=causal)[0, 0].numpy()


def check_s1_per_bin_softmax(orc, n=200, d=8):
    """s = 1: T~ is softmax attention run independently inside each bin (plain loop)."""
    q, k, v = _rand_qkv(n, d, 3)
    table = np.array([[[7.3, 2.1]]])
    ids = orc.bin_ids(table, n)[0]
    for causal in (False, True):
        O, R = orc.approx_attention(q, k, v, ids, causal)
        want = np.empty((n, d))
        want_r = np.empty(n)
        for i in range(n):
            js = [j for j in range(n) if ids[0, j] == ids[0, i] and (not causal or j <= i)]
            logits = np.array([q[i] @ k[j] / math.sqrt(d) for j in js])
            mx = logits.max()
            w = np.exp(logits - mx)
            want[i] = (w[:, None] * v[js]).sum(0) / w.sum()
            want_r[i] = math.log(w.sum()) + mx
        np.testing.assert_allclose(O, want, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(R, want_r, rtol=1e-12, atol=1e-12)


def check_one_bin_dense(orc, n=257, d=16):
    """delta = 2n, u = 0 for every hash: one bin, so T~ is dense softmax attention (SDPA)."""
    q, k, v = _rand_qkv(n, d, 4)
    table = np.array([[[2.0 * n, 0.0]] * 5])
    ids = orc.bin_ids(table, n)[0]
    for causal in (False, True):
        O, R = orc.approx_attention(q, k, v, ids, causal)
        np.testing.assert_allclose(O, _sdpa(q, k, v, causal=causal), rtol=1e-10, atol=1e-12)
        S = q @ k.T / math.sqrt(d)
        if causal:
            S = np.where(np.tril(np.ones((n, n))) > 0, S, -np.inf)
        lse = torch.logsumexp(torch.from_numpy(S), dim=1).numpy()
        np.testing.assert_allclose(R, lse, rtol=1e-12, atol=1e-12)


def check_singleton_bins(orc, n=100, d=8):
    """delta < 1: every position alone in its bin, so O = V and row_sum = S_ii."""
    q, k, v = _rand_qkv(n, d, 5)
    table = np.array([[[0.5, 0.25], [0.9, 0.1], [0.3, 0.2]]])
    ids = orc.bin_ids(table, n)[0]
    for causal in (False, True):
        O, R = orc.approx_attention(q, k, v, ids, causal)
        np.testing.assert_array_equal(O, v)
        np.testing.assert_allclose(R, (q * k).sum(1) / math.sqrt(d), rtol=0, atol=1e-13)


def check_exact_alibi_sdpa(orc, n=300, d=16, sigma=9.0):
    """T* = softmax(QK^T/sqrt d - |i-j|/sigma) V: ALiBi as an additive bias (SDPA float mask)."""
    q, k, v = _rand_qkv(n, d, 6)
    dist = np.abs(np.arange(n)[:, None] - np.arange(n)[None, :]).astype(float)
    bias = -dist / sigma
    for causal in (False, True):
        O, _ = orc.exact_attention(q, k, v, sigma, causal)
        mask = np.where(np.tril(np.ones((n, n))) > 0, bias, -np.inf) if causal else bias
        np.testing.assert_allclose(O, _sdpa(q, k, v, mask=mask), rtol=1e-10, atol=1e-12)


def check_convergence(orc, n=256, d=16, sigma=8.0, s_list=(4, 16, 64, 256), tables=8):
    """||T* - T~||_max falls toward 0 as s grows, about like 1/sqrt(s) ([nl R] convergence)."""
    q, k, v = _rand_qkv(n, d, 7)
    Ostar, _ = orc.exact_attention(q, k, v, sigma, False)
    med = []
    for s in s_list:
        errs = []
        for t in range(tables):
            table = orc.draw_table(3000 + t, [sigma], s)
            O, _ = orc.approx_attention(q, k, v, orc.bin_ids(table, n)[0], False)
            errs.append(np.abs(O - Ostar).max())
        med.append(np.median(errs))
    slope = np.polyfit(np.log(s_list), np.log(med), 1)[0]
    assert all(a > b for a, b in zip(med, med[1:])), med
    assert -0.75 <= slope <= -0.3, (slope, med)


def check_rows_and_gqa(orc, n=160, d=8):
    """Sampled rows equal the full computation's rows; GQA equals MHA on repeated K/V."""
    r = np.random.default_rng(8)
    B, H, Hkv = 2, 4, 2
    Q = r.standard_normal((B, H, n, d))
    K = r.standard_normal((B, Hkv, n, d))
    V = r.standard_normal((B, Hkv, n, d))
    table = orc.draw_table(9, [2.0, 5.0, 11.0, 30.0], 6)
    rows = [0, 5, 77, 128, 159]
    for causal in (False, True):
        O, R = orc.forward(Q, K, V, table, causal)
        Orow, Rrow = orc.forward(Q, K, V, table, causal, rows)
        np.testing.assert_allclose(Orow, O[:, :, rows], rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(Rrow, R[:, :, rows], rtol=1e-13, atol=1e-13)
        Krep = np.repeat(K, H // Hkv, axis=1)
        Vrep = np.repeat(V, H // Hkv, axis=1)
        O2, R2 = orc.forward(Q, Krep, Vrep, table, causal)
        np.testing.assert_allclose(O2, O, rtol=1e-13, atol=1e-13)
        # head 1 reads KV head 0, head 2 reads KV head 1
        O1, _ = orc.approx_attention(Q[0, 2], K[0, 1], V[0, 1], orc.bin_ids(table, n)[2], causal)
        np.testing.assert_allclose(O[0, 2], O1, rtol=1e-13, atol=1e-13)


def check_forward_exact_gqa(orc, n=140, d=8):
    """Multi-head exact ALiBi T* with grouped KV heads equals torch SDPA's own grouped-query
    attention (enable_gqa) with the additive bias -|i-j|/sigma_h per head ([nl M1]: ALiBi's bias
    matrix); sampled rows equal the full computation's rows."""
    r = np.random.default_rng(10)
    B, H, Hkv = 2, 4, 2
    Q = r.standard_normal((B, H, n, d))
    K = r.standard_normal((B, Hkv, n, d))
    V = r.standard_normal((B, Hkv, n, d))
    sigma = [1.5, 4.0, 12.0, 40.0]
    rows = [0, 3, 64, 139]
    dist = np.abs(np.arange(n)[:, None] - np.arange(n)[None, :]).astype(float)
    bias = np.stack([-dist / sg for sg in sigma])
    for causal in (False, True):
        O = orc.forward_exact(Q, K, V, sigma, causal)
        mask = np.where(np.tril(np.ones((n, n))) > 0, bias, -np.inf) if causal else bias
        want = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(Q), torch.from_numpy(K), torch.from_numpy(V),
            attn_mask=torch.from_numpy(mask)[None], enable_gqa=True).numpy()
        np.testing.assert_allclose(O, want, rtol=1e-10, atol=1e-12)
        Orow = orc.forward_exact(Q, K, V, sigma, causal, rows)
        np.testing.assert_allclose(Orow, O[:, :, rows], rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------------------
# Gradients
# ---------------------------------------------------------------------------

def _counts_by_definition(ids_hs):
    """c_ij = number of hashes putting positions i and j in one bin, by direct comparison."""
    return sum((row[:, None] == row[None, :]).astype(np.float64) for row in ids_hs)


def check_grad_autograd(orc, n=150, d=8):
    """Gradients against torch autograd of softmax(S + ln c) V: T~ is that softmax attention for
    any table (ln 0 = -inf drops the pair), so the library's reverse mode gives the exact answer."""
    r = np.random.default_rng(21)
    q, k, v, do = (r.standard_normal((n, d)) for _ in range(4))
    for sigma, s in ((3.0, 5), (20.0, 12), (0.7, 3)):
        ids = orc.bin_ids(orc.draw_table(31 + s, [sigma], s), n)[0]
        W = _counts_by_definition(ids)
        for causal in (False, True):
            Wc = np.tril(W) if causal else W
            tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
            bias = torch.from_numpy(np.where(Wc > 0, np.log(np.where(Wc > 0, Wc, 1.0)), -np.inf))
            att = torch.softmax(tq @ tk.T / math.sqrt(d) + bias, dim=1)
            (att @ tv).backward(torch.from_numpy(do))
            dq, dk, dv = orc.approx_attention_grad(q, k, v, do, ids, causal)
            np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-10, atol=1e-12)
            np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=1e-10, atol=1e-12)
            np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=1e-10, atol=1e-12)


def check_grad_finite_differences(orc, n=12, d=3, eps=1e-6):
    """Central differences of f = <dO, T~> computed with the oracle's forward."""
    r = np.random.default_rng(22)
    q, k, v, do = (r.standard_normal((n, d)) for _ in range(4))
    ids = orc.bin_ids(orc.draw_table(5, [2.5], 4), n)[0]
    for causal in (False, True):
        grads = orc.approx_attention_grad(q, k, v, do, ids, causal)
        for which in range(3):
            for (i, e) in ((0, 0), (5, 1), (11, 2), (7, 0)):
                xs = [q.copy(), k.copy(), v.copy()]
                xs[which][i, e] += eps
                fp = (orc.approx_attention(*xs, ids, causal)[0] * do).sum()
                xs[which][i, e] -= 2 * eps
                fm = (orc.approx_attention(*xs, ids, causal)[0] * do).sum()
                fd = (fp - fm) / (2 * eps)
                assert abs(fd - grads[which][i, e]) <= 1e-7 * max(1.0, abs(fd)), (which, i, e, fd,
                                                                                  grads[which][i, e])


def check_grad_singleton_bins(orc, n=60, d=8):
    """delta < 1: T~ = V whatever Q and K are, so dV = dO and dQ = dK = 0."""
    r = np.random.default_rng(23)
    q, k, v, do = (r.standard_normal((n, d)) for _ in range(4))
    ids = orc.bin_ids(np.array([[[0.5, 0.25], [0.9, 0.1]]]), n)[0]
    for causal in (False, True):
        dq, dk, dv = orc.approx_attention_grad(q, k, v, do, ids, causal)
        np.testing.assert_allclose(dv, do, rtol=0, atol=1e-14)
        assert np.abs(dq).max() <= 1e-14 and np.abs(dk).max() <= 1e-14


def check_backward_gqa(orc, n=90, d=6):
    """Multi-head gradients: GQA equals MHA on repeated K/V with the group's dK, dV summed."""
    r = np.random.default_rng(24)
    B, H, Hkv = 2, 4, 2
    Q, dO = r.standard_normal((B, H, n, d)), r.standard_normal((B, H, n, d))
    K, V = r.standard_normal((B, Hkv, n, d)), r.standard_normal((B, Hkv, n, d))
    table = orc.draw_table(25, [2.0, 5.0, 11.0, 30.0], 6)
    for causal in (False, True):
        dQ, dK, dV = orc.backward(Q, K, V, dO, table, causal)
        dQr, dKr, dVr = orc.backward(Q, np.repeat(K, 2, axis=1), np.repeat(V, 2, axis=1), dO, table, causal)
        np.testing.assert_allclose(dQ, dQr, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(dK, dKr[:, 0::2] + dKr[:, 1::2], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(dV, dVr[:, 0::2] + dVr[:, 1::2], rtol=1e-12, atol=1e-13)
        # query head 3 reads KV head 1
        ids3 = orc.bin_ids(table, n)[3]
        dq3, _, _ = orc.approx_attention_grad(Q[1, 3], K[1, 1], V[1, 1], dO[1, 3], ids3, causal)
        np.testing.assert_allclose(dQ[1, 3], dq3, rtol=1e-13, atol=1e-13)


def check_grad_sampled_equals_full(orc, n=700, d=8):
    """The sampled gradients equal the full ones on the same rows and keys (small chunks force
    several passes over the reaching rows)."""
    r = np.random.default_rng(26)
    q, k, v, do = (r.standard_normal((n, d)) for _ in range(4))
    rows = [0, 1, 128, 350, 699]
    keys = [0, 5, 300, 640, 699]
    for sigma in (3.0, 40.0):
        ids = orc.bin_ids(orc.draw_table(27, [sigma], 7), n)[0]
        for causal in (False, True):
            dq, dk, dv = orc.approx_attention_grad(q, k, v, do, ids, causal)
            sq_, sk, sv = orc.approx_attention_grad_sampled(q, k, v, do, ids, causal, rows, keys, chunk=64)
            np.testing.assert_allclose(sq_, dq[rows], rtol=1e-10, atol=1e-12)
            np.testing.assert_allclose(sk, dk[keys], rtol=1e-10, atol=1e-12)
            np.testing.assert_allclose(sv, dv[keys], rtol=1e-10, atol=1e-12)
