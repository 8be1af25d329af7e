"""Glue between the CUDA path (through the C-ABI binding) and the CPU oracle.

Runs the library on seeded inputs and returns numpy copies of everything it
produced; runs the oracle on the same bits. The two sides share nothing but
the seeded inputs from workloads.py.
"""
from __future__ import annotations

from typing import Optional, Sequence

import numpy as np
import torch

import oracle
import workloads


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def run_gpu(B, H, H_kv, n, d, s, causal, sigma, seed, q, k, v, table: Optional[np.ndarray] = None,
            varlen: bool = False):
    """The whole path through the C-ABI; q, k, v are CPU tensors (copied to cuda:0).

    varlen=True runs the per-sample comparator (plsh_attention_varlen_fwd) for the attention step
    and also returns its per-hash windows.
    """
    from alibi_positional_lsh_b200 import PlshForward
    plan = PlshForward(B, H, H_kv, n, d, s, causal, sigma, seed, q.dtype, "cuda:0")
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    # poison the outputs so a row the kernel never writes cannot pass
    plan.O.fill_(float("nan"))
    plan.row_sum.fill_(float("nan"))
    if varlen:
        plan.prepare(table=table)
        plan.attend_varlen(qd, kd, vd)
    else:
        plan(qd, kd, vd, table=table)
    errs = plan.device_errors()
    out = dict(
        errors=errs,
        table=plan.table_host.numpy().copy(),
        ids=plan.ids.cpu().numpy().astype(np.int64),
        bmax=plan.bmax.cpu().numpy().astype(np.int64),
        spans=plan.spans.cpu().numpy().astype(np.int64),
        bmask=(plan.bmask.cpu().numpy().view(np.uint32) if s <= 32 else plan.bmask.cpu().numpy().view(np.uint64)),
        O=f64(plan.O),
        row_sum=plan.row_sum.cpu().numpy().astype(np.float64),
    )
    if varlen:
        T = (n + 127) // 128
        out["varlen_spans"] = plan.scratch.cpu().numpy().astype(np.int64)[: H * s * T * 2].reshape(H, s, T, 2)
    return out


def oracle_window_checks(table, n, causal, gpu, tiles_per_head: Optional[int] = None):
    """Compares ids, boundary masks, b_max and tile windows bit for bit."""
    H, s, _ = table.shape
    ids = oracle.bin_ids(table, n)
    assert np.array_equal(gpu["ids"], ids), "bin ids differ"
    T = (n + 127) // 128
    for h in range(H):
        bm = oracle.boundary_bits(ids[h])
        assert np.array_equal(gpu["bmask"][h].astype(np.uint64), bm), f"bmask differs at head {h}"
        assert gpu["bmax"][h] == oracle.bmax(ids[h]), f"b_max differs at head {h}"
        if tiles_per_head is None or tiles_per_head >= T:
            want = oracle.tile_spans(ids[h], causal)
            assert np.array_equal(gpu["spans"][h], want), f"spans differ at head {h}"
        else:
            rng = np.random.default_rng(h)
            pick = sorted(set([0, T - 1] + list(rng.choice(T, tiles_per_head, replace=False))))
            for t in pick:
                sub = _span_one_tile(ids[h], causal, t, n)
                assert tuple(gpu["spans"][h, t]) == sub, (h, t, gpu["spans"][h, t], sub)
    return ids


def _span_one_tile(ids_hs, causal, t, n):
    rows = np.arange(t * 128, min(n, t * 128 + 128))
    c = oracle.counts_rows(ids_hs, rows)
    if causal:
        c[np.arange(n)[None, :] > rows[:, None]] = 0
    nz = np.nonzero(c.sum(axis=0))[0]
    return (int(nz.min()), int(nz.max()))


def oracle_rows(q, k, v, table, causal, rows: Optional[Sequence[int]], batches: Optional[Sequence[int]] = None,
                chunk: int = 64):
    """Oracle T~ and row_sum on the given rows (all rows if None), in float64."""
    Q, K, V = f64(q), f64(k), f64(v)
    B, H, n, d = Q.shape
    group = H // K.shape[1]
    ids = oracle.bin_ids(table, n)
    rows = list(range(n)) if rows is None else list(rows)
    batches = list(range(B)) if batches is None else list(batches)
    O = np.empty((len(batches), H, len(rows), d))
    R = np.empty((len(batches), H, len(rows)))
    for bi, b in enumerate(batches):
        for h in range(H):
            for c0 in range(0, len(rows), chunk):
                rr = rows[c0:c0 + chunk]
                o, r = oracle.approx_attention(Q[b, h], K[b, h // group], V[b, h // group], ids[h], causal, rr)
                O[bi, h, c0:c0 + len(rr)] = o
                R[bi, h, c0:c0 + len(rr)] = r
    return O, R


def tolerance(dtype: torch.dtype, v: torch.Tensor):
    """(O tolerance, row_sum tolerance).

    O: 1e-5 absolute for fp32 inputs, 2e-2 * max|V| for bf16 inputs.
    row_sum: fp32 path 1e-5 (fp32 sums of positive terms, relative error a
    few ulp times the log's argument scale); bf16 path 1e-3 (bf16 inputs are
    exact in the oracle; the tensor-core QK^T accumulates in fp32 and the
    sum of weights stays fp32, so only fp32 rounding and the exp2
    approximation enter).
    """
    if dtype == torch.float32:
        return 1e-5, 1e-5
    return 2e-2 * float(v.abs().max()), 1e-3


def assert_close(gpu_O, gpu_R, want_O, want_R, o_tol, r_tol, what=""):
    assert np.all(np.isfinite(gpu_O)), f"{what}: non-finite O"
    assert np.all(np.isfinite(gpu_R)), f"{what}: non-finite row_sum"
    eo = np.abs(gpu_O - want_O).max()
    er = np.abs(gpu_R - want_R).max()
    assert eo <= o_tol, f"{what}: max|dO| = {eo:.3e} > {o_tol:.3e}"
    assert er <= r_tol, f"{what}: max|d row_sum| = {er:.3e} > {r_tol:.3e}"
    return eo, er
