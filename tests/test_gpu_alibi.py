"""Exact banded ALiBi (plsh_alibi_banded_fwd) against the oracle's exact T* (needs a B200).

The band |i - j| <= ceil(sigma_h ln(1/eps)) drops keys whose ALiBi weight is
below eps relative to the diagonal; with eps = 1e-12 that is far below the
tolerances, so O and row_sum must match oracle.exact_attention (the full
T* = D*^{-1} (exp(QK^T/sqrt d) o L*) V, pinned against additive-bias softmax)
within the same bars as the approximation: max|dO| <= 1e-5 for fp32 inputs,
<= 2e-2 * max|V| for bf16; row_sum within 1e-5 / 1e-3.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests import plsh_harness as PH

pytestmark = pytest.mark.gpu


def _run(B, H, H_kv, n, d, dtype, causal, sigma, eps, seed):
    from alibi_positional_lsh_b200 import PlshForward
    w = workloads.Workload("case", B, H, H_kv, n, d, "f32" if dtype == torch.float32 else "bf16", causal, 1, seed)
    q, k, v = workloads.make_qkv(w)
    plan = PlshForward(B, H, H_kv, n, d, 1, causal, sigma, 0, dtype, "cuda:0")
    plan.O.fill_(float("nan"))
    plan.row_sum.fill_(float("nan"))
    plan.attend_alibi(q.cuda(), k.cuda(), v.cuda(), eps)
    errs = plan.device_errors()
    return q, k, v, PH.f64(plan.O), plan.row_sum.cpu().numpy().astype(np.float64), errs


def _oracle(q, k, v, sigma, causal, rows=None):
    Q, K, V = PH.f64(q), PH.f64(k), PH.f64(v)
    B, H, n, d = Q.shape
    group = H // K.shape[1]
    nr = n if rows is None else len(rows)
    O = np.empty((B, H, nr, d))
    R = np.empty((B, H, nr))
    for b in range(B):
        for h in range(H):
            O[b, h], R[b, h] = oracle.exact_attention(Q[b, h], K[b, h // group], V[b, h // group], float(sigma[h]),
                                                      causal, rows)
    return O, R


CASES = [
    # B, H, H_kv, n, d, dtype, causal, sigmas
    (1, 2, 1, 1000, 128, torch.bfloat16, True, [3.0, 90.0]),
    (2, 4, 2, 700, 128, torch.bfloat16, False, [1.5, 8.0, 40.0, 300.0]),
    (1, 1, 1, 129, 128, torch.bfloat16, True, [5000.0]),
    (1, 2, 1, 1, 128, torch.bfloat16, False, [2.0, 2.0]),
    (1, 2, 2, 777, 64, torch.float32, True, [4.0, 60.0]),
    (1, 2, 1, 640, 128, torch.float32, False, [0.7, 25.0]),
]


@pytest.mark.parametrize("B,H,H_kv,n,d,dtype,causal,sigma", CASES,
                         ids=[f"B{c[0]}H{c[1]}kv{c[2]}n{c[3]}d{c[4]}{'f32' if c[5] == torch.float32 else 'bf16'}"
                              f"{'c' if c[6] else 'nc'}" for c in CASES])
def test_banded_alibi_small_full_oracle(B, H, H_kv, n, d, dtype, causal, sigma):
    q, k, v, O, R, errs = _run(B, H, H_kv, n, d, dtype, causal, sigma, 1e-12, 500 + n)
    assert errs == []
    Ow, Rw = _oracle(q, k, v, sigma, causal)
    to, tr = PH.tolerance(dtype, v)
    PH.assert_close(O, R, Ow, Rw, to, tr, "banded alibi")


def test_banded_alibi_full_size_sampled_rows():
    w = workloads.WORKLOADS["qwen3_0p6b_n32k"]
    sigma = w.sigmas()
    q, k, v, O, R, errs = _run(w.B, w.H, w.H_kv, w.n, w.d, w.torch_dtype, w.causal, sigma, 1e-10, w.seed)
    assert errs == []
    rows = sorted(set(workloads.sample_rows(w.n, 24, w.seed + 7)) | {0, 127, 128, w.n - 1})
    Ow, Rw = _oracle(q, k, v, sigma, w.causal, rows)
    to, tr = PH.tolerance(w.torch_dtype, v)
    PH.assert_close(O[:, :, rows], R[:, :, rows], Ow, Rw, to, tr, "banded alibi n=32k")


def test_banded_alibi_band_cut_is_eps():
    """A coarse eps drops far keys (here from 384 positions on, weight e^{-384/200} ~ 0.15): the
    result moves toward T* as eps shrinks."""
    sigma = [200.0]
    q, k, v, O1, _, e1 = _run(1, 1, 1, 2000, 128, torch.float32, False, sigma, 0.3, 9)
    _, _, _, O2, _, e2 = _run(1, 1, 1, 2000, 128, torch.float32, False, sigma, 1e-12, 9)
    assert e1 == [] and e2 == []
    Ow, _ = _oracle(q, k, v, sigma, False)
    err1, err2 = np.abs(O1 - Ow).max(), np.abs(O2 - Ow).max()
    assert err2 <= 1e-5 < err1
