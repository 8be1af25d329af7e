"""The oracle checks the long-context and Mistral-7B-shaped workloads ask for (needs a B200).

long_n128k (B=1, 40 query / 8 KV heads, n=131072, d=128, bf16, causal, s=16): on 512 sampled
query rows of every head, T~ from plsh_attention_fwd against the oracle's T~, and exact T* from
plsh_alibi_banded_fwd against the oracle's exact ALiBi attention.

mistral7b_n16k (B=1, 32 query / 8 KV heads, n=16384, d=128, bf16, causal): ||T* - T~|| on 256
sampled rows of every head for s = 10, 20, 40, with T~ from the GPU and T* from the oracle. The
convergence statement of the pages (T~ approaches T* as s grows) says the error falls with s;
the test checks that and prints the figures.
"""
import json

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests import plsh_harness as PH

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _rows_f64(x: torch.Tensor, b: int, h: int, rows=None) -> np.ndarray:
    t = x[b, h] if rows is None else x[b, h, rows]
    return t.to(torch.float64).numpy()


def test_long_context_512_rows_approx_and_exact():
    from alibi_positional_lsh_b200 import PlshForward
    w = workloads.WORKLOADS["long_n128k"]
    q, k, v = workloads.make_qkv(w)
    rows = sorted(set(workloads.sample_rows(w.n, w.oracle_rows, w.seed)) | {127, 128, w.n - 128, w.n - 129})
    plan = PlshForward(w.B, w.H, w.H_kv, w.n, w.d, w.s, w.causal, w.sigmas(), w.seed, w.torch_dtype, "cuda:0")
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    for fill in (plan.O, plan.row_sum):
        fill.fill_(float("nan"))
    plan(qd, kd, vd)
    assert plan.device_errors() == []
    O_t = plan.O[:, :, rows].double().cpu().numpy()
    R_t = plan.row_sum[:, :, rows].double().cpu().numpy()
    plan.O.fill_(float("nan"))
    plan.row_sum.fill_(float("nan"))
    plan.attend_alibi(qd, kd, vd, 1e-10)
    assert plan.device_errors() == []
    O_s = plan.O[:, :, rows].double().cpu().numpy()
    R_s = plan.row_sum[:, :, rows].double().cpu().numpy()
    del qd, kd, vd
    table = oracle.draw_table(w.seed, w.sigmas(), w.s)
    ids = oracle.bin_ids(table, w.n)
    group = w.H // w.H_kv
    to, tr = PH.tolerance(w.torch_dtype, v)
    for h in range(w.H):
        Qr = _rows_f64(q, 0, h)
        Kh, Vh = _rows_f64(k, 0, h // group), _rows_f64(v, 0, h // group)
        for c0 in range(0, len(rows), 128):
            rr = rows[c0:c0 + 128]
            Oo, Ro = oracle.approx_attention(Qr, Kh, Vh, ids[h], True, rr)
            PH.assert_close(O_t[0, h, c0:c0 + len(rr)], R_t[0, h, c0:c0 + len(rr)], Oo, Ro, to, tr, f"T~ head {h}")
            Oe, Re = oracle.exact_attention(Qr, Kh, Vh, float(w.sigmas()[h]), True, rr)
            PH.assert_close(O_s[0, h, c0:c0 + len(rr)], R_s[0, h, c0:c0 + len(rr)], Oe, Re, to, tr, f"T* head {h}")


def test_mistral_error_to_exact_alibi_falls_with_s():
    from alibi_positional_lsh_b200 import PlshForward
    base = workloads.WORKLOADS["mistral7b_n16k"]
    q, k, v = workloads.make_qkv(base)
    rows = workloads.sample_rows(base.n, base.oracle_rows, base.seed)
    group = base.H // base.H_kv
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    approx = {}
    for s in workloads.MISTRAL_S_SWEEP:
        plan = PlshForward(base.B, base.H, base.H_kv, base.n, base.d, s, True, base.sigmas(), base.seed,
                           base.torch_dtype, "cuda:0")
        plan(qd, kd, vd)
        assert plan.device_errors() == []
        approx[s] = plan.O[0, :, rows].double().cpu().numpy()
    exact = np.empty((base.H, len(rows), base.d))
    for h in range(base.H):
        exact[h], _ = oracle.exact_attention(_rows_f64(q, 0, h), _rows_f64(k, 0, h // group),
                                             _rows_f64(v, 0, h // group), float(base.sigmas()[h]), True, rows)
    report = {}
    for s in workloads.MISTRAL_S_SWEEP:
        diff = np.abs(approx[s] - exact)            # [H][rows][d]
        per_row_max = diff.max(axis=2)
        per_row_mean = diff.mean(axis=2)
        report[s] = {"max": float(per_row_max.max()), "mean_of_row_max": float(per_row_max.mean()),
                     "mean_abs": float(per_row_mean.mean())}
    print("||T* - T~|| on", len(rows), "rows x", base.H, "heads:", json.dumps(report))
    s_list = list(workloads.MISTRAL_S_SWEEP)
    for a, b in zip(s_list, s_list[1:]):
        assert report[b]["mean_of_row_max"] < report[a]["mean_of_row_max"], report
        assert report[b]["mean_abs"] < report[a]["mean_abs"], report
