"""The per-sample comparator (K4) through the C-ABI against the CPU oracle (needs a B200).

plsh_attention_varlen_fwd computes the same T~ and row_sum as the fused
kernel, as a sum of s block-diagonal attentions (Theorem 2.2's construction,
Methodology 3). Its per-hash windows must be bit-exact with
oracle.varlen_spans; O and row_sum must meet the same tolerances as K3
(max|dO| <= 1e-5 for fp32 inputs, <= 2e-2 * max|V| for bf16 inputs).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests import plsh_harness as PH

pytestmark = pytest.mark.gpu

W = workloads.WORKLOADS


def _inputs(B, H, H_kv, n, d, dtype, seed):
    w = workloads.Workload("case", B, H, H_kv, n, d, "f32" if dtype == torch.float32 else "bf16", False, 1, seed)
    return workloads.make_qkv(w)


def _tolerance(dtype, v, s, n):
    """K3's tolerances, except fp32 row_sum: the comparator folds s separate passes into the
    running sum, each chunk of 32 keys possibly rescaling it by a float exp and every key adding
    to it, so its relative error is bounded by (s * ceil(n/32) + n) * 2^-24 rather than a few ulp."""
    to, tr = PH.tolerance(dtype, v)
    if dtype == torch.float32:
        tr = max(tr, (s * ((n + 31) // 32) + n) * 2.0 ** -24)
    return to, tr


def _check_varlen_spans(gpu, n, causal, tiles_per_head=None):
    ids = gpu["ids"]
    H, s, _ = ids.shape
    T = (n + 127) // 128
    for h in range(H):
        if tiles_per_head is None or tiles_per_head >= T:
            pick = None
        else:
            rng = np.random.default_rng(100 + h)
            pick = sorted(set([0, T - 1] + list(rng.choice(T, tiles_per_head, replace=False))))
        want = oracle.varlen_spans(ids[h], causal, tiles=pick)
        got = gpu["varlen_spans"][h]
        sel = slice(None) if pick is None else pick
        assert np.array_equal(got[:, sel], want[:, sel]), f"per-hash windows differ at head {h}"


SMALL = [
    # B, H, H_kv, n, d, dtype, causal, s, sigma_kind
    (1, 2, 1, 1000, 128, torch.bfloat16, True, 20, "mixed"),
    (1, 2, 2, 1000, 128, torch.bfloat16, False, 10, "mixed"),
    (2, 4, 2, 700, 128, torch.bfloat16, True, 33, "mixed"),
    (1, 2, 1, 1300, 64, torch.bfloat16, True, 7, "mixed"),
    (1, 2, 1, 777, 128, torch.float32, True, 16, "mixed"),
    (1, 2, 2, 640, 64, torch.float32, False, 40, "mixed"),
    (1, 1, 1, 1, 128, torch.bfloat16, True, 4, "mixed"),
    (1, 1, 1, 129, 128, torch.bfloat16, False, 4, "mixed"),
    (1, 2, 2, 384, 128, torch.bfloat16, True, 1, "mixed"),
    (1, 2, 1, 600, 128, torch.bfloat16, False, 20, "huge"),
    (1, 2, 1, 600, 128, torch.bfloat16, True, 20, "tiny"),
]


def _sigmas(kind, H):
    if kind == "huge":
        return [5000.0] * H
    if kind == "tiny":
        return [0.3] * H
    return [2.0 ** (1 + 8.0 * h / max(1, H - 1)) for h in range(H)]


@pytest.mark.parametrize("B,H,H_kv,n,d,dtype,causal,s,kind", SMALL,
                         ids=[f"B{c[0]}H{c[1]}kv{c[2]}n{c[3]}d{c[4]}{'f32' if c[5] == torch.float32 else 'bf16'}"
                              f"{'c' if c[6] else 'nc'}s{c[7]}{c[8]}" for c in SMALL])
def test_varlen_small_full_oracle(B, H, H_kv, n, d, dtype, causal, s, kind):
    q, k, v = _inputs(B, H, H_kv, n, d, dtype, 300 + n + s)
    gpu = PH.run_gpu(B, H, H_kv, n, d, s, causal, _sigmas(kind, H), 17 + s, q, k, v, varlen=True)
    assert gpu["errors"] == []
    _check_varlen_spans(gpu, n, causal)
    O, R = PH.oracle_rows(q, k, v, gpu["table"], causal, None)
    to, tr = _tolerance(dtype, v, s, n)
    PH.assert_close(gpu["O"], gpu["row_sum"], O, R, to, tr, "varlen small")


def test_varlen_single_head_fp32_workload():
    w = W["single_head_n1024"]
    q, k, v = workloads.make_qkv(w)
    gpu = PH.run_gpu(w.B, w.H, w.H_kv, w.n, w.d, w.s, w.causal, w.sigmas(), w.seed, q, k, v, varlen=True)
    assert gpu["errors"] == []
    _check_varlen_spans(gpu, w.n, w.causal)
    O, R = PH.oracle_rows(q, k, v, gpu["table"], w.causal, None)
    to, tr = _tolerance(torch.float32, v, w.s, w.n)
    PH.assert_close(gpu["O"], gpu["row_sum"], O, R, to, tr, "varlen fp32 n=1024")


VARLEN_ROWS = {"mha8_n8192": 48, "qwen3_0p6b_n32k": 32}


@pytest.mark.parametrize("name", list(VARLEN_ROWS))
def test_varlen_full_size_sampled_rows_and_fused_agreement(name):
    w = W[name]
    q, k, v = workloads.make_qkv(w)
    gpu = PH.run_gpu(w.B, w.H, w.H_kv, w.n, w.d, w.s, w.causal, w.sigmas(), w.seed, q, k, v, varlen=True)
    assert gpu["errors"] == []
    _check_varlen_spans(gpu, w.n, w.causal, tiles_per_head=4)
    rows = sorted(set(workloads.sample_rows(w.n, VARLEN_ROWS[name], w.seed + 1)) | {127, 128, w.n - 1})
    O, R = PH.oracle_rows(q, k, v, gpu["table"], w.causal, rows)
    to, tr = _tolerance(w.torch_dtype, v, w.s, w.n)
    PH.assert_close(gpu["O"][:, :, rows], gpu["row_sum"][:, :, rows], O, R, to, tr, name)
    # every row: the comparator and the fused kernel compute the same T~
    fused = PH.run_gpu(w.B, w.H, w.H_kv, w.n, w.d, w.s, w.causal, w.sigmas(), w.seed, q, k, v)
    assert fused["errors"] == []
    assert np.abs(gpu["O"] - fused["O"]).max() <= 2 * to
    assert np.abs(gpu["row_sum"] - fused["row_sum"]).max() <= 2 * tr


def test_varlen_scratch_size_is_checked():
    from alibi_positional_lsh_b200 import PlshError, PLSH_BF16, plsh_attention_varlen_fwd, plsh_varlen_scratch_bytes
    from alibi_positional_lsh_b200 import PlshForward
    n, s = 300, 5
    plan = PlshForward(1, 1, 1, n, 128, s, True, [4.0], 1, torch.bfloat16, "cuda:0")
    plan.prepare()
    q, k, v = (t.cuda() for t in _inputs(1, 1, 1, n, 128, torch.bfloat16, 2))
    need = plsh_varlen_scratch_bytes(1, s, n)
    assert need == 8 * s * 3
    small = torch.empty((need // 4 - 1,), dtype=torch.int32, device="cuda:0")
    with pytest.raises(PlshError) as ei:
        plsh_attention_varlen_fwd(q, k, v, PLSH_BF16, 1, 1, 1, n, 128, plan.sigma_dev, s, plan.table_dev, plan.ids,
                                  plan.bmask, 1, small, plan.O, plan.row_sum, plan.err)
    assert ei.value.code == 1
    assert plan.device_errors() == []
