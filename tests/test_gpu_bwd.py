"""plsh_attention_bwd through the C-ABI against the CPU oracle (needs a B200).

The forward runs on the GPU (its O and row_sum feed the backward, as in
training); the oracle computes dQ, dK, dV from the same inputs and table in
float64. Tolerances, relative to the largest reference entry of each tensor:
  fp32 inputs: 1e-4. Every P_ij is recomputed from S and the forward's row_sum
    with a few fp32 roundings (relative error a few 1e-7), D_i from the fp32 O;
    the sums over a row's or key's window then cancel (sum_j dS_ij = 0), which
    can magnify that error against the result by one or two orders.
  bf16 inputs: 2e-2 (the forward's bound for O): dQ, dK, dV are rounded to
    bf16 (2^-9) and D_i = dO_i . O_i uses the bf16 O.
The scale has a floor of 1e-3: where the exact gradient is 0 (n = 1, a single
key: dS = P (dP - D) = 0) the GPU's value is the fp32 rounding of dP - D.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests import plsh_harness as PH

pytestmark = pytest.mark.gpu

W = workloads.WORKLOADS


def _sigmas(kind, H):
    if kind == "huge":
        return [5000.0] * H
    if kind == "tiny":
        return [0.3] * H
    return [2.0 ** (1 + 8.0 * h / max(1, H - 1)) for h in range(H)]


def _grad_out(shape, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=torch.float32).to(dtype)


def _run(B, H, H_kv, n, d, dtype, causal, s, sigma, seed):
    from alibi_positional_lsh_b200 import PlshForward
    w = workloads.Workload("case", B, H, H_kv, n, d, "f32" if dtype == torch.float32 else "bf16", causal, s, seed)
    q, k, v = workloads.make_qkv(w)
    dO = _grad_out((B, H, n, d), dtype, seed + 7)
    plan = PlshForward(B, H, H_kv, n, d, s, causal, sigma, seed + 1, dtype, "cuda:0")
    qd, kd, vd, dOd = q.cuda(), k.cuda(), v.cuda(), dO.cuda()
    plan(qd, kd, vd)
    dQ, dK, dV = plan.backward(qd, kd, vd, dOd)
    assert plan.device_errors() == []
    return (q, k, v, dO), plan, (PH.f64(dQ), PH.f64(dK), PH.f64(dV))


def _tol(dtype):
    return 1e-4 if dtype == torch.float32 else 2e-2


def _assert_grads(got, want, dtype, what):
    for name, g, w in zip(("dQ", "dK", "dV"), got, want):
        assert np.all(np.isfinite(g)), f"{what}: non-finite {name}"
        err = np.abs(g - w).max()
        scale = max(np.abs(w).max(), 1e-3)
        assert err <= _tol(dtype) * scale, f"{what}: max|d{name}| = {err:.3e} > {_tol(dtype)} * {scale:.3e}"


SMALL = [
    # B, H, H_kv, n, d, dtype, causal, s, sigma_kind
    (1, 2, 1, 1000, 128, torch.bfloat16, True, 20, "mixed"),
    (1, 2, 2, 1000, 128, torch.bfloat16, False, 10, "mixed"),
    (2, 4, 2, 700, 128, torch.bfloat16, True, 33, "mixed"),
    (1, 2, 1, 1300, 64, torch.bfloat16, False, 7, "mixed"),
    (1, 2, 1, 777, 128, torch.float32, True, 16, "mixed"),
    (1, 2, 2, 640, 64, torch.float32, False, 40, "mixed"),
    (1, 1, 1, 1, 128, torch.bfloat16, True, 4, "mixed"),
    (1, 1, 1, 129, 128, torch.float32, False, 64, "mixed"),
    (1, 2, 1, 600, 128, torch.float32, True, 20, "huge"),
    (1, 2, 1, 600, 128, torch.float32, False, 20, "tiny"),
]


@pytest.mark.parametrize("B,H,H_kv,n,d,dtype,causal,s,kind", SMALL,
                         ids=[f"B{c[0]}H{c[1]}kv{c[2]}n{c[3]}d{c[4]}{'f32' if c[5] == torch.float32 else 'bf16'}"
                              f"{'c' if c[6] else 'nc'}s{c[7]}{c[8]}" for c in SMALL])
def test_backward_small_full_oracle(B, H, H_kv, n, d, dtype, causal, s, kind):
    (q, k, v, dO), plan, got = _run(B, H, H_kv, n, d, dtype, causal, s, _sigmas(kind, H), 600 + n + s)
    want = oracle.backward(PH.f64(q), PH.f64(k), PH.f64(v), PH.f64(dO), plan.table_host.numpy(), causal)
    _assert_grads(got, want, dtype, "backward small")


def test_backward_singleton_bins_give_dv_equal_do():
    """delta < 1 for every hash: T~ = V, so dV = dO (summed over the group) and dQ = dK = 0."""
    from alibi_positional_lsh_b200 import PlshForward
    B, H, H_kv, n, d, s = 1, 2, 1, 300, 128, 3
    w = workloads.Workload("case", B, H, H_kv, n, d, "f32", True, s, 5)
    q, k, v = (t.cuda() for t in workloads.make_qkv(w))
    dO = _grad_out((B, H, n, d), torch.float32, 9).cuda()
    plan = PlshForward(B, H, H_kv, n, d, s, True, [1.0, 1.0], 1, torch.float32, "cuda:0")
    plan(q, k, v, table=np.tile(np.array([[0.5, 0.25], [0.9, 0.1], [0.3, 0.2]]), (H, 1, 1)))
    dQ, dK, dV = plan.backward(q, k, v, dO)
    assert plan.device_errors() == []
    # dS_ii = dP_ii - D_i is 0 in exact arithmetic; in fp32 the two dot products round differently,
    # by at most about d * 2^-24 * max|dO| * max|V| each, and dQ, dK multiply that by K or Q / sqrt d
    bound = 4 * d * 2.0 ** -24 * float(dO.abs().max() * v.abs().max()) * float(max(q.abs().max(), k.abs().max()))
    bound /= d ** 0.5
    assert float(dQ.abs().max()) <= bound and float(dK.abs().max()) <= bound, bound
    # P_ii = exp(S_ii / sqrt d - L_i) = 1 up to the fp32 rounding of the forward's row_sum L_i = S_ii / sqrt d
    torch.testing.assert_close(dV[:, 0], dO.sum(dim=1), rtol=2e-5, atol=2e-5)


def test_backward_headline_sampled():
    """The headline shape (B=2, GQA 16/8, n=32768, s=20, causal): dQ on sampled rows of every head,
    dK and dV on sampled keys of KV heads 1 and 5 (query heads 2, 3 and 10, 11) of batch 0."""
    w = W["qwen3_0p6b_n32k"]
    (q, k, v, dO), plan, (dQ, dK, dV) = _run(w.B, w.H, w.H_kv, w.n, w.d, w.torch_dtype, w.causal, w.s,
                                             w.sigmas(), w.seed)
    ids = oracle.bin_ids(plan.table_host.numpy(), w.n)
    Q, K, V, G = PH.f64(q), PH.f64(k), PH.f64(v), PH.f64(dO)
    group = w.H // w.H_kv
    rows = sorted(set(workloads.sample_rows(w.n, 6, w.seed + 2)) | {0, 127, 128, w.n - 1})
    keys = sorted(set(workloads.sample_rows(w.n, 3, w.seed + 3)) | {0, w.n - 1})
    got_q, want_q = [], []
    for b in range(w.B):
        for h in range(w.H):
            g = h // group
            dq, _, _ = oracle.approx_attention_grad_sampled(Q[b, h], K[b, g], V[b, g], G[b, h], ids[h], w.causal,
                                                            rows, [])
            got_q.append(dQ[b, h, rows])
            want_q.append(dq)
    got_k, want_k, got_v, want_v = [], [], [], []
    for g in (1, 5):
        dk = np.zeros((len(keys), w.d))
        dv = np.zeros((len(keys), w.d))
        for h in range(g * group, (g + 1) * group):
            _, a, c = oracle.approx_attention_grad_sampled(Q[0, h], K[0, g], V[0, g], G[0, h], ids[h], w.causal,
                                                           [], keys)
            dk += a
            dv += c
        got_k.append(dK[0, g, keys])
        want_k.append(dk)
        got_v.append(dV[0, g, keys])
        want_v.append(dv)
    _assert_grads((np.stack(got_q), np.stack(got_k), np.stack(got_v)),
                  (np.stack(want_q), np.stack(want_k), np.stack(want_v)), w.torch_dtype, "backward headline")


def test_backward_single_head_fp32_workload():
    """fp32, d = 64, non-causal, n = 1024, s = 8: the full oracle."""
    w = W["single_head_n1024"]
    (q, k, v, dO), plan, got = _run(w.B, w.H, w.H_kv, w.n, w.d, w.torch_dtype, w.causal, w.s, w.sigmas(), w.seed)
    want = oracle.backward(PH.f64(q), PH.f64(k), PH.f64(v), PH.f64(dO), plan.table_host.numpy(), w.causal)
    _assert_grads(got, want, w.torch_dtype, "backward single_head_n1024")


def test_backward_mha8_sampled_non_causal():
    """bf16, 8 heads, n = 8192, non-causal (both sides of every key): dQ on sampled rows of every head,
    dK and dV on sampled keys of heads 0 and 5."""
    w = W["mha8_n8192"]
    (q, k, v, dO), plan, (dQ, dK, dV) = _run(w.B, w.H, w.H_kv, w.n, w.d, w.torch_dtype, w.causal, w.s,
                                             w.sigmas(), w.seed)
    ids = oracle.bin_ids(plan.table_host.numpy(), w.n)
    Q, K, V, G = PH.f64(q), PH.f64(k), PH.f64(v), PH.f64(dO)
    rows = sorted(set(workloads.sample_rows(w.n, 8, w.seed + 4)) | {0, 63, 64, w.n - 1})
    keys = sorted(set(workloads.sample_rows(w.n, 4, w.seed + 5)) | {0, w.n - 1})
    got, want = ([], [], []), ([], [], [])
    for h in range(w.H):
        dq, _, _ = oracle.approx_attention_grad_sampled(Q[0, h], K[0, h], V[0, h], G[0, h], ids[h], w.causal, rows, [])
        got[0].append(dQ[0, h, rows])
        want[0].append(dq)
    for h in (0, 5):
        _, dk, dv = oracle.approx_attention_grad_sampled(Q[0, h], K[0, h], V[0, h], G[0, h], ids[h], w.causal, [], keys)
        got[1].append(dK[0, h, keys])
        want[1].append(dk)
        got[2].append(dV[0, h, keys])
        want[2].append(dv)
    _assert_grads(tuple(np.stack(x) for x in got), tuple(np.stack(x) for x in want), w.torch_dtype,
                  "backward mha8_n8192")


# ---------------------------------------------------------------- the tcgen05 kernels (bf16, d = 128)

TC_MORE = [
    (1, 2, 1, 600, 128, torch.bfloat16, False, 20, "tiny"),
    (1, 2, 1, 600, 128, torch.bfloat16, True, 20, "huge"),
    (1, 2, 2, 129, 128, torch.bfloat16, False, 64, "mixed"),
    (2, 4, 1, 1000, 128, torch.bfloat16, False, 40, "mixed"),
    (1, 4, 2, 2000, 128, torch.bfloat16, True, 12, "mixed"),
]


@pytest.mark.parametrize("B,H,H_kv,n,d,dtype,causal,s,kind", TC_MORE,
                         ids=[f"B{c[0]}H{c[1]}kv{c[2]}n{c[3]}{'c' if c[6] else 'nc'}s{c[7]}{c[8]}" for c in TC_MORE])
def test_backward_tensor_cores_full_oracle(B, H, H_kv, n, d, dtype, causal, s, kind):
    """bf16 with d = 128 takes the tcgen05 kernels (plsh_attention_bwd_tc): tiny and huge length
    scales, 64-bit masks, grouped heads both ways, ragged n."""
    (q, k, v, dO), plan, got = _run(B, H, H_kv, n, d, dtype, causal, s, _sigmas(kind, H), 900 + n + s)
    want = oracle.backward(PH.f64(q), PH.f64(k), PH.f64(v), PH.f64(dO), plan.table_host.numpy(), causal)
    _assert_grads(got, want, dtype, "backward tensor cores")


@pytest.mark.parametrize("causal", [True, False])
def test_backward_tensor_cores_agree_with_cuda_core_path(causal):
    """The tcgen05 kernels and the fp32 CUDA-core kernels on the same inputs: within the bf16 bar of
    each other (both are within it of the oracle)."""
    from alibi_positional_lsh_b200 import PlshForward
    B, H, H_kv, n, d, s = 1, 4, 2, 3000, 128, 20
    w = workloads.Workload("case", B, H, H_kv, n, d, "bf16", causal, s, 71)
    q, k, v = (t.cuda() for t in workloads.make_qkv(w))
    dO = _grad_out((B, H, n, d), torch.bfloat16, 72).cuda()
    plan = PlshForward(B, H, H_kv, n, d, s, causal, _sigmas("mixed", H), 73, torch.bfloat16, "cuda:0")
    plan(q, k, v)
    tc = [t.double().clone() for t in plan.backward(q, k, v, dO, path="tc")]
    simt = [t.double().clone() for t in plan.backward(q, k, v, dO, path="simt")]
    assert plan.device_errors() == []
    for name, a, b in zip(("dQ", "dK", "dV"), tc, simt):
        assert float((a - b).abs().max()) <= 2e-2 * max(float(b.abs().max()), 1e-3), name
