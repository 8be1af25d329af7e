"""plsh_decode_fwd through the C-ABI against the CPU oracle (needs a B200).

A decode call computes chosen rows of the same T~ as the fused kernel: the
query row at position i against the whole key cache (j <= i when causal),
weighted by the M~ counts (Methodology 2 and 3). The oracle computes the same
rows from the bin ids in float64; tolerances are the fused kernel's
(max|dO| <= 1e-5 for fp32 inputs, <= 2e-2 * max|V| for bf16 inputs; row_sum
1e-5 / 1e-3).
"""
import numpy as np
import pytest
import torch

import workloads
from tests import plsh_harness as PH

pytestmark = pytest.mark.gpu

W = workloads.WORKLOADS


def _sigmas(H):
    return [2.0 ** (1 + 8.0 * h / max(1, H - 1)) for h in range(H)]


def _run(B, H, H_kv, n, d, dtype, causal, s, sigma, seed, rows):
    from alibi_positional_lsh_b200 import PlshForward
    w = workloads.Workload("case", B, H, H_kv, n, d, "f32" if dtype == torch.float32 else "bf16", causal, s, seed)
    q, k, v = workloads.make_qkv(w)
    plan = PlshForward(B, H, H_kv, n, d, s, causal, sigma, seed + 1, dtype, "cuda:0")
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    plan(qd, kd, vd)                                   # masks, and the fused kernel's T~ on every row
    pos = torch.tensor(rows, dtype=torch.int32, device="cuda:0")
    O, R = plan.decode(qd[:, :, rows].contiguous(), pos, kd, vd)
    assert plan.device_errors() == []
    return q, k, v, plan, PH.f64(O), R.cpu().numpy().astype(np.float64)


SMALL = [
    # B, H, H_kv, n, d, dtype, causal, s
    (1, 2, 1, 1000, 128, torch.bfloat16, True, 20),
    (1, 2, 2, 1000, 128, torch.bfloat16, False, 10),
    (2, 4, 2, 700, 128, torch.bfloat16, True, 33),
    (1, 2, 1, 1300, 64, torch.bfloat16, False, 7),
    (1, 2, 1, 777, 128, torch.float32, True, 16),
    (1, 2, 2, 640, 64, torch.float32, False, 40),
    (1, 1, 1, 1, 128, torch.bfloat16, True, 4),
    (1, 1, 1, 300, 128, torch.bfloat16, False, 1),
]


@pytest.mark.parametrize("B,H,H_kv,n,d,dtype,causal,s", SMALL,
                         ids=[f"B{c[0]}H{c[1]}kv{c[2]}n{c[3]}d{c[4]}{'f32' if c[5] == torch.float32 else 'bf16'}"
                              f"{'c' if c[6] else 'nc'}s{c[7]}" for c in SMALL])
def test_decode_rows_match_oracle_and_fused(B, H, H_kv, n, d, dtype, causal, s):
    rng = np.random.default_rng(n + s)
    rows = sorted(set([0, n - 1, n // 2] + list(rng.integers(0, n, 8))))
    rows = rows + [rows[-1]]                           # a repeated position
    q, k, v, plan, O, R = _run(B, H, H_kv, n, d, dtype, causal, s, _sigmas(H), 500 + n, rows)
    want_O, want_R = PH.oracle_rows(q, k, v, plan.table_host.numpy(), causal, rows)
    to, tr = PH.tolerance(dtype, v)
    PH.assert_close(O, R, want_O, want_R, to, tr, "decode")
    # the fused kernel's rows of the same T~
    fO, fR = PH.f64(plan.O)[:, :, rows], plan.row_sum.cpu().numpy().astype(np.float64)[:, :, rows]
    assert np.abs(O - fO).max() <= 2 * to
    assert np.abs(R - fR).max() <= 2 * tr


@pytest.mark.parametrize("sigma", [0.3, 5000.0])
def test_decode_extreme_block_sizes(sigma):
    # tiny sigma: nearly every block a single position (only the own key weighs much);
    # huge sigma: blocks span the whole sequence (the walk runs to the ends)
    n, H = 900, 2
    rows = [0, 1, 450, 898, 899]
    for causal in (True, False):
        q, k, v, plan, O, R = _run(1, H, 1, n, 128, torch.bfloat16, causal, 20, [sigma] * H, 77, rows)
        want_O, want_R = PH.oracle_rows(q, k, v, plan.table_host.numpy(), causal, rows)
        to, tr = PH.tolerance(torch.bfloat16, v)
        PH.assert_close(O, R, want_O, want_R, to, tr, f"decode sigma={sigma} causal={causal}")


def test_decode_headline_last_positions():
    """The headline shape (GQA 16/8, n = 32768, s = 20, causal): the newest positions against the full cache."""
    w = W["qwen3_0p6b_n32k"]
    rows = [w.n - 1, w.n - 2, w.n - 129, 16383, 0]
    q, k, v, plan, O, R = _run(w.B, w.H, w.H_kv, w.n, w.d, w.torch_dtype, w.causal, w.s, w.sigmas(), w.seed, rows)
    want_O, want_R = PH.oracle_rows(q, k, v, plan.table_host.numpy(), w.causal, rows)
    to, tr = PH.tolerance(w.torch_dtype, v)
    PH.assert_close(O, R, want_O, want_R, to, tr, "decode headline")


def test_decode_position_out_of_range_sets_error_bit():
    from alibi_positional_lsh_b200 import PlshForward
    n, H = 256, 2
    plan = PlshForward(1, H, 1, n, 128, 8, True, _sigmas(H), 3, torch.bfloat16, "cuda:0")
    plan.prepare()
    k = torch.zeros((1, 1, n, 128), dtype=torch.bfloat16, device="cuda:0")
    q = torch.zeros((1, H, 2, 128), dtype=torch.bfloat16, device="cuda:0")
    pos = torch.tensor([5, n], dtype=torch.int32, device="cuda:0")   # n is one past the cache
    O, R = plan.decode(q, pos, k, k)
    assert plan.device_errors() == ["POSITION"]
    plan.reset_errors()
    assert bool(torch.isfinite(O[:, :, 0].float()).all())


def test_decode_repeated_calls_agree_and_leave_counters_zero():
    """The last CTA of each row merges the partials and resets the row's counter: repeated calls give the
    same rows bit for bit, and the counters at the end of the scratch are zero after every call."""
    from alibi_positional_lsh_b200 import PlshForward, plsh_decode_scratch_bytes
    n, H, d = 2000, 4, 128
    w = workloads.Workload("case", 1, H, 2, n, d, "bf16", True, 20, 31)
    q, k, v = (t.cuda() for t in workloads.make_qkv(w))
    plan = PlshForward(1, H, 2, n, d, 20, True, _sigmas(H), 4, torch.bfloat16, "cuda:0")
    plan.prepare()
    rows = [n - 1, 1000, 3]
    pos = torch.tensor(rows, dtype=torch.int32, device="cuda:0")
    qr = q[:, :, rows].contiguous()
    first = plan.decode(qr, pos, k, v)
    first = (first[0].clone(), first[1].clone())
    m = len(rows)
    n_rows = 1 * H * m
    for _ in range(3):
        O, R = plan.decode(qr, pos, k, v)
        torch.cuda.synchronize()
        assert torch.equal(O, first[0]) and torch.equal(R, first[1])
        counters = plan.decode_scratch[plsh_decode_scratch_bytes(1, H, m, d) // 4 - n_rows:]
        assert int(counters.view(torch.int32).abs().max()) == 0
    assert plan.device_errors() == []


def test_decode_mha8_non_causal_both_sides():
    """8 heads, n = 8192, non-causal: each row's walk runs below and above its position."""
    w = W["mha8_n8192"]
    rows = [0, 4095, 4096, w.n - 1]
    q, k, v, plan, O, R = _run(w.B, w.H, w.H_kv, w.n, w.d, w.torch_dtype, w.causal, w.s, w.sigmas(), w.seed, rows)
    want_O, want_R = PH.oracle_rows(q, k, v, plan.table_host.numpy(), w.causal, rows)
    to, tr = PH.tolerance(w.torch_dtype, v)
    PH.assert_close(O, R, want_O, want_R, to, tr, "decode mha8")


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_decode_long_runs_both_sides(dtype, d):
    """Blocks much longer than the sequence (sigma = 1e6) and not causal: every row's runs reach both ends
    of a 20,000-key cache, so the range pass takes several 2,048-key steps, each side gets several work
    units of many segments, and every unit but the first starts from a carry."""
    n, H = 20000, 2
    rows = [0, 137, 9999, 19998, 19999]
    q, k, v, plan, O, R = _run(1, H, 1, n, d, dtype, False, 20, [1.0e6, 3.0e3], 2024, rows)
    want_O, want_R = PH.oracle_rows(q, k, v, plan.table_host.numpy(), False, rows)
    to, tr = PH.tolerance(dtype, v)
    PH.assert_close(O, R, want_O, want_R, to, tr, "decode long runs")
