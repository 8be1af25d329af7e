"""Failure detection of the fused attention kernel: a bounded wait runs out (needs a B200).

With a 1 ms wait limit and the tensor-core issuer told to issue nothing, no tile of scores ever
arrives: the softmax warps' waits run out, PLSH_DEVERR_TIMEOUT is set, every role leaves its loop,
the copies in flight are drained and Tensor Memory is freed, and the launch returns. Nothing traps
or hangs. The next normal call on the same stream must then match the oracle.
"""
import numpy as np
import pytest
import torch

import workloads
from tests import plsh_harness as PH

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_the_next_call_is_correct():
    from alibi_positional_lsh_b200 import PlshForward, plsh_set_wait_limit_ns, plsh_test_withhold_mma
    B, H, H_kv, n, d, s, causal = 1, 2, 1, 300, 128, 12, True
    w = workloads.Workload("case", B, H, H_kv, n, d, "bf16", causal, s, 31)
    q, k, v = workloads.make_qkv(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    sigma = [4.0, 50.0]
    plan = PlshForward(B, H, H_kv, n, d, s, causal, sigma, 5, torch.bfloat16, "cuda:0")
    plan.prepare()
    torch.cuda.synchronize()
    plsh_set_wait_limit_ns(1_000_000)
    plsh_test_withhold_mma(True)
    try:
        plan.attend(qd, kd, vd)
        torch.cuda.synchronize()
    finally:
        plsh_test_withhold_mma(False)
        plsh_set_wait_limit_ns(0)
    assert "TIMEOUT" in plan.device_errors()
    # the context is usable and the kernel correct again
    plan.reset_errors()
    plan.O.fill_(float("nan"))
    plan.row_sum.fill_(float("nan"))
    plan.attend(qd, kd, vd)
    torch.cuda.synchronize()
    assert plan.device_errors() == []
    O, R = PH.oracle_rows(q, k, v, plan.table_host.numpy(), causal, None)
    to, tr = PH.tolerance(torch.bfloat16, v)
    PH.assert_close(PH.f64(plan.O), plan.row_sum.cpu().numpy().astype(np.float64), O, R, to, tr, "after timeout")


def test_decode_bounded_wait_runs_out_and_the_next_call_is_correct():
    """The decode kernel's producer warp told to issue nothing: the compute warps' waits for a segment
    run out (1 ms), PLSH_DEVERR_TIMEOUT is set and the launch returns. The next normal call on the same
    scratch must match the oracle and leave the per-row counters at zero."""
    from alibi_positional_lsh_b200 import (PlshForward, plsh_decode_scratch_bytes, plsh_set_wait_limit_ns,
                                           plsh_test_withhold_mma)
    B, H, H_kv, n, d, s, causal = 1, 2, 1, 600, 128, 12, True
    w = workloads.Workload("case", B, H, H_kv, n, d, "bf16", causal, s, 41)
    q, k, v = workloads.make_qkv(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    plan = PlshForward(B, H, H_kv, n, d, s, causal, [6.0, 300.0], 9, torch.bfloat16, "cuda:0")
    plan.prepare()
    rows = [n - 1, 250]
    pos = torch.tensor(rows, dtype=torch.int32, device="cuda:0")
    qr = qd[:, :, rows].contiguous()
    torch.cuda.synchronize()
    plsh_set_wait_limit_ns(1_000_000)
    plsh_test_withhold_mma(True)
    try:
        plan.decode(qr, pos, kd, vd)
        torch.cuda.synchronize()
    finally:
        plsh_test_withhold_mma(False)
        plsh_set_wait_limit_ns(0)
    assert "TIMEOUT" in plan.device_errors()
    plan.reset_errors()
    O, R = plan.decode(qr, pos, kd, vd)
    torch.cuda.synchronize()
    assert plan.device_errors() == []
    want_O, want_R = PH.oracle_rows(q, k, v, plan.table_host.numpy(), causal, rows)
    to, tr = PH.tolerance(torch.bfloat16, v)
    PH.assert_close(PH.f64(O), R.cpu().numpy().astype(np.float64), want_O, want_R, to, tr, "decode after timeout")
    n_rows = B * H * len(rows)
    counters = plan.decode_scratch[plsh_decode_scratch_bytes(B, H, len(rows), d) // 4 - n_rows:]
    assert int(counters.view(torch.int32).abs().max()) == 0
