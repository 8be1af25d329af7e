"""plsh_attention_varlen_fwd_static against plsh_attention_varlen_fwd (needs a B200).

The static entry point keeps the comparator's per-hash windows in the
library's own file-scope device buffer instead of caller scratch. It runs the
same kernels on the same windows, so two calls in a row must reproduce the
caller-scratch entry point's O and row_sum bit for bit; a problem whose windows
do not fit the buffer is refused on the host before anything is launched.
The file name sorts last, so in a full run these tests also follow every other
GPU test in the same process.
"""
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

CASES = [
    # B, H, H_kv, n, d, dtype, causal, s
    (1, 2, 1, 1000, 128, torch.bfloat16, True, 20),
    (2, 4, 2, 700, 128, torch.bfloat16, False, 33),
    (1, 2, 2, 640, 64, torch.float32, False, 40),
]


@pytest.mark.parametrize("B,H,H_kv,n,d,dtype,causal,s", CASES)
def test_static_buffer_matches_caller_scratch_twice(B, H, H_kv, n, d, dtype, causal, s):
    from alibi_positional_lsh_b200 import PlshForward, plsh_attention_varlen_fwd_static
    w = workloads.Workload("case", B, H, H_kv, n, d, "f32" if dtype == torch.float32 else "bf16", causal, s, 40 + n)
    q, k, v = (t.cuda() for t in workloads.make_qkv(w))
    sigma = [2.0 ** (1 + 8.0 * h / max(1, H - 1)) for h in range(H)]
    plan = PlshForward(B, H, H_kv, n, d, s, causal, sigma, 9 + s, dtype, "cuda:0")
    plan.prepare()
    O_ref, R_ref = (t.clone() for t in plan.attend_varlen(q, k, v))
    for _ in range(2):
        O = torch.full_like(O_ref, float("nan"))
        R = torch.full_like(R_ref, float("nan"))
        plsh_attention_varlen_fwd_static(q, k, v, plan.dtype_code, B, H, H_kv, n, d, plan.sigma_dev, s,
                                         plan.table_dev, plan.ids, plan.bmask, int(causal), O, R, plan.err)
        torch.cuda.synchronize()
        assert torch.equal(O, O_ref)
        assert torch.equal(R, R_ref)
    assert plan.device_errors() == []


def test_static_buffer_refuses_oversize_before_launch():
    from alibi_positional_lsh_b200 import (PLSH_BF16, PLSH_VARLEN_STATIC_SCRATCH_BYTES, PlshError,
                                           plsh_attention_varlen_fwd_static, plsh_varlen_scratch_bytes)
    H, s, n = 40, 64, 131072
    assert plsh_varlen_scratch_bytes(H, s, n) > PLSH_VARLEN_STATIC_SCRATCH_BYTES
    # the size check comes before any launch, so small stand-in buffers are never touched
    t = torch.zeros((256,), dtype=torch.bfloat16, device="cuda:0")
    i = torch.zeros((256,), dtype=torch.int32, device="cuda:0")
    f = torch.zeros((256,), dtype=torch.float32, device="cuda:0")
    with pytest.raises(PlshError) as ei:
        plsh_attention_varlen_fwd_static(t, t, t, PLSH_BF16, 1, H, 8, n, 128, None, s, None, i, i, 1, t, f, i)
    assert ei.value.code == 3
    assert "static buffer" in str(ei.value)
    torch.cuda.synchronize()


def _static_call(plan, q, k, v, B, H, H_kv, n, d, s, causal, O, R):
    from alibi_positional_lsh_b200 import plsh_attention_varlen_fwd_static
    plsh_attention_varlen_fwd_static(q, k, v, plan.dtype_code, B, H, H_kv, n, d, plan.sigma_dev, s,
                                     plan.table_dev, plan.ids, plan.bmask, int(causal), O, R, plan.err)


def test_static_buffer_call_allocates_nothing():
    """After a first call (which loads the module in this context), a call changes neither the
    bytes torch has allocated nor the device's free bytes."""
    from alibi_positional_lsh_b200 import PlshForward
    B, H, H_kv, n, d, s, causal = 1, 2, 1, 900, 128, 20, True
    w = workloads.Workload("case", B, H, H_kv, n, d, "bf16", causal, s, 77)
    q, k, v = (t.cuda() for t in workloads.make_qkv(w))
    plan = PlshForward(B, H, H_kv, n, d, s, causal, [3.0, 40.0], 5, torch.bfloat16, "cuda:0")
    plan.prepare()
    plan.ensure_ids()
    O = torch.empty_like(q)
    R = torch.empty((B, H, n), dtype=torch.float32, device="cuda:0")
    _static_call(plan, q, k, v, B, H, H_kv, n, d, s, causal, O, R)
    torch.cuda.synchronize()
    alloc0, free0 = torch.cuda.memory_allocated(), torch.cuda.mem_get_info()[0]
    for _ in range(3):
        _static_call(plan, q, k, v, B, H, H_kv, n, d, s, causal, O, R)
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == alloc0
    assert torch.cuda.mem_get_info()[0] == free0
    assert plan.device_errors() == []


def test_static_buffer_exact_limit_accepted_one_tile_more_refused():
    """8 H s ceil(n/128) equal to the buffer size runs and matches the caller-scratch entry point;
    one query tile more is refused with PLSH_ERR_RANGE before any launch."""
    from alibi_positional_lsh_b200 import (PLSH_BF16, PLSH_VARLEN_STATIC_SCRATCH_BYTES, PlshError, PlshForward,
                                           plsh_attention_varlen_fwd_static, plsh_varlen_scratch_bytes)
    B, H, H_kv, d, s, causal = 1, 8, 8, 128, 64, True
    n = (PLSH_VARLEN_STATIC_SCRATCH_BYTES // (8 * H * s)) * 128
    assert plsh_varlen_scratch_bytes(H, s, n) == PLSH_VARLEN_STATIC_SCRATCH_BYTES
    g = torch.Generator(device="cuda:0").manual_seed(3)
    q = torch.randn((B, H, n, d), generator=g, device="cuda:0").to(torch.bfloat16)
    k = torch.randn((B, H_kv, n, d), generator=g, device="cuda:0").to(torch.bfloat16)
    v = torch.randn((B, H_kv, n, d), generator=g, device="cuda:0").to(torch.bfloat16)
    # short length scales: every hash's blocks are a few positions long, so the comparator's
    # 64 passes per query tile stay near the diagonal
    plan = PlshForward(B, H, H_kv, n, d, s, causal, [0.7 + 0.3 * h for h in range(H)], 11, torch.bfloat16, "cuda:0")
    plan.prepare()
    O_ref, R_ref = (t.clone() for t in plan.attend_varlen(q, k, v))
    O = torch.full_like(O_ref, float("nan"))
    R = torch.full_like(R_ref, float("nan"))
    _static_call(plan, q, k, v, B, H, H_kv, n, d, s, causal, O, R)
    torch.cuda.synchronize()
    assert torch.equal(O, O_ref)
    assert torch.equal(R, R_ref)
    assert plan.device_errors() == []
    # one more query tile: refused on the host, nothing launched (stand-in buffers are never touched)
    n2 = n + 1
    assert plsh_varlen_scratch_bytes(H, s, n2) > PLSH_VARLEN_STATIC_SCRATCH_BYTES
    t = torch.zeros((256,), dtype=torch.bfloat16, device="cuda:0")
    i = torch.zeros((256,), dtype=torch.int32, device="cuda:0")
    f = torch.zeros((256,), dtype=torch.float32, device="cuda:0")
    with pytest.raises(PlshError) as ei:
        plsh_attention_varlen_fwd_static(t, t, t, PLSH_BF16, B, H, H_kv, n2, d, None, s, None, i, i, 1, t, f, i)
    assert ei.value.code == 3
    torch.cuda.synchronize()
