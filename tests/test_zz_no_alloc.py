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
