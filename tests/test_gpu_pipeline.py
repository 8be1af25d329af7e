"""HostPipeline against PlshForward.run_host (needs a B200).

The pipeline runs the same kernels on the same table as run_host, only with
the copies of neighbouring steps overlapped on their own streams, so every
step's O and row_sum must equal run_host's for the same batch bit for bit,
whatever the overlap.
"""
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("causal", [True, False])
def test_pipeline_matches_run_host_per_batch(causal):
    from alibi_positional_lsh_b200 import HostPipeline, PlshForward
    B, H, H_kv, n, d, s = 1, 4, 2, 1500, 128, 20
    sigma = [2.0 ** (1 + 8.0 * h / (H - 1)) for h in range(H)]
    plan = PlshForward(B, H, H_kv, n, d, s, causal, sigma, 5, torch.bfloat16, "cuda:0")
    batches = []
    for t in range(5):
        w = workloads.Workload("case", B, H, H_kv, n, d, "bf16", causal, s, 70 + t)
        batches.append([x.pin_memory() for x in workloads.make_qkv(w)])
    # run_host, one batch at a time
    want = []
    qd, kd, vd = (torch.empty(x.shape, dtype=x.dtype, device="cuda:0") for x in batches[0])
    for qh, kh, vh in batches:
        oh = torch.empty(plan.O.shape, dtype=plan.O.dtype).pin_memory()
        rh = torch.empty(plan.row_sum.shape, dtype=torch.float32).pin_memory()
        plan.run_host(qh, kh, vh, qd, kd, vd, oh, rh)
        torch.cuda.synchronize()
        want.append((oh.clone(), rh.clone()))
    # the pipeline, all batches enqueued back to back
    pipe = HostPipeline(plan)
    outs = [(torch.full(plan.O.shape, float("nan"), dtype=plan.O.dtype).pin_memory(),
             torch.full(plan.row_sum.shape, float("nan"), dtype=torch.float32).pin_memory()) for _ in batches]
    for (qh, kh, vh), (oh, rh) in zip(batches, outs):
        pipe.step(qh, kh, vh, oh, rh)
    pipe.wait()
    torch.cuda.synchronize()
    assert plan.device_errors() == []
    for t, ((o, r), (wo, wr)) in enumerate(zip(outs, want)):
        assert torch.equal(o, wo), f"O differs at step {t}"
        assert torch.equal(r, wr), f"row_sum differs at step {t}"
