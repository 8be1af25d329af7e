"""CUDA path against the CPU oracle, through the C-ABI (needs a B200).

Bin ids, boundary masks, b_max and tile windows must be bit-exact; O and
row_sum must be within the stated tolerance (max|dO| <= 1e-5 for fp32
inputs, <= 2e-2 * max|V| for bf16 inputs). Every case runs on seeded
inputs; outputs are poisoned with NaN before the run so unwritten rows fail.
"""
import math

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


# ---------------------------------------------------------------- K1 + K2

@pytest.mark.parametrize("name", list(W))
def test_bins_masks_windows_bit_exact(name):
    w = W[name]
    n = w.n
    # the preparation steps (table, K1, K2) at full n
    from alibi_positional_lsh_b200 import PlshForward
    plan = PlshForward(1, w.H, w.H_kv, n, w.d, w.s, w.causal, w.sigmas(), w.seed, w.torch_dtype, "cuda:0")
    plan.prepare()
    assert plan.device_errors() == []
    gpu = dict(ids=plan.ids.cpu().numpy().astype(np.int64), bmax=plan.bmax.cpu().numpy(),
               spans=plan.spans.cpu().numpy().astype(np.int64),
               bmask=plan.bmask.cpu().numpy().view(np.uint32 if w.s <= 32 else np.uint64))
    table = oracle.draw_table(w.seed, w.sigmas(), w.s)
    assert plan.table_host.numpy().tobytes() == table.tobytes()
    PH.oracle_window_checks(table, n, w.causal, gpu, tiles_per_head=None if n <= 8192 else 6)


@pytest.mark.parametrize("s", workloads.MISTRAL_S_SWEEP)
def test_bins_masks_windows_s_sweep(s):
    w = W["mistral7b_n16k"].with_(s=s)
    from alibi_positional_lsh_b200 import PlshForward
    plan = PlshForward(1, w.H, w.H_kv, w.n, w.d, s, True, w.sigmas(), w.seed, w.torch_dtype, "cuda:0")
    plan.prepare()
    assert plan.device_errors() == []
    gpu = dict(ids=plan.ids.cpu().numpy().astype(np.int64), bmax=plan.bmax.cpu().numpy(),
               spans=plan.spans.cpu().numpy().astype(np.int64),
               bmask=plan.bmask.cpu().numpy().view(np.uint32 if s <= 32 else np.uint64))
    PH.oracle_window_checks(oracle.draw_table(w.seed, w.sigmas(), s), w.n, True, gpu, tiles_per_head=4)


def test_bins_extreme_tables():
    """Hand-made tables: pitch below 1 (singleton bins), pitch above n (one bin), a tie at an integer."""
    n = 1000
    table = np.array([[[0.5, 0.25], [0.3, 0.0], [2.0 * n, 0.0], [3.0, 2.0], [1.0, 0.0], [128.0, 0.0],
                       [7.25, 7.0], [1e-3, 0.0]]])
    H, s = 1, table.shape[1]
    q, k, v = _inputs(1, 1, 1, n, 128, torch.bfloat16, 5)
    gpu = PH.run_gpu(1, H, 1, n, 128, s, False, [4.0], 0, q, k, v, table=table)
    assert gpu["errors"] == []
    PH.oracle_window_checks(table, n, False, gpu)


def test_bin_id_overflow_is_reported():
    n = 4096
    table = np.array([[[1e-7, 0.0]]])   # (n-1)/delta overflows int32
    q, k, v = _inputs(1, 1, 1, n, 128, torch.bfloat16, 6)
    from alibi_positional_lsh_b200 import PlshForward
    plan = PlshForward(1, 1, 1, n, 128, 1, False, [1.0], 0, torch.bfloat16, "cuda:0")
    plan.prepare(table=table)
    assert "RANGE" in plan.device_errors()


# ---------------------------------------------------------------- K3: full oracle on small cases

def test_single_head_fp32_workload_full():
    w = W["single_head_n1024"]
    q, k, v = workloads.make_qkv(w)
    gpu = PH.run_gpu(w.B, w.H, w.H_kv, w.n, w.d, w.s, w.causal, w.sigmas(), w.seed, q, k, v)
    assert gpu["errors"] == []
    O, R = PH.oracle_rows(q, k, v, gpu["table"], w.causal, None)
    to, tr = PH.tolerance(torch.float32, v)
    PH.assert_close(gpu["O"], gpu["row_sum"], O, R, to, tr, "fp32 n=1024")


SMALL = [
    # B, H, H_kv, n, d, dtype, causal, s, sigma_kind
    (1, 2, 1, 1000, 128, torch.bfloat16, True, 20, "mixed"),
    (1, 2, 2, 1000, 128, torch.bfloat16, False, 10, "mixed"),
    (2, 4, 2, 700, 128, torch.bfloat16, True, 33, "mixed"),
    (1, 2, 1, 1300, 64, torch.bfloat16, True, 7, "mixed"),
    (1, 2, 2, 900, 64, torch.bfloat16, False, 40, "mixed"),
    (1, 2, 1, 777, 128, torch.float32, True, 16, "mixed"),
    (1, 2, 2, 640, 64, torch.float32, False, 64, "mixed"),
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
def test_attention_small_full_oracle(B, H, H_kv, n, d, dtype, causal, s, kind):
    q, k, v = _inputs(B, H, H_kv, n, d, dtype, 100 + n + s)
    sig = _sigmas(kind, H)
    gpu = PH.run_gpu(B, H, H_kv, n, d, s, causal, sig, 7 + s, q, k, v)
    assert gpu["errors"] == []
    PH.oracle_window_checks(gpu["table"], n, causal, gpu)
    O, R = PH.oracle_rows(q, k, v, gpu["table"], causal, None)
    to, tr = PH.tolerance(dtype, v)
    PH.assert_close(gpu["O"], gpu["row_sum"], O, R, to, tr, "small")


_UNDERFLOW = pytest.mark.xfail(
    strict=False,
    reason="known limitation of the fused kernel: its reference maximum is taken over every key of "
           "a live chunk pair, weighted or not, so a row whose weighted scores all lie more than "
           "about 87 (natural log) below a zero-weight score in those pairs underflows; with Q x 32 "
           "row 0 of a causal head (one weighted key beside 31 masked ones) does")


@pytest.mark.parametrize("scale,causal", [(8.0, True), pytest.param(32.0, True, marks=_UNDERFLOW),
                                          pytest.param(32.0, False, marks=_UNDERFLOW)])
def test_attention_large_scores_full_oracle(scale, causal):
    """Q scaled by a power of two (exact in bf16): scores spread over tens of log2 units, so a
    row's maximum rises from tile to tile by more than the kernel's rescale margin. The output
    must still match the float64 oracle, which works on the same scaled inputs."""
    B, H, H_kv, n, d, s = 1, 2, 1, 1000, 128, 20
    q, k, v = _inputs(B, H, H_kv, n, d, torch.bfloat16, 4242 + int(scale))
    q = (q.float() * scale).to(torch.bfloat16)
    sig = _sigmas("mixed", H)
    gpu = PH.run_gpu(B, H, H_kv, n, d, s, causal, sig, 11, q, k, v)
    assert gpu["errors"] == []
    O, R = PH.oracle_rows(q, k, v, gpu["table"], causal, None)
    to, tr = PH.tolerance(torch.bfloat16, v)
    PH.assert_close(gpu["O"], gpu["row_sum"], O, R, to, tr, f"scores x{scale}")


def test_singleton_bins_give_v_and_one_bin_gives_softmax():
    n, d = 500, 128
    q, k, v = _inputs(1, 2, 2, n, d, torch.bfloat16, 9)
    table = np.array([[[0.5, 0.25]] * 3, [[2.0 * n, 0.0]] * 3])
    for causal in (False, True):
        gpu = PH.run_gpu(1, 2, 2, n, d, 3, causal, [1.0, 1.0], 0, q, k, v, table=table)
        vf = PH.f64(v)
        assert np.abs(gpu["O"][0, 0] - vf[0, 0]).max() <= 2e-2 * np.abs(vf).max()
        sd = torch.nn.functional.scaled_dot_product_attention(
            q[:, 1:2].double(), k[:, 1:2].double(), v[:, 1:2].double(), is_causal=causal)[0, 0].numpy()
        assert np.abs(gpu["O"][0, 1] - sd).max() <= 2e-2 * np.abs(vf).max()


# ---------------------------------------------------------------- K3: full-size workloads, sampled rows

FULL_ROWS = {"mha8_n8192": 64, "qwen3_0p6b_n32k": 48, "mistral7b_n16k": 32, "long_n128k": 24}


@pytest.mark.parametrize("name", list(FULL_ROWS))
def test_attention_full_size_sampled_rows(name):
    w = W[name]
    q, k, v = workloads.make_qkv(w)
    gpu = PH.run_gpu(w.B, w.H, w.H_kv, w.n, w.d, w.s, w.causal, w.sigmas(), w.seed, q, k, v)
    assert gpu["errors"] == []
    rows = workloads.sample_rows(w.n, FULL_ROWS[name], w.seed)
    # also rows at tile edges
    rows = sorted(set(rows) | {127, 128, w.n - 128, w.n - 129})
    O, R = PH.oracle_rows(q, k, v, gpu["table"], w.causal, rows)
    to, tr = PH.tolerance(w.torch_dtype, v)
    PH.assert_close(gpu["O"][:, :, rows], gpu["row_sum"][:, :, rows], O, R, to, tr, name)
    assert np.all(np.isfinite(gpu["O"])) and np.all(np.isfinite(gpu["row_sum"]))


def test_mistral_s_sweep_sampled_rows():
    base = W["mistral7b_n16k"]
    q, k, v = workloads.make_qkv(base)
    rows = workloads.sample_rows(base.n, 16, 3)
    for s in workloads.MISTRAL_S_SWEEP:
        gpu = PH.run_gpu(base.B, base.H, base.H_kv, base.n, base.d, s, True, base.sigmas(), base.seed, q, k, v)
        assert gpu["errors"] == []
        O, R = PH.oracle_rows(q, k, v, gpu["table"], True, rows)
        to, tr = PH.tolerance(base.torch_dtype, v)
        PH.assert_close(gpu["O"][:, :, rows], gpu["row_sum"][:, :, rows], O, R, to, tr, f"s={s}")


# ---------------------------------------------------------------- the fixed-blocks baseline

@pytest.mark.parametrize("causal", [False, True])
def test_fixed_blocks_baseline(causal):
    """A deterministic table (s = 1, pitch = block, offset 0) through the same kernels: each row
    attends inside its own block of `block` positions (the fixed-blocks comparison)."""
    from alibi_positional_lsh_b200 import fixed_blocks_table
    B, H, H_kv, n, d, block = 1, 2, 1, 1000, 128, 96
    q, k, v = _inputs(B, H, H_kv, n, d, torch.bfloat16, 77)
    table = fixed_blocks_table(H, block)
    gpu = PH.run_gpu(B, H, H_kv, n, d, 1, causal, [float(block)] * H, 0, q, k, v, table=table)
    assert gpu["errors"] == []
    ids = oracle.bin_ids(table, n)
    assert np.array_equal(ids[0, 0], np.arange(n) // block)
    PH.oracle_window_checks(table, n, causal, gpu)
    O, R = PH.oracle_rows(q, k, v, table, causal, None)
    to, tr = PH.tolerance(torch.bfloat16, v)
    PH.assert_close(gpu["O"], gpu["row_sum"], O, R, to, tr, "fixed blocks")
    # per-block softmax, written out directly
    Qf, Kf, Vf = PH.f64(q)[0, 0], PH.f64(k)[0, 0], PH.f64(v)[0, 0]
    for i in (0, block - 1, block, n - 1):
        lo = (i // block) * block
        hi = i if causal else min(n, lo + block) - 1
        sc = Qf[i] @ Kf[lo:hi + 1].T / math.sqrt(d)
        w = np.exp(sc - sc.max())
        assert np.abs(gpu["O"][0, 0, i] - (w @ Vf[lo:hi + 1]) / w.sum()).max() <= to
