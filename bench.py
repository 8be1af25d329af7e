"""Throughput of Positional-LSH approximate ALiBi attention on B200.

One step = the whole forward path on one batch of synthetic inputs already in
HBM: table draw (host) + its copy, bin ids (K1), windows and boundary masks
(K2), fused attention (K3). Metric: query tokens per second (B * n per step,
summed over ranks), plus the roofline fraction of the attention kernel.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   (the CPU oracle on a bounded sample)

Multi-GPU (torchrun, one rank per GPU): every rank runs its own independent
problem of the same shape (the path has no exchange step), so per-GPU work is
fixed and scaling is weak; the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
TILE = 128
ATTN_KERNEL_SRC = [os.path.join(ROOT, "alibi_positional_lsh_b200", "csrc", f) for f in
                   ("plsh_attn_tc.cu", "plsh_sm100.cuh", "plsh_tile_common.cuh", "plsh_internal.h")]
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "attn_tc_qwen3_0p6b_n32k.md")


# ---------------------------------------------------------------- helpers

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in PEAKS_FALLBACK}, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def kernel_source_hash() -> str:
    """Hash of the attention kernel's source and the headers it is built from."""
    h = hashlib.sha256()
    for path in ATTN_KERNEL_SRC:
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes per launch of the attention kernel from the committed ncu summary,
    or None when absent or taken on a different kernel source."""
    if not os.path.exists(PROFILE_SUMMARY):
        return None
    text = open(PROFILE_SUMMARY).read()
    mh = re.search(r"kernel_source_sha256_16:\s*([0-9a-f]+)", text)
    mt = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not mh or not mt or mh.group(1) != kernel_source_hash():
        return None
    return float(mt.group(1))


class ClockSampler:
    """SM clock and clock-event reasons sampled through NVML every ~2 ms while the timed region runs."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, local_index: int, period_s: float = 0.002):
        self.local_index = local_index
        self.period = period_s
        self.samples = []
        self.error = None
        self._stop = None
        self._thread = None

    def _handle(self):
        import pynvml
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.local_index)
        bus = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
        return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)

    def __enter__(self):
        import threading
        try:
            self.nvml, self.h = self._handle()
            self.max_mhz = self.nvml.nvmlDeviceGetMaxClockInfo(self.h, self.nvml.NVML_CLOCK_SM)
        except Exception as e:  # pragma: no cover - no NVML on this host
            self.error = f"nvml unavailable: {e}"
            return self
        self._stop = threading.Event()

        def loop():
            while not self._stop.is_set():
                try:
                    mhz = self.nvml.nvmlDeviceGetClockInfo(self.h, self.nvml.NVML_CLOCK_SM)
                    rs = self.nvml.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                    self.samples.append((mhz, rs))
                except Exception as e:  # pragma: no cover
                    self.error = str(e)
                    return
                time.sleep(self.period)

        # the timed loop's host work (the table draw, the launches) holds the GIL; a short switch
        # interval lets the sampling thread in every few hundred microseconds
        self._switch = sys.getswitchinterval()
        sys.setswitchinterval(0.0002)
        self._thread = threading.Thread(target=loop, daemon=True)
        self._thread.start()
        time.sleep(0.02)
        return self

    def __exit__(self, *a):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=2)
            sys.setswitchinterval(self._switch)

    def summary(self):
        if self.error or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.error or "no samples"], "samples": 0,
                    "source": "nvml"}
        mhz = [m for m, _ in self.samples]
        reasons = sorted({name for _, rs in self.samples for name, bit in self.REASONS.items() if rs & bit})
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(self.samples), "source": "nvml, every 2 ms during the timed region"}


def alibi_spans(sigma, eps: float, n: int, causal: bool) -> np.ndarray:
    """[H][T][2] key windows of exact banded ALiBi (the kernel's own rule)."""
    T = (n + TILE - 1) // TILE
    out = np.empty((len(sigma), T, 2), dtype=np.int64)
    for h, sg in enumerate(sigma):
        reach = min(n, int(np.ceil(sg * np.log(1.0 / eps))))
        for t in range(T):
            i0, last = t * TILE, min(n, (t + 1) * TILE) - 1
            out[h, t] = (max(0, i0 - reach), last if causal else min(n - 1, last + reach))
    return out


def issued_tiles(spans: np.ndarray, causal: bool) -> int:
    """Key tiles of 128 the fused kernel's window covers, summed over heads and query tiles:
    ceil((hi - lo + 1) / 128) per query tile (the span rounded to the MMA N granularity)."""
    lo = spans[..., 0].astype(np.int64)
    hi = spans[..., 1].astype(np.int64)
    return int(np.sum((hi - lo + 1 + TILE - 1) // TILE))


def kernel_tiles(spans: np.ndarray, causal: bool) -> int:
    """Key tiles the fused kernel actually visits (128-aligned around the diagonal)."""
    T = spans.shape[1]
    i0 = (np.arange(T) * TILE)[None, :]
    lo = spans[..., 0].astype(np.int64)
    hi = spans[..., 1].astype(np.int64)
    below = (i0 - lo + TILE - 1) // TILE
    above = 0 if causal else (hi - i0) // TILE
    return int(np.sum(1 + below + above))


# ---------------------------------------------------------------- distributed plumbing

def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    return rank, world, local


def dist_max(x: float, world: int) -> float:
    """Max over ranks (a CUDA tensor under NCCL, a CPU tensor under gloo)."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def rank_workload(w: workloads.Workload, rank: int) -> workloads.Workload:
    """Each rank solves an independent problem of the same shape (its own seed)."""
    return w.with_(seed=w.seed + 1000 * rank)


def job_value(tokens_per_rank: int, world: int, ms_step_max: float) -> float:
    """Whole-job query-tokens/s: the tokens every rank processed over the slowest rank's step time."""
    return tokens_per_rank * world / (ms_step_max * 1e-3)


L2_BYTES = 126 * 2 ** 20          # B200 L2
FLUSH_BYTES = 256 * 2 ** 20       # written between timed steps when the inputs fit in L2


def qkv_bytes(w: workloads.Workload) -> int:
    return (w.B * w.H * w.n * w.d + 2 * w.B * w.H_kv * w.n * w.d) * (2 if w.dtype == "bf16" else 4)


def needs_l2_flush(w: workloads.Workload) -> bool:
    """Inputs that fit in L2 would stay cached from one timed step to the next: flush between steps."""
    return qkv_bytes(w) <= L2_BYTES


def config_of(w: workloads.Workload, world: int) -> dict:
    qkv = qkv_bytes(w)
    l2 = (f"flushed: Q+K+V = {qkv / 1e6:.0f} MB fits in the 126 MB L2, so a {FLUSH_BYTES >> 20} MB buffer is "
          "written between timed steps, outside the per-step events" if needs_l2_flush(w) else
          f"no flush: Q+K+V = {qkv / 1e6:.0f} MB per step, larger than the 126 MB L2")
    return {"workload": w.name, "B": w.B, "H": w.H, "H_kv": w.H_kv, "n": w.n, "d": w.d, "s": w.s,
            "causal": w.causal, "global_batch": w.B * world, "seq_len": w.n,
            "parallelism": f"independent problem per GPU x{world}",
            "l2": l2}


def barrier(world: int):
    if world > 1:
        torch.distributed.barrier()


# ---------------------------------------------------------------- CPU oracle (baseline and reference arm)

class OracleSampler:
    """The CPU oracle on query rows of batch element 0, all heads, of one workload.

    Inputs, table and bin ids are prepared once; run(budget_s) then computes
    rows (8 at a time, every head) until the budget is spent and returns the
    equivalent query-tokens/s = (row, head) units / time / H.
    """

    def __init__(self, w: workloads.Workload):
        import oracle
        self.oracle = oracle
        self.w = w
        g = torch.Generator().manual_seed(w.seed)
        self.q = torch.randn(1, w.H, w.n, w.d, generator=g).to(w.torch_dtype).double().numpy()
        self.k = torch.randn(1, w.H_kv, w.n, w.d, generator=g).to(w.torch_dtype).double().numpy()
        self.v = torch.randn(1, w.H_kv, w.n, w.d, generator=g).to(w.torch_dtype).double().numpy()
        self.table = oracle.draw_table(w.seed, w.sigmas(), w.s)
        self.ids = oracle.bin_ids(self.table, w.n)
        self.rows = workloads.sample_rows(w.n, min(w.n, 4096), w.seed)
        self.next = 0
        self.cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)

    def run(self, budget_s: float):
        from threadpoolctl import threadpool_limits
        w = self.w
        group = w.H // w.H_kv
        units = 0
        with threadpool_limits(limits=self.cores):
            t0 = time.perf_counter()
            while True:
                rows = self.rows[self.next:self.next + 8]
                self.next = (self.next + 8) % len(self.rows)
                for h in range(w.H):
                    self.oracle.approx_attention(self.q[0, h], self.k[0, h // group], self.v[0, h // group],
                                                 self.ids[h], w.causal, rows)
                    units += len(rows)
                if time.perf_counter() - t0 >= budget_s:
                    break
            dt = time.perf_counter() - t0
        rate = units / dt / w.H
        desc = (f"{units // w.H} query rows x all {w.H} heads of batch element 0 of {w.name} "
                f"({units} row-head units in {dt:.1f} s, float64 numpy on {self.cores} cores); "
                f"query-tokens/s = units / time / H")
        return rate, desc


# ---------------------------------------------------------------- our arm

def decode_keys(bmask: np.ndarray, s: int, i: int, causal: bool) -> int:
    """Keys with a nonzero count c_ij for the query at position i, summed over heads: the rows of K
    and V plsh_decode_fwd reads. c_ij = s - popcount(OR of the masks over (min, max])."""
    H, n = bmask.shape
    full = (1 << s) - 1
    total = 0
    for h in range(H):
        bm = bmask[h].astype(np.uint64)
        below = np.bitwise_or.accumulate(bm[i:0:-1]) if i > 0 else np.zeros(0, np.uint64)   # keys i-1 .. 0
        total += 1 + int(np.count_nonzero(below != full))
        if not causal and i + 1 < n:
            above = np.bitwise_or.accumulate(bm[i + 1:])                                        # keys i+1 .. n-1
            total += int(np.count_nonzero(above != full))
    return total


BWD_TILE = 64
FP32_LANES_PER_SM = 128   # fp32 FMA lanes per SM (4 sub-partitions x 32)


def bwd_chunk_pairs(ids: np.ndarray, causal: bool, group: int) -> tuple:
    """(query-tile x key-chunk pairs of bwd_dq_kernel, key-tile x query-chunk pairs of bwd_dkdv_kernel) for one
    batch element: per 64-position tile the range of positions sharing a block with it in some hash (first
    position of the first row's block to the last of the last row's block, widest over the hashes), walked in
    chunks of 64. ids: [H][s][n]."""
    H, s, n = ids.shape
    T = (n + BWD_TILE - 1) // BWD_TILE
    a = np.arange(T) * BWD_TILE
    b = np.minimum(n - 1, a + BWD_TILE - 1)
    dq = dkdv = 0
    for h in range(H):
        lo = np.full(T, n, np.int64)
        hi = np.full(T, -1, np.int64)
        for k in range(s):
            row = ids[h, k]
            lo = np.minimum(lo, np.searchsorted(row, row[a], "left"))
            hi = np.maximum(hi, np.searchsorted(row, row[b], "right") - 1)
        hq = np.minimum(hi, b) if causal else hi          # dQ: keys j <= i
        lk = np.maximum(lo, a) if causal else lo          # dK, dV: rows i >= j
        dq += int(((hq - lo) // BWD_TILE + 1).sum())
        dkdv += int(((hi - lk) // BWD_TILE + 1).sum())
    return dq, dkdv


def bwd_tc_tiles(spans: np.ndarray, key_spans: np.ndarray, causal: bool) -> tuple:
    """(key tiles the tensor-core dQ kernel visits, query tiles the dK/dV kernel walks) for one batch
    element. spans: the forward's windows [H][T][2]; key_spans: the non-causal ones (the query rows
    that reach each key tile). The dK/dV kernel walks, per head and key tile, the key tile's own
    tile, the tiles before it (non-causal only) and the tiles after it up to the window's end."""
    dq = kernel_tiles(spans, causal)
    H, T, _ = key_spans.shape
    j0 = (np.arange(T) * TILE)[None, :]
    lo = np.minimum(key_spans[..., 0].astype(np.int64), j0)
    hi = key_spans[..., 1].astype(np.int64)
    below = 0 if causal else (j0 - lo + TILE - 1) // TILE
    dkdv = int(np.sum(1 + below + (hi - j0) // TILE))
    return dq, dkdv


def bwd_timing(plan, q, k, v, stream, w, sm_count: int, sm_max_mhz: float, bf16_peak: float):
    """plsh_attention_bwd on the step's inputs with a seeded dO: device time per call (L2 flushed before
    each) of the tcgen05 kernels (bf16, d = 128) and of the fp32 CUDA-core kernels. The tensor-core roofline counts 3 MMAs
    of 128 x 128 x 128 per dQ tile (S, dP, dQ += dS K) and 4 per dK/dV tile (S^T, dP^T, dV, dK)
    against the dense bf16 peak; the CUDA-core figure counts its 64 x 64 pairs (S, dP and dQ; S, dP,
    dV and dK; 2d each) against the fp32 FMA peak derived from the SM count and maximum clock."""
    g = torch.Generator(device=q.device).manual_seed(w.seed + 99)
    dO = torch.randn(q.shape, generator=g, device=q.device, dtype=torch.float32).to(q.dtype)
    plan.attend(q, k, v, stream)             # O and row_sum of these inputs
    tc_ok = w.dtype == "bf16" and w.d == 128

    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=q.device)

    def timed(path):
        for _ in range(2):
            plan.backward(q, k, v, dO, stream, path=path)
        ts = []
        for _ in range(5):
            flush.fill_(2)                   # L2 cold at the start of every timed call
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            plan.backward(q, k, v, dO, stream, path=path)
            b.record(stream)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        errs = plan.device_errors()
        if errs:
            raise RuntimeError(f"device errors in backward ({path}): {errs}")
        return float(np.median(ts))

    ms_simt = timed("simt")
    ids = plan.ids.cpu().numpy()
    dq_pairs, dkdv_pairs = bwd_chunk_pairs(ids, w.causal, w.H // w.H_kv)
    per_pair = 2.0 * w.d * BWD_TILE * BWD_TILE
    flops = (3 * dq_pairs + 4 * dkdv_pairs) * per_pair * w.B
    peak = sm_count * FP32_LANES_PER_SM * 2 * sm_max_mhz * 1e6 / 1e12
    achieved = flops / (ms_simt * 1e-3) / 1e12
    simt = {"path": "plsh_attention_bwd: fp32 CUDA-core arithmetic",
            "kernels": ["bwd_delta_kernel", "bwd_dkdv_kernel", "bwd_dq_kernel"], "ms_per_call": ms_simt,
            "issued_fp32_flops": flops, "achieved_TFLOPs": achieved,
            "roofline": {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak,
                         "peak_source": f"derived: {sm_count} SMs x {FP32_LANES_PER_SM} fp32 lanes x 2 x "
                                        f"{sm_max_mhz:.0f} MHz"}}
    if not tc_ok:
        return dict(simt, path="backward (" + simt["path"] + ")")
    ms = timed("tc")
    dq_tiles, dkdv_tiles = bwd_tc_tiles(plan.spans.cpu().numpy(), plan.key_spans().cpu().numpy(), w.causal)
    mma = 2.0 * TILE * TILE * w.d
    tflops = (3 * dq_tiles + 4 * dkdv_tiles) * mma * w.B
    ach = tflops / (ms * 1e-3) / 1e12
    return {"path": "backward (plsh_attention_bwd_tc): dQ, dK, dV of T~ on the tcgen05 tensor cores",
            "kernels": ["bwd_delta_kernel", "bwd_dq_tc_kernel", "bwd_dkdv_tc_kernel"], "ms_per_call": ms,
            "dq_tiles_per_batch": dq_tiles, "dkdv_tiles_per_batch": dkdv_tiles, "issued_tensor_flops": tflops,
            "roofline": {"bound": "tensor", "achieved": ach, "peak": bf16_peak, "unit": "TFLOP/s",
                         "frac": ach / bf16_peak},
            "cuda_core_path": simt, "speedup_over_cuda_core_path": ms_simt / ms}


def graph_call_us(call, stream, reps: int) -> dict:
    """Device time of one call, from CUDA graphs replayed back to back (one call timed alone on an
    idle GPU would include the host's launch latency). `warm_us`: the call's graph replayed `reps`
    times, so what one call reads may still sit in L2 for the next. `cold_us`: a graph of an L2 flush
    (a write of FLUSH_BYTES) followed by the call, minus a graph of the flush alone. Medians of 5."""
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=torch.device("cuda", torch.cuda.current_device()))
    graphs = {}
    for name in ("warm", "flush_call", "flush"):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            if name != "warm":
                flush.fill_(1)
            if name != "flush":
                call()
        graphs[name] = g
    out = {}
    for name, g in graphs.items():
        g.replay()
        ts = []
        for _ in range(5):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(reps):
                g.replay()
            b.record(stream)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b) * 1e3 / reps)
        out[name] = float(np.median(ts))
    del graphs, flush
    return {"warm_us": out["warm"], "cold_us": out["flush_call"] - out["flush"], "flush_us": out["flush"]}


def decode_timing(plan, q, k, v, stream, w):
    """plsh_decode_fwd on the newest position (one query row per (b, h) at i = n-1) against the whole
    cache: device time per call and the K/V bytes it must read (the weighted keys' rows)."""
    i = w.n - 1
    pos = torch.tensor([i], dtype=torch.int32, device=q.device)
    q1 = q[:, :, i:i + 1].contiguous()
    for _ in range(3):
        plan.decode(q1, pos, k, v, stream)
    torch.cuda.synchronize()
    t = graph_call_us(lambda: plan.decode(q1, pos, k, v), stream, 50)
    errs = plan.device_errors()
    if errs:
        raise RuntimeError(f"device errors in decode: {errs}")
    bm = plan.bmask.cpu().numpy()
    bm = bm.view(np.uint32) if w.s <= 32 else bm.view(np.uint64)
    keys = decode_keys(bm, w.s, i, w.causal) * w.B
    elt = 2 if w.dtype == "bf16" else 4
    kv_bytes = keys * 2 * w.d * elt
    us = t["cold_us"]
    return {"path": "decode (plsh_decode_fwd), one query row per (b, h) at position n-1, whole cache",
            "kernels": ["decode_range_kernel", "decode_unit_kernel"], "us_per_call": us,
            "timing": "L2 flushed before each call: CUDA graph of (flush, call) minus graph of the flush, "
                      "50 replays, median of 5",
            "us_per_call_l2_warm": t["warm_us"], "weighted_keys": keys, "kv_bytes": kv_bytes,
            "achieved_GBps": kv_bytes / (us * 1e-6) / 1e9}


def decode_batched_timing(w, stream, peak_gbs: float, batch: int = 64):
    """plsh_decode_fwd for a batch of `batch` sequences of the workload's shape (one query row per
    (b, h) at the newest position n-1, B*H rows, each against its own cache): device time per call
    and the K/V rows of the weighted keys, which no two rows share, against the HBM peak."""
    from alibi_positional_lsh_b200 import PlshForward
    wb = w.with_(B=batch)
    dev = torch.device("cuda", torch.cuda.current_device())
    g = torch.Generator(device=dev).manual_seed(w.seed + 7)
    dt = wb.torch_dtype
    k = torch.randn((batch, w.H_kv, w.n, w.d), generator=g, device=dev, dtype=torch.float32).to(dt)
    v = torch.randn((batch, w.H_kv, w.n, w.d), generator=g, device=dev, dtype=torch.float32).to(dt)
    q1 = torch.randn((batch, w.H, 1, w.d), generator=g, device=dev, dtype=torch.float32).to(dt)
    plan = PlshForward(batch, w.H, w.H_kv, w.n, w.d, w.s, w.causal, w.sigmas(), w.seed, dt, str(dev))
    plan.prepare(stream)
    i = w.n - 1
    pos = torch.tensor([i], dtype=torch.int32, device=dev)
    for _ in range(3):
        plan.decode(q1, pos, k, v, stream)
    torch.cuda.synchronize()
    t = graph_call_us(lambda: plan.decode(q1, pos, k, v), stream, 20)
    errs = plan.device_errors()
    if errs:
        raise RuntimeError(f"device errors in batched decode: {errs}")
    bm = plan.bmask.cpu().numpy()
    bm = bm.view(np.uint32) if w.s <= 32 else bm.view(np.uint64)
    keys = decode_keys(bm, w.s, i, w.causal) * batch
    elt = 2 if w.dtype == "bf16" else 4
    kv_bytes = keys * 2 * w.d * elt
    us = t["cold_us"]
    gbs = kv_bytes / (us * 1e-6) / 1e9
    del k, v, q1, plan
    torch.cuda.empty_cache()
    return {"path": f"batched decode (plsh_decode_fwd), {batch} sequences x {w.H} heads = {batch * w.H} rows at "
                    "position n-1, each against its own cache", "rows": batch * w.H, "us_per_call": us,
            "timing": "L2 flushed before each call: CUDA graph of (flush, call) minus graph of the flush, "
                      "20 replays, median of 5",
            "us_per_call_l2_warm": t["warm_us"],
            "weighted_keys": keys, "kv_bytes": kv_bytes, "achieved_GBps": gbs, "hbm_peak_GBps": peak_gbs,
            "frac_of_hbm": gbs / peak_gbs}


def run_ours(args, rank, world, local):
    from alibi_positional_lsh_b200 import PlshForward
    import alibi_positional_lsh_b200 as plsh_mod  # noqa: F401

    w = workloads.WORKLOADS[args.workload]
    if args.batch:
        w = w.with_(B=args.batch)
    if args.s:
        w = w.with_(s=args.s)
    dev = f"cuda:{local}"
    torch.cuda.set_device(local)
    wr = rank_workload(w, rank)                      # independent problem per rank
    q, k, v = workloads.make_qkv_device(wr, dev)
    plan = PlshForward(w.B, w.H, w.H_kv, w.n, w.d, w.s, w.causal, w.sigmas(), wr.seed, w.torch_dtype, dev)
    stream = torch.cuda.current_stream()

    varlen = args.path == "varlen"
    alibi = args.path == "alibi"

    def attend():
        if varlen:
            plan.attend_varlen(q, k, v, stream)
        elif alibi:
            plan.attend_alibi(q, k, v, args.eps, stream)
        else:
            plan.attend(q, k, v, stream)

    def step(ev=None):
        if not alibi:       # exact banded ALiBi needs no table, ids or masks
            plan.prepare(stream)
        if ev is not None:
            ev[0].record(stream)
        attend()
        if ev is not None:
            ev[1].record(stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    errs = plan.device_errors()
    if errs:
        raise RuntimeError(f"device errors during warm-up: {errs}")
    if varlen:   # per-hash windows [H][s][T][2]: every hash's window is visited
        T = (w.n + TILE - 1) // TILE
        spans = plan.scratch.cpu().numpy()[: w.H * w.s * T * 2].reshape(w.H * w.s, T, 2)
    elif alibi:  # bands |i - j| <= ceil(sigma_h ln(1/eps)) around each query tile
        spans = alibi_spans(w.sigmas(), args.eps, w.n, w.causal)
    else:
        spans = plan.spans.cpu().numpy()
    tiles_min = issued_tiles(spans, w.causal)
    tiles_run = kernel_tiles(spans, w.causal)

    # timed region: K steps, device-timed, inputs already resident; inputs that fit in L2 are
    # evicted between steps by a write larger than L2, which each step's own events leave out
    K = args.steps
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev) if needs_l2_flush(w) else None
    ev_k = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    ev_s = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize()
        start.record(stream)
        for i in range(K):
            if flush is not None:
                flush.fill_(i & 255)
            ev_s[i][0].record(stream)
            step(ev_k[i])
            ev_s[i][1].record(stream)
        end.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    ms_total = (sum(a.elapsed_time(b) for a, b in ev_s) if flush is not None else start.elapsed_time(end))
    attn_ms = [a.elapsed_time(b) for a, b in ev_k]
    ms_total = dist_max(ms_total, world)
    ms_step = ms_total / K
    attn_avg = dist_max(sum(attn_ms) / K, world)
    clocks = clk.summary()
    errs = plan.device_errors()
    if errs:
        raise RuntimeError(f"device errors during the timed region: {errs}")

    # end to end through the public API: pinned host Q/K/V in, host O and row_sum out
    qh = q.cpu().pin_memory()
    kh = k.cpu().pin_memory()
    vh = v.cpu().pin_memory()
    oh = torch.empty_like(plan.O, device="cpu").pin_memory()
    rh = torch.empty_like(plan.row_sum, device="cpu").pin_memory()
    qd, kd, vd = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)

    def run_host(qh_, kh_, vh_, qd_, kd_, vd_, oh_, rh_):
        if alibi:   # no table or masks: copy in, attend, copy out
            with torch.cuda.stream(stream):
                qd_.copy_(qh_, non_blocking=True)
                kd_.copy_(kh_, non_blocking=True)
                vd_.copy_(vh_, non_blocking=True)
                plan.attend_alibi(qd_, kd_, vd_, args.eps, stream)
                oh_.copy_(plan.O, non_blocking=True)
                rh_.copy_(plan.row_sum, non_blocking=True)
        else:
            plan.run_host(qh_, kh_, vh_, qd_, kd_, vd_, oh_, rh_, stream, varlen=varlen)
    for _ in range(3):
        run_host(qh, kh, vh, qd, kd, vd, oh, rh)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    Ke = max(3, min(K, 20))
    barrier(world)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(Ke):
        run_host(qh, kh, vh, qd, kd, vd, oh, rh)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = dist_max(e0.elapsed_time(e1) / Ke, world)
    h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh)) + plan.table_host.numel() * 8
    d2h = oh.numel() * oh.element_size() + rh.numel() * 4
    # the same steps through HostPipeline: step t+1's inputs copied in while step t computes and copies out
    pipe_ms = None
    if not alibi and not varlen:
        from alibi_positional_lsh_b200 import HostPipeline
        pipe = HostPipeline(plan)
        for _ in range(3):
            pipe.step(qh, kh, vh, oh, rh, stream)
        pipe.wait(stream)
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(Ke):
            pipe.step(qh, kh, vh, oh, rh, stream)
        pipe.wait(stream)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        pipe_ms = dist_max(e0.elapsed_time(e1) / Ke, world)
        errs = plan.device_errors()
        if errs:
            raise RuntimeError(f"device errors in the pipelined end-to-end steps: {errs}")
        del pipe

    # the other attention paths on the same plan and inputs, for comparison (not part of the step)
    others = []
    if world == 1:
        paths = {"fused": ("fused (plsh_attention_fwd)", lambda: plan.attend(q, k, v, stream)),
                 "varlen": ("per-sample comparator (plsh_attention_varlen_fwd)",
                            lambda: plan.attend_varlen(q, k, v, stream)),
                 "alibi": (f"exact banded ALiBi, eps={args.eps:g} (plsh_alibi_banded_fwd)",
                           lambda: plan.attend_alibi(q, k, v, args.eps, stream))}
        plan.prepare(stream)
        for key, (label, run) in paths.items():
            if key == args.path:
                continue
            for _ in range(2):
                run()
            ts = []
            for _ in range(5):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                run()
                b.record(stream)
                torch.cuda.synchronize()
                ts.append(a.elapsed_time(b))
            errs = plan.device_errors()
            if errs:
                raise RuntimeError(f"device errors in the comparison path {key}: {errs}")
            others.append({"path": label, "attention_ms": float(np.median(ts)),
                           "this_path_speedup": float(np.median(ts)) / attn_avg})

    decode = decode_timing(plan, q, k, v, stream, w) if (world == 1 and not alibi) else None
    decode_batched = None
    if world == 1 and not alibi and w.dtype == "bf16" and w.n <= 32768:   # 64 caches of up to 8.6 GB
        decode_batched = decode_batched_timing(w, stream, load_peaks()[0]["hbm_gbs"], args.decode_batch)
    bwd = None
    if world == 1 and not alibi and not args.no_backward:
        props = torch.cuda.get_device_properties(local)
        bwd = bwd_timing(plan, q, k, v, stream, w, props.multi_processor_count,
                         float(clocks.get("sm_max_mhz") or 1965), load_peaks()[0]["bf16_tflops"])

    tokens = w.B * w.n * world
    value = job_value(w.B * w.n, world, ms_step)
    peaks, peak_src = load_peaks()
    elt = 2 if w.dtype == "bf16" else 4
    qkvo_bytes = (w.B * w.H * w.n * w.d * 2 + 2 * w.B * w.H_kv * w.n * w.d) * elt
    flops = 4.0 * w.d * TILE * TILE * tiles_min * w.B
    t_mem = qkvo_bytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops / (peaks["bf16_tflops"] * 1e12)
    attn_s = attn_avg * 1e-3
    if t_mem >= t_tc:
        roof = {"bound": "hbm", "achieved": qkvo_bytes / attn_s / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": flops / attn_s / 1e12, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = profiled_traffic()
    roof.update({
        "peak_source": f"{peak_src} (burst figures of MEASURED_PEAKS.json)" if peak_src == "measured" else "fallback",
        "kernel": "attn_tc_kernel" if (w.dtype == "bf16" and w.d == 128) else "attn_simt_kernel",
        "kernel_ms": attn_avg,
        "algorithmic_bytes": qkvo_bytes,
        "issued_tensor_flops": flops,
        "roofline_ms": max(t_mem, t_tc) * 1e3,
        "t_mem_ms": t_mem * 1e3,
        "t_tensor_ms": t_tc * 1e3,
        "frac_vs_sustained_tensor": (max(t_mem, flops / (peaks["bf16_tflops_sustained"] * 1e12)) / attn_s),
        "key_tiles_per_batch": tiles_min,
        "key_tiles_visited_per_batch": tiles_run,
    })

    line = {
        "metric": "PLSH-ALiBi fwd query-tokens/s at n=32k, s=20; achieved % of roofline",
        "path": ("per-sample comparator (plsh_attention_varlen_fwd)" if varlen else
                 f"exact banded ALiBi, eps={args.eps:g} (plsh_alibi_banded_fwd)" if alibi else
                 "fused (plsh_attention_fwd)"),
        "value": value,
        "unit": "query-tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": max(3, args.warmup),
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic (iid N(0,1) Q/K/V drawn on the device, seeded per rank)",
        "config": config_of(w, world),
        "roofline": roof,
        "e2e": ({"value": tokens / (pipe_ms * 1e-3), "unit": "query-tokens/s", "ms_per_step": pipe_ms,
                 "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                 "path": "HostPipeline.step: pinned host Q/K/V -> device -> table, fused K1+K2, K3 -> host O, row_sum, "
                         "copies of neighbouring steps overlapped (two device buffer sets)",
                 "sequential": {"value": tokens / (e2e_ms * 1e-3), "ms_per_step": e2e_ms,
                                "path": "PlshForward.run_host, one step at a time on one stream"}}
                if pipe_ms is not None else
                {"value": tokens / (e2e_ms * 1e-3), "unit": "query-tokens/s", "ms_per_step": e2e_ms,
                 "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                 "path": ("pinned host Q/K/V -> device -> exact banded ALiBi -> host O, row_sum" if alibi else
                          "PlshForward.run_host: pinned host Q/K/V -> device -> table, fused K1+K2, "
                          + ("K1 ids, K4" if varlen else "K3") + " -> host O, row_sum")}),
        "gpu_launches": (1 if alibi else 5 if varlen else 3) * K,
        "gpu_launches_per_step": ({roof["kernel"]: 1} if alibi else
                                  dict({"mask_bmax_kernel": 1, "spans_kernel": 1, roof["kernel"]: 1},
                                       **({"sample_bins_kernel": 1, "varlen_spans_kernel": 1} if varlen else {}))),
        "step_breakdown_ms": {"attention": attn_avg, "table+window": ms_step - attn_avg},
        "clocks": clocks,
    }
    if others:
        line["comparison"] = others
    if decode:
        line["decode"] = decode
    if decode_batched:
        line["decode_batched"] = decode_batched
    if bwd:
        line["backward"] = bwd
    if rank == 0 and not args.no_cpu_baseline:
        sampler = OracleSampler(w)
        rate, desc = sampler.run(args.cpu_seconds)
        line["cpu_baseline"] = {"value": rate, "unit": "query-tokens/s", "cores": sampler.cores, "kind": "oracle",
                                "sample": desc}
    return line


def run_reference(args, rank, world):
    """The CPU oracle as the reference arm: rank 0 only, a bounded sample per step."""
    w = workloads.WORKLOADS[args.workload]
    if args.s:
        w = w.with_(s=args.s)
    if rank != 0:
        return None
    sampler = OracleSampler(w)
    per_step = min(5.0, max(0.5, args.cpu_seconds / max(1, args.steps)))
    for _ in range(args.warmup):
        sampler.run(0.2)
    rates = []
    t0 = time.perf_counter()
    desc = ""
    for _ in range(args.steps):
        r, desc = sampler.run(per_step)
        rates.append(r)
    dt = time.perf_counter() - t0
    value = statistics.mean(rates)
    return {
        "impl": "reference",
        "metric": "PLSH-ALiBi fwd query-tokens/s at n=32k, s=20; achieved % of roofline",
        "value": value,
        "unit": "query-tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": dt * 1e3 / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (iid N(0,1) Q/K/V, seeded)",
        "config": config_of(w, world),
        "cpu_baseline": {"value": value, "unit": "query-tokens/s", "cores": sampler.cores, "kind": "oracle",
                         "sample": f"each step: {desc}"},
        "e2e": {"value": value, "unit": "query-tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=workloads.HEADLINE, choices=list(workloads.WORKLOADS))
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-backward", action="store_true", help="skip timing plsh_attention_bwd beside the step")
    ap.add_argument("--path", choices=["fused", "varlen", "alibi"], default="fused",
                    help="attention path timed: the fused kernel (K3), the per-sample comparator (K4) or "
                         "exact banded ALiBi")
    ap.add_argument("--eps", type=float, default=1e-4,
                    help="band cut-off of exact banded ALiBi (keys lighter than eps are left out)")
    ap.add_argument("--s", type=int, default=None, help="hashes per head instead of the workload's own")
    ap.add_argument("--decode-batch", type=int, default=64,
                    help="sequences of the batched decode timing (64; fewer for a small profiling case)")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (smaller cases for profiling)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    rank, world, local = dist_setup(args.gpus) if args.impl == "ours" else (
        int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), 0)
    try:
        if args.impl == "reference":
            line = run_reference(args, rank, world)
        else:
            line = run_ours(args, rank, world, local)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if args.impl == "ours" and world > 1 and torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
