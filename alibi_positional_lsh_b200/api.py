"""User-facing forward pass built on the C entry points.

PlshForward owns the device buffers of one problem shape (allocated once
with torch) and runs the whole path:
  a1 plsh_draw_table   (host)   -> (delta, u) table, copied to the device
  a2+a3 plsh_window_from_table (K1 + K2 fused) -> b_max, tile windows, boundary masks
  a2 plsh_sample_bins  (K1)     -> bin ids, computed when something needs them (the comparator,
                                   the backward, a caller reading .ids)
  a4 plsh_attention_fwd (K3)    -> O, row_sum
  a5 plsh_attention_varlen_fwd (K4, the per-sample comparator) -> the same O, row_sum
  plsh_decode_fwd (single query rows against the cached K, V) -> rows of T~, row_sum
  plsh_attention_bwd (training) -> dQ, dK, dV of T~ with the table fixed
  plsh_alibi_banded_fwd (exact banded ALiBi, what the method approximates) -> T*, row_sum
All arithmetic of a2..a5 runs in libplsh's CUDA kernels.
"""
from __future__ import annotations

from typing import Optional, Sequence, Tuple

import numpy as np
import torch

from . import (PLSH_BF16, PLSH_F32, PLSH_TILE, PlshError, decode_device_error, plsh_alibi_banded_fwd,
               plsh_attention_bwd, plsh_attention_bwd_tc, plsh_attention_fwd, plsh_attention_varlen_fwd, plsh_decode_fwd,
               plsh_decode_scratch_bytes, plsh_draw_table_heads, plsh_sample_bins,
               plsh_window_from_table, plsh_varlen_scratch_bytes)


class PlshForward:
    """Positional-LSH approximate ALiBi attention for one (B, H, H_kv, n, d, s) shape."""

    def __init__(self, B: int, H: int, H_kv: int, n: int, d: int, s: int, causal: bool,
                 sigma: Sequence[float], seed: int, dtype: torch.dtype = torch.bfloat16,
                 device: str = "cuda", head_offset: int = 0):
        """head_offset: the plan's heads are global heads head_offset .. head_offset + H - 1 of a
        larger problem (a slice of a head partition, see head_partition): its table rows are drawn
        from those heads' counters, so the slices of all ranks make up the whole problem's table."""
        if dtype not in (torch.bfloat16, torch.float32):
            raise ValueError("dtype must be torch.bfloat16 or torch.float32")
        self.B, self.H, self.H_kv, self.n, self.d, self.s = B, H, H_kv, n, d, s
        self.causal = bool(causal)
        self.seed = int(seed)
        self.head_offset = int(head_offset)
        self.dtype = dtype
        self.dtype_code = PLSH_BF16 if dtype == torch.bfloat16 else PLSH_F32
        self.device = torch.device(device)
        self.sigma_host = np.ascontiguousarray(sigma, dtype=np.float64)
        if self.sigma_host.shape != (H,):
            raise ValueError("sigma must hold one value per query head")
        T = (n + PLSH_TILE - 1) // PLSH_TILE
        dev = self.device
        self.table_host = torch.empty((H, s, 2), dtype=torch.float64).pin_memory()
        self._table_copied = None  # event after the last host->device table copy
        self.table_dev = torch.empty((H, s, 2), dtype=torch.float64, device=dev)
        self.sigma_dev = torch.from_numpy(self.sigma_host.copy()).to(dev)
        self._ids = torch.empty((H, s, n), dtype=torch.int32, device=dev)
        self._ids_ok = False  # whether _ids holds the bin ids of the current table
        self.bmax = torch.empty((H,), dtype=torch.int32, device=dev)
        self.spans = torch.empty((H, T, 2), dtype=torch.int32, device=dev)
        self.bmask = torch.empty((H, n), dtype=torch.int32 if s <= 32 else torch.int64, device=dev)
        self.err = torch.zeros((4,), dtype=torch.int32, device=dev)
        self.O = torch.empty((B, H, n, d), dtype=dtype, device=dev)
        self.row_sum = torch.empty((B, H, n), dtype=torch.float32, device=dev)
        self.scratch = None  # per-hash windows of the comparator, allocated on first use
        self.grads = None    # (delta, dQ, dK, dV) of backward(), allocated on first use
        self._kspans = None  # (non-causal windows, their b_max and masks) for the tensor-core backward
        self._kspans_ok = False
        self.decode_scratch = None  # partial results of decode(), grown on demand

    # a1 + a2 + a3
    def prepare(self, stream: Optional[torch.cuda.Stream] = None, table: Optional[np.ndarray] = None) -> None:
        """Draws the table (or takes `table`, float64 [H][s][2]) and builds ids, windows and masks."""
        if self._table_copied is not None:
            self._table_copied.synchronize()   # the pinned buffer may still be in flight
        if table is None:
            plsh_draw_table_heads(self.seed, self.head_offset, self.H, self.s, self.sigma_host, self.table_host.numpy())
        else:
            t = np.ascontiguousarray(table, dtype=np.float64)
            if t.shape != (self.H, self.s, 2):
                raise ValueError("table must be float64 [H][s][2]")
            self.table_host.numpy()[...] = t
        st = torch.cuda.current_stream() if stream is None else stream
        with torch.cuda.stream(st):
            self.table_dev.copy_(self.table_host, non_blocking=True)
            self._table_copied = torch.cuda.Event()
            self._table_copied.record(st)
        plsh_window_from_table(self.table_dev, self.H, self.s, self.n, int(self.causal), self.bmax, self.spans,
                               self.bmask, self.err, st)
        self._ids_ok = False
        self._kspans_ok = False

    def ensure_ids(self, stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
        """The bin ids [H][s][n] of the current table (K1, run on `stream` the first time they are needed).

        K1 reads the device copy of the table that prepare() enqueued on its own stream: with the default
        (current) stream on both sides the order is implicit; with different streams, order them."""
        if not self._ids_ok:
            st = torch.cuda.current_stream() if stream is None else stream
            plsh_sample_bins(self.table_dev, self.H, self.s, self.n, self._ids, self.err, st)
            self._ids_ok = True
        return self._ids

    @property
    def ids(self) -> torch.Tensor:
        return self.ensure_ids()

    # a4
    def attend(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
               stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor]:
        B, H, H_kv, n, d = self.B, self.H, self.H_kv, self.n, self.d
        if q.shape != (B, H, n, d) or k.shape != (B, H_kv, n, d) or v.shape != (B, H_kv, n, d):
            raise ValueError("q/k/v shapes do not match the plan")
        for t, nm in ((q, "q"), (k, "k"), (v, "v")):
            if t.dtype != self.dtype or t.device != self.O.device:
                raise ValueError(f"{nm} must be {self.dtype} on {self.O.device}")
        st = torch.cuda.current_stream() if stream is None else stream
        plsh_attention_fwd(q, k, v, self.dtype_code, B, H, H_kv, n, d, self.sigma_dev, self.s, self.table_dev,
                           self.spans, self.bmask, int(self.causal), self.O, self.row_sum, self.err, st)
        return self.O, self.row_sum

    # a5
    def attend_varlen(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                      stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor]:
        """The per-sample comparator (K4): the same T~ from s block-diagonal attentions."""
        B, H, H_kv, n, d = self.B, self.H, self.H_kv, self.n, self.d
        if q.shape != (B, H, n, d) or k.shape != (B, H_kv, n, d) or v.shape != (B, H_kv, n, d):
            raise ValueError("q/k/v shapes do not match the plan")
        for t, nm in ((q, "q"), (k, "k"), (v, "v")):
            if t.dtype != self.dtype or t.device != self.O.device:
                raise ValueError(f"{nm} must be {self.dtype} on {self.O.device}")
        if self.scratch is None:
            nbytes = plsh_varlen_scratch_bytes(H, self.s, n)
            self.scratch = torch.empty((nbytes // 4,), dtype=torch.int32, device=self.O.device)
        st = torch.cuda.current_stream() if stream is None else stream
        plsh_attention_varlen_fwd(q, k, v, self.dtype_code, B, H, H_kv, n, d, self.sigma_dev, self.s,
                                  self.table_dev, self.ensure_ids(st), self.bmask, int(self.causal), self.scratch,
                                  self.O, self.row_sum, self.err, st)
        return self.O, self.row_sum

    def attend_alibi(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, eps: float = 1e-4,
                     stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor]:
        """Exact ALiBi attention T* over the band |i - j| <= ceil(sigma_h ln(1/eps)) (needs no prepare())."""
        B, H, H_kv, n, d = self.B, self.H, self.H_kv, self.n, self.d
        if q.shape != (B, H, n, d) or k.shape != (B, H_kv, n, d) or v.shape != (B, H_kv, n, d):
            raise ValueError("q/k/v shapes do not match the plan")
        for t, nm in ((q, "q"), (k, "k"), (v, "v")):
            if t.dtype != self.dtype or t.device != self.O.device:
                raise ValueError(f"{nm} must be {self.dtype} on {self.O.device}")
        st = torch.cuda.current_stream() if stream is None else stream
        plsh_alibi_banded_fwd(q, k, v, self.dtype_code, B, H, H_kv, n, d, self.sigma_dev, float(eps),
                              int(self.causal), self.O, self.row_sum, self.err, st)
        return self.O, self.row_sum

    def key_spans(self, stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
        """[H][T][2] non-causal windows of the current table: by the symmetry of the counts, the query rows
        that reach each 128-key tile (the windows themselves when the plan is not causal)."""
        if not self.causal:
            return self.spans
        if not self._kspans_ok:
            if self._kspans is None:
                dev = self.O.device
                T = self.spans.shape[1]
                self._kspans = (torch.empty((self.H, T, 2), dtype=torch.int32, device=dev),
                                torch.empty((self.H,), dtype=torch.int32, device=dev), torch.empty_like(self.bmask))
            st = torch.cuda.current_stream() if stream is None else stream
            spans, bmax, bmask = self._kspans
            plsh_window_from_table(self.table_dev, self.H, self.s, self.n, 0, bmax, spans, bmask, self.err, st)
            self._kspans_ok = True
        return self._kspans[0]

    def backward(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, dO: torch.Tensor,
                 stream: Optional[torch.cuda.Stream] = None,
                 path: str = "auto") -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
        """dQ, dK, dV of <dO, T~> for the inputs of the last attend() (its O and row_sum, the same table).

        path: "tc" the tcgen05 kernels (bf16, d = 128), "simt" the fp32 CUDA-core kernels, "auto" the
        former where it applies."""
        B, H, H_kv, n, d = self.B, self.H, self.H_kv, self.n, self.d
        if q.shape != (B, H, n, d) or dO.shape != (B, H, n, d) or k.shape != (B, H_kv, n, d) \
                or v.shape != (B, H_kv, n, d):
            raise ValueError("q/k/v/dO shapes do not match the plan")
        for t, nm in ((q, "q"), (k, "k"), (v, "v"), (dO, "dO")):
            if t.dtype != self.dtype or t.device != self.O.device:
                raise ValueError(f"{nm} must be {self.dtype} on {self.O.device}")
        if self.grads is None:
            dev = self.O.device
            self.grads = (torch.empty((B, H, n), dtype=torch.float32, device=dev), torch.empty_like(self.O),
                          torch.empty((B, H_kv, n, d), dtype=self.dtype, device=dev),
                          torch.empty((B, H_kv, n, d), dtype=self.dtype, device=dev))
        delta, dQ, dK, dV = self.grads
        st = torch.cuda.current_stream() if stream is None else stream
        tc_ok = self.dtype == torch.bfloat16 and d == 128
        if path not in ("auto", "tc", "simt") or (path == "tc" and not tc_ok):
            raise ValueError("path must be 'auto', 'simt' or (bf16 with d = 128) 'tc'")
        if path == "tc" or (path == "auto" and tc_ok):
            plsh_attention_bwd_tc(q, k, v, self.O, dO, self.row_sum, B, H, H_kv, n, d, self.s, self.bmask, self.spans,
                                  self.key_spans(st), int(self.causal), delta, dQ, dK, dV, self.err, st)
        else:
            plsh_attention_bwd(q, k, v, self.O, dO, self.row_sum, self.dtype_code, B, H, H_kv, n, d, self.s,
                               self.ensure_ids(st), int(self.causal), delta, dQ, dK, dV, self.err, st)
        return dQ, dK, dV

    def decode(self, q_rows: torch.Tensor, pos: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
               stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor]:
        """Rows pos (int32 [m] on the device) of T~ for query rows q_rows [B,H,m,d] against the cache k, v
        [B,H_kv,n,d], with the masks of the last prepare(). Returns new tensors O [B,H,m,d], row_sum [B,H,m]."""
        B, H, H_kv, n, d = self.B, self.H, self.H_kv, self.n, self.d
        m = int(pos.shape[0]) if pos.dim() == 1 else -1
        if m < 1 or pos.dtype != torch.int32 or pos.device != self.O.device:
            raise ValueError(f"pos must be a non-empty int32 vector on {self.O.device}")
        if q_rows.shape != (B, H, m, d) or k.shape != (B, H_kv, n, d) or v.shape != (B, H_kv, n, d):
            raise ValueError("q_rows/k/v shapes do not match the plan")
        for t, nm in ((q_rows, "q_rows"), (k, "k"), (v, "v")):
            if t.dtype != self.dtype or t.device != self.O.device:
                raise ValueError(f"{nm} must be {self.dtype} on {self.O.device}")
        O = torch.empty((B, H, m, d), dtype=self.dtype, device=self.O.device)
        R = torch.empty((B, H, m), dtype=torch.float32, device=self.O.device)
        need = plsh_decode_scratch_bytes(B, H, m, d)
        if self.decode_scratch is None or self.decode_scratch.numel() * 4 < need:
            # zero once: the per-row counters at its end must start at zero (every call leaves them so)
            self.decode_scratch = torch.zeros((need // 4,), dtype=torch.float32, device=self.O.device)
        st = torch.cuda.current_stream() if stream is None else stream
        plsh_decode_fwd(q_rows, pos, m, k, v, self.dtype_code, B, H, H_kv, n, d, self.s, self.bmask,
                        int(self.causal), self.decode_scratch, O, R, self.err, st)
        return O, R

    def __call__(self, q, k, v, stream=None, table=None):
        self.prepare(stream, table)
        return self.attend(q, k, v, stream)

    def run_host(self, q_host: torch.Tensor, k_host: torch.Tensor, v_host: torch.Tensor,
                 q_dev: torch.Tensor, k_dev: torch.Tensor, v_dev: torch.Tensor,
                 o_host: torch.Tensor, rs_host: Optional[torch.Tensor] = None,
                 stream=None, varlen: bool = False) -> None:
        """End to end from (pinned) host inputs to host outputs on one stream (varlen: the comparator)."""
        st = torch.cuda.current_stream() if stream is None else stream
        with torch.cuda.stream(st):
            q_dev.copy_(q_host, non_blocking=True)
            k_dev.copy_(k_host, non_blocking=True)
            v_dev.copy_(v_host, non_blocking=True)
            self.prepare(st)
            if varlen:
                self.attend_varlen(q_dev, k_dev, v_dev, st)
            else:
                self.attend(q_dev, k_dev, v_dev, st)
            o_host.copy_(self.O, non_blocking=True)
            if rs_host is not None:
                rs_host.copy_(self.row_sum, non_blocking=True)

    def reset_errors(self) -> None:
        self.err.zero_()

    def device_errors(self) -> list:
        """Synchronises and decodes the device error word."""
        torch.cuda.synchronize(self.O.device)
        return decode_device_error(int(self.err[0].item()) & 0xFFFFFFFF)

    def check(self) -> None:
        errs = self.device_errors()
        if errs:
            raise PlshError(-1, "device reported " + ",".join(errs))


class HostPipeline:
    """T~ for a stream of batches that live in pinned host memory, with the copies overlapped.

    Each step copies one batch's Q, K, V in, runs the table draw, fused K1 + K2 and K3,
    and copies O and row_sum out. Two device buffer sets alternate, so the
    host->device copy of step t+1 runs while step t computes and while its
    outputs travel device->host (the link carries both directions at once).
    Every step draws its table from the plan's seed, as PlshForward.run_host does.
    """

    def __init__(self, plan: PlshForward):
        self.plan = plan
        dev = plan.O.device
        B, H, H_kv, n, d = plan.B, plan.H, plan.H_kv, plan.n, plan.d
        self.sets = [dict(q=torch.empty((B, H, n, d), dtype=plan.dtype, device=dev),
                          k=torch.empty((B, H_kv, n, d), dtype=plan.dtype, device=dev),
                          v=torch.empty((B, H_kv, n, d), dtype=plan.dtype, device=dev),
                          O=torch.empty_like(plan.O), R=torch.empty_like(plan.row_sum)) for _ in range(2)]
        self.copy_in = torch.cuda.Stream(dev)
        self.copy_out = torch.cuda.Stream(dev)
        self.inputs_ready = [torch.cuda.Event() for _ in range(2)]
        self.computed = [torch.cuda.Event() for _ in range(2)]
        self.copied_out = [torch.cuda.Event() for _ in range(2)]
        self.t = 0

    def step(self, q_host: torch.Tensor, k_host: torch.Tensor, v_host: torch.Tensor, o_host: torch.Tensor,
             rs_host: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None) -> None:
        """Enqueues one batch: pinned host Q, K, V in; O (and row_sum) written to the pinned host buffers once the
        step's copy-out has run (after synchronize(), or after the next steps' events)."""
        plan, i = self.plan, self.t % 2
        buf = self.sets[i]
        compute = torch.cuda.current_stream() if stream is None else stream
        if self.t >= 2:
            self.copy_in.wait_event(self.computed[i])   # step t-2 has finished reading this set's inputs
            compute.wait_event(self.copied_out[i])      # and copied this set's outputs out
        with torch.cuda.stream(self.copy_in):
            buf["q"].copy_(q_host, non_blocking=True)
            buf["k"].copy_(k_host, non_blocking=True)
            buf["v"].copy_(v_host, non_blocking=True)
            self.inputs_ready[i].record(self.copy_in)
        compute.wait_event(self.inputs_ready[i])
        plan.prepare(compute)
        plsh_attention_fwd(buf["q"], buf["k"], buf["v"], plan.dtype_code, plan.B, plan.H, plan.H_kv, plan.n, plan.d,
                           plan.sigma_dev, plan.s, plan.table_dev, plan.spans, plan.bmask, int(plan.causal),
                           buf["O"], buf["R"], plan.err, compute)
        self.computed[i].record(compute)
        self.copy_out.wait_event(self.computed[i])
        with torch.cuda.stream(self.copy_out):
            o_host.copy_(buf["O"], non_blocking=True)
            if rs_host is not None:
                rs_host.copy_(buf["R"], non_blocking=True)
            self.copied_out[i].record(self.copy_out)
        self.t += 1

    def wait(self, stream: Optional[torch.cuda.Stream] = None) -> None:
        """Makes `stream` (default: the current stream) wait for every enqueued step's copy-out."""
        st = torch.cuda.current_stream() if stream is None else stream
        for t in range(max(0, self.t - 2), self.t):
            st.wait_event(self.copied_out[t % 2])


def head_partition(H: int, H_kv: int, world: int, rank: int) -> Tuple[int, int]:
    """Query heads [h0, h1) of `rank` when one problem is split over `world` devices by heads.

    Whole GQA groups stay together: the KV heads are dealt out as evenly as possible (the first
    H_kv % world ranks take one more), and each rank takes the query heads that read its KV
    heads. Every (batch, head) is independent given the table, so the ranks exchange nothing;
    with head_offset=h0 each rank's PlshForward draws exactly its rows of the whole table.
    A rank left without KV heads (world > H_kv) gets an empty range.
    """
    if H_kv < 1 or H % H_kv or world < 1 or not 0 <= rank < world:
        raise ValueError("need H_kv >= 1 dividing H and 0 <= rank < world")
    group = H // H_kv
    base, extra = divmod(H_kv, world)
    g0 = rank * base + min(rank, extra)
    g1 = g0 + base + (1 if rank < extra else 0)
    return g0 * group, g1 * group


def fixed_blocks_table(H: int, block: float) -> np.ndarray:
    """Table of the "fixed blocks" baseline: one hash per head with pitch `block` and offset 0, so
    positions [k*block, (k+1)*block) form the blocks and every row attends inside its own block
    (Results, Mistral-7B bullet: the fixed-blocks comparison). Pass it to PlshForward.prepare
    (table=...) or __call__ with s = 1."""
    if not block > 0:
        raise ValueError("block must be > 0")
    t = np.zeros((H, 1, 2), dtype=np.float64)
    t[:, 0, 0] = float(block)
    return t


def forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, sigma: Sequence[float], s: int, seed: int,
            causal: bool) -> Tuple[torch.Tensor, torch.Tensor]:
    """One-shot T~ and row_sum for CUDA tensors q [B,H,n,d], k, v [B,H_kv,n,d]."""
    B, H, n, d = q.shape
    plan = PlshForward(B, H, k.shape[1], n, d, s, causal, sigma, seed, q.dtype, str(q.device))
    O, R = plan(q.contiguous(), k.contiguous(), v.contiguous())
    plan.check()
    return O.clone(), R.clone()
