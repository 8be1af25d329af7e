"""Python binding of libplsh (Positional-LSH approximate ALiBi attention, B200).

Argument marshalling only: each function here has the name of the C entry
point it calls (include/plsh.h), checks that tensors sit where the C side
expects them, passes raw pointers and the current CUDA stream, and turns a
nonzero status into PlshError. Every step of the computation runs in the
library's CUDA kernels; importing this package fails loudly if libplsh.so
is missing, and there is no other code path.

PyTorch is used for device memory and streams only.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libplsh.so")

PLSH_OK = 0
PLSH_BF16 = 0
PLSH_F32 = 1
PLSH_TILE = 128
PLSH_MAX_S = 64
PLSH_VARLEN_STATIC_SCRATCH_BYTES = 4 << 20
DEVERR_BITS = {1: "RANGE", 2: "TABLE", 4: "WINDOW", 8: "TIMEOUT", 16: "SIGMA", 32: "POSITION"}


class PlshError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"libplsh error {code}: {msg}")
        self.code = code


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built: run `python alibi_positional_lsh_b200/build.py` "
                          "(or __graft_entry__.build()) first")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, u64, dp = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint64, ctypes.c_void_p
    lib.plsh_last_error.restype = ctypes.c_char_p
    lib.plsh_last_error.argtypes = []
    lib.plsh_version.restype = i32
    lib.plsh_version.argtypes = []
    lib.plsh_set_wait_limit_ns.restype = i32
    lib.plsh_set_wait_limit_ns.argtypes = [u64]
    lib.plsh_test_withhold_mma.restype = i32
    lib.plsh_test_withhold_mma.argtypes = [i32]
    lib.plsh_draw_table.restype = i32
    lib.plsh_draw_table.argtypes = [u64, i32, i32, dp, dp]
    lib.plsh_draw_table_heads.restype = i32
    lib.plsh_draw_table_heads.argtypes = [u64, i32, i32, i32, dp, dp]
    lib.plsh_sample_bins.restype = i32
    lib.plsh_sample_bins.argtypes = [vp, i32, i32, i32, vp, vp, vp]
    lib.plsh_window.restype = i32
    lib.plsh_window.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, vp, vp]
    lib.plsh_window_from_table.restype = i32
    lib.plsh_window_from_table.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, vp, vp]
    lib.plsh_attention_fwd.restype = i32
    lib.plsh_attention_fwd.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, i32, vp, vp, vp, i32,
                                       vp, vp, vp, vp]
    lib.plsh_varlen_scratch_bytes.restype = ctypes.c_size_t
    lib.plsh_varlen_scratch_bytes.argtypes = [i32, i32, i32]
    lib.plsh_varlen_spans.restype = i32
    lib.plsh_varlen_spans.argtypes = [vp, i32, i32, i32, i32, vp, vp]
    lib.plsh_attention_varlen_fwd.restype = i32
    lib.plsh_attention_varlen_fwd.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, i32, vp, vp, vp, i32,
                                              vp, ctypes.c_size_t, vp, vp, vp, vp]
    lib.plsh_alibi_banded_fwd.restype = i32
    lib.plsh_alibi_banded_fwd.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, ctypes.c_double, i32, vp, vp,
                                          vp, vp]
    lib.plsh_attention_varlen_fwd_static.restype = i32
    lib.plsh_attention_varlen_fwd_static.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, i32, vp, vp,
                                                     vp, i32, vp, vp, vp, vp]
    lib.plsh_attention_bwd.restype = i32
    lib.plsh_attention_bwd.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, vp, i32, vp, vp,
                                       vp, vp, vp, vp]
    lib.plsh_attention_bwd_tc.restype = i32
    lib.plsh_attention_bwd_tc.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, vp, vp, i32,
                                          vp, vp, vp, vp, vp, vp]
    lib.plsh_decode_fwd.restype = i32
    lib.plsh_decode_fwd.argtypes = [vp, vp, i32, vp, vp, i32, i32, i32, i32, i32, i32, i32, vp, i32, vp,
                                    ctypes.c_size_t, vp, vp, vp, vp]
    lib.plsh_decode_scratch_bytes.restype = ctypes.c_size_t
    lib.plsh_decode_scratch_bytes.argtypes = [i32, i32, i32, i32]
    return lib


_lib = _load()


def _check(rc: int) -> None:
    if rc != PLSH_OK:
        raise PlshError(rc, _lib.plsh_last_error().decode(errors="replace"))


def _dev_ptr(t, name: str):
    """Pointer of a contiguous CUDA tensor (None passes NULL)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def plsh_last_error() -> str:
    return _lib.plsh_last_error().decode(errors="replace")


def plsh_version() -> int:
    return _lib.plsh_version()


def plsh_set_wait_limit_ns(limit_ns: int) -> None:
    _check(_lib.plsh_set_wait_limit_ns(ctypes.c_uint64(int(limit_ns))))


def plsh_test_withhold_mma(on: bool) -> None:
    _check(_lib.plsh_test_withhold_mma(1 if on else 0))


def plsh_draw_table(seed: int, H: int, s: int, sigma_host: np.ndarray, table_host: np.ndarray) -> None:
    """Host call: fills table_host float64 [H][s][2] with (delta, u)."""
    sig = np.ascontiguousarray(sigma_host, dtype=np.float64)
    if sig.shape != (H,):
        raise ValueError("sigma_host must have shape [H]")
    if table_host.dtype != np.float64 or table_host.shape != (H, s, 2) or not table_host.flags.c_contiguous:
        raise ValueError("table_host must be a contiguous float64 array [H][s][2]")
    _check(_lib.plsh_draw_table(ctypes.c_uint64(seed & (2 ** 64 - 1)), H, s,
                                sig.ctypes.data_as(ctypes.c_void_p), table_host.ctypes.data_as(ctypes.c_void_p)))


def plsh_draw_table_heads(seed: int, h0: int, H: int, s: int, sigma_host: np.ndarray, table_host: np.ndarray) -> None:
    """Host call: rows of global heads h0 .. h0 + H - 1 of the table, float64 [H][s][2]."""
    sig = np.ascontiguousarray(sigma_host, dtype=np.float64)
    if sig.shape != (H,):
        raise ValueError("sigma_host must have shape [H]")
    if table_host.dtype != np.float64 or table_host.shape != (H, s, 2) or not table_host.flags.c_contiguous:
        raise ValueError("table_host must be a contiguous float64 array [H][s][2]")
    _check(_lib.plsh_draw_table_heads(ctypes.c_uint64(seed & (2 ** 64 - 1)), h0, H, s,
                                      sig.ctypes.data_as(ctypes.c_void_p), table_host.ctypes.data_as(ctypes.c_void_p)))


def plsh_sample_bins(table_dev, H: int, s: int, n: int, ids_dev, err_dev, stream=None) -> None:
    _check(_lib.plsh_sample_bins(_dev_ptr(table_dev, "table_dev"), H, s, n, _dev_ptr(ids_dev, "ids_dev"),
                                 _dev_ptr(err_dev, "err_dev"), _stream_ptr(stream)))


def plsh_window(ids_dev, H: int, s: int, n: int, causal: int, bmax_dev, tile_span_dev, bmask_dev, err_dev,
                stream=None) -> None:
    _check(_lib.plsh_window(_dev_ptr(ids_dev, "ids_dev"), H, s, n, int(causal), _dev_ptr(bmax_dev, "bmax_dev"),
                            _dev_ptr(tile_span_dev, "tile_span_dev"), _dev_ptr(bmask_dev, "bmask_dev"),
                            _dev_ptr(err_dev, "err_dev"), _stream_ptr(stream)))


def plsh_window_from_table(table_dev, H: int, s: int, n: int, causal: int, bmax_dev, spans_dev, bmask_dev, err_dev,
                           stream=None) -> None:
    _check(_lib.plsh_window_from_table(_dev_ptr(table_dev, "table_dev"), H, s, n, int(causal),
                                       _dev_ptr(bmax_dev, "bmax_dev"), _dev_ptr(spans_dev, "spans_dev"),
                                       _dev_ptr(bmask_dev, "bmask_dev"), _dev_ptr(err_dev, "err_dev"),
                                       _stream_ptr(stream)))


def plsh_attention_fwd(Q, K, V, dtype: int, B: int, H: int, H_kv: int, n: int, d: int, sigma_dev, s: int,
                       table_dev, tile_span_dev, bmask_dev, causal: int, O, row_sum, err_dev,
                       stream=None) -> None:
    _check(_lib.plsh_attention_fwd(_dev_ptr(Q, "Q"), _dev_ptr(K, "K"), _dev_ptr(V, "V"), dtype, B, H, H_kv, n, d,
                                   _dev_ptr(sigma_dev, "sigma_dev"), s, _dev_ptr(table_dev, "table_dev"),
                                   _dev_ptr(tile_span_dev, "tile_span_dev"), _dev_ptr(bmask_dev, "bmask_dev"),
                                   int(causal), _dev_ptr(O, "O"), _dev_ptr(row_sum, "row_sum"),
                                   _dev_ptr(err_dev, "err_dev"), _stream_ptr(stream)))


def plsh_varlen_scratch_bytes(H: int, s: int, n: int) -> int:
    return int(_lib.plsh_varlen_scratch_bytes(H, s, n))


def plsh_varlen_spans(ids_dev, H: int, s: int, n: int, causal: int, spans_dev, stream=None) -> None:
    _check(_lib.plsh_varlen_spans(_dev_ptr(ids_dev, "ids_dev"), H, s, n, int(causal),
                                  _dev_ptr(spans_dev, "spans_dev"), _stream_ptr(stream)))


def plsh_attention_varlen_fwd(Q, K, V, dtype: int, B: int, H: int, H_kv: int, n: int, d: int, sigma_dev, s: int,
                              table_dev, ids_dev, bmask_dev, causal: int, scratch_dev, O, row_sum, err_dev,
                              stream=None) -> None:
    nbytes = 0 if scratch_dev is None else scratch_dev.numel() * scratch_dev.element_size()
    _check(_lib.plsh_attention_varlen_fwd(_dev_ptr(Q, "Q"), _dev_ptr(K, "K"), _dev_ptr(V, "V"), dtype, B, H, H_kv,
                                          n, d, _dev_ptr(sigma_dev, "sigma_dev"), s,
                                          _dev_ptr(table_dev, "table_dev"), _dev_ptr(ids_dev, "ids_dev"),
                                          _dev_ptr(bmask_dev, "bmask_dev"), int(causal),
                                          _dev_ptr(scratch_dev, "scratch_dev"), ctypes.c_size_t(nbytes),
                                          _dev_ptr(O, "O"), _dev_ptr(row_sum, "row_sum"),
                                          _dev_ptr(err_dev, "err_dev"), _stream_ptr(stream)))


def plsh_attention_varlen_fwd_static(Q, K, V, dtype: int, B: int, H: int, H_kv: int, n: int, d: int, sigma_dev,
                                     s: int, table_dev, ids_dev, bmask_dev, causal: int, O, row_sum, err_dev,
                                     stream=None) -> None:
    _check(_lib.plsh_attention_varlen_fwd_static(
        _dev_ptr(Q, "Q"), _dev_ptr(K, "K"), _dev_ptr(V, "V"), dtype, B, H, H_kv, n, d,
        _dev_ptr(sigma_dev, "sigma_dev"), s, _dev_ptr(table_dev, "table_dev"), _dev_ptr(ids_dev, "ids_dev"),
        _dev_ptr(bmask_dev, "bmask_dev"), int(causal), _dev_ptr(O, "O"), _dev_ptr(row_sum, "row_sum"),
        _dev_ptr(err_dev, "err_dev"), _stream_ptr(stream)))


def plsh_alibi_banded_fwd(Q, K, V, dtype: int, B: int, H: int, H_kv: int, n: int, d: int, sigma_dev, eps: float,
                          causal: int, O, row_sum, err_dev, stream=None) -> None:
    _check(_lib.plsh_alibi_banded_fwd(_dev_ptr(Q, "Q"), _dev_ptr(K, "K"), _dev_ptr(V, "V"), dtype, B, H, H_kv, n, d,
                                      _dev_ptr(sigma_dev, "sigma_dev"), ctypes.c_double(eps), int(causal),
                                      _dev_ptr(O, "O"), _dev_ptr(row_sum, "row_sum"), _dev_ptr(err_dev, "err_dev"),
                                      _stream_ptr(stream)))


def plsh_decode_scratch_bytes(B: int, H: int, m: int, d: int) -> int:
    return int(_lib.plsh_decode_scratch_bytes(B, H, m, d))


def plsh_decode_fwd(Q, pos_dev, m: int, K, V, dtype: int, B: int, H: int, H_kv: int, n: int, d: int, s: int,
                    bmask_dev, causal: int, scratch_dev, O, row_sum, err_dev, stream=None) -> None:
    nbytes = 0 if scratch_dev is None else scratch_dev.numel() * scratch_dev.element_size()
    _check(_lib.plsh_decode_fwd(_dev_ptr(Q, "Q"), _dev_ptr(pos_dev, "pos_dev"), m, _dev_ptr(K, "K"),
                                _dev_ptr(V, "V"), dtype, B, H, H_kv, n, d, s, _dev_ptr(bmask_dev, "bmask_dev"),
                                int(causal), _dev_ptr(scratch_dev, "scratch_dev"), ctypes.c_size_t(nbytes),
                                _dev_ptr(O, "O"), _dev_ptr(row_sum, "row_sum"), _dev_ptr(err_dev, "err_dev"),
                                _stream_ptr(stream)))


def plsh_attention_bwd(Q, K, V, O, dO, row_sum, dtype: int, B: int, H: int, H_kv: int, n: int, d: int, s: int,
                       ids_dev, causal: int, delta_dev, dQ, dK, dV, err_dev, stream=None) -> None:
    _check(_lib.plsh_attention_bwd(_dev_ptr(Q, "Q"), _dev_ptr(K, "K"), _dev_ptr(V, "V"), _dev_ptr(O, "O"),
                                   _dev_ptr(dO, "dO"), _dev_ptr(row_sum, "row_sum"), dtype, B, H, H_kv, n, d, s,
                                   _dev_ptr(ids_dev, "ids_dev"), int(causal), _dev_ptr(delta_dev, "delta_dev"),
                                   _dev_ptr(dQ, "dQ"), _dev_ptr(dK, "dK"), _dev_ptr(dV, "dV"),
                                   _dev_ptr(err_dev, "err_dev"), _stream_ptr(stream)))


def plsh_attention_bwd_tc(Q, K, V, O, dO, row_sum, B: int, H: int, H_kv: int, n: int, d: int, s: int, bmask_dev,
                          tile_span_dev, key_span_dev, causal: int, delta_dev, dQ, dK, dV, err_dev, stream=None) -> None:
    _check(_lib.plsh_attention_bwd_tc(_dev_ptr(Q, "Q"), _dev_ptr(K, "K"), _dev_ptr(V, "V"), _dev_ptr(O, "O"),
                                      _dev_ptr(dO, "dO"), _dev_ptr(row_sum, "row_sum"), B, H, H_kv, n, d, s,
                                      _dev_ptr(bmask_dev, "bmask_dev"), _dev_ptr(tile_span_dev, "tile_span_dev"),
                                      _dev_ptr(key_span_dev, "key_span_dev"), int(causal),
                                      _dev_ptr(delta_dev, "delta_dev"), _dev_ptr(dQ, "dQ"), _dev_ptr(dK, "dK"),
                                      _dev_ptr(dV, "dV"), _dev_ptr(err_dev, "err_dev"), _stream_ptr(stream)))


def decode_device_error(word: int) -> list:
    return [name for bit, name in DEVERR_BITS.items() if word & bit]


from .api import HostPipeline, PlshForward, fixed_blocks_table, forward, head_partition  # noqa: E402,F401
