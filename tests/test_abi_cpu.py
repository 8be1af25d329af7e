"""The C-ABI library without a GPU: it loads, exports every symbol the header
declares, its host-side table sampler matches the oracle bit for bit, and
its host-side argument checks return the documented codes before any
device work."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "plsh.h")


def _declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(plsh_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def plsh():
    import alibi_positional_lsh_b200 as m
    return m


def test_header_declares_the_path():
    syms = _declared_symbols()
    for want in ("plsh_draw_table", "plsh_sample_bins", "plsh_window", "plsh_attention_fwd", "plsh_last_error"):
        assert want in syms, syms


def test_library_exports_every_declared_symbol(plsh):
    lib = ctypes.CDLL(plsh.LIB_PATH)
    for name in _declared_symbols():
        assert hasattr(lib, name), name


def test_version(plsh):
    assert plsh.plsh_version() >= 100


@pytest.mark.parametrize("seed,sigma,s", [
    (0, [16.0], 8),
    (1, [2.0 ** (h + 1) for h in range(8)], 10),
    (2, [2.0 ** ((h + 1) / 2) for h in range(16)], 20),
    (3, [2.0 ** ((h + 1) / 4) for h in range(32)], 40),
    (4, [2.0 ** (8 * (h + 1) / 40) for h in range(40)], 16),
    (2 ** 64 - 1, [1e-3, 1e6], 64),
])
def test_draw_table_bit_exact_with_oracle(plsh, seed, sigma, s):
    H = len(sigma)
    got = np.empty((H, s, 2), dtype=np.float64)
    plsh.plsh_draw_table(seed, H, s, np.asarray(sigma), got)
    want = oracle.draw_table(seed, sigma, s)
    assert got.tobytes() == want.tobytes()


def test_draw_table_for_every_workload(plsh):
    for w in workloads.WORKLOADS.values():
        got = np.empty((w.H, w.s, 2))
        plsh.plsh_draw_table(w.seed, w.H, w.s, np.asarray(w.sigmas()), got)
        assert got.tobytes() == oracle.draw_table(w.seed, w.sigmas(), w.s).tobytes()


def test_draw_table_rejects_bad_arguments(plsh):
    t = np.empty((1, 4, 2))
    for sigma in ([0.0], [-1.0], [float("nan")], [float("inf")]):
        with pytest.raises(plsh.PlshError) as e:
            plsh.plsh_draw_table(1, 1, 4, np.asarray(sigma), t)
        assert e.value.code == 1
    with pytest.raises(plsh.PlshError):
        plsh.plsh_draw_table(1, 1, 65, np.asarray([1.0]), np.empty((1, 65, 2)))


def test_entry_points_reject_bad_sizes_before_any_launch(plsh):
    lib = plsh._lib
    null = None
    # invalid sizes or null pointers: INVALID_ARG (1), returned by host checks
    assert lib.plsh_sample_bins(null, 1, 0, 10, null, null, null) == 1
    assert lib.plsh_sample_bins(null, 1, 4, 10, null, null, null) == 1
    assert lib.plsh_window(null, 1, 4, 10, 2, null, null, null, null, null) == 1
    assert lib.plsh_window(null, 0, 4, 10, 0, null, null, null, null, null) == 1
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the checks fail first
    # head dim without a kernel: UNSUPPORTED (2)
    rc = lib.plsh_attention_fwd(fake, fake, fake, 0, 1, 1, 1, 128, 96, null, 4, null, fake, fake, 0, fake, fake,
                                fake, null)
    assert rc == 2 and "head dim" in plsh.plsh_last_error()
    # H_kv not dividing H
    rc = lib.plsh_attention_fwd(fake, fake, fake, 0, 1, 6, 4, 128, 128, null, 4, null, fake, fake, 0, fake, fake,
                                fake, null)
    assert rc == 1
    # misaligned Q
    rc = lib.plsh_attention_fwd(ctypes.c_void_p((1 << 20) + 8), fake, fake, 0, 1, 1, 1, 128, 128, null, 4, null,
                                fake, fake, 0, fake, fake, fake, null)
    assert rc == 1 and "aligned" in plsh.plsh_last_error()
    # unknown dtype
    rc = lib.plsh_attention_fwd(fake, fake, fake, 7, 1, 1, 1, 128, 128, null, 4, null, fake, fake, 0, fake, fake,
                                fake, null)
    assert rc == 2


def test_banded_alibi_rejects_bad_arguments_before_any_launch(plsh):
    lib = plsh._lib
    null = None
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the checks fail first
    args = lambda eps, sigma=fake, d=128, causal=1: (fake, fake, fake, 0, 1, 2, 1, 256, d, sigma,
                                                     ctypes.c_double(eps), causal, fake, fake, fake, null)
    assert lib.plsh_alibi_banded_fwd(*args(0.0)) == 1 and "eps" in plsh.plsh_last_error()
    assert lib.plsh_alibi_banded_fwd(*args(1.0)) == 1
    assert lib.plsh_alibi_banded_fwd(*args(float("nan"))) == 1
    assert lib.plsh_alibi_banded_fwd(*args(1e-4, sigma=null)) == 1 and "null" in plsh.plsh_last_error()
    assert lib.plsh_alibi_banded_fwd(*args(1e-4, d=96)) == 2
    assert lib.plsh_alibi_banded_fwd(*args(1e-4, causal=3)) == 1


def test_varlen_entry_points_reject_bad_arguments_before_any_launch(plsh):
    lib = plsh._lib
    null = None
    fake = ctypes.c_void_p(1 << 20)
    assert lib.plsh_varlen_scratch_bytes(16, 20, 32768) == 8 * 16 * 20 * 256
    assert lib.plsh_varlen_scratch_bytes(0, 20, 32768) == 0
    assert lib.plsh_varlen_spans(null, 1, 4, 100, 0, fake, null) == 1
    assert lib.plsh_varlen_spans(fake, 1, 4, 100, 2, fake, null) == 1
    # scratch smaller than needed
    rc = lib.plsh_attention_varlen_fwd(fake, fake, fake, 0, 1, 1, 1, 300, 128, null, 5, null, fake, fake, 1, fake,
                                       ctypes.c_size_t(8), fake, fake, fake, null)
    assert rc == 1 and "scratch" in plsh.plsh_last_error()
    # the static-buffer entry point refuses windows larger than its buffer
    rc = lib.plsh_attention_varlen_fwd_static(fake, fake, fake, 0, 1, 40, 8, 131072, 128, null, 64, null, fake,
                                              fake, 1, fake, fake, fake, null)
    assert rc == 3 and "static buffer" in plsh.plsh_last_error()


def test_decode_rejects_bad_arguments_before_any_launch(plsh):
    lib = plsh._lib
    null = None
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the checks fail first
    args = lambda m=4, pos=fake, d=128, H_kv=1, causal=1, nbytes=1 << 30: (
        fake, pos, m, fake, fake, 0, 1, 2, H_kv, 256, d, 20, fake, causal, fake, ctypes.c_size_t(nbytes), fake, fake,
        fake, null)
    assert lib.plsh_decode_scratch_bytes(1, 2, 4, 128) == 2 * 4 * (32 * 130 + 260) + 16
    assert lib.plsh_decode_fwd(*args(nbytes=100)) == 1 and "scratch" in plsh.plsh_last_error()
    assert lib.plsh_decode_fwd(*args(m=0)) == 1 and "m >= 1" in plsh.plsh_last_error()
    assert lib.plsh_decode_fwd(*args(pos=null)) == 1 and "null" in plsh.plsh_last_error()
    assert lib.plsh_decode_fwd(*args(d=96)) == 2
    assert lib.plsh_decode_fwd(*args(H_kv=3)) == 1
    assert lib.plsh_decode_fwd(*args(causal=2)) == 1


def test_backward_rejects_bad_arguments_before_any_launch(plsh):
    lib = plsh._lib
    null = None
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the checks fail first
    args = lambda d=128, H_kv=1, causal=1, ids=fake, dtype=0, Q=fake: (Q, fake, fake, fake, fake, fake, dtype, 1, 2,
                                                                        H_kv, 256, d, 20, ids, causal, fake, fake,
                                                                        fake, fake, fake, null)
    assert lib.plsh_attention_bwd(*args(ids=null)) == 1 and "null" in plsh.plsh_last_error()
    assert lib.plsh_attention_bwd(*args(d=96)) == 2
    assert lib.plsh_attention_bwd(*args(H_kv=3)) == 1
    assert lib.plsh_attention_bwd(*args(causal=2)) == 1
    assert lib.plsh_attention_bwd(*args(dtype=9)) == 2
    assert lib.plsh_attention_bwd(*args(Q=ctypes.c_void_p((1 << 20) + 4))) == 1 and "aligned" in plsh.plsh_last_error()


def test_window_from_table_rejects_bad_arguments_before_any_launch(plsh):
    lib = plsh._lib
    null = None
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the checks fail first
    assert lib.plsh_window_from_table(null, 1, 4, 100, 0, fake, fake, fake, fake, null) == 1
    assert "null" in plsh.plsh_last_error()
    assert lib.plsh_window_from_table(fake, 1, 4, 100, 2, fake, fake, fake, fake, null) == 1
    assert lib.plsh_window_from_table(fake, 1, 0, 100, 0, fake, fake, fake, fake, null) == 1
    assert lib.plsh_window_from_table(fake, 1, 65, 100, 0, fake, fake, fake, fake, null) == 1
    assert lib.plsh_window_from_table(fake, 0, 4, 100, 0, fake, fake, fake, fake, null) == 1


def test_wait_limit_setting_checks_its_range(plsh):
    from alibi_positional_lsh_b200 import PlshError, plsh_set_wait_limit_ns, plsh_test_withhold_mma
    plsh_set_wait_limit_ns(5_000_000)
    plsh_set_wait_limit_ns(0)          # back to the default
    with pytest.raises(PlshError) as ei:
        plsh_set_wait_limit_ns(61_000_000_000)
    assert ei.value.code == 3
    plsh_test_withhold_mma(True)
    plsh_test_withhold_mma(False)
