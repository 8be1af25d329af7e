"""plsh_window_from_table against plsh_sample_bins + plsh_window (needs a B200).

The fused path evaluates every bin id it needs with K1's own float64 steps
instead of reading them back from memory, so b_max, the tile windows and the
boundary masks must be the same bit for bit, and a bad table entry or an id
overflow must set the same device error bits.
"""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

CASES = [
    # H, s, n, causal, sigmas
    (4, 20, 32768, True, [1.4, 8.0, 45.0, 256.0]),
    (2, 20, 5003, False, [3.0, 120.0]),
    (3, 64, 2049, True, [0.3, 17.0, 5000.0]),
    (2, 33, 130, False, [2.0, 9.0]),
    (1, 4, 1, True, [3.0]),
    (2, 1, 777, False, [50.0, 0.7]),
]


def _two_step(table_dev, H, s, n, causal):
    from alibi_positional_lsh_b200 import plsh_sample_bins, plsh_window
    dev = "cuda:0"
    T = (n + 127) // 128
    ids = torch.empty((H, s, n), dtype=torch.int32, device=dev)
    bmax = torch.empty((H,), dtype=torch.int32, device=dev)
    spans = torch.empty((H, T, 2), dtype=torch.int32, device=dev)
    bmask = torch.empty((H, n), dtype=torch.int32 if s <= 32 else torch.int64, device=dev)
    err = torch.zeros((4,), dtype=torch.int32, device=dev)
    plsh_sample_bins(table_dev, H, s, n, ids, err)
    plsh_window(ids, H, s, n, int(causal), bmax, spans, bmask, err)
    return bmax, spans, bmask, err


def _fused(table_dev, H, s, n, causal):
    from alibi_positional_lsh_b200 import plsh_window_from_table
    dev = "cuda:0"
    T = (n + 127) // 128
    bmax = torch.full((H,), -7, dtype=torch.int32, device=dev)
    spans = torch.full((H, T, 2), -7, dtype=torch.int32, device=dev)
    bmask = torch.full((H, n), -7, dtype=torch.int32 if s <= 32 else torch.int64, device=dev)
    err = torch.zeros((4,), dtype=torch.int32, device=dev)
    plsh_window_from_table(table_dev, H, s, n, int(causal), bmax, spans, bmask, err)
    return bmax, spans, bmask, err


@pytest.mark.parametrize("H,s,n,causal,sigmas", CASES,
                         ids=[f"H{c[0]}s{c[1]}n{c[2]}{'c' if c[3] else 'nc'}" for c in CASES])
def test_fused_window_equals_two_step(H, s, n, causal, sigmas):
    table = oracle.draw_table(1000 + n + s, sigmas, s)
    table_dev = torch.from_numpy(table).cuda()
    a = _two_step(table_dev, H, s, n, causal)
    b = _fused(table_dev, H, s, n, causal)
    torch.cuda.synchronize()
    for name, x, y in zip(("bmax", "spans", "bmask", "err"), a, b):
        assert torch.equal(x, y), f"{name} differs"
    assert int(b[3][0]) == 0


def test_fused_window_reports_the_same_errors():
    n, s = 3000, 3
    table = oracle.draw_table(5, [4.0, 4.0], s)
    table[0, 1, 0] = float("nan")       # a bad pitch: TABLE, ids 0 for that hash
    table[1, 2, 0] = 1e-7               # ids past 2^31: RANGE
    table_dev = torch.from_numpy(table).cuda()
    a = _two_step(table_dev, 2, s, n, True)
    b = _fused(table_dev, 2, s, n, True)
    torch.cuda.synchronize()
    assert int(a[3][0]) == int(b[3][0]) == (2 | 1)
    for name, x, y in zip(("bmax", "spans", "bmask"), a[:3], b[:3]):
        assert torch.equal(x, y), f"{name} differs"
