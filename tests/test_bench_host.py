"""bench.py's host-side work counts against brute force from the oracle's definitions (no GPU).

The decode and backward roofline figures divide counted work by measured
time: decode_keys counts the keys a decode row gives weight to, and
bwd_chunk_pairs the 64 x 64 tile pairs the backward kernels walk. Both are
recounted here from c_ij by direct comparison of bin ids.
"""
import numpy as np
import pytest

import bench
import oracle


def _table_ids(n, sigmas, s, seed):
    return oracle.bin_ids(oracle.draw_table(seed, sigmas, s), n)


@pytest.mark.parametrize("causal", [True, False])
def test_decode_keys_counts_weighted_keys(causal):
    n, s = 500, 6
    ids = _table_ids(n, [2.0, 30.0, 7.0], s, 3)
    bm = np.stack([oracle.boundary_bits(ids[h]) for h in range(ids.shape[0])])
    for i in (0, 1, 250, 499):
        want = 0
        for h in range(ids.shape[0]):
            c = (ids[h][:, i][:, None] == ids[h]).sum(axis=0)
            if causal:
                c[i + 1:] = 0
            want += int((c > 0).sum())
        assert bench.decode_keys(bm, s, i, causal) == want


@pytest.mark.parametrize("causal", [True, False])
def test_bwd_chunk_pairs_match_block_ranges(causal):
    n = 700
    ids = _table_ids(n, [2.0, 30.0, 5.0], 6, 4)
    dq = dkdv = 0
    for h in range(ids.shape[0]):
        C = oracle.match_counts(ids[h])
        for t in range(0, n, bench.BWD_TILE):
            rows = np.arange(t, min(n, t + bench.BWD_TILE))
            nz = np.nonzero(C[rows].sum(axis=0))[0]
            lo, hi = int(nz.min()), int(nz.max())
            hq = min(hi, int(rows[-1])) if causal else hi        # dQ: keys j <= i
            lk = max(lo, t) if causal else lo                    # dK, dV: rows i >= j
            dq += (hq - lo) // bench.BWD_TILE + 1
            dkdv += (hi - lk) // bench.BWD_TILE + 1
    assert bench.bwd_chunk_pairs(ids, causal, 1) == (dq, dkdv)


@pytest.mark.parametrize("causal", [True, False])
def test_issued_and_visited_key_tiles(causal):
    """The headline roofline counts issued tensor work as 128-key tiles: per query tile, the span of keys
    with weight rounded up to whole tiles (issued_tiles), and the 128-aligned tiles the kernel walks around
    the diagonal (kernel_tiles). Both recounted from c_ij."""
    n, T = 1000, 8
    ids = _table_ids(n, [3.0, 60.0, 400.0], 5, 6)
    spans = np.stack([oracle.tile_spans(ids[h], causal) for h in range(ids.shape[0])])
    issued = visited = 0
    for h in range(ids.shape[0]):
        C = oracle.match_counts(ids[h])
        if causal:
            C = np.tril(C)
        for t in range(T):
            rows = np.arange(t * 128, min(n, t * 128 + 128))
            nz = np.nonzero(C[rows].sum(axis=0))[0]
            lo, hi = int(nz.min()), int(nz.max())
            issued += -(-(hi - lo + 1) // 128)
            visited += sum(1 for j0 in range(0, n, 128) if j0 + 127 >= lo and j0 <= hi)
    assert bench.issued_tiles(spans, causal) == issued
    assert bench.kernel_tiles(spans, causal) == visited


@pytest.mark.parametrize("causal", [True, False])
def test_tensor_core_backward_tiles(causal):
    """The tensor-core backward's work counts, recounted from c_ij: the dQ kernel visits the forward's
    tiles; the dK/dV kernel walks, per head and 128-key tile, every 128-row query tile holding a row that
    shares a block with one of the keys (only rows at or after the tile's first key when causal)."""
    n, T = 1000, 8
    ids = _table_ids(n, [3.0, 60.0, 400.0], 5, 7)
    spans = np.stack([oracle.tile_spans(ids[h], causal) for h in range(ids.shape[0])])
    kspans = np.stack([oracle.tile_spans(ids[h], False) for h in range(ids.shape[0])])
    walked = 0
    for h in range(ids.shape[0]):
        C = oracle.match_counts(ids[h])
        for t in range(T):
            keys = np.arange(t * 128, min(n, t * 128 + 128))
            rows = np.nonzero(C[:, keys].sum(axis=1))[0]
            if causal:
                rows = rows[rows >= t * 128]
            walked += len({int(r) // 128 for r in rows} | {t})
    assert bench.bwd_tc_tiles(spans, kspans, causal) == (bench.kernel_tiles(spans, causal), walked)


def test_profiled_traffic_follows_the_kernel_source(tmp_path, monkeypatch):
    """The committed DRAM traffic is used only while the attention kernel's source and headers
    hash to the value recorded beside it; a change to any of them drops it (reported as null)."""
    srcs = []
    for name in ("kernel.cu", "a.cuh", "b.h"):
        p = tmp_path / name
        p.write_text(f"// {name}\n")
        srcs.append(str(p))
    monkeypatch.setattr(bench, "ATTN_KERNEL_SRC", srcs)
    summary = tmp_path / "summary.md"
    summary.write_text(f"kernel_source_sha256_16: {bench.kernel_source_hash()}\ntraffic_bytes_per_launch: 12345\n")
    monkeypatch.setattr(bench, "PROFILE_SUMMARY", str(summary))
    assert bench.profiled_traffic() == 12345.0
    (tmp_path / "a.cuh").write_text("// a.cuh, changed\n")
    assert bench.profiled_traffic() is None
