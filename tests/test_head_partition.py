"""One problem split over ranks by heads, on CPU (no GPU): two gloo ranks.

Every (batch, head) is independent given the (delta, u) table, so a head partition needs no
exchange step. Each rank takes whole GQA groups (head_partition) and draws only its rows of the
table (plsh_draw_table_heads, the counters of its global heads). The ranks' slices, gathered over
gloo, must equal the whole problem's table bit for bit, and the oracle's bin ids, boundary masks,
b_max and tile windows built from each slice must equal the whole problem's rows.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
import workloads


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_head_partition_keeps_gqa_groups_whole():
    from alibi_positional_lsh_b200 import head_partition
    for H, H_kv in ((16, 8), (32, 8), (40, 8), (8, 8), (12, 3)):
        for world in (1, 2, 3, 4, 8):
            parts = [head_partition(H, H_kv, world, r) for r in range(world)]
            assert parts[0][0] == 0 and parts[-1][1] == H
            for (a0, a1), (b0, b1) in zip(parts, parts[1:]):
                assert a1 == b0
            group = H // H_kv
            for h0, h1 in parts:
                assert h0 % group == 0 and h1 % group == 0        # whole groups only
            sizes = [h1 - h0 for h0, h1 in parts]
            assert max(sizes) - min(sizes) <= group               # as even as whole groups allow
    with pytest.raises(ValueError):
        head_partition(16, 5, 2, 0)


def test_draw_table_heads_slices_the_whole_table():
    from alibi_positional_lsh_b200 import plsh_draw_table_heads
    w = workloads.WORKLOADS["long_n128k"]
    sig = np.array(w.sigmas())
    whole = oracle.draw_table(w.seed, sig, w.s)
    for h0, h1 in ((0, 5), (5, 40), (17, 18)):
        t = np.empty((h1 - h0, w.s, 2))
        plsh_draw_table_heads(w.seed, h0, h1 - h0, w.s, sig[h0:h1], t)
        assert t.tobytes() == whole[h0:h1].tobytes()


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from alibi_positional_lsh_b200 import head_partition, plsh_draw_table_heads
        w = workloads.WORKLOADS["qwen3_0p6b_n32k"]
        sig = np.array(w.sigmas())
        h0, h1 = head_partition(w.H, w.H_kv, world, rank)
        mine = np.empty((h1 - h0, w.s, 2))
        plsh_draw_table_heads(w.seed, h0, h1 - h0, w.s, sig[h0:h1], mine)
        sizes = [None] * world
        torch.distributed.all_gather_object(sizes, (h0, h1))
        gathered = [torch.empty(((b - a), w.s, 2), dtype=torch.float64) for a, b in sizes]
        torch.distributed.all_gather(gathered, torch.from_numpy(mine))
        if rank == 0:
            np.save(out, torch.cat(gathered).numpy())
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks_tables_concatenate_to_the_whole(tmp_path):
    world = 2
    out = str(tmp_path / "table.npy")
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
    w = workloads.WORKLOADS["qwen3_0p6b_n32k"]
    whole = oracle.draw_table(w.seed, w.sigmas(), w.s)
    got = np.load(out)
    assert got.tobytes() == whole.tobytes()
    # the window inputs built from the slices are the whole problem's rows (oracle, a short prefix of n)
    n = 4096
    ids_whole = oracle.bin_ids(whole, n)
    from alibi_positional_lsh_b200 import head_partition
    for rank in range(world):
        h0, h1 = head_partition(w.H, w.H_kv, world, rank)
        ids = oracle.bin_ids(got[h0:h1], n)
        assert np.array_equal(ids, ids_whole[h0:h1])
        for h in range(h1 - h0):
            assert np.array_equal(oracle.boundary_bits(ids[h]), oracle.boundary_bits(ids_whole[h0 + h]))
            assert oracle.bmax(ids[h]) == oracle.bmax(ids_whole[h0 + h])
            assert np.array_equal(oracle.tile_spans(ids[h], True), oracle.tile_spans(ids_whole[h0 + h], True))
