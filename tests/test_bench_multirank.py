"""bench.py's multi-rank host logic on CPU: two gloo ranks (no GPU).

With N ranks every rank solves its own problem of the headline shape (weak
scaling, no data-path collective); the step time is the max over ranks and
the whole-job value counts every rank's tokens. The reference arm runs on
rank 0 alone; the other ranks exit without work.
"""
import json
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import bench
import workloads


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 1.0 + 2.5 * rank                      # rank 1 is the slow one
        ms_max = bench.dist_max(local_ms, world)
        bench.barrier(world)
        w = workloads.WORKLOADS[workloads.HEADLINE]
        wr = bench.rank_workload(w, rank)
        res = {"ms_max": ms_max, "seed": wr.seed, "shape": [wr.B, wr.H, wr.H_kv, wr.n, wr.d, wr.s],
               "value": bench.job_value(w.B * w.n, world, ms_max)}
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump(res, f)
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks_max_time_and_whole_job_value(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    w = workloads.WORKLOADS[workloads.HEADLINE]
    for r in res:
        assert r["ms_max"] == pytest.approx(3.5)         # the slowest rank's time, on every rank
        assert r["value"] == pytest.approx(w.B * w.n * world / 3.5e-3)
        assert r["shape"] == [w.B, w.H, w.H_kv, w.n, w.d, w.s]
    assert res[0]["seed"] != res[1]["seed"]              # independent problems


def test_single_rank_needs_no_process_group():
    assert bench.dist_max(2.0, 1) == 2.0
    bench.barrier(1)
    assert bench.job_value(1000, 1, 1.0) == pytest.approx(1e6)


def test_reference_arm_runs_on_rank_0_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    bench.main(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"])
    assert capsys.readouterr().out == ""


def test_reference_line_carries_the_contract_keys(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    bench.main(["--impl", "reference", "--workload", "single_head_n1024", "--steps", "1", "--warmup", "3",
                "--cpu-seconds", "0.5"])
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "query-tokens/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["config"] == bench.config_of(workloads.WORKLOADS["single_head_n1024"], 1)
