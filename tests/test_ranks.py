"""Host logic of the multi-rank bench path, on CPU: two gloo ranks (no GPU).

The fine stage has no exchange step, so N GPUs run N independent replicas: each
rank draws its own seeded problem, and the ranks' timings are combined as the
maximum over ranks (one all-reduce) before rank 0 prints the line.
"""
from __future__ import annotations

import json
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str) -> None:
    sys.path.insert(0, ROOT)
    import bench

    torch.distributed.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                                         world_size=world, timeout=__import__("datetime").timedelta(seconds=60))
    try:
        got = bench.max_over_ranks([1.0 + rank, 5.0 - rank, 0.25 * (rank + 1)], "cpu")
        cfg = bench.problem_config(rank)
        small = bench.problem_config(rank, heads=8)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"max": got, "seed": cfg.seed, "H": cfg.H, "small_H": small.H, "small_seed": small.seed}, f)
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks_combine_timings_and_draw_distinct_problems(tmp_path):
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    r = [json.load(open(tmp_path / f"rank{i}.json")) for i in range(2)]
    for x in r:
        assert x["max"] == [2.0, 5.0, 0.5]  # the max over ranks, on every rank
    assert [x["seed"] for x in r] == [0, 1]  # an independent problem per rank
    assert r[0]["H"] == r[1]["H"] == 40 and r[0]["small_H"] == 8 and r[1]["small_seed"] == 1


def test_single_process_reduction_is_the_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert not torch.distributed.is_initialized()
    assert bench.max_over_ranks([3.0, 1.5], "cpu") == [3.0, 1.5]


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    """Under torchrun the oracle arm runs and prints on rank 0 alone; the other
    ranks return at once without work or output."""
    sys.path.insert(0, ROOT)
    import bench

    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("LOCAL_RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1"])
    bench.main()
    assert capsys.readouterr().out == ""


def test_bench_bitmaps_are_the_oracle_format():
    """The bench's bitmap input (the routed lists as packed words) is the format the
    oracle defines: the same words as the lists' BSR rows written out as bitmaps."""
    import numpy as np

    import bench
    import oracle
    import synth

    for nq in (37, 64, 624):
        idx = np.sort(synth.random_topk(nq, 1, 2, nq, 9), axis=-1).astype(np.int32)
        got = bench.lists_to_bitmask(torch.from_numpy(idx)).numpy().view(np.uint32)
        want = oracle.bsr_to_bitmask(*oracle.lists_to_bsr(idx), 1, 2, nq)
        assert np.array_equal(got, want)
