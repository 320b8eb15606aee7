"""The multi-rank path of bench.py on CPU: two gloo ranks on 127.0.0.1 take disjoint token rows and agree
on the slowest rank's time, from which the whole-job throughput is formed (no GPU, no data-path
collective: the layer runs as independent replicas)."""

import json
import os
import socket
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        T, steps = 8, 5
        local_ms = [12.5, 20.0][rank]                    # rank 1 is the slower one
        total = bench.max_over_ranks(local_ms, dist, "cpu")
        rows = list(range(bench.rank_first_row(rank, T), bench.rank_first_row(rank, T) + T))
        gathered = [None] * world
        dist.all_gather_object(gathered, rows)
        with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
            f.write(f"{total} {bench.job_tokens_per_s(world, T, steps, total)} {json.dumps(gathered)}\n")
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    lines = [open(tmp_path / f"rank{r}.txt").read().split(" ", 2) for r in range(world)]
    for total, value, rows in lines:
        assert float(total) == 20.0                       # both ranks report the slowest rank's time
        assert float(value) == pytest.approx(2 * 8 * 5 / 0.020)
        ranks_rows = json.loads(rows)
        assert set(ranks_rows[0]).isdisjoint(ranks_rows[1]) and len(ranks_rows[0]) == 8


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.rank_first_row(0, 2048) == 0
