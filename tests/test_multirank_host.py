"""The benchmark's multi-rank host logic on CPU with the gloo backend,
world size 2: timings combine as the maximum over ranks, the job rate counts
every rank's units, and the reference arm runs on rank 0 only.  No GPU."""
import io
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        mine = [10.0 + 5.0 * rank, 3.0 - rank]          # rank 1 slower in the first value only
        got = bench.max_over_ranks(dist, mine, "cpu")
        rate = bench.job_rate(world, 1000, 4, got[0])
        # the reference arm prints on rank 0 only; other ranks return at once
        os.environ["RANK"] = str(rank)
        os.environ["WORLD_SIZE"] = str(world)
        buf = io.StringIO()
        printed = None
        if rank != 0:
            with redirect_stdout(buf):
                bench.run_reference(type("A", (), {"steps": 1, "warmup": 3})(), bench.WORKLOADS["modal32k"])
            printed = buf.getvalue()
        dist.barrier()
        with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
            f.write(repr((got, rate, printed)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_combine_as_maximum(tmp_path):
    import torch.multiprocessing as mp
    port = free_port()
    mp.spawn(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    res = [eval(open(tmp_path / f"rank{r}.txt").read()) for r in range(2)]
    for got, rate, _ in res:
        assert got == [15.0, 3.0]                       # element-wise maximum over both ranks
        assert rate == pytest.approx(2 * 1000 * 4 / 0.015)
    assert res[1][2] == ""                              # rank 1 printed nothing for the reference arm


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(None, [2.5, 7], "cpu") == [2.5, 7.0]
    assert bench.job_rate(1, 10, 3, 1000.0) == 30.0
