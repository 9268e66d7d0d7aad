"""The benchmark's multi-rank plumbing on the CPU with two gloo ranks: the per-step time it
reports is the slowest rank's, and the reference arm runs on rank 0 only (the others exit
without work).  The GPU arm shards nothing but replicas (no collective on the data path), so
this host logic is all that runs across ranks."""
import contextlib
import io
import multiprocessing as mp
import os
import socket
import sys
from pathlib import Path

ROOT = Path(__file__).resolve().parents[1]


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, port: int, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE="2",
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, str(ROOT))
    import datetime

    import torch
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=2, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        slowest = bench.max_over_ranks(10.0 + 5.0 * rank, torch.device("cpu"))
        out = io.StringIO()
        if rank == 1:   # a non-zero rank of the reference arm prints nothing and returns
            with contextlib.redirect_stdout(out):
                bench.run_reference(bench.parse(["--impl", "reference", "--gpus", "2"]))
        dist.barrier()
        q.put((rank, slowest, out.getvalue()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_report_the_slowest_and_one_reference_line():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[1] for r in res] == [15.0, 15.0]      # both ranks see the slower rank's time
    assert res[1][2] == ""                           # rank 1 of the reference arm: no output
