"""Multi-rank host logic of bench.py on CPU: two gloo ranks (no GPU).

The decode step shards by batch with no data-path collective; the only
cross-rank operations are the barrier around the timed region and the
max-over-ranks of the measured times.  These run here as two processes.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from synthetic import config, make_inputs
        # every rank joins the same collectives in the same order
        dist.barrier()
        got = bench.max_over_ranks(1.5 + rank, world, torch.device("cpu"))
        cfg = config(1)
        mine = config(1, seed=bench.rank_seed(cfg.seed, rank), B=1, head_dim=64)
        inp = make_inputs(mine, lengths=[256])
        dist.barrier()
        out[rank] = (got, mine.seed, int(inp.q.astype("int64").sum()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_and_shards():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    assert set(res) == {0, 1}
    # the slowest rank's time on every rank
    assert res[0][0] == pytest.approx(2.5) and res[1][0] == pytest.approx(2.5)
    # each rank decodes its own batch: distinct seeds, distinct inputs
    assert res[0][1] != res[1][1]
    assert res[0][2] != res[1][2]


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.25, 1, torch.device("cpu")) == 3.25
    assert bench.rank_seed(100, 0) == 100
