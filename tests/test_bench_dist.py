"""Host logic of bench.py's multi-rank mode on CPU ranks (gloo, world size 2).

bench.py runs one replica of the workload per rank; the job time is the
maximum of the per-rank device times and the job rate counts every rank's
tokens. The reference arm runs on rank 0 only.
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


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_dir):
    import datetime
    import io
    import contextlib
    import types
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # per-rank step and attention times; rank 1 is the slower on the first
        mine = [1.5 + rank, 0.75 - 0.25 * rank]
        got = bench.max_over_ranks(mine, dist, torch.device("cpu"), world)
        rate = bench.whole_job_rate(world, 64, got[0])
        # the reference arm: only rank 0 works and prints
        args = types.SimpleNamespace(workload="v3", steps=1, warmup=0, gpus=world)
        buf = io.StringIO()
        if rank != 0:
            with contextlib.redirect_stdout(buf):
                rc = bench.run_reference(args, rank, world)
        else:
            rc = 0
        with open(os.path.join(out_dir, f"r{rank}.txt"), "w") as f:
            f.write(f"{got[0]} {got[1]} {rate} {rc} {len(buf.getvalue())}\n")
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_rate_gloo(tmp_path):
    world = 2
    port = _free_port()
    mp.start_processes(_worker, args=(world, port, str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    for r in range(world):
        t_step, t_attn, rate, rc, printed = (tmp_path / f"r{r}.txt").read_text().split()
        assert float(t_step) == pytest.approx(2.5)      # max(1.5, 2.5)
        assert float(t_attn) == pytest.approx(0.75)     # max(0.75, 0.5)
        assert float(rate) == pytest.approx(2 * 64 / 2.5e-3)
        assert int(rc) == 0
        assert int(printed) == 0                        # non-zero ranks print nothing


def test_single_rank_untouched():
    import bench
    assert bench.max_over_ranks([3.0, 1.0], None, None, 1) == [3.0, 1.0]
    assert bench.whole_job_rate(1, 64, 1.0) == pytest.approx(64000.0)
