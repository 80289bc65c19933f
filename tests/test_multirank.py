"""The N > 1 host logic of bench.py on two gloo ranks (CPU only): the
max-over-ranks reduction of the device time, the barrier, and the
reference arm running on rank 0 alone."""
import io
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks(3.0 * rank + 1.0, world)
        bench.barrier(world)
        buf = io.StringIO()
        with redirect_stdout(buf):
            rc = bench.run_reference(None, world, rank) if rank != 0 else 0
        with open(os.path.join(out_dir, f"r{rank}.txt"), "w") as f:
            f.write(f"{got} {rc} {len(buf.getvalue())}\n")
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    for rank in range(world):
        got, rc, printed = open(tmp_path / f"r{rank}.txt").read().split()
        assert float(got) == 3.0 * (world - 1) + 1.0   # every rank sees the slowest rank's time
        assert int(rc) == 0
        assert int(printed) == 0                      # only rank 0 prints a bench line
