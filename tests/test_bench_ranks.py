"""bench.py with more than one rank: two gloo processes on the CPU stand in for two GPUs.
Each rank reports its own time; every rank must end with the slowest rank's time, and the
whole-job value counts both ranks' work over that time."""
import os
import socket

import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(100.0 + 25.0 * rank, "cpu")
        with open(os.path.join(out_dir, f"r{rank}.txt"), "w") as f:
            f.write(repr(ms))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    got = [float((tmp_path / f"r{r}.txt").read_text()) for r in range(world)]
    assert got == [125.0, 125.0]


def test_one_rank_keeps_its_own_time_and_the_value_counts_every_rank():
    assert bench.max_over_ranks(3.5, "cpu") == 3.5        # no process group
    # 2 TFLOP of work per rank and step, 4 ranks, 8 ms per step: 1000 TFLOP/s for the job
    assert abs(bench.whole_job_tflops(2e12, 4, 8.0) - 1000.0) < 1e-9
