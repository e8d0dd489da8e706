"""The multi-replica host logic of bench.py on CPU: two gloo ranks take the
maximum of their timings, and the whole-job throughput scales with the ranks
(weak scaling: each rank runs its own canvases)."""

import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        # rank r "measured" 10 + r ms for the device pass and 20 - r ms end to end
        got = bench.max_over_ranks([10.0 + rank, 20.0 - rank], world, torch.device("cpu"))
        with open(os.path.join(out_dir, f"r{rank}.txt"), "w") as f:
            f.write(" ".join(repr(v) for v in got))
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks_take_the_max(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn")
    for r in range(world):
        vals = [float(v) for v in (tmp_path / f"r{r}.txt").read_text().split()]
        assert vals == [11.0, 20.0]


def test_single_rank_passes_values_through():
    assert bench.max_over_ranks([3.5, 7], 1, None) == [3.5, 7.0]


def test_throughput_is_weak_scaling():
    # one replica: 256 tokens per 8-pass block, 200 passes in 1.6 s -> 4000 tok/s
    one = bench.canvas_throughput(1, 1, 256, 200, 8, 1600.0)
    assert one == pytest.approx(4000.0)
    # two replicas taking the same time finalise twice the tokens
    assert bench.canvas_throughput(2, 1, 256, 200, 8, 1600.0) == pytest.approx(2 * one)
