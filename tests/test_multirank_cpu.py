"""The multi-GPU path's host logic on CPU: two gloo ranks (one process each,
rendezvous on 127.0.0.1) agree on the slowest rank's time, compute the
whole-job throughput from it, and draw distinct batches.  The path is
data-parallel replicas (weak scaling): no data-path collective exists, only
the timing all-reduce(max) exercised here."""
import os
import socket
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import bench
    from nvfp4_w4a4_quantized_09_b200 import synth
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        local_ms = 10.0 * (rank + 1)                      # rank 1 is the slow one
        total = bench.max_over_ranks(local_ms, world, torch.device("cpu"))
        value = bench.job_throughput(world, 2.0e12, 4, total)
        x = synth.student_t_activations(4, 64, seed=bench.rank_seed(rank))
        gathered = [torch.empty_like(x.float()) for _ in range(world)]
        dist.all_gather(gathered, x.float())
        out[rank] = (total, value, not torch.equal(gathered[0], gathered[1]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_job_value():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world,
                       start_method="spawn", join=True)
    assert set(out.keys()) == {0, 1}
    for r in range(world):
        total, value, distinct = out[r]
        assert total == 20.0                             # max over ranks
        assert abs(value - world * 2.0e12 * 4 / 20e-3 / 1e12) < 1e-9
        assert distinct                                  # each rank its own batch


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(7.5, 1, torch.device("cpu")) == 7.5
    assert bench.job_throughput(1, 1e12, 10, 1000.0) == 10.0
