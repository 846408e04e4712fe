"""The multi-process (one rank per GPU) host logic of bench.py, run as two
gloo ranks on the CPU: each rank works on its own requests (different seeds)
and the job's time is the slowest rank's."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    from compressed_sparse_attention_hca_b200 import workloads as W
    my_ms = [3.0, 5.0][rank]
    total = bench.max_over_ranks(my_ms, dist, torch.device("cpu"))
    # each rank's requests come from its own seed (independent replicas)
    cfg = dict(W.CONFIGS["tiny_prefill_f32"])
    cfg["seed"] += 1000 * rank
    x = W.attention_inputs(cfg, "cpu")
    gathered = [torch.zeros_like(x["Q"]) for _ in range(world)]
    dist.all_gather(gathered, x["Q"])
    out[rank] = (total, bench.job_throughput(world, 4, total), not torch.equal(gathered[0], gathered[1]))
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_own_requests():
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(2, _free_port(), out), nprocs=2, start_method="spawn", join=True)
    for rank in range(2):
        total, value, distinct = out[rank]
        assert total == 5.0                   # max over ranks
        assert value == pytest.approx(2 * 4 / 5e-3)  # whole-job units per second
        assert distinct                       # the ranks' requests differ
