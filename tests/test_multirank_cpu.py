"""The multi-rank logic of bench.py on CPU: gloo, world size 2.  Every rank is an
independent replica on its own tokens; the job time is the slowest rank's."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from sparse_mixture_experts_ffn_b200 import inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        elapsed = 10.0 + 5.0 * rank  # rank 1 is the slow one
        got = bench.max_over_ranks(elapsed, dist, torch.device("cpu"))
        cfg = bench.rank_config(inputs.small_config(T=8, H=64, E=8, top_k=2, I=128, I_shared=128), rank)
        x, _, _ = inputs.make_routing_inputs(cfg)
        out[rank] = (got, float(x.float().sum()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time_and_own_tokens():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    assert out[0][0] == out[1][0] == 15.0
    assert out[0][1] != out[1][1]  # different tokens per rank
    base = inputs.small_config(T=8, H=64, E=8, top_k=2, I=128, I_shared=128)
    assert out[0][1] == float(inputs.make_routing_inputs(base)[0].float().sum())  # rank 0 = the workload


def test_weak_scaling_value():
    # 2 ranks x 4 tokens x 10 steps in 2 ms -> 40 000 tokens/s
    assert bench.job_tokens_per_s(4, 2, 10, 2.0) == pytest.approx(40000.0)
    assert bench.max_over_ranks(3.0, None, None) == 3.0
