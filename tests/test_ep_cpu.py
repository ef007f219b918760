"""Expert parallelism's exchange logic on CPU process groups (gloo, world size 2 and 3):
all-gather of the tokens, each rank's share over its expert range and its own rows of the
shared expert, reduce-scatter of the shares.  The ranks' local computation is the oracle
here (the library's kernels need a GPU); the result on every rank must equal the oracle's
output of the whole layer for that rank's tokens."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import sparse_mixture_experts_ffn_b200 as moe
from sparse_mixture_experts_ffn_b200 import inputs

T_RANK = 5


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _cfg(world):
    return inputs.small_config(T=T_RANK * world, H=64, E=7, top_k=3, I=32, I_shared=32, dtype="bf16",
                               w_std=0.1, seed=5)


def _oracle_share(d, e0, e1, top_k):
    """The oracle's version of one rank's fp32 share (used as the local computation)."""
    import oracle
    from conftest import to_oracle

    def f(X, expert_begin, shared_rows):
        assert expert_begin == e0
        xo = to_oracle(X)
        s = oracle.router_scores(xo, to_oracle(d["W_router"]))
        idx, _, w64 = oracle.route(s, top_k)
        mine = (idx >= e0) & (idx < e1)
        idx_l = np.where(mine, idx - e0, 0).astype(np.int32)
        w_l = np.where(mine, w64, 0.0)
        Wgu, Wd = to_oracle(d["W_gate_up"][e0:e1]), to_oracle(d["W_down"][e0:e1])
        out = oracle.moe_tokens(xo, idx_l, w_l, Wgu, Wd)
        s0, s1 = shared_rows
        if s1 > s0:
            out[s0:s1] += oracle.moe_tokens(xo, idx_l, np.zeros_like(w_l), Wgu, Wd, to_oracle(d["Ws_gate_up"]),
                                            to_oracle(d["Ws_down"]), tokens=np.arange(s0, s1))
        return torch.from_numpy(out)
    return f


def _worker(rank, world, port, out):
    import sys
    here = os.path.dirname(os.path.abspath(__file__))
    sys.path.insert(0, here)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from sparse_mixture_experts_ffn_b200.ep import ExpertParallelMoE
        cfg = _cfg(world)
        d = inputs.make_inputs(cfg)
        e0, e1 = moe.expert_range(cfg.E, world, rank)
        layer = ExpertParallelMoE(d["W_router"], d["W_gate_up"][e0:e1], d["W_down"][e0:e1], d["Ws_gate_up"],
                                  d["Ws_down"], top_k=cfg.top_k, local_forward=_oracle_share(d, e0, e1, cfg.top_k),
                                  finish=lambda own, dtype: own)
        x_mine = d["x"][rank * T_RANK:(rank + 1) * T_RANK]
        out[rank] = layer.forward(x_mine).numpy()
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_expert_parallel_exchange_gives_the_whole_layer(world):
    import oracle
    from conftest import to_oracle
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    cfg = _cfg(world)
    d = inputs.make_inputs(cfg)
    ref = oracle.moe_forward(*(to_oracle(d[k]) for k in ("x", "W_router", "W_gate_up", "W_down", "Ws_gate_up",
                                                          "Ws_down")), top_k=cfg.top_k)["y"]
    for r in range(world):
        got = out[r]
        want = ref[r * T_RANK:(r + 1) * T_RANK]
        assert np.abs(got - want).max() <= 1e-12 * np.abs(want).max(), r


@pytest.mark.parametrize("E,world", [(288, 8), (288, 3), (7, 2), (5, 5), (16, 1)])
def test_expert_ranges_partition_the_experts(E, world):
    ranges = [moe.expert_range(E, world, r) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == E
    assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
    sizes = [b - a for a, b in ranges]
    assert min(sizes) >= 1 and max(sizes) - min(sizes) <= 1
