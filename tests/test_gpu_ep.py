"""Expert parallelism on one GPU: the ranks' shares (moe_layer_forward_ep), run one after
another with each rank's slice of the expert weights, added by moe_layer_sum_partials, must
give the layer's output (oracle tolerance), with the routing of every share bit-exact."""
import numpy as np
import pytest
import torch

import sparse_mixture_experts_ffn_b200 as moe
from helpers import assert_routing_exact, assert_y_close, oracle_routing, oracle_y, tile_class_tokens, to_device
from sparse_mixture_experts_ffn_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _library():
    from sparse_mixture_experts_ffn_b200 import build
    build.build()
    moe.load_library()


def shares(d, cfg, world, **kw):
    """Each rank's share over all T tokens, rank r taking the shared expert on its slice."""
    T = cfg.T
    parts, routings = [], []
    for r in range(world):
        e0, e1 = moe.expert_range(cfg.E, world, r)
        rows = (r * T // world, (r + 1) * T // world)
        part, rt = moe.moe_layer_forward_ep(d["x"], d["W_router"], d["W_gate_up"][e0:e1].contiguous(),
                                            d["W_down"][e0:e1].contiguous(), d.get("Ws_gate_up"), d.get("Ws_down"),
                                            top_k=cfg.top_k, expert_begin=e0, shared_rows=rows,
                                            router_bias=d.get("bias"), routing=True, **kw)
        parts.append(part)
        routings.append(rt)
    y = moe.sum_partials(parts, torch.empty(T, cfg.H, dtype=d["x"].dtype, device=d["x"].device))
    return y, parts, routings


CASES = [
    dict(T=300, H=256, E=16, top_k=4, I=256, I_shared=256, world=2),    # 128-token tiles (x_perm gather)
    dict(T=3, H=512, E=16, top_k=4, I=128, I_shared=128, world=4),      # 16-token tiles, split gate/up
    dict(T=700, H=256, E=8, top_k=4, I=256, I_shared=128, world=3),     # 256-token down tiles, uneven ranges
    dict(T=200, H=512, E=40, top_k=6, I=384, I_shared=0, world=5),      # no shared expert
    dict(T=700, H=256, E=8, top_k=4, I=256, I_shared=256, world=3),     # tiles over pairs of SMs
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "T{T}_E{E}_G{world}".format(**c))
def test_shares_add_up_to_the_layer(case):
    case = dict(case)
    world = case.pop("world")
    cfg = inputs.small_config(**case)
    d = to_device(inputs.make_inputs(cfg, "cuda", shared=cfg.I_shared > 0))
    y, parts, routings = shares(d, cfg, world)
    torch.cuda.synchronize()
    ref = oracle_routing(d, cfg.top_k)
    for rt in routings:
        assert_routing_exact(rt, ref, cfg.E)
    assert_y_close(y, oracle_y(d, ref), f"{world} shares")
    # each share holds only its experts' contributions: a share without the shared expert
    # and without routed tokens is exactly zero
    y_full, _ = moe.moe_layer_forward(d["x"], d["W_router"], d["W_gate_up"], d["W_down"], d.get("Ws_gate_up"),
                                      d.get("Ws_down"), top_k=cfg.top_k)
    assert_y_close(y, oracle_y(d, ref), "shares")
    diff = (y.float() - y_full.float()).abs().max().item()
    assert diff <= 2e-2 * y_full.float().abs().max().item()


def test_a_share_of_experts_no_token_chose_is_zero():
    cfg = inputs.small_config(T=40, H=256, E=16, top_k=2, I=128, I_shared=128)
    d = inputs.make_inputs(cfg, "cuda")
    b = torch.full((cfg.E,), -30.0)
    b[:8] = 0.0  # no token can choose experts 8..15
    d["bias"] = b
    d = to_device(d)
    part, rt = moe.moe_layer_forward_ep(d["x"], d["W_router"], d["W_gate_up"][8:].contiguous(),
                                        d["W_down"][8:].contiguous(), d["Ws_gate_up"], d["Ws_down"],
                                        top_k=cfg.top_k, expert_begin=8, shared_rows=(0, 0),
                                        router_bias=d["bias"], routing=True)
    torch.cuda.synchronize()
    assert int(rt.counts[8:].sum()) == 0
    assert torch.count_nonzero(part) == 0


def test_sum_partials_adds_in_order():
    g = torch.Generator(device="cuda").manual_seed(3)
    parts = [torch.randn(37, 96, generator=g, device="cuda") for _ in range(5)]
    y32 = moe.sum_partials(parts, torch.empty(37, 96, device="cuda"))
    want = parts[0].clone()
    for p in parts[1:]:
        want += p
    assert torch.equal(y32, want)
    yb = moe.sum_partials(parts, torch.empty(37, 96, dtype=torch.bfloat16, device="cuda"))
    assert torch.equal(yb, want.to(torch.bfloat16))


@pytest.mark.parametrize("name,world", [("decode_t4", 8), ("prefill_t4096", 8)])
def test_full_size_shares(name, world):
    """The decode and prefill workloads split over 8 ranks (36 experts each)."""
    cfg = inputs.CONFIGS[name]
    d = to_device(inputs.make_inputs(cfg, "cuda"))
    y, parts, routings = shares(d, cfg, world)
    torch.cuda.synchronize()
    ref = oracle_routing(d, cfg.top_k)
    for rt in routings:
        assert_routing_exact(rt, ref, cfg.E)
    tokens = np.arange(cfg.T) if cfg.T <= 128 else tile_class_tokens(ref, cfg.T, cfg.top_k, 20, cfg.seed)
    y_ref = oracle_y(d, ref, tokens=tokens)
    assert_y_close(y[torch.as_tensor(tokens, device=y.device)], y_ref, name + " shares")
