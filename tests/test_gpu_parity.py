"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the same seeded
inputs.  Expert indices, counts, offsets and the permutation must match bit for bit;
outputs within max|err| <= 2e-2 * max|y_ref| and relative L2 <= 1e-2."""
import numpy as np
import pytest
import torch

import sparse_mixture_experts_ffn_b200 as moe
from helpers import (assert_routing_exact, assert_y_close, oracle_routing, oracle_y, tile_class_tokens,
                     to_device)
from sparse_mixture_experts_ffn_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _library():
    from sparse_mixture_experts_ffn_b200 import build
    build.build()
    moe.load_library()


def run(d, top_k, **kw):
    y, r = moe.moe_layer_forward(d["x"], d["W_router"], d["W_gate_up"], d["W_down"], d.get("Ws_gate_up"),
                                 d.get("Ws_down"), top_k=top_k, router_bias=d.get("bias"), **kw)
    return y, r


def check_full(d, top_k, what):
    ws = moe.alloc_workspace(moe.make_shape(d["x"].shape[0], d["x"].shape[1], d["W_router"].shape[0],
                                            d["W_gate_up"].shape[1] // 2,
                                            0 if d.get("Ws_gate_up") is None else d["Ws_gate_up"].shape[0] // 2,
                                            top_k, d["x"].dtype), d["x"].device)
    y, r = run(d, top_k, workspace=ws)
    assert moe.check_status(ws) == moe.MOE_OK
    ref = oracle_routing(d, top_k)
    assert_routing_exact(r, ref, d["W_router"].shape[0])
    y_ref = oracle_y(d, ref)
    return assert_y_close(y, y_ref, what), moe.route_stats(ws)


SMALL = [
    dict(T=300, H=256, E=16, top_k=4, I=256, I_shared=256),
    dict(T=1, H=256, E=16, top_k=4, I=128, I_shared=128),
    dict(T=129, H=384, E=12, top_k=1, I=128, I_shared=256),
    dict(T=77, H=256, E=8, top_k=8, I=128, I_shared=128),
    dict(T=200, H=512, E=40, top_k=6, I=384, I_shared=0),
    dict(T=1000, H=256, E=64, top_k=8, I=128, I_shared=128),
    # router reduction split over blocks: 2 chunks; 3 chunks with a ragged last slice and a
    # ragged last expert tile
    dict(T=30, H=1024, E=96, top_k=6, I=128, I_shared=128),
    dict(T=3, H=2176, E=200, top_k=8, I=128, I_shared=128),
    # 16-token tiles (both GEMMs in one launch) without a shared expert, the gate/up
    # reduction split: fewer items than blocks, so blocks start on down tiles and wait
    dict(T=5, H=256, E=32, top_k=4, I=256, I_shared=0),
    # router reduction split over 4 chunks for 100 tokens: the partials added by a separate
    # grid-wide kernel rather than by each tile's last block
    dict(T=100, H=1024, E=96, top_k=6, I=128, I_shared=128),
    # 256-token tiles (about 350 tokens per expert: one full and one ragged tile each)
    dict(T=700, H=256, E=8, top_k=4, I=256, I_shared=128),
    # 256 x 256 tiles over pairs of SMs (widths multiples of 256): ragged token tiles, a
    # shared expert of one weight tile; no shared expert and two weight tiles per expert
    dict(T=700, H=256, E=8, top_k=4, I=256, I_shared=256),
    dict(T=1100, H=512, E=6, top_k=2, I=512, I_shared=0),
]


@pytest.mark.parametrize("sz", SMALL, ids=lambda s: "T{T}_H{H}_E{E}_k{top_k}_I{I}_Is{I_shared}".format(**s))
def test_small_bf16_parity(sz):
    cfg = inputs.small_config(**sz)
    d = to_device(inputs.make_inputs(cfg, "cuda", shared=sz["I_shared"] > 0))
    check_full(d, cfg.top_k, cfg.name)


LIMIT_CASES = [
    # 16-token tiles with the gate/up reduction split (the last slice applies the clamp)
    dict(T=3, H=512, E=16, top_k=4, I=128, I_shared=128),
    # 128-token gate/up tiles (staged epilogue), 128- and 256-token down tiles
    dict(T=300, H=256, E=16, top_k=4, I=256, I_shared=128),
    dict(T=700, H=256, E=8, top_k=4, I=256, I_shared=128),
    dict(T=45, H=72, E=10, top_k=3, I=40, I_shared=24, dtype="f32", r_std=0.1),
]


@pytest.mark.parametrize("sz", LIMIT_CASES, ids=lambda s: "T{T}_H{H}_E{E}".format(**s) + s.get("dtype", ""))
def test_swiglu_limits(sz):
    """SwiGLU limits 0.3 (routed) and 0.2 (shared): gate <= L, up in [-L, L] before SiLU*up."""
    cfg = inputs.small_config(**sz)
    d = to_device(inputs.make_inputs(cfg, "cuda"))
    y, r = run(d, cfg.top_k, swiglu_limit=0.3, swiglu_limit_shared=0.2)
    ref = oracle_routing(d, cfg.top_k)
    assert_routing_exact(r, ref, cfg.E)
    y_ref = oracle_y(d, ref, swiglu_limit=0.3, swiglu_limit_shared=0.2)
    assert_y_close(y, y_ref, "swiglu limits")
    y_free = oracle_y(d, ref)
    assert np.abs(y_ref - y_free).max() > 0.05 * np.abs(y_free).max()  # the clamps are active


SIGMOID_CASES = [
    dict(T=257, H=256, E=32, top_k=4, I=128, I_shared=128),                  # tensor-core scores
    dict(T=3, H=2176, E=200, top_k=8, I=128, I_shared=128),                  # split reduction
    dict(T=45, H=72, E=10, top_k=3, I=40, I_shared=24, dtype="f32", r_std=0.1),  # fp64 scores
]


@pytest.mark.parametrize("with_bias", [False, True])
@pytest.mark.parametrize("sz", SIGMOID_CASES, ids=lambda s: "T{T}_H{H}_E{E}".format(**s) + s.get("dtype", ""))
def test_sigmoid_router(sz, with_bias):
    """The router as configured: p = sigma32(s), bias for the selection only, weights
    3 * p / sum p; indices, counts, offsets and perm bit-exact against the oracle."""
    cfg = inputs.small_config(**sz)
    d = inputs.make_inputs(cfg, "cuda")
    if with_bias:
        d["bias"] = torch.linspace(-0.2, 0.2, cfg.E, dtype=torch.float32)
    d = to_device(d)
    y, r = run(d, cfg.top_k, router="sigmoid", routed_scaling_factor=3.0)
    ref = oracle_routing(d, cfg.top_k, router="sigmoid", scale=3.0)
    assert_routing_exact(r, ref, cfg.E)
    assert_y_close(y, oracle_y(d, ref), "sigmoid router")
    assert torch.allclose(r.topk_w.sum(1), torch.full((cfg.T,), 3.0, device=r.topk_w.device), rtol=1e-5)


FP32_ROUTER_CASES = [
    dict(T=257, H=256, E=32, top_k=4, I=128, I_shared=128),    # unsplit tensor-core scores
    dict(T=3, H=2176, E=200, top_k=8, I=128, I_shared=128),    # reduction split over blocks
    dict(T=60, H=1024, E=96, top_k=6, I=128, I_shared=128),    # split, grid-wide reduce kernel
]


@pytest.mark.parametrize("router", ["softmax", "sigmoid"])
@pytest.mark.parametrize("sz", FP32_ROUTER_CASES, ids=lambda s: "T{T}_H{H}_E{E}".format(**s))
def test_fp32_router_weights(sz, router):
    """bf16 layer with fp32 router weights (need_fp32_gate): the scores are the exact dots of
    bf16 tokens and fp32 weights; indices bit-exact against the oracle."""
    cfg = inputs.small_config(**sz)
    d = inputs.make_inputs(cfg, "cuda")
    g = torch.Generator().manual_seed(cfg.seed + 31)
    d["W_router"] = torch.randn(cfg.E, cfg.H, generator=g) * cfg.r_std  # fp32, not bf16-rounded
    if router == "sigmoid":
        d["bias"] = torch.linspace(-0.1, 0.1, cfg.E, dtype=torch.float32)
    d = to_device(d)
    scale = 3.0 if router == "sigmoid" else 1.0
    y, r = run(d, cfg.top_k, router=router, routed_scaling_factor=scale)
    ref = oracle_routing(d, cfg.top_k, router=router, scale=scale)
    assert_routing_exact(r, ref, cfg.E)
    assert_y_close(y, oracle_y(d, ref), "fp32 router weights")


EDGE_CASES = [
    dict(T=40, H=256, E=1024, top_k=8, I=128, I_shared=128),   # the most experts: fp64 router kernel
    dict(T=33, H=256, E=513, top_k=4, I=128, I_shared=0),      # one past the tensor-core router
    dict(T=33, H=256, E=512, top_k=4, I=128, I_shared=128),    # the largest tensor-core router
    dict(T=50, H=256, E=1, top_k=1, I=128, I_shared=128),      # a single expert
    dict(T=3, H=512, E=16, top_k=4, I=256, I_shared=0),        # split decode GEMM, no shared expert
    dict(T=2, H=128, E=16, top_k=4, I=128, I_shared=128),      # two k-blocks: the split stops at 2
]


@pytest.mark.parametrize("router", ["softmax", "sigmoid"])
@pytest.mark.parametrize("sz", EDGE_CASES, ids=lambda s: "T{T}_E{E}_k{top_k}_Is{I_shared}".format(**s))
def test_edge_shapes(sz, router):
    cfg = inputs.small_config(**sz)
    d = to_device(inputs.make_inputs(cfg, "cuda", shared=sz["I_shared"] > 0))
    scale = 3.0 if router == "sigmoid" else 1.0
    shape = moe.make_shape(cfg.T, cfg.H, cfg.E, cfg.I, cfg.I_shared, cfg.top_k, torch.bfloat16)
    ws = moe.alloc_workspace(shape, "cuda")
    y, r = run(d, cfg.top_k, workspace=ws, router=router, routed_scaling_factor=scale)
    assert moe.check_status(ws) == moe.MOE_OK
    ref = oracle_routing(d, cfg.top_k, router=router, scale=scale)
    assert_routing_exact(r, ref, cfg.E)
    assert_y_close(y, oracle_y(d, ref), f"edge {sz} {router}")


def test_small_bf16_with_router_bias():
    cfg = inputs.small_config(T=257, H=256, E=32, top_k=4, I=128, I_shared=128)
    d = inputs.make_inputs(cfg, "cuda")
    d["bias"] = torch.linspace(-1.0, 1.0, cfg.E, dtype=torch.float32)
    check_full(to_device(d), cfg.top_k, "bias")


def test_tiny_fp32_workload():
    cfg = inputs.CONFIGS["tiny_f32_t64"]
    d = to_device(inputs.make_inputs(cfg, "cuda"))
    check_full(d, cfg.top_k, cfg.name)


def test_fp32_ragged_sizes():
    cfg = inputs.small_config(T=45, H=72, E=10, top_k=3, I=40, I_shared=24, dtype="f32", r_std=0.1)
    d = to_device(inputs.make_inputs(cfg, "cuda"))
    check_full(d, cfg.top_k, "fp32 ragged")


def test_group_sizes_at_tile_edges():
    """Top-1 routing forced through the router: expert e gets exactly sizes[e] tokens."""
    sizes = [0, 1, 15, 16, 17, 127, 128, 129, 255, 257, 2, 0]
    E, H, I = len(sizes), 256, 128
    T = sum(sizes)
    owner = np.concatenate([np.full(n, e) for e, n in enumerate(sizes)])
    rng = np.random.default_rng(0)
    owner = owner[rng.permutation(T)]
    x = torch.randn(T, H) * 0.01
    x[torch.arange(T), torch.tensor(owner)] += 4.0  # token t points along axis owner[t]
    Wr = torch.zeros(E, H)
    Wr[torch.arange(E), torch.arange(E)] = 1.0
    cfg = inputs.small_config(T=T, H=H, E=E, top_k=1, I=I, I_shared=I)
    d = inputs.make_inputs(cfg, "cuda")
    d["x"] = x.to(torch.bfloat16)
    d["W_router"] = Wr.to(torch.bfloat16)
    d = to_device(d)
    y, r = run(d, 1)
    assert np.array_equal(r.counts.cpu().numpy(), np.array(sizes))
    ref = oracle_routing(d, 1)
    assert_routing_exact(r, ref, E)
    assert_y_close(y, oracle_y(d, ref), "tile edges")


def test_decode_forward_launch_count():
    """16-token tiles with bf16 weights run five launches: router GEMM, selection, dispatch, one
    launch of both expert GEMMs, combine (the decode shape: 4 tokens, 288 experts, top-8)."""
    cfg = inputs.small_config(T=4, H=512, E=288, top_k=8, I=128, I_shared=128)
    d = to_device(inputs.make_inputs(cfg, "cuda", shared=True))
    ws = moe.alloc_workspace(moe.make_shape(cfg.T, cfg.H, cfg.E, cfg.I, cfg.I_shared, cfg.top_k, torch.bfloat16), "cuda")
    run(d, cfg.top_k, workspace=ws)  # first call: one-time setup launches, if any
    torch.cuda.synchronize()
    n0 = moe.launch_count()
    y, r = run(d, cfg.top_k, workspace=ws)
    torch.cuda.synchronize()
    assert moe.launch_count() - n0 == 5
    assert moe.check_status(ws) == moe.MOE_OK
    ref = oracle_routing(d, cfg.top_k)
    assert_routing_exact(r, ref, cfg.E)
    assert_y_close(y, oracle_y(d, ref), cfg.name)


def test_ties_and_zero_input():
    cfg = inputs.small_config(T=64, H=256, E=16, top_k=4, I=128, I_shared=128)
    d = inputs.make_inputs(cfg, "cuda")
    d["W_router"][7] = d["W_router"][3]   # exact ties between experts 3 and 7
    d["W_router"][12] = d["W_router"][3]
    d["x"][:8] = 0                          # all keys 0: experts 0..3 with weight 1/4
    d = to_device(d)
    y, r = run(d, 4)
    ref = oracle_routing(d, 4)
    assert_routing_exact(r, ref, cfg.E)
    assert np.array_equal(r.topk_idx[:8].cpu().numpy(), np.tile(np.arange(4), (8, 1)))
    assert torch.all(r.topk_w[:8] == 0.25)
    assert torch.all(y[:8] == 0)
    assert_y_close(y, oracle_y(d, ref), "ties")


def test_empty_batch_is_a_no_op():
    cfg = inputs.small_config(T=0, H=256, E=16, top_k=4, I=128, I_shared=128)
    d = to_device(inputs.make_inputs(cfg, "cuda"))
    y, r = run(d, 4)
    assert y.shape == (0, 256)


def test_repeat_runs_are_bitwise_identical():
    cfg = inputs.small_config(T=500, H=256, E=32, top_k=8, I=256, I_shared=256)
    d = to_device(inputs.make_inputs(cfg, "cuda"))
    y1, r1 = run(d, 8)
    y2, r2 = run(d, 8)
    assert torch.equal(y1, y2)
    assert torch.equal(r1.perm, r2.perm) and torch.equal(r1.topk_w, r2.topk_w)


def test_intermediate_activation_matches_oracle():
    """Per-kernel check of the gate/up GEMM + SiLU*up epilogue on the rows of x_perm."""
    import oracle
    from conftest import to_oracle
    cfg = inputs.small_config(T=150, H=256, E=8, top_k=2, I=256, I_shared=128)
    d = to_device(inputs.make_inputs(cfg, "cuda"))
    shape = moe.make_shape(cfg.T, cfg.H, cfg.E, cfg.I, cfg.I_shared, cfg.top_k, torch.bfloat16)
    ws = moe.alloc_workspace(shape, "cuda")
    y, r = run(d, cfg.top_k, workspace=ws)
    torch.cuda.synchronize()
    lay = moe.workspace_layout(shape)
    P = cfg.T * cfg.top_k
    h = ws[lay.h:lay.h + P * cfg.I * 2].view(torch.bfloat16).view(P, cfg.I).float().cpu().numpy()
    perm = r.perm.cpu().numpy()
    idx = r.topk_idx.cpu().numpy()
    xo = to_oracle(d["x"])
    for pos in [0, 1, P // 3, P // 2, P - 1]:
        a = perm[pos]
        t, j = a // cfg.top_k, a % cfg.top_k
        e = idx[t, j]
        ref = oracle.expert_act(xo[t], to_oracle(d["W_gate_up"][e]))
        err = np.abs(h[pos] - ref).max() / np.abs(ref).max()
        assert err < 2e-2, (pos, err)


# ------------------------------------------------------------------------------------
# the full-size workloads
# ------------------------------------------------------------------------------------
FULL = ["decode_t4", "decode_t128", "prefill_t4096", "prefill_t16384_skew"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_workload(name):
    cfg = inputs.CONFIGS[name]
    d = to_device(inputs.make_inputs(cfg, "cuda"))
    shape = moe.make_shape(cfg.T, cfg.H, cfg.E, cfg.I, cfg.I_shared, cfg.top_k, torch.bfloat16)
    ws = moe.alloc_workspace(shape, "cuda")
    y, r = run(d, cfg.top_k, workspace=ws)
    assert moe.check_status(ws) == moe.MOE_OK
    stats = moe.route_stats(ws)
    ref = oracle_routing(d, cfg.top_k)
    assert_routing_exact(r, ref, cfg.E)
    tokens = np.arange(cfg.T) if cfg.T <= 128 else tile_class_tokens(ref, cfg.T, cfg.top_k, 40, cfg.seed)
    y_ref = oracle_y(d, ref, tokens=tokens)
    assert_y_close(y[torch.as_tensor(tokens, device=y.device)], y_ref, name)
    print(name, "route stats", stats)


@pytest.mark.parametrize("name", ["decode_t4", "prefill_t16384_skew"])
def test_full_size_layer_as_configured(name):
    """The last layers as configured: fp32 router weights, sigmoid router with the routing
    factor 3 and a bias for the selection, SwiGLU limits 7 (routed) and 16 (shared)."""
    cfg = inputs.CONFIGS[name]
    d = inputs.make_inputs(cfg, "cuda")
    if d.get("bias") is None:
        d["bias"] = torch.linspace(-0.05, 0.05, cfg.E, dtype=torch.float32)
    # need_fp32_gate: fp32 router weights
    g = torch.Generator().manual_seed(cfg.seed + 31)
    d["W_router"] = torch.randn(cfg.E, cfg.H, generator=g) * cfg.r_std
    d = to_device(d)
    opts = dict(router="sigmoid", routed_scaling_factor=3.0, swiglu_limit=7.0, swiglu_limit_shared=16.0)
    shape = moe.make_shape(cfg.T, cfg.H, cfg.E, cfg.I, cfg.I_shared, cfg.top_k, torch.bfloat16)
    ws = moe.alloc_workspace(shape, "cuda")
    y, r = run(d, cfg.top_k, workspace=ws, **opts)
    assert moe.check_status(ws) == moe.MOE_OK
    ref = oracle_routing(d, cfg.top_k, router="sigmoid", scale=3.0)
    assert_routing_exact(r, ref, cfg.E)
    tokens = np.arange(cfg.T) if cfg.T <= 128 else tile_class_tokens(ref, cfg.T, cfg.top_k, 20, cfg.seed)
    y_ref = oracle_y(d, ref, tokens=tokens, swiglu_limit=7.0, swiglu_limit_shared=16.0)
    assert_y_close(y[torch.as_tensor(tokens, device=y.device)], y_ref, name + " as configured")
    print(name, "as configured, route stats", moe.route_stats(ws))


# ------------------------------------------------------------------------------------
# FP8 expert weights (E4M3 codes, one E8M0 scale per 128 x 128 block)
# ------------------------------------------------------------------------------------
def fp8_inputs(cfg, shared=True):
    x, Wr, bias = inputs.make_routing_inputs(cfg)
    d = to_device(dict(x=x, W_router=Wr, bias=bias))
    d["fp8"] = inputs.make_fp8_expert_weights(cfg, "cuda", shared=shared)
    return d


def oracle_y_fp8(d, routing, tokens=None, swiglu_limit=0.0, swiglu_limit_shared=0.0):
    import oracle
    from conftest import to_oracle

    def host(pair):
        return None if pair is None else tuple(t.cpu().numpy() for t in pair)

    w = d["fp8"]
    return oracle.moe_tokens_fp8(to_oracle(d["x"]), routing["idx"], routing["w64"], host(w["W_gate_up"]),
                                 host(w["W_down"]), host(w["Ws_gate_up"]), host(w["Ws_down"]), tokens=tokens,
                                 swiglu_limit=swiglu_limit, swiglu_limit_shared=swiglu_limit_shared)


def run_fp8(d, top_k, tokens=None, what="", **kw):
    x = d["x"]
    w = d["fp8"]
    I = w["W_gate_up"][0].shape[1] // 2
    Is = 0 if w.get("Ws_gate_up") is None else w["Ws_gate_up"][0].shape[0] // 2
    ws = moe.alloc_workspace(moe.make_shape(x.shape[0], x.shape[1], d["W_router"].shape[0], I, Is, top_k,
                                            x.dtype), x.device)
    y, r = moe.moe_layer_forward_fp8(x, d["W_router"], w, top_k=top_k, router_bias=d.get("bias"),
                                     workspace=ws, **kw)
    assert moe.check_status(ws) == moe.MOE_OK
    ref = oracle_routing(d, top_k)
    assert_routing_exact(r, ref, d["W_router"].shape[0])
    limits = {k: kw[k] for k in ("swiglu_limit", "swiglu_limit_shared") if k in kw}
    y_ref = oracle_y_fp8(d, ref, tokens=tokens, **limits)
    yt = y if tokens is None else y[torch.as_tensor(tokens, device=y.device)]
    return assert_y_close(yt, y_ref, what)


FP8_CASES = [
    # 16-token tiles, gate/up reduction split in 4 (each slice two k-blocks of one scale block)
    dict(T=3, H=512, E=16, top_k=4, I=128, I_shared=128),
    # 17 scale blocks along H, 200 experts, split reduction with ragged slices
    dict(T=3, H=2176, E=200, top_k=8, I=128, I_shared=128),
    # 128-token tiles; 3 scale blocks along H, 2 row blocks per gate and up half
    dict(T=129, H=384, E=12, top_k=1, I=256, I_shared=256),
    dict(T=300, H=256, E=16, top_k=4, I=256, I_shared=128),
    # long-prefill grouping (the bf16 down GEMM would take 256-token tiles; FP8 keeps 128)
    dict(T=700, H=256, E=8, top_k=4, I=256, I_shared=128),
    # no shared expert, 3 row blocks per half
    dict(T=200, H=512, E=40, top_k=6, I=384, I_shared=0),
    # one scale block along H, split reduction of two k-blocks
    dict(T=2, H=128, E=16, top_k=4, I=128, I_shared=128),
]


@pytest.mark.parametrize("sz", FP8_CASES, ids=lambda s: "T{T}_H{H}_E{E}_k{top_k}_I{I}_Is{I_shared}".format(**s))
def test_fp8_weights_parity(sz):
    cfg = inputs.small_config(**sz)
    d = fp8_inputs(cfg, shared=sz["I_shared"] > 0)
    run_fp8(d, cfg.top_k, what=cfg.name + " fp8")


def test_fp8_weights_with_swiglu_limits():
    cfg = inputs.small_config(T=300, H=256, E=16, top_k=4, I=256, I_shared=128)
    d = fp8_inputs(cfg)
    run_fp8(d, cfg.top_k, what="fp8 limits", swiglu_limit=0.3, swiglu_limit_shared=0.2)


@pytest.mark.parametrize("T", [3, 300])
def test_fp8_subnormal_and_zero_codes(T):
    """Weights made only of E4M3 subnormals (exponent field 0) and zeros, with scales far
    from 1: the output is nonzero only if the conversion keeps the subnormals."""
    cfg = inputs.small_config(T=T, H=256, E=16, top_k=4, I=128, I_shared=128)
    d = fp8_inputs(cfg)
    g = torch.Generator(device="cuda").manual_seed(5)
    for k, (q, sc) in list(d["fp8"].items()):
        codes = torch.randint(0, 8, q.shape, generator=g, device="cuda", dtype=torch.int32)  # m, e = 0
        sign = torch.randint(0, 2, q.shape, generator=g, device="cuda", dtype=torch.int32) << 7
        scale = torch.randint(125, 134, sc.shape, generator=g, device="cuda", dtype=torch.int32)
        d["fp8"][k] = ((codes | sign).to(torch.uint8), scale.to(torch.uint8))
    rel_max, _ = run_fp8(d, cfg.top_k, what="fp8 subnormals")
    y, _ = moe.moe_layer_forward_fp8(d["x"], d["W_router"], d["fp8"], top_k=cfg.top_k, routing=False)
    assert float(y.float().abs().max()) > 0


@pytest.mark.parametrize("name", ["decode_t4", "decode_t128", "prefill_t4096"])
def test_fp8_full_size_workload(name):
    cfg = inputs.CONFIGS[name]
    d = fp8_inputs(cfg)
    if cfg.T <= 128:
        tokens = None
    else:
        tokens = tile_class_tokens(oracle_routing(d, cfg.top_k), cfg.T, cfg.top_k, 20, cfg.seed, tiles=(16, 128))
    run_fp8(d, cfg.top_k, tokens=tokens, what=name + " fp8")


# ------------------------------------------------------------------------------------
# the tensor-core router's error bound
# ------------------------------------------------------------------------------------
def _tc_router_error_ratio(d, top_k):
    """max |s^ - s| / (L 2^-23 ||x|| ||w||) of the tensor-core router score estimates kept in
    the workspace (fp32 accumulation over slices of L products), against the oracle's exact
    scores.  The certified selection assumes this ratio is at most 2."""
    import oracle
    from conftest import to_oracle
    T, H = d["x"].shape
    E = d["W_router"].shape[0]
    shape = moe.make_shape(T, H, E, d["W_gate_up"].shape[1] // 2, d["Ws_gate_up"].shape[0] // 2, top_k,
                           torch.bfloat16)
    ws = moe.alloc_workspace(shape, "cuda")
    y, r = run(d, top_k, workspace=ws)
    assert moe.check_status(ws) == moe.MOE_OK
    torch.cuda.synchronize()
    lay = moe.workspace_layout(shape)
    assert lay.scores_slice > 0
    s_hat = ws[lay.scores:lay.scores + T * E * 8].view(torch.float64).view(T, E).cpu().numpy()
    s = oracle.router_scores(to_oracle(d["x"]), to_oracle(d["W_router"])).astype(np.float64)
    xf, wf = d["x"].double().cpu().numpy(), d["W_router"].double().cpu().numpy()
    bound = lay.scores_slice * 2.0 ** -23 * np.outer(np.linalg.norm(xf, axis=1), np.linalg.norm(wf, axis=1))
    ulp = np.spacing(np.abs(s).astype(np.float32)).astype(np.float64)  # s is already RN32(exact)
    return float(((np.abs(s_hat - s) - 0.5 * ulp) / bound).max()), r, ws


def test_tensor_core_router_error_is_far_inside_the_certified_band():
    cfg = inputs.small_config(T=1024, H=4096, E=288, top_k=8, I=128, I_shared=128)
    d = to_device(inputs.make_inputs(cfg, "cuda"))
    ratio, r, ws = _tc_router_error_ratio(d, cfg.top_k)
    print("tensor-core router error / (L 2^-23 |x||w|):", ratio, moe.route_stats(ws))
    assert ratio < 0.25  # the selection assumes <= 2


def test_tensor_core_router_wide_dynamic_range():
    """Inputs spanning many binades with cancellation: the accumulation error is still
    inside the band and the routing still matches the exact one."""
    cfg = inputs.small_config(T=640, H=1024, E=96, top_k=8, I=128, I_shared=128)
    d = inputs.make_inputs(cfg, "cuda")
    g = torch.Generator().manual_seed(5)
    scale = torch.pow(2.0, torch.randint(-20, 12, (cfg.T, cfg.H), generator=g).float())
    x = (torch.randn(cfg.T, cfg.H, generator=g) * scale)
    x[:, 1::2] = -x[:, 0::2] * (1 + 2.0 ** -7)  # near-cancelling pairs
    d["x"] = x.to(torch.bfloat16)
    d = to_device(d)
    ratio, r, ws = _tc_router_error_ratio(d, cfg.top_k)
    print("wide-range router error ratio:", ratio, moe.route_stats(ws))
    assert ratio < 0.5
    ref = oracle_routing(d, cfg.top_k)
    # the keys of experts chosen for certain come from the fp32-accumulated estimate; with
    # sum|x w| far above |s| their weights are checked at the looser 1e-3
    assert_routing_exact(r, ref, cfg.E, w_tol=1e-3)


def test_decode_tiles_with_popular_experts():
    """16-token tiles (few tokens per expert) with a bias that sends most tokens to four
    experts, so those experts and the shared expert span many tiles."""
    cfg = inputs.small_config(T=90, H=256, E=64, top_k=4, I=256, I_shared=128)
    d = inputs.make_inputs(cfg, "cuda")
    b = torch.zeros(cfg.E, dtype=torch.float32)
    b[:4] = 3.0
    d["bias"] = b
    d = to_device(d)
    y, r = run(d, cfg.top_k)
    assert int(r.counts.max()) > 40
    ref = oracle_routing(d, cfg.top_k)
    assert_routing_exact(r, ref, cfg.E)
    assert_y_close(y, oracle_y(d, ref), "popular experts, 16-token tiles")


def test_bounded_wait_times_out_with_a_readable_status():
    """A wait on a barrier that nothing completes gives up (about 2 s), the status word
    reads MOE_ERR_DEVICE_TIMEOUT, and the context still runs the layer correctly."""
    import ctypes
    import time
    lib = moe.load_library()
    lib.moe_layer_selftest_wait_timeout.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    lib.moe_layer_selftest_wait_timeout.restype = ctypes.c_int
    ws = torch.zeros(1 << 12, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    t0 = time.perf_counter()
    rc = lib.moe_layer_selftest_wait_timeout(ctypes.c_void_p(ws.data_ptr()), ws.numel(),
                                             ctypes.c_void_p(stream.cuda_stream))
    assert rc == moe.MOE_OK
    assert moe.check_status(ws) == 5  # MOE_ERR_DEVICE_TIMEOUT
    assert 1.5 < time.perf_counter() - t0 < 30.0
    cfg = inputs.small_config(T=64, H=256, E=16, top_k=4, I=128, I_shared=128)
    check_full(to_device(inputs.make_inputs(cfg, "cuda")), cfg.top_k, "after a timeout")


def test_fp8_weights_layer_as_configured_decode():
    """FP8 expert weights under the last layers' configuration at decode size: fp32 router
    weights, sigmoid router with the routing factor 3 and a selection bias, SwiGLU limits 7
    (routed) and 16 (shared)."""
    import oracle
    from conftest import to_oracle
    cfg = inputs.CONFIGS["decode_t4"]
    d = fp8_inputs(cfg)
    d["bias"] = torch.linspace(-0.05, 0.05, cfg.E, dtype=torch.float32, device="cuda")
    g = torch.Generator().manual_seed(cfg.seed + 31)
    d["W_router"] = (torch.randn(cfg.E, cfg.H, generator=g) * cfg.r_std).cuda()
    opts = dict(router="sigmoid", routed_scaling_factor=3.0, swiglu_limit=7.0, swiglu_limit_shared=16.0)
    y, r = moe.moe_layer_forward_fp8(d["x"], d["W_router"], d["fp8"], top_k=cfg.top_k, router_bias=d["bias"],
                                     **opts)
    ref = oracle_routing(d, cfg.top_k, router="sigmoid", scale=3.0)
    assert_routing_exact(r, ref, cfg.E)
    y_ref = oracle_y_fp8(d, ref, swiglu_limit=7.0, swiglu_limit_shared=16.0)
    assert_y_close(y, y_ref, "decode_t4 fp8 as configured")
