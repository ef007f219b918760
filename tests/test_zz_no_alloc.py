"""The workspace-free routing entry point (moe_layer_route_noalloc), through the C ABI.

It serves callers that cannot allocate device memory; its scratch is a fixed array inside
the library.  Its routing must equal the routing of moe_layer_forward() on the same inputs,
on two calls in a row (the second call reuses the array left by the first).  This file is
collected last so that a run stopping at the first failure has run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import sparse_mixture_experts_ffn_b200 as moe
from helpers import W_REL_TOL
from sparse_mixture_experts_ffn_b200 import build, inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    build.build()
    lib = moe.load_library()
    P = ctypes.c_void_p
    lib.moe_layer_route_noalloc.argtypes = [ctypes.POINTER(moe.MoEShape), P, P, P, P, P, P]
    lib.moe_layer_route_noalloc.restype = ctypes.c_int
    return lib


CASES = [
    dict(T=300, H=512, E=64, top_k=8, I=128, I_shared=128, dtype="bf16"),
    dict(T=4, H=4096, E=288, top_k=8, I=128, I_shared=128, dtype="bf16"),
    dict(T=2000, H=4096, E=288, top_k=8, I=128, I_shared=128, dtype="bf16"),  # near the scratch limit
    dict(T=64, H=256, E=16, top_k=2, I=128, I_shared=128, dtype="f32", r_std=0.1, rms_norm=False),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "T{T}_H{H}_E{E}_{dtype}".format(**c))
def test_noalloc_routing_matches_forward(lib, case):
    cfg = inputs.small_config(**case)
    d = inputs.make_inputs(cfg, "cuda")
    _, ref = moe.moe_layer_forward(d["x"], d["W_router"], d["W_gate_up"], d["W_down"], d["Ws_gate_up"],
                                   d["Ws_down"], top_k=cfg.top_k, router_bias=d["bias"])
    shape = moe.make_shape(cfg.T, cfg.H, cfg.E, cfg.I, cfg.I_shared, cfg.top_k, cfg.torch_dtype)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        idx = torch.full((cfg.T, cfg.top_k), -1, dtype=torch.int32, device="cuda")
        w = torch.full((cfg.T, cfg.top_k), -1.0, dtype=torch.float32, device="cuda")
        rc = lib.moe_layer_route_noalloc(ctypes.byref(shape), ctypes.c_void_p(d["x"].data_ptr()),
                                         ctypes.c_void_p(d["W_router"].data_ptr()), None,
                                         ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(w.data_ptr()),
                                         stream)
        assert rc == moe.MOE_OK, moe.status_string(rc)
        torch.cuda.synchronize()
        assert torch.equal(idx, ref.topk_idx), f"call {call}: indices differ"
        rel = (w - ref.topk_w).abs() / ref.topk_w.abs().clamp_min(1e-30)
        assert float(rel.max()) <= W_REL_TOL, f"call {call}: weights differ by {float(rel.max()):.2e}"


def test_noalloc_routing_with_a_router_bias_matches_the_oracle(lib):
    """The skewed long-prefill workload's router bias (added to the scores, for the selection
    and the weights) on a decode-sized batch: indices bit-exact against the oracle's exact
    routing, weights within the routing-weight tolerance, on two calls in a row."""
    from helpers import oracle_routing
    big = inputs.CONFIGS["prefill_t16384_skew"]
    cfg = inputs.with_sizes(big, T=4)
    x, Wr, bias = inputs.make_routing_inputs(cfg)
    assert bias is not None
    d = dict(x=x.cuda(), W_router=Wr.cuda(), bias=bias.cuda())
    ref = oracle_routing(d, cfg.top_k)
    shape = moe.make_shape(cfg.T, cfg.H, cfg.E, cfg.I, cfg.I_shared, cfg.top_k, cfg.torch_dtype)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        idx = torch.full((cfg.T, cfg.top_k), -1, dtype=torch.int32, device="cuda")
        w = torch.full((cfg.T, cfg.top_k), -1.0, dtype=torch.float32, device="cuda")
        rc = lib.moe_layer_route_noalloc(ctypes.byref(shape), ctypes.c_void_p(d["x"].data_ptr()),
                                         ctypes.c_void_p(d["W_router"].data_ptr()),
                                         ctypes.c_void_p(d["bias"].data_ptr()),
                                         ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(w.data_ptr()), stream)
        assert rc == moe.MOE_OK, moe.status_string(rc)
        torch.cuda.synchronize()
        assert np.array_equal(idx.cpu().numpy(), ref["idx"]), f"call {call}: indices differ"
        rel = np.abs(w.cpu().numpy().astype(np.float64) - ref["w64"]) / np.abs(ref["w64"])
        assert float(rel.max()) <= W_REL_TOL, f"call {call}: weights differ by {float(rel.max()):.2e}"


def test_noalloc_rejects_batches_beyond_its_scratch(lib):
    shape = moe.make_shape(100000, 4096, 288, 1280, 1280, 8, torch.bfloat16)
    P = ctypes.c_void_p
    rc = lib.moe_layer_route_noalloc(ctypes.byref(shape), P(16), P(16), None, P(16), P(16), None)
    assert rc == 3  # MOE_ERR_WORKSPACE_TOO_SMALL, before anything is enqueued
