"""Shared helpers of the test suite: running the CUDA path and the oracle on the same
seeded inputs, and the parity criteria."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from conftest import to_oracle

# output tolerance of the layer: max|err| <= 2e-2 * max|y_ref| and relative L2 <= 1e-2
Y_MAX_TOL = 2e-2
Y_REL_L2_TOL = 1e-2
# routing weights (fp32 softmax of the chosen keys) against the oracle's fp64 softmax of
# the exact keys.  Keys of experts chosen for certain come from the score estimate (fp64
# accumulation, or fp32 slices of 256 products added in fp64 on the tensor-core path),
# whose error on these workloads is a few 1e-6 of a logit.
W_REL_TOL = 2e-5


def y_errors(y_gpu, y_ref: np.ndarray):
    yg = y_gpu.detach().float().cpu().numpy().astype(np.float64)
    d = yg - y_ref
    max_err = float(np.abs(d).max()) if d.size else 0.0
    scale = float(np.abs(y_ref).max()) if y_ref.size else 0.0
    rel_l2 = float(np.linalg.norm(d) / max(np.linalg.norm(y_ref), 1e-300)) if d.size else 0.0
    return max_err, scale, rel_l2


def assert_y_close(y_gpu, y_ref: np.ndarray, what=""):
    max_err, scale, rel_l2 = y_errors(y_gpu, y_ref)
    assert max_err <= Y_MAX_TOL * scale + 1e-30, f"{what}: max|err| {max_err:.3e} > 2e-2 * {scale:.3e}"
    assert rel_l2 <= Y_REL_L2_TOL, f"{what}: relative L2 {rel_l2:.3e} > 1e-2"
    return max_err / max(scale, 1e-300), rel_l2


def oracle_arrays(d: dict):
    return {k: to_oracle(v) if v is not None else None for k, v in d.items()}


def oracle_routing(d: dict, top_k: int, router: str = "softmax", scale: float = 1.0):
    """Exact routing of every token by the oracle."""
    a = oracle_arrays({"x": d["x"], "W_router": d["W_router"]})
    s = oracle.router_scores(a["x"], a["W_router"])
    bias = None if d.get("bias") is None else d["bias"].detach().cpu().numpy().astype(np.float32)
    idx, w, w64 = oracle.route(s, top_k, bias, router=router, scale=scale)
    counts, offsets, perm, inv = oracle.dispatch(idx, d["W_router"].shape[0])
    return dict(scores=s, idx=idx, w=w, w64=w64, counts=counts, offsets=offsets, perm=perm, inv_perm=inv)


def oracle_y(d: dict, routing: dict, tokens=None, swiglu_limit=0.0, swiglu_limit_shared=0.0):
    a = oracle_arrays({k: d.get(k) for k in ("x", "W_gate_up", "W_down", "Ws_gate_up", "Ws_down")})
    return oracle.moe_tokens(a["x"], routing["idx"], routing["w64"], a["W_gate_up"], a["W_down"],
                             a["Ws_gate_up"], a["Ws_down"], tokens=tokens, swiglu_limit=swiglu_limit,
                             swiglu_limit_shared=swiglu_limit_shared)


def assert_routing_exact(r_gpu, r_ref: dict, E: int, w_tol: float = None):
    idx = r_gpu.topk_idx.cpu().numpy()
    assert np.array_equal(idx, r_ref["idx"]), (
        f"topk_idx differs on {int((idx != r_ref['idx']).any(1).sum())} tokens")
    assert np.array_equal(r_gpu.counts.cpu().numpy(), r_ref["counts"])
    assert np.array_equal(r_gpu.offsets.cpu().numpy(), r_ref["offsets"])
    assert np.array_equal(r_gpu.perm.cpu().numpy(), r_ref["perm"])
    w = r_gpu.topk_w.cpu().numpy().astype(np.float64)
    rel = np.abs(w - r_ref["w64"]) / np.maximum(np.abs(r_ref["w64"]), 1e-30)
    tol = W_REL_TOL if w_tol is None else w_tol
    assert float(rel.max()) <= tol, f"topk_w relative error {float(rel.max()):.3e}"


def to_device(d: dict, device="cuda"):
    return {k: (v.to(device).contiguous() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


def tile_class_tokens(ref: dict, T: int, top_k: int, n_random: int, seed: int, top: int = 5,
                      tiles=(16, 128, 256)):
    """Tokens whose outputs a full-size test checks, chosen from the exact routing so that
    every kind of expert-GEMM tile is hit: for each of the `top` most-loaded experts and
    each token-tile width in `tiles`, the last row of its last (ragged) tile and the first
    row of that tile; the rows at the starts of 256-token tiles of the most-loaded expert;
    the first and the last token (the shared expert's first and ragged last tiles); and
    `n_random` random tokens."""
    counts, offsets, perm = ref["counts"], ref["offsets"], ref["perm"]
    picks = [0, T - 1]
    for e in np.argsort(-counts, kind="stable")[:top]:
        c = int(counts[e])
        if c == 0:
            continue
        for bn in tiles:
            last = (c - 1) // bn * bn
            for r in (last, c - 1):
                picks.append(int(perm[offsets[e] + r]) // top_k)
    e0 = int(np.argmax(counts))
    for r in range(0, int(counts[e0]), 256):
        picks.append(int(perm[offsets[e0] + r]) // top_k)
    rng = np.random.default_rng(seed)
    picks += rng.choice(T, min(n_random, T), replace=False).tolist()
    return np.unique(np.asarray(picks, np.int64))
