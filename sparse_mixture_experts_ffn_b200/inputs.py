"""Seeded synthetic inputs for the Step-3.5-Flash routed-expert MoE layer.

This module holds random-number recipes only -- none of the layer's arithmetic -- so the
CUDA path and the CPU oracle can be fed identical tensors.

Shapes follow the llm-atlas page "Step-3.5-Flash", table "Champs bruts du config.json":
hidden_size 4096, moe_num_experts 288, moe_top_k 8, moe_intermediate_size 1280,
share_expert_dim 1280, torch_dtype bfloat16.  The page prints no weights; every tensor
here is random.

Recipe (fixed order, one generator per role):
* routing inputs on the CPU, ``torch.Generator().manual_seed(seed)``: x, then W_router;
* (skewed workload only) the expert rank permutation of the router bias on the CPU,
  ``torch.Generator().manual_seed(seed + 104729)``;
* expert weights on the target device, ``torch.Generator(device).manual_seed(seed + 7919)``:
  W_gate_up expert by expert, then W_down expert by expert, then the shared expert's
  gate/up and down matrices.
x ~ N(0,1); for the bf16 workloads each row is scaled to unit RMS (a unit-gain
pre-norm, in line with ``zero_centered true`` on the same page) and rounded to bf16.
Weights ~ N(0, w_std), router ~ N(0, r_std), rounded to the working dtype.

Skewed workload: b_e = beta * ln(r_e^-1.1 / sum_r r^-1.1) with r a seeded permutation of
the ranks 1..E; beta is set so that the 10% most-loaded experts take about half of all
assignments on this workload (a plain Zipf(1.1) would give them about 70%).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

# beta of the skewed workload's router bias.  Written by tests/golden/calibrate_skew_bias.py,
# which bisects beta on this workload's x and W_router with the CPU oracle's routing so that
# the 29 most-loaded of 288 experts hold 0.50 of the 131072 assignments.
SKEW_BETA = 0.511585
ZIPF_S = 1.1


@dataclass(frozen=True)
class MoEConfig:
    name: str
    seed: int
    T: int
    H: int
    E: int
    top_k: int
    I: int
    I_shared: int
    dtype: str  # "f32" or "bf16"
    x_std: float = 1.0
    w_std: float = 0.02
    r_std: float = 0.02
    rms_norm: bool = True
    skew: bool = False

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


CONFIGS = {
    c.name: c
    for c in [
        MoEConfig("tiny_f32_t64", seed=0, T=64, H=256, E=16, top_k=2, I=128, I_shared=128,
                  dtype="f32", r_std=0.1, rms_norm=False),
        MoEConfig("decode_t4", seed=1, T=4, H=4096, E=288, top_k=8, I=1280, I_shared=1280,
                  dtype="bf16"),
        MoEConfig("decode_t128", seed=2, T=128, H=4096, E=288, top_k=8, I=1280, I_shared=1280,
                  dtype="bf16"),
        MoEConfig("prefill_t4096", seed=3, T=4096, H=4096, E=288, top_k=8, I=1280, I_shared=1280,
                  dtype="bf16"),
        MoEConfig("prefill_t16384_skew", seed=4, T=16384, H=4096, E=288, top_k=8, I=1280,
                  I_shared=1280, dtype="bf16", skew=True),
    ]
}


def small_config(name: str = "small_bf16", seed: int = 11, T: int = 300, H: int = 256, E: int = 16,
                 top_k: int = 4, I: int = 256, I_shared: int = 256, dtype: str = "bf16",
                 **kw) -> MoEConfig:
    """A reduced workload with the same value distributions (for fast parity tests)."""
    return MoEConfig(name, seed=seed, T=T, H=H, E=E, top_k=top_k, I=I, I_shared=I_shared,
                     dtype=dtype, **kw)


def skew_bias(cfg: MoEConfig, beta: float = SKEW_BETA) -> torch.Tensor:
    gen = torch.Generator().manual_seed(cfg.seed + 104729)
    ranks = (torch.randperm(cfg.E, generator=gen) + 1).to(torch.float64)
    z = ranks.pow(-ZIPF_S)
    z = z / z.sum()
    return (beta * torch.log(z)).to(torch.float32)


def make_routing_inputs(cfg: MoEConfig, beta: float | None = None, router_fp32: bool = False):
    """x [T,H], W_router [E,H] (working dtype; fp32 with router_fp32, the same draws unrounded)
    and router bias [E] fp32 or None, on the CPU."""
    g = torch.Generator().manual_seed(cfg.seed)
    x = torch.randn(cfg.T, cfg.H, generator=g, dtype=torch.float32) * cfg.x_std
    if cfg.rms_norm:
        x = x * torch.rsqrt(x.pow(2).mean(dim=-1, keepdim=True) + 1e-6)
    x = x.to(cfg.torch_dtype)
    Wr = torch.randn(cfg.E, cfg.H, generator=g, dtype=torch.float32) * cfg.r_std
    if not router_fp32:
        Wr = Wr.to(cfg.torch_dtype)
    bias = skew_bias(cfg, SKEW_BETA if beta is None else beta) if cfg.skew else None
    return x, Wr, bias


def make_expert_weights(cfg: MoEConfig, device="cpu", shared: bool = True):
    """W_gate_up [E,2I,H] (gate rows then up rows), W_down [E,H,I], and the shared expert's
    Ws_gate_up [2Is,H], Ws_down [H,Is] (None when ``shared`` is False), on ``device``."""
    device = torch.device(device)
    g = torch.Generator(device=device).manual_seed(cfg.seed + 7919)
    dt = cfg.torch_dtype
    E, H, I, Is = cfg.E, cfg.H, cfg.I, cfg.I_shared
    Wgu = torch.empty(E, 2 * I, H, dtype=dt, device=device)
    Wd = torch.empty(E, H, I, dtype=dt, device=device)
    for e in range(E):
        Wgu[e] = torch.randn(2 * I, H, generator=g, device=device) * cfg.w_std
    for e in range(E):
        Wd[e] = torch.randn(H, I, generator=g, device=device) * cfg.w_std
    if not shared:
        return Wgu, Wd, None, None
    Wsgu = (torch.randn(2 * Is, H, generator=g, device=device) * cfg.w_std).to(dt)
    Wsd = (torch.randn(H, Is, generator=g, device=device) * cfg.w_std).to(dt)
    return Wgu, Wd, Wsgu, Wsd


FP8_BLOCK = 128  # one E8M0 scale per 128 x 128 block of an FP8 weight matrix


def fp8_blockwise(w: torch.Tensor):
    """(codes uint8 [R, K], scales uint8 [ceil(R/128), ceil(K/128)]) of a weight matrix in the
    blockwise FP8 format: E4M3 codes by torch's own cast, and per block the E8M0 scale
    2^ceil(log2(amax / 448)) that brings the block's largest magnitude within E4M3's range."""
    R, K = w.shape
    rb, kb = -(-R // FP8_BLOCK), -(-K // FP8_BLOCK)
    wf = torch.zeros(rb * FP8_BLOCK, kb * FP8_BLOCK, dtype=torch.float32, device=w.device)
    wf[:R, :K] = w.float()
    blocks = wf.view(rb, FP8_BLOCK, kb, FP8_BLOCK)
    amax = blocks.abs().amax(dim=(1, 3)).clamp_min(2.0 ** -100)
    exp = torch.ceil(torch.log2(amax / 448.0)).clamp(-127, 127)
    scaled = blocks * torch.exp2(-exp)[:, None, :, None]
    codes = scaled.view(rb * FP8_BLOCK, kb * FP8_BLOCK)[:R, :K].to(torch.float8_e4m3fn)
    return codes.view(torch.uint8).contiguous(), (exp + 127).to(torch.uint8).contiguous()


def make_fp8_expert_weights(cfg: MoEConfig, device="cpu", shared: bool = True):
    """The expert weights of ``make_expert_weights`` (same draws) in the blockwise FP8 format:
    a dict of (codes, scales) pairs W_gate_up ([E,2I,H], [E,ceil(2I/128),ceil(H/128)]),
    W_down ([E,H,I], [E,ceil(H/128),ceil(I/128)]) and, with ``shared``, Ws_gate_up and
    Ws_down.  Drawn and converted one expert at a time."""
    device = torch.device(device)
    g = torch.Generator(device=device).manual_seed(cfg.seed + 7919)
    E, H, I, Is = cfg.E, cfg.H, cfg.I, cfg.I_shared
    dt = cfg.torch_dtype

    def stack(rows, cols):
        q = torch.empty(E, rows, cols, dtype=torch.uint8, device=device)
        s = torch.empty(E, -(-rows // FP8_BLOCK), -(-cols // FP8_BLOCK), dtype=torch.uint8, device=device)
        for e in range(E):
            q[e], s[e] = fp8_blockwise((torch.randn(rows, cols, generator=g, device=device) * cfg.w_std).to(dt))
        return q, s

    out = {"W_gate_up": stack(2 * I, H), "W_down": stack(H, I)}
    if shared:
        out["Ws_gate_up"] = fp8_blockwise((torch.randn(2 * Is, H, generator=g, device=device) * cfg.w_std).to(dt))
        out["Ws_down"] = fp8_blockwise((torch.randn(H, Is, generator=g, device=device) * cfg.w_std).to(dt))
    else:
        out["Ws_gate_up"] = out["Ws_down"] = None
    return out


def make_inputs(cfg: MoEConfig, device="cpu", shared: bool = True):
    """All inputs of one workload as a dict of tensors on ``device``."""
    x, Wr, bias = make_routing_inputs(cfg)
    Wgu, Wd, Wsgu, Wsd = make_expert_weights(cfg, device, shared)
    device = torch.device(device)
    return dict(x=x.to(device), W_router=Wr.to(device),
                bias=None if bias is None else bias.to(device),
                W_gate_up=Wgu, W_down=Wd, Ws_gate_up=Wsgu, Ws_down=Wsd)


def with_sizes(cfg: MoEConfig, **kw) -> MoEConfig:
    return replace(cfg, **kw)
