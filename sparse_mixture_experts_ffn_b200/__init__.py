"""Python binding of the sm_100a MoE layer library (``libmoe_layer.so``, C ABI in
``include/moe_layer.h``).

Argument marshalling only: every step of the layer runs in the library's CUDA kernels.
PyTorch provides device memory and the current stream.  There is no fallback: if the
library is missing the call raises.

    from sparse_mixture_experts_ffn_b200 import moe_layer_forward
    y, routing = moe_layer_forward(x, W_router, W_gate_up, W_down, Ws_gate_up, Ws_down, top_k=8)
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_layer.so")

MOE_OK = 0
MOE_F32, MOE_BF16 = 0, 1
STATUS_NAMES = {
    0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED_SHAPE",
    3: "MOE_ERR_WORKSPACE_TOO_SMALL", 4: "MOE_ERR_CUDA", 5: "MOE_ERR_DEVICE_TIMEOUT",
    6: "MOE_ERR_DEVICE_BOUNDS",
}
EXPORTED = ("moe_layer_workspace_bytes", "moe_layer_forward", "moe_layer_forward_ex", "moe_layer_forward_fp8",
            "moe_layer_forward_ep", "moe_layer_sum_partials", "moe_layer_check_status",
            "moe_layer_route_stats", "moe_layer_workspace_layout", "moe_layer_profile_enable",
            "moe_layer_profile_read", "moe_layer_launch_count", "moe_status_string")
STAGES = ("routing", "dispatch", "gate_up", "down", "combine")


class MoEShape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("H", ctypes.c_int32), ("E", ctypes.c_int32),
                ("I", ctypes.c_int32), ("I_shared", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("dtype", ctypes.c_int32)]


class MoEOptions(ctypes.Structure):
    _fields_ = [("swiglu_limit", ctypes.c_float), ("swiglu_limit_shared", ctypes.c_float),
                ("router", ctypes.c_int32), ("routed_scaling_factor", ctypes.c_float),
                ("router_weights_fp32", ctypes.c_int32)]


ROUTERS = {"softmax": 0, "sigmoid": 1}


class MoEFp8Weights(ctypes.Structure):
    _fields_ = [("W_gate_up", ctypes.c_void_p), ("W_gate_up_scale", ctypes.c_void_p),
                ("W_down", ctypes.c_void_p), ("W_down_scale", ctypes.c_void_p),
                ("Ws_gate_up", ctypes.c_void_p), ("Ws_gate_up_scale", ctypes.c_void_p),
                ("Ws_down", ctypes.c_void_p), ("Ws_down_scale", ctypes.c_void_p)]


class MoEEpRange(ctypes.Structure):
    _fields_ = [("expert_begin", ctypes.c_int32), ("expert_end", ctypes.c_int32),
                ("shared_begin", ctypes.c_int64), ("shared_end", ctypes.c_int64)]


class MoERoutingOut(ctypes.Structure):
    _fields_ = [("topk_idx", ctypes.c_void_p), ("topk_w", ctypes.c_void_p),
                ("counts", ctypes.c_void_p), ("offsets", ctypes.c_void_p),
                ("perm", ctypes.c_void_p)]


class MoERouteStats(ctypes.Structure):
    _fields_ = [("n_refined", ctypes.c_int64), ("n_exact", ctypes.c_int64),
                ("n_tokens_refined", ctypes.c_int64), ("n_weight_keys", ctypes.c_int64)]


class MoEWorkspaceLayout(ctypes.Structure):
    _fields_ = [("x_perm", ctypes.c_size_t), ("h", ctypes.c_size_t), ("h_shared", ctypes.c_size_t),
                ("o", ctypes.c_size_t), ("o_shared", ctypes.c_size_t), ("row_w", ctypes.c_size_t),
                ("scores", ctypes.c_size_t), ("scores_slice", ctypes.c_int32)]


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


_lib = None


def load_library(path: str = LIB_PATH):
    """Load the CUDA library (no fallback: raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} not found: build it with `python -m sparse_mixture_experts_ffn_b200.build`")
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    lib.moe_layer_workspace_bytes.argtypes = [ctypes.POINTER(MoEShape)]
    lib.moe_layer_workspace_bytes.restype = ctypes.c_size_t
    lib.moe_layer_forward.argtypes = [ctypes.POINTER(MoEShape), P, P, P, P, P, P, P, P,
                                      ctypes.POINTER(MoERoutingOut), P, ctypes.c_size_t, P]
    lib.moe_layer_forward.restype = ctypes.c_int
    lib.moe_layer_forward_ex.argtypes = [ctypes.POINTER(MoEShape), P, P, P, P, P, P, P, P,
                                         ctypes.POINTER(MoERoutingOut), ctypes.POINTER(MoEOptions), P,
                                         ctypes.c_size_t, P]
    lib.moe_layer_forward_ex.restype = ctypes.c_int
    lib.moe_layer_forward_fp8.argtypes = [ctypes.POINTER(MoEShape), P, P, P, ctypes.POINTER(MoEFp8Weights), P,
                                          ctypes.POINTER(MoERoutingOut), ctypes.POINTER(MoEOptions), P,
                                          ctypes.c_size_t, P]
    lib.moe_layer_forward_fp8.restype = ctypes.c_int
    lib.moe_layer_forward_ep.argtypes = [ctypes.POINTER(MoEShape), P, P, P, P, P, P, P, ctypes.POINTER(MoEEpRange),
                                         P, ctypes.POINTER(MoERoutingOut), ctypes.POINTER(MoEOptions), P,
                                         ctypes.c_size_t, P]
    lib.moe_layer_forward_ep.restype = ctypes.c_int
    lib.moe_layer_sum_partials.argtypes = [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                           ctypes.POINTER(ctypes.c_void_p), P, P]
    lib.moe_layer_sum_partials.restype = ctypes.c_int
    lib.moe_layer_check_status.argtypes = [P, P]
    lib.moe_layer_check_status.restype = ctypes.c_int
    lib.moe_layer_route_stats.argtypes = [P, ctypes.POINTER(MoERouteStats), P]
    lib.moe_layer_route_stats.restype = ctypes.c_int
    lib.moe_layer_workspace_layout.argtypes = [ctypes.POINTER(MoEShape), ctypes.POINTER(MoEWorkspaceLayout)]
    lib.moe_layer_workspace_layout.restype = ctypes.c_int
    lib.moe_layer_profile_enable.argtypes = [ctypes.c_int]
    lib.moe_layer_profile_enable.restype = ctypes.c_int
    lib.moe_layer_profile_read.argtypes = [ctypes.POINTER(ctypes.c_float), ctypes.c_int]
    lib.moe_layer_profile_read.restype = ctypes.c_int
    lib.moe_layer_launch_count.argtypes = []
    lib.moe_layer_launch_count.restype = ctypes.c_int64
    lib.moe_status_string.argtypes = [ctypes.c_int]
    lib.moe_status_string.restype = ctypes.c_char_p
    _lib = lib
    return lib


def make_shape(T, H, E, I, I_shared, top_k, dtype) -> MoEShape:
    import torch
    code = MOE_BF16 if dtype == torch.bfloat16 else MOE_F32 if dtype == torch.float32 else -1
    if code < 0:
        raise TypeError(f"unsupported dtype {dtype}")
    return MoEShape(int(T), int(H), int(E), int(I), int(I_shared), int(top_k), code)


def workspace_bytes(shape: MoEShape) -> int:
    return int(load_library().moe_layer_workspace_bytes(ctypes.byref(shape)))


def workspace_layout(shape: MoEShape) -> MoEWorkspaceLayout:
    out = MoEWorkspaceLayout()
    rc = load_library().moe_layer_workspace_layout(ctypes.byref(shape), ctypes.byref(out))
    if rc != MOE_OK:
        raise MoEError(rc, "moe_layer_workspace_layout")
    return out


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


@dataclass
class Routing:
    topk_idx: "object"
    topk_w: "object"
    counts: "object"
    offsets: "object"
    perm: "object"


def alloc_workspace(shape: MoEShape, device):
    import torch
    nbytes = workspace_bytes(shape)
    if nbytes == 0:
        raise MoEError(1, "moe_layer_workspace_bytes")
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def moe_layer_forward(x, W_router, W_gate_up, W_down, Ws_gate_up=None, Ws_down=None, *, top_k,
                      router_bias=None, y=None, workspace=None, routing=True, stream=None,
                      swiglu_limit=0.0, swiglu_limit_shared=0.0, router="softmax",
                      routed_scaling_factor=1.0):
    """Run the MoE layer on the device.  Returns (y, Routing or None).

    Shapes: x [T,H], W_router [E,H], W_gate_up [E,2I,H], W_down [E,H,I], Ws_gate_up
    [2Is,H], Ws_down [H,Is] (or both None), router_bias [E] fp32 or None.  All CUDA,
    contiguous, on x's device, same dtype (bf16 or fp32); W_router may be fp32 with bf16
    tokens (fp32 router weights).  Mismatched shapes, dtypes or devices raise ValueError
    before anything is launched.  swiglu_limit / swiglu_limit_shared: SwiGLU
    limits of the routed / shared experts (gate <= L, up in [-L, L]; 0 = none).
    router="sigmoid": sigmoid scores, router_bias for the selection only, weights
    routed_scaling_factor * p / sum p (the default "softmax" ignores the factor).
    """
    if W_gate_up.dim() != 3 or (Ws_gate_up is not None and Ws_gate_up.dim() != 2):
        raise ValueError("W_gate_up must be [E, 2I, H] and Ws_gate_up [2Is, H]")
    I = W_gate_up.shape[1] // 2
    Is = 0 if Ws_gate_up is None else Ws_gate_up.shape[0] // 2
    return _forward("moe_layer_forward_ex", (W_gate_up, W_down, Ws_gate_up, Ws_down), x, W_router, I, Is,
                    top_k, router_bias, y, workspace, routing, stream, swiglu_limit, swiglu_limit_shared, router,
                    routed_scaling_factor)


def moe_layer_forward_fp8(x, W_router, weights, *, top_k, router_bias=None, y=None, workspace=None,
                          routing=True, stream=None, swiglu_limit=0.0, swiglu_limit_shared=0.0,
                          router="softmax", routed_scaling_factor=1.0):
    """moe_layer_forward with expert weights in the blockwise FP8 format.

    ``weights``: a dict with W_gate_up, W_down, Ws_gate_up, Ws_down, each a pair (codes
    uint8, scales uint8) -- E4M3 codes of the matrix and one E8M0 scale per 128 x 128 block,
    shapes as in include/moe_layer.h (the shared pairs may be None) -- as made by
    ``inputs.fp8_blockwise``.  x and W_router bf16 (W_router may be fp32).
    """
    import torch
    gu, dn = weights["W_gate_up"], weights["W_down"]
    sgu, sdn = weights.get("Ws_gate_up"), weights.get("Ws_down")
    for pair in (gu, dn, sgu, sdn):
        if pair is not None and (pair[0].dtype != torch.uint8 or pair[1].dtype != torch.uint8):
            raise ValueError("FP8 weights are (codes, scales) pairs of uint8 tensors")
    if gu[0].dim() != 3 or (sgu is not None and sgu[0].dim() != 2):
        raise ValueError("W_gate_up codes must be [E, 2I, H] and Ws_gate_up codes [2Is, H]")
    I = gu[0].shape[1] // 2
    Is = 0 if sgu is None else sgu[0].shape[0] // 2
    return _forward("moe_layer_forward_fp8", (gu, dn, sgu, sdn), x, W_router, I, Is, top_k, router_bias, y,
                    workspace, routing, stream, swiglu_limit, swiglu_limit_shared, router,
                    routed_scaling_factor)


def expert_range(E: int, world: int, rank: int) -> tuple:
    """The routed experts [begin, end) that rank `rank` of `world` holds under expert
    parallelism: contiguous, sizes differing by at most one."""
    return rank * E // world, (rank + 1) * E // world


def moe_layer_forward_ep(x, W_router, W_gate_up, W_down, Ws_gate_up=None, Ws_down=None, *, top_k,
                         expert_begin, shared_rows=(0, 0), router_bias=None, y_partial=None, workspace=None,
                         routing=False, stream=None, swiglu_limit=0.0, swiglu_limit_shared=0.0,
                         router="softmax", routed_scaling_factor=1.0):
    """One rank's fp32 share of the layer under expert parallelism (moe_layer_forward_ep in
    include/moe_layer.h).  W_gate_up [n, 2I, H] and W_down [n, H, I] hold the routed experts
    [expert_begin, expert_begin + n) only; W_router holds all E.  The shared expert is added
    on the token rows [shared_rows[0], shared_rows[1]).  Returns (y_partial fp32 [T, H],
    Routing or None); the shares of ranks whose expert and shared ranges partition the
    experts and the tokens add up to the layer's output."""
    import torch
    if W_gate_up.dim() != 3 or W_down.dim() != 3 or (Ws_gate_up is not None and Ws_gate_up.dim() != 2):
        raise ValueError("W_gate_up must be [n, 2I, H], W_down [n, H, I] and Ws_gate_up [2Is, H]")
    if x.dtype != torch.bfloat16:
        raise ValueError("expert parallelism runs bf16 layers")
    n = W_gate_up.shape[0]
    E = W_router.shape[0]
    e0 = int(expert_begin)
    if not (0 <= e0 and e0 + n <= E and n >= 1):
        raise ValueError(f"experts [{e0}, {e0 + n}) outside [0, {E})")
    I = W_gate_up.shape[1] // 2
    Is = 0 if Ws_gate_up is None else Ws_gate_up.shape[0] // 2
    _check_args(x, W_router[e0:e0 + n], router_bias[e0:e0 + n] if router_bias is not None else None, None,
                (W_gate_up, W_down, Ws_gate_up, Ws_down), I, Is, False)
    if router_bias is not None and (router_bias.dtype != torch.float32 or tuple(router_bias.shape) != (E,)):
        raise ValueError(f"router_bias must be fp32 [{E}]")
    T, H = x.shape
    s0, s1 = int(shared_rows[0]), int(shared_rows[1])
    if not (0 <= s0 <= s1 <= T):
        raise ValueError(f"shared rows [{s0}, {s1}) outside [0, {T}]")
    if y_partial is None:
        y_partial = torch.empty(T, H, dtype=torch.float32, device=x.device)
    elif y_partial.dtype != torch.float32 or tuple(y_partial.shape) != (T, H) or y_partial.device != x.device:
        raise ValueError(f"y_partial must be fp32 [{T}, {H}] on x's device")
    lib = load_library()
    shape = make_shape(T, H, E, I, Is, top_k, x.dtype)
    if workspace is None:
        workspace = alloc_workspace(shape, x.device)
    r, rout = _routing_buffers(T, E, top_k, x.device) if routing else (None, None)
    if stream is None:
        stream = torch.cuda.current_stream(x.device)
    w32 = 1 if W_router.dtype == torch.float32 else 0
    opts = MoEOptions(float(swiglu_limit), float(swiglu_limit_shared), ROUTERS[router],
                      float(routed_scaling_factor), w32)
    rng = MoEEpRange(e0, e0 + n, s0, s1)
    rc = lib.moe_layer_forward_ep(ctypes.byref(shape), _ptr(x), _ptr(W_router), _ptr(router_bias), _ptr(W_gate_up),
                                  _ptr(W_down), _ptr(Ws_gate_up), _ptr(Ws_down), ctypes.byref(rng), _ptr(y_partial),
                                  ctypes.byref(rout) if rout is not None else None, ctypes.byref(opts),
                                  _ptr(workspace), workspace.numel(), ctypes.c_void_p(stream.cuda_stream))
    if rc != MOE_OK:
        raise MoEError(rc, "moe_layer_forward_ep")
    return y_partial, r


def sum_partials(parts, y, stream=None):
    """y = parts[0] + parts[1] + ... (fp32, in order), stored in y's dtype (bf16 or fp32).
    Each part is an fp32 tensor of y's shape on y's device."""
    import torch
    if not parts or len(parts) > 16:
        raise ValueError("1 to 16 parts")
    for t in parts:
        if t.dtype != torch.float32 or t.shape != y.shape or t.device != y.device or not t.is_contiguous():
            raise ValueError("parts must be contiguous fp32 tensors of y's shape on y's device")
    if y.dim() != 2 or not y.is_contiguous() or y.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("y must be a contiguous bf16 or fp32 [T, H] tensor")
    if stream is None:
        stream = torch.cuda.current_stream(y.device)
    arr = (ctypes.c_void_p * len(parts))(*[t.data_ptr() for t in parts])
    rc = load_library().moe_layer_sum_partials(y.shape[0], y.shape[1], MOE_BF16 if y.dtype == torch.bfloat16
                                               else MOE_F32, len(parts), arr, _ptr(y),
                                               ctypes.c_void_p(stream.cuda_stream))
    if rc != MOE_OK:
        raise MoEError(rc, "moe_layer_sum_partials")
    return y


def _routing_buffers(T, E, top_k, dev):
    import torch
    r = Routing(torch.empty(T, top_k, dtype=torch.int32, device=dev),
                torch.empty(T, top_k, dtype=torch.float32, device=dev),
                torch.empty(E, dtype=torch.int32, device=dev),
                torch.empty(E + 1, dtype=torch.int32, device=dev),
                torch.empty(T * top_k, dtype=torch.int32, device=dev))
    return r, MoERoutingOut(r.topk_idx.data_ptr(), r.topk_w.data_ptr(), r.counts.data_ptr(),
                            r.offsets.data_ptr(), r.perm.data_ptr())


def _check_args(x, W_router, router_bias, y, weights, I, Is, fp8: bool):
    """Validate shapes, dtypes and devices before anything reaches the C ABI, which sees only
    pointers: a mismatch there would make the kernels read past an allocation.  Raises
    ValueError.  ``weights`` are (W_gate_up, W_down, Ws_gate_up, Ws_down): tensors in x's
    dtype, or (codes, scales) uint8 pairs for FP8 weights (shared pair None without a
    shared expert)."""
    import torch

    def shape_of(t):
        return tuple(t.shape)

    if x.dim() != 2:
        raise ValueError(f"x must be [T, H], got {shape_of(x)}")
    T, H = x.shape
    if x.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError(f"x must be bf16 or fp32, got {x.dtype}")
    if fp8 and x.dtype != torch.bfloat16:
        raise ValueError("FP8 expert weights need bf16 tokens")
    if W_router.dim() != 2 or W_router.shape[1] != H:
        raise ValueError(f"W_router must be [E, {H}], got {shape_of(W_router)}")
    E = W_router.shape[0]
    router_dtypes = (x.dtype, torch.float32) if x.dtype == torch.bfloat16 else (x.dtype,)
    if W_router.dtype not in router_dtypes:
        raise ValueError(f"W_router must be {x.dtype}" + (" or fp32" if len(router_dtypes) > 1 else "") +
                         f", got {W_router.dtype}")
    if router_bias is not None and (router_bias.dtype != torch.float32 or shape_of(router_bias) != (E,)):
        raise ValueError(f"router_bias must be fp32 [{E}], got {router_bias.dtype} {shape_of(router_bias)}")
    if y is not None and (y.dtype != x.dtype or shape_of(y) != (T, H)):
        raise ValueError(f"y must be {x.dtype} [{T}, {H}], got {y.dtype} {shape_of(y)}")
    Wgu, Wd, Wsgu, Wsd = weights
    if (Wsgu is None) != (Wsd is None):
        raise ValueError("give both shared-expert matrices or neither")
    mats = [("W_gate_up", Wgu, (E, 2 * I, H)), ("W_down", Wd, (E, H, I))]
    if Wsgu is not None:
        mats += [("Ws_gate_up", Wsgu, (2 * Is, H)), ("Ws_down", Wsd, (H, Is))]
    checked = [("x", x), ("W_router", W_router), ("router_bias", router_bias), ("y", y)]
    for name, w, want in mats:
        if w is None:
            raise ValueError(f"{name} is required")
        if fp8:
            codes, scales = w
            sshape = want[:-2] + tuple(-(-n // 128) for n in want[-2:])
            for part, t, shp in (("codes", codes, want), ("scales", scales, sshape)):
                if t.dtype != torch.uint8 or shape_of(t) != shp:
                    raise ValueError(f"{name} {part} must be uint8 {list(shp)}, got {t.dtype} {shape_of(t)}")
            checked += [(name, codes), (name + "_scale", scales)]
        else:
            if w.dtype != x.dtype or shape_of(w) != want:
                raise ValueError(f"{name} must be {x.dtype} {list(want)}, got {w.dtype} {shape_of(w)}")
            checked.append((name, w))
    for name, t in checked:
        if t is None:
            continue
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if t.device != x.device:
            raise ValueError(f"{name} is on {t.device}, x on {x.device}")
    if not x.is_cuda:
        raise ValueError("the tensors must be CUDA tensors (the layer runs only on the GPU)")


def _forward(entry, weights, x, W_router, I, Is, top_k, router_bias, y, workspace, routing, stream,
             swiglu_limit, swiglu_limit_shared, router, routed_scaling_factor):
    import torch
    _check_args(x, W_router, router_bias, y, weights, I, Is, entry == "moe_layer_forward_fp8")
    if workspace is not None and (workspace.device != x.device or workspace.dtype != torch.uint8
                                  or not workspace.is_contiguous()):
        raise ValueError("workspace must be a contiguous uint8 tensor on x's device")
    lib = load_library()
    T, H = x.shape
    E = W_router.shape[0]
    shape = make_shape(T, H, E, I, Is, top_k, x.dtype)
    if y is None:
        y = torch.empty_like(x)
    if workspace is None:
        workspace = alloc_workspace(shape, x.device)
    r, rout = _routing_buffers(T, E, top_k, x.device) if routing else (None, None)
    if stream is None:
        stream = torch.cuda.current_stream(x.device)
    w32 = 1 if (x.dtype == torch.bfloat16 and W_router.dtype == torch.float32) else 0
    opts = MoEOptions(float(swiglu_limit), float(swiglu_limit_shared), ROUTERS[router],
                      float(routed_scaling_factor), w32)
    common = (ctypes.byref(shape), _ptr(x), _ptr(W_router), _ptr(router_bias))
    tail = (_ptr(y), ctypes.byref(rout) if rout is not None else None, ctypes.byref(opts), _ptr(workspace),
            workspace.numel(), ctypes.c_void_p(stream.cuda_stream))
    if entry == "moe_layer_forward_fp8":
        fw = MoEFp8Weights(*[None if pr is None else pr[i].data_ptr() for pr in weights for i in (0, 1)])
        rc = lib.moe_layer_forward_fp8(*common, ctypes.byref(fw), *tail)
    else:
        rc = lib.moe_layer_forward_ex(*common, *(_ptr(w) for w in weights), *tail)
    if rc != MOE_OK:
        raise MoEError(rc, entry)
    return y, r


def check_status(workspace, stream=None) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(workspace.device)
    return int(load_library().moe_layer_check_status(_ptr(workspace), ctypes.c_void_p(stream.cuda_stream)))


def route_stats(workspace, stream=None) -> dict:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(workspace.device)
    out = MoERouteStats()
    rc = load_library().moe_layer_route_stats(_ptr(workspace), ctypes.byref(out), ctypes.c_void_p(stream.cuda_stream))
    if rc != MOE_OK:
        raise MoEError(rc, "moe_layer_route_stats")
    return dict(n_refined=out.n_refined, n_exact=out.n_exact, n_tokens_refined=out.n_tokens_refined,
                n_weight_keys=out.n_weight_keys)


def status_string(status: int) -> str:
    return load_library().moe_status_string(int(status)).decode()


def profile_enable(enable: bool = True) -> None:
    load_library().moe_layer_profile_enable(1 if enable else 0)


def profile_read() -> tuple[int, dict]:
    """(forward calls covered, {stage: total ms}) since the previous read."""
    ms = (ctypes.c_float * len(STAGES))()
    calls = load_library().moe_layer_profile_read(ms, len(STAGES))
    if calls < 0:
        raise MoEError(4, "moe_layer_profile_read")
    return calls, {name: float(ms[i]) for i, name in enumerate(STAGES)}


def launch_count() -> int:
    return int(load_library().moe_layer_launch_count())
