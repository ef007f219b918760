"""CPU oracle of the Step-3.5-Flash routed-expert MoE FFN layer (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
import this package.  The CUDA library never does, and the two share no code: the
oracle's arithmetic lives in ``moe_oracle.c`` (plain C, OpenMP over tokens), written from
the definition of the layer; this module only marshals numpy arrays into it.

Definition followed (llm-atlas page "Step-3.5-Flash", table "Champs bruts du
config.json": moe_num_experts, moe_top_k, norm_expert_weight, need_fp32_gate,
moe_intermediate_size, share_expert_dim; "FFN / MoE" paragraph of the same page):

* router score  s[t,e] = exact sum_h x[t,h] W_r[e,h], rounded once to fp32;
* key[t,e]      = fp32(s[t,e] + b[e]) with an optional router bias b;
* selection     = the top_k keys, ties toward the lower expert index, stored ascending;
* weights       = softmax over the selected keys (renormalised to sum to 1), fp64;
* output        y_t = sum_j w_j SiLU(x W_g^T) * (x W_u^T) W_d^T + shared expert, fp64;
* FP8 weights   (the low-precision expert weights for decode) E4M3 codes with one E8M0
                power-of-two scale per 128 x 128 block, decoded exactly (``dequant_e4m3``,
                ``moe_tokens_fp8``).

bf16 arrays are passed as ``numpy.uint16`` bit patterns; fp32 as ``numpy.float32``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libmoe_oracle.so")

F32, BF16 = 0, 1

_lib = None


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into oracle/_build/libmoe_oracle.so with gcc -O2 -fopenmp
    (-ffp-contract=off: the fixed-sequence exponential fuses only where it says so)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fopenmp", "-fPIC",
                               "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        lib.oracle_exact_dot.argtypes = [ctypes.c_int, ctypes.c_int, P, P, P]
        lib.oracle_router_scores.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                             P, P, P, ctypes.c_int]
        lib.oracle_route.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, P, P, P, P, P]
        lib.oracle_dispatch.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, P, P, P, P, P]
        D = ctypes.c_double
        lib.oracle_route_mode.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, P, P, ctypes.c_int, D,
                                          P, P, P]
        lib.oracle_sigmoid32.argtypes = [ctypes.c_int64, P, P]
        lib.oracle_exact_dot_mixed.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P]
        lib.oracle_router_scores_mixed.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_int,
                                                   ctypes.c_int, P, P, P, ctypes.c_int]
        lib.oracle_expert_act.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, D, P]
        lib.oracle_moe_tokens.argtypes = [ctypes.c_int, ctypes.c_int64, P, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P, P, P, P,
                                          P, D, D, P, ctypes.c_int]
        lib.oracle_dequant_e4m3.argtypes = [ctypes.c_int64, ctypes.c_int, P, P, P]
        lib.oracle_moe_tokens_fp8.argtypes = [ctypes.c_int64, P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_int, ctypes.c_int, P, P, P, P, P, P, P, P, P, P, P,
                                              D, D, P, ctypes.c_int]
        for f in (lib.oracle_exact_dot, lib.oracle_router_scores, lib.oracle_route,
                  lib.oracle_dispatch, lib.oracle_expert_act, lib.oracle_moe_tokens,
                  lib.oracle_route_mode, lib.oracle_sigmoid32, lib.oracle_exact_dot_mixed,
                  lib.oracle_router_scores_mixed, lib.oracle_dequant_e4m3, lib.oracle_moe_tokens_fp8):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.uint16:
        return BF16
    if a.dtype == np.float32:
        return F32
    raise TypeError(f"oracle inputs are bf16 bit patterns (uint16) or float32, got {a.dtype}")


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype=None):
    if a is None:
        return None
    return np.ascontiguousarray(a if dtype is None else a.astype(dtype, copy=False))


def nthreads_default() -> int:
    return len(os.sched_getaffinity(0))


def exact_dot(x: np.ndarray, w: np.ndarray) -> np.float32:
    """Exact sum_h x[h]*w[h] rounded once to fp32 (nearest, ties to even); each of x and w
    bf16 (uint16 bit patterns) or float32."""
    x, w = _c(x), _c(w)
    assert x.shape == w.shape and x.ndim == 1
    out = np.zeros(1, np.float32)
    rc = _load().oracle_exact_dot_mixed(_dtype_code(x), _dtype_code(w), x.shape[0], _p(x), _p(w), _p(out))
    if rc != 0:
        raise ValueError("exact_dot: non-finite input")
    return out[0]


def router_scores(x: np.ndarray, Wr: np.ndarray, nthreads: int = 0) -> np.ndarray:
    """s[t,e] = RN32(exact x[t] . Wr[e]) for every token t and expert e -> float32 [T,E]
    (x and Wr each bf16 or float32: fp32 router weights with bf16 tokens are allowed)."""
    x, Wr = _c(x), _c(Wr)
    T, H = x.shape
    E, H2 = Wr.shape
    assert H == H2
    s = np.empty((T, E), np.float32)
    rc = _load().oracle_router_scores_mixed(_dtype_code(x), _dtype_code(Wr), T, H, E, _p(x), _p(Wr), _p(s),
                                            nthreads or nthreads_default())
    if rc != 0:
        raise ValueError("router_scores: non-finite input")
    return s


ROUTERS = {"softmax": 0, "sigmoid": 1}


def route(scores: np.ndarray, top_k: int, bias: np.ndarray | None = None, router: str = "softmax",
          scale: float = 1.0):
    """Top-k routing of every token -> (idx int32 [T,k] ascending, w fp32 [T,k], w fp64 [T,k]).

    router="softmax": key = s (+ bias), w = softmax of the chosen keys.
    router="sigmoid": p = sigma32(s), key = p (+ bias, selection only), w = scale * p / sum p."""
    s = _c(scores, np.float32)
    T, E = s.shape
    b = _c(bias, np.float32)
    idx = np.empty((T, top_k), np.int32)
    w = np.empty((T, top_k), np.float32)
    w64 = np.empty((T, top_k), np.float64)
    rc = _load().oracle_route_mode(T, E, top_k, _p(s), _p(b), ROUTERS[router], float(scale), _p(idx),
                                   _p(w), _p(w64))
    if rc != 0:
        raise ValueError("route: top_k must be in [1, E]")
    return idx, w, w64


def sigmoid32(scores: np.ndarray) -> np.ndarray:
    """fp32(1 / (1 + e^-s)) by the oracle's fixed-sequence exponential (0 below -110, 1 above 40)."""
    s = _c(np.asarray(scores), np.float32)
    p = np.empty_like(s)
    _load().oracle_sigmoid32(s.size, _p(s), _p(p))
    return p


def dispatch(idx: np.ndarray, E: int):
    """(counts [E], offsets [E+1], perm [T*k], inv_perm [T*k]) of a routing, all int32."""
    idx = _c(idx, np.int32)
    T, k = idx.shape
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    perm = np.empty(T * k, np.int32)
    inv = np.empty(T * k, np.int32)
    rc = _load().oracle_dispatch(T, E, k, _p(idx), _p(counts), _p(offsets), _p(perm), _p(inv))
    if rc != 0:
        raise ValueError("dispatch: expert index out of range")
    return counts, offsets, perm, inv


def expert_act(xrow: np.ndarray, Wgu_e: np.ndarray, swiglu_limit: float = 0.0) -> np.ndarray:
    """SiLU(x W_g^T) * (x W_u^T) of one token through one expert, fp64 [I]; a SwiGLU limit
    L > 0 first clamps gate to <= L and up to [-L, L]."""
    xrow, Wgu_e = _c(xrow), _c(Wgu_e)
    twoI, H = Wgu_e.shape
    out = np.empty(twoI // 2, np.float64)
    _load().oracle_expert_act(_dtype_code(xrow), H, twoI // 2, _p(xrow), _p(Wgu_e),
                              float(swiglu_limit), _p(out))
    return out


def moe_tokens(x, idx, w64, Wgu, Wd, Wsgu=None, Wsd=None, tokens=None, nthreads: int = 0,
               swiglu_limit: float = 0.0, swiglu_limit_shared: float = 0.0):
    """Layer output (fp64 [n, H]) for the listed tokens (all tokens when ``tokens`` is None).
    swiglu_limit / swiglu_limit_shared: SwiGLU limits of the routed / shared experts (0: none)."""
    x, Wgu, Wd = _c(x), _c(Wgu), _c(Wd)
    Wsgu, Wsd = _c(Wsgu), _c(Wsd)
    idx = _c(idx, np.int32)
    w64 = _c(w64, np.float64)
    T, H = x.shape
    E, twoI, H2 = Wgu.shape
    assert H2 == H and Wd.shape == (E, H, twoI // 2)
    k = idx.shape[1]
    Is = 0
    if Wsgu is not None:
        Is = Wsgu.shape[0] // 2
        assert Wsgu.shape == (2 * Is, H) and Wsd.shape == (H, Is)
    tok = np.arange(T, dtype=np.int64) if tokens is None else _c(np.asarray(tokens), np.int64)
    y = np.empty((tok.shape[0], H), np.float64)
    rc = _load().oracle_moe_tokens(_dtype_code(x), tok.shape[0], _p(tok), H, E, k, twoI // 2, Is,
                                   _p(x), _p(idx), _p(w64), _p(Wgu), _p(Wd), _p(Wsgu), _p(Wsd),
                                   float(swiglu_limit), float(swiglu_limit_shared),
                                   _p(y), nthreads or nthreads_default())
    if rc != 0:
        raise ValueError("moe_tokens: expert index out of range")
    return y


def fp8_scale_shape(R: int, K: int):
    """Shape of the scale table of an FP8 weight matrix [R, K]: one scale per 128 x 128 block."""
    return ((R + 127) // 128, (K + 127) // 128)


def dequant_e4m3(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """The fp64 weights [R, K] that FP8 E4M3 codes q [R, K] (uint8) with E8M0 block scales
    s [ceil(R/128), ceil(K/128)] (uint8) stand for: e4m3(q[r, c]) * 2^(s[r//128, c//128] - 127)."""
    q, s = _c(q, np.uint8), _c(s, np.uint8)
    R, K = q.shape
    assert s.shape == fp8_scale_shape(R, K)
    out = np.empty((R, K), np.float64)
    _load().oracle_dequant_e4m3(R, K, _p(q), _p(s), _p(out))
    return out


def moe_tokens_fp8(x, idx, w64, Wgu, Wd, Wsgu=None, Wsd=None, tokens=None, nthreads: int = 0,
                   swiglu_limit: float = 0.0, swiglu_limit_shared: float = 0.0):
    """moe_tokens with bf16 tokens and FP8 expert weights.  Each weight argument is a pair
    (codes uint8, scales uint8): Wgu ([E, 2I, H], [E, ceil(2I/128), ceil(H/128)]),
    Wd ([E, H, I], [E, ceil(H/128), ceil(I/128)]), Wsgu ([2Is, H], ...), Wsd ([H, Is], ...)."""
    x = _c(x)
    assert x.dtype == np.uint16, "tokens are bf16 bit patterns"
    (gq, gs), (dq, ds) = Wgu, Wd
    gq, gs, dq, ds = (_c(a, np.uint8) for a in (gq, gs, dq, ds))
    T, H = x.shape
    E, twoI, H2 = gq.shape
    I = twoI // 2
    assert H2 == H and dq.shape == (E, H, I)
    assert gs.shape == (E,) + fp8_scale_shape(twoI, H) and ds.shape == (E,) + fp8_scale_shape(H, I)
    sgq = sgs = sdq = sds = None
    Is = 0
    if Wsgu is not None:
        (sgq, sgs), (sdq, sds) = Wsgu, Wsd
        sgq, sgs, sdq, sds = (_c(a, np.uint8) for a in (sgq, sgs, sdq, sds))
        Is = sgq.shape[0] // 2
        assert sgq.shape == (2 * Is, H) and sdq.shape == (H, Is)
        assert sgs.shape == fp8_scale_shape(2 * Is, H) and sds.shape == fp8_scale_shape(H, Is)
    idx = _c(idx, np.int32)
    w64 = _c(w64, np.float64)
    k = idx.shape[1]
    tok = np.arange(T, dtype=np.int64) if tokens is None else _c(np.asarray(tokens), np.int64)
    y = np.empty((tok.shape[0], H), np.float64)
    rc = _load().oracle_moe_tokens_fp8(tok.shape[0], _p(tok), H, E, k, I, Is, _p(x), _p(idx), _p(w64),
                                       _p(gq), _p(gs), _p(dq), _p(ds), _p(sgq), _p(sgs), _p(sdq), _p(sds),
                                       float(swiglu_limit), float(swiglu_limit_shared), _p(y),
                                       nthreads or nthreads_default())
    if rc != 0:
        raise ValueError("moe_tokens_fp8: expert index out of range")
    return y


def moe_forward(x, Wr, Wgu, Wd, Wsgu=None, Wsd=None, top_k=8, bias=None, tokens=None,
                nthreads: int = 0, swiglu_limit: float = 0.0, swiglu_limit_shared: float = 0.0,
                router: str = "softmax", routed_scale: float = 1.0):
    """The whole layer: routing for every token, output for ``tokens`` (default all).

    Returns a dict with scores, idx, w, w64, counts, offsets, perm, inv_perm and y (fp64).
    """
    s = router_scores(x, Wr, nthreads)
    idx, w, w64 = route(s, top_k, bias, router=router, scale=routed_scale)
    counts, offsets, perm, inv = dispatch(idx, Wr.shape[0])
    y = moe_tokens(x, idx, w64, Wgu, Wd, Wsgu, Wsd, tokens=tokens, nthreads=nthreads,
                   swiglu_limit=swiglu_limit, swiglu_limit_shared=swiglu_limit_shared)
    return dict(scores=s, idx=idx, w=w, w64=w64, counts=counts, offsets=offsets, perm=perm,
                inv_perm=inv, y=y)
