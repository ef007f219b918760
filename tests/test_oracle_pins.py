"""Pins of the CPU oracle against what the pages and the mathematics fix (CPU only).

Each test checks the oracle against something other than itself: exact rational
arithmetic, brute-force enumeration, closed forms, special cases that reduce to a library
routine, or invariants that the definition implies.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from conftest import to_oracle
from sparse_mixture_experts_ffn_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# --------------------------------------------------------------------------------------
# exact rational helpers (independent of the oracle's integer-bin algorithm)
# --------------------------------------------------------------------------------------
def frac_to_f32(q: Fraction) -> np.float32:
    """Round a rational to the nearest fp32, ties to even, subnormals included."""
    if q == 0:
        return np.float32(0.0)
    neg = q < 0
    q = abs(q)
    e = q.numerator.bit_length() - q.denominator.bit_length()
    while Fraction(2) ** e > q:
        e -= 1
    while Fraction(2) ** (e + 1) <= q:
        e += 1
    lsb = max(e - 23, -149)
    scaled = q / Fraction(2) ** lsb
    n = scaled.numerator // scaled.denominator
    rem = scaled - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    v = math.ldexp(n, lsb)
    if v > float(np.finfo(np.float32).max):
        v = math.inf
    f = np.float32(v)
    return -f if neg else f


def exact_value(bits_or_f32) -> Fraction:
    a = np.asarray(bits_or_f32)
    if a.dtype == np.uint16:
        f = (a.astype(np.uint32) << 16).view(np.float32)
    else:
        f = a.astype(np.float32)
    return Fraction(float(f))


def bf16_bits(values) -> np.ndarray:
    t = torch.tensor(np.asarray(values, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def brute_dot(x, w) -> np.float32:
    return frac_to_f32(sum((exact_value(a) * exact_value(b) for a, b in zip(x, w)), Fraction(0)))


def random_wide_vector(rng, n, dtype):
    """Values spanning many binades, with subnormals of the dtype and some cancellation."""
    mant = rng.standard_normal(n)
    lo = -140 if dtype == "bf16" else -155
    expo = rng.integers(lo, 60, size=n)
    v = np.ldexp(mant, expo)
    if n >= 4:  # exact cancelling pairs
        v[: n // 4] = -v[n // 4: 2 * (n // 4)]
    if dtype == "bf16":
        return bf16_bits(v.astype(np.float32))
    return v.astype(np.float32)


# --------------------------------------------------------------------------------------
# exact router dot product
# --------------------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_exact_dot_matches_rational_sum(dtype):
    rng = np.random.default_rng(1234)
    for trial in range(300):
        n = int(rng.integers(1, 80))
        x = random_wide_vector(rng, n, dtype)
        w = random_wide_vector(rng, n, dtype)
        got = oracle.exact_dot(x, w)
        want = brute_dot(x, w)
        assert got.tobytes() == want.tobytes() or (got == 0 and want == 0), (trial, got, want)


def test_exact_dot_mixed_bf16_tokens_fp32_router_weights():
    """need_fp32_gate read as fp32 router weights with bf16 tokens: the exact sum of bf16 x
    fp32 products (subnormals, extreme exponents, cancellation) against rational arithmetic."""
    rng = np.random.default_rng(4321)
    for trial in range(300):
        n = int(rng.integers(1, 80))
        x = random_wide_vector(rng, n, "bf16")
        w = random_wide_vector(rng, n, "f32")
        got = oracle.exact_dot(x, w)
        want = brute_dot(x, w)
        assert got.tobytes() == want.tobytes() or (got == 0 and want == 0), (trial, got, want)
    # router scores with fp32 weights are the same exact dots
    xs = np.stack([random_wide_vector(rng, 48, "bf16") for _ in range(3)])
    ws = np.stack([random_wide_vector(rng, 48, "f32") for _ in range(5)])
    s = oracle.router_scores(xs, ws)
    for t in range(3):
        for e in range(5):
            assert s[t, e].tobytes() == brute_dot(xs[t], ws[e]).tobytes() or (s[t, e] == 0 and brute_dot(xs[t], ws[e]) == 0)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_exact_dot_router_like_vectors(dtype):
    rng = np.random.default_rng(99)
    for _ in range(20):
        xv = rng.standard_normal(512).astype(np.float32)
        wv = (rng.standard_normal(512) * 0.02).astype(np.float32)
        x = bf16_bits(xv) if dtype == "bf16" else xv
        w = bf16_bits(wv) if dtype == "bf16" else wv
        assert oracle.exact_dot(x, w).tobytes() == brute_dot(x, w).tobytes()


def test_exact_dot_rounding_cases():
    one = np.float32(1.0)
    ones = np.ones(3, np.float32)
    # 1 + 2^-24 is the midpoint between 1 and 1+2^-23: ties to even -> 1
    assert oracle.exact_dot(np.array([1.0, 2.0 ** -24], np.float32), ones[:2]) == one
    # 1 + 3*2^-24 lies between 1+2^-23 and 1+2^-22 at their midpoint -> even is 1+2^-22
    assert oracle.exact_dot(np.array([1.0, 3 * 2.0 ** -24], np.float32), ones[:2]) == np.float32(1 + 2 ** -22)
    # a sticky bit far below breaks the tie upward
    got = oracle.exact_dot(np.array([1.0, 2.0 ** -24, 2.0 ** -60], np.float32), ones)
    assert got == np.float32(1 + 2 ** -23)
    # a sequential fp32 sum would lose the small terms; the exact sum keeps them
    v = np.array([2.0 ** 24, 1.0, 1.0], np.float32)
    assert oracle.exact_dot(v, ones) == np.float32(2 ** 24 + 2)
    # exact cancellation gives +0
    z = oracle.exact_dot(np.array([3.0, -3.0], np.float32), np.ones(2, np.float32))
    assert z == 0 and not np.signbit(z)
    # subnormal results: 2^-140 * 2^-10 = 2^-150 is half the smallest subnormal -> ties to 0
    tiny = np.array([2.0 ** -140], np.float32)
    assert oracle.exact_dot(tiny, np.array([2.0 ** -10], np.float32)) == 0
    # 3 * 2^-150 = 1.5 * 2^-149 -> ties to even -> 2 * 2^-149
    assert oracle.exact_dot(tiny, np.array([3 * 2.0 ** -10], np.float32)) == np.float32(2 * 2.0 ** -149)
    # bf16 products are exact: (1+2^-7)^2 = 1 + 2^-6 + 2^-14, representable in fp32
    b = bf16_bits([1 + 2 ** -7])
    assert oracle.exact_dot(b, b) == np.float32(1 + 2 ** -6 + 2 ** -14)


def test_router_scores_are_exact_dots():
    rng = np.random.default_rng(5)
    x = bf16_bits(rng.standard_normal((3, 40)))
    Wr = bf16_bits(rng.standard_normal((5, 40)) * 0.02)
    s = oracle.router_scores(x, Wr)
    for t in range(3):
        for e in range(5):
            assert s[t, e].tobytes() == brute_dot(x[t], Wr[e]).tobytes()


# --------------------------------------------------------------------------------------
# top-k selection and renormalised softmax
# --------------------------------------------------------------------------------------
def brute_force_set(key, k, bias=None):
    E = len(key)
    kk = [np.float32(key[e] + bias[e]) if bias is not None else np.float32(key[e]) for e in range(E)]
    found = []
    for S in itertools.combinations(range(E), k):
        Sset = set(S)
        ok = all(kk[a] > kk[b] or (kk[a] == kk[b] and a < b)
                 for a in S for b in range(E) if b not in Sset)
        if ok:
            found.append(S)
    assert len(found) == 1  # the order (key desc, index asc) is total
    return list(found[0])


@pytest.mark.parametrize("E", [2, 3, 5, 8])
def test_selection_brute_force_with_ties(E):
    rng = np.random.default_rng(E)
    T = 60
    # few distinct values so that ties are frequent
    levels = rng.standard_normal(3).astype(np.float32)
    s = levels[rng.integers(0, 3, size=(T, E))]
    bias = rng.choice(np.array([0.0, 0.5, -0.25], np.float32), size=E)
    for k in range(1, E + 1):
        for b in (None, bias):
            idx, w, w64 = oracle.route(s, k, b)
            for t in range(T):
                assert list(idx[t]) == brute_force_set(s[t], k, b)
                assert np.all(np.diff(idx[t]) > 0)


def test_selection_prefers_lower_index_on_equal_keys():
    s = np.zeros((1, 6), np.float32)
    idx, w, _ = oracle.route(s, 3)
    assert list(idx[0]) == [0, 1, 2]
    assert np.allclose(w, 1 / 3, rtol=0, atol=1e-7)


def test_weights_sum_to_one_and_k1():
    rng = np.random.default_rng(3)
    s = (rng.standard_normal((200, 288)) * 1.28).astype(np.float32)
    idx, w, w64 = oracle.route(s, 8)
    assert np.all(np.abs(w.astype(np.float64).sum(1) - 1) <= 8 * 2.0 ** -23)
    assert np.all(np.abs(w64.sum(1) - 1) <= 1e-14)
    # the selected experts are the 8 largest scores (no ties in continuous data)
    ref = np.sort(np.argsort(-s, axis=1, kind="stable")[:, :8], axis=1)
    assert np.array_equal(idx, ref)
    idx1, w1, _ = oracle.route(s, 1)
    assert np.all(w1 == 1.0)
    assert np.array_equal(idx1[:, 0], np.argmax(s, axis=1))


def test_softmax_closed_form():
    # keys 0 and ln 3: renormalised weights 1/4 and 3/4; higher key gets more weight
    ln3 = np.float32(math.log(3.0))
    s = np.array([[0.0, ln3, -5.0]], np.float32)
    idx, w, w64 = oracle.route(s, 2)
    assert list(idx[0]) == [0, 1]
    assert abs(w64[0, 0] - 0.25) < 1e-7 and abs(w64[0, 1] - 0.75) < 1e-7
    # the third expert's key cancels out of the renormalised weights
    s2 = np.array([[0.0, ln3, 4.0]], np.float32)
    idx2, _, w2 = oracle.route(s2, 2)
    assert list(idx2[0]) == [1, 2]
    assert abs(w2[0, 0] - 1 / (1 + math.exp(4.0 - float(ln3)))) < 1e-12


def test_bias_shifts_selection():
    s = np.zeros((1, 4), np.float32)
    bias = np.array([0.0, 0.0, 1.0, 0.5], np.float32)
    idx, w, w64 = oracle.route(s, 2, bias)
    assert list(idx[0]) == [2, 3]
    assert abs(w64[0, 1] / w64[0, 0] - math.exp(-0.5)) < 1e-12


# --------------------------------------------------------------------------------------
# dispatch bookkeeping
# --------------------------------------------------------------------------------------
def test_dispatch_against_library_sort():
    rng = np.random.default_rng(8)
    T, E, k = 97, 12, 3
    idx = np.stack([np.sort(rng.choice(E, size=k, replace=False)) for _ in range(T)]).astype(np.int32)
    counts, offsets, perm, inv = oracle.dispatch(idx, E)
    assert np.array_equal(counts, np.bincount(idx.ravel(), minlength=E))
    assert offsets[0] == 0 and np.array_equal(offsets[1:], np.cumsum(counts))
    order = sorted(range(T * k), key=lambda a: (idx.ravel()[a], a // k))
    assert list(perm) == order
    assert np.array_equal(inv[perm], np.arange(T * k))


# --------------------------------------------------------------------------------------
# expert FFNs and the combine
# --------------------------------------------------------------------------------------
def silu(z):
    return z / (1.0 + np.exp(-z))


def test_silu_gate_up_closed_form():
    ln3 = np.float32(math.log(3.0))
    x = np.array([1.0], np.float32)
    for g, want_silu in ((ln3, 0.75 * float(ln3)), (-ln3, -0.25 * float(ln3)), (np.float32(0), 0.0)):
        Wgu = np.array([[g], [2.0]], np.float32)  # gate row, then up row
        act = oracle.expert_act(x, Wgu)
        assert abs(act[0] - 2.0 * want_silu) < 1e-7
    # gate and up are not interchangeable: SiLU(2)*ln3 != SiLU(ln3)*2
    act = oracle.expert_act(x, np.array([[2.0], [ln3]], np.float32))
    assert abs(act[0] - 2.0 / (1 + math.exp(-2.0)) * float(ln3)) < 1e-7
    assert abs(act[0] - 1.5 * float(ln3)) > 0.1


def test_swiglu_limit_closed_form():
    """The SwiGLU limit L (llm-atlas page "Step-3.5-Flash", table "Champs bruts du
    config.json": swiglu_limits, swiglu_limits_shared; values only) read as a clamp of the
    activation inputs: gate <- min(gate, L), up <- clip(up, -L, L); L = 0 is no clamp."""
    x = np.array([1.0], np.float32)
    s7 = 7.0 / (1.0 + math.exp(-7.0))  # SiLU(7)
    cases = [  # gate, up, L, expected
        (10.0, 10.0, 7.0, s7 * 7.0),                                  # both clamped
        (10.0, -10.0, 7.0, s7 * -7.0),                                # up clamped from below
        (-10.0, 3.0, 7.0, -10.0 / (1.0 + math.exp(10.0)) * 3.0),     # gate has no lower clamp
        (5.0, 5.0, 7.0, 5.0 / (1.0 + math.exp(-5.0)) * 5.0),         # inside the limit
        (10.0, 10.0, 0.0, 10.0 / (1.0 + math.exp(-10.0)) * 10.0),    # L = 0: no clamp
    ]
    for g, u, L, want in cases:
        act = oracle.expert_act(x, np.array([[g], [u]], np.float32), swiglu_limit=L)
        assert abs(act[0] - want) <= 1e-12 * max(1.0, abs(want)), (g, u, L, act[0], want)


def _numpy_ffn(x, Wgu, Wd, limit=0.0):
    """Dense gated FFN with numpy fp64 matmuls (a library routine, not the oracle)."""
    I = Wgu.shape[0] // 2
    g = x @ Wgu[:I].T
    u = x @ Wgu[I:].T
    if limit > 0:
        g, u = np.minimum(g, limit), np.clip(u, -limit, limit)
    return (silu(g) * u) @ Wd.T


def _f64(t):
    return t.to(torch.float64).numpy()


def _small(dtype="f32", **kw):
    base = dict(T=24, H=64, E=6, top_k=2, I=32, I_shared=32, r_std=0.1, rms_norm=False)
    base.update(kw)
    return inputs.small_config(dtype=dtype, **base)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_identical_experts_reduce_to_one_dense_ffn(dtype):
    cfg = _small(dtype)
    d = inputs.make_inputs(cfg)
    Wgu = d["W_gate_up"][:1].expand(cfg.E, -1, -1).contiguous()
    Wd = d["W_down"][:1].expand(cfg.E, -1, -1).contiguous()
    r = oracle.moe_forward(to_oracle(d["x"]), to_oracle(d["W_router"]), to_oracle(Wgu), to_oracle(Wd),
                           to_oracle(d["Ws_gate_up"]), to_oracle(d["Ws_down"]), top_k=cfg.top_k)
    x = _f64(d["x"])
    want = _numpy_ffn(x, _f64(Wgu[0]), _f64(Wd[0])) + _numpy_ffn(x, _f64(d["Ws_gate_up"]), _f64(d["Ws_down"]))
    assert np.allclose(r["y"], want, rtol=1e-10, atol=1e-12)


def test_swiglu_limits_of_routed_and_shared_experts():
    """Identical routed experts with limit 0.3 and a shared expert with limit 0.2 reduce to
    two dense clamped FFNs (numpy); swapping the two limits would fail."""
    cfg = _small("f32", w_std=0.2)
    d = inputs.make_inputs(cfg)
    Wgu = d["W_gate_up"][:1].expand(cfg.E, -1, -1).contiguous()
    Wd = d["W_down"][:1].expand(cfg.E, -1, -1).contiguous()
    r = oracle.moe_forward(to_oracle(d["x"]), to_oracle(d["W_router"]), to_oracle(Wgu), to_oracle(Wd),
                           to_oracle(d["Ws_gate_up"]), to_oracle(d["Ws_down"]), top_k=cfg.top_k,
                           swiglu_limit=0.3, swiglu_limit_shared=0.2)
    x = _f64(d["x"])
    want = _numpy_ffn(x, _f64(Wgu[0]), _f64(Wd[0]), 0.3) + _numpy_ffn(x, _f64(d["Ws_gate_up"]),
                                                                        _f64(d["Ws_down"]), 0.2)
    assert np.allclose(r["y"], want, rtol=1e-10, atol=1e-12)
    unclamped = _numpy_ffn(x, _f64(Wgu[0]), _f64(Wd[0])) + _numpy_ffn(x, _f64(d["Ws_gate_up"]),
                                                                       _f64(d["Ws_down"]))
    assert np.abs(want - unclamped).max() > 1e-3  # the clamps are active on these inputs


def test_top_k_equal_E_is_the_full_softmax_mixture():
    cfg = _small("f32", top_k=6)
    d = inputs.make_inputs(cfg)
    r = oracle.moe_forward(to_oracle(d["x"]), to_oracle(d["W_router"]), to_oracle(d["W_gate_up"]),
                           to_oracle(d["W_down"]), to_oracle(d["Ws_gate_up"]), to_oracle(d["Ws_down"]),
                           top_k=cfg.E)
    x = _f64(d["x"])
    logits = x @ _f64(d["W_router"]).T  # fp64 library matmul, rounding differences << 1e-6
    p = np.exp(logits - logits.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    want = _numpy_ffn(x, _f64(d["Ws_gate_up"]), _f64(d["Ws_down"]))
    for e in range(cfg.E):
        want += p[:, e:e + 1] * _numpy_ffn(x, _f64(d["W_gate_up"][e]), _f64(d["W_down"][e]))
    assert np.allclose(r["y"], want, rtol=1e-6, atol=1e-9)
    assert np.array_equal(r["idx"], np.tile(np.arange(cfg.E, dtype=np.int32), (cfg.T, 1)))


def test_zero_down_projection_leaves_the_shared_expert():
    cfg = _small("bf16")
    d = inputs.make_inputs(cfg)
    Wd0 = torch.zeros_like(d["W_down"])
    r = oracle.moe_forward(to_oracle(d["x"]), to_oracle(d["W_router"]), to_oracle(d["W_gate_up"]),
                           to_oracle(Wd0), to_oracle(d["Ws_gate_up"]), to_oracle(d["Ws_down"]),
                           top_k=cfg.top_k)
    want = _numpy_ffn(_f64(d["x"]), _f64(d["Ws_gate_up"]), _f64(d["Ws_down"]))
    assert np.allclose(r["y"], want, rtol=1e-10, atol=1e-12)
    r2 = oracle.moe_forward(to_oracle(d["x"]), to_oracle(d["W_router"]), to_oracle(d["W_gate_up"]),
                            to_oracle(Wd0), None, None, top_k=cfg.top_k)
    assert np.all(r2["y"] == 0.0)


def test_zero_input():
    cfg = _small("bf16")
    d = inputs.make_inputs(cfg)
    x0 = torch.zeros_like(d["x"])
    r = oracle.moe_forward(to_oracle(x0), to_oracle(d["W_router"]), to_oracle(d["W_gate_up"]),
                           to_oracle(d["W_down"]), to_oracle(d["Ws_gate_up"]), to_oracle(d["Ws_down"]),
                           top_k=cfg.top_k)
    assert np.all(r["scores"] == 0)
    assert np.array_equal(r["idx"], np.tile(np.arange(cfg.top_k, dtype=np.int32), (cfg.T, 1)))
    assert np.all(r["w"] == np.float32(1.0 / cfg.top_k))
    assert np.all(r["y"] == 0.0)


def test_duplicated_router_rows_tie_toward_lower_index():
    cfg = _small("bf16", E=8, top_k=3)
    d = inputs.make_inputs(cfg)
    Wr = d["W_router"].clone()
    Wr[5] = Wr[2]  # experts 2 and 5 always tie exactly
    r = oracle.moe_forward(to_oracle(d["x"]), to_oracle(Wr), to_oracle(d["W_gate_up"]),
                           to_oracle(d["W_down"]), None, None, top_k=cfg.top_k)
    assert np.array_equal(r["scores"][:, 2], r["scores"][:, 5])
    for t in range(cfg.T):
        chosen = set(r["idx"][t])
        assert not (5 in chosen and 2 not in chosen)


def test_token_permutation_equivariance():
    cfg = _small("bf16", T=30)
    d = inputs.make_inputs(cfg)
    args = [to_oracle(d[k]) for k in ("W_router", "W_gate_up", "W_down", "Ws_gate_up", "Ws_down")]
    r = oracle.moe_forward(to_oracle(d["x"]), *args, top_k=cfg.top_k)
    p = np.random.default_rng(0).permutation(cfg.T)
    rp = oracle.moe_forward(to_oracle(d["x"])[p], *args, top_k=cfg.top_k)
    assert np.array_equal(rp["idx"], r["idx"][p])
    assert np.array_equal(rp["w"], r["w"][p])
    assert np.array_equal(rp["y"], r["y"][p])


def test_token_subset_matches_full_output():
    cfg = _small("f32", T=20)
    d = inputs.make_inputs(cfg)
    args = [to_oracle(d[k]) for k in ("W_router", "W_gate_up", "W_down", "Ws_gate_up", "Ws_down")]
    r = oracle.moe_forward(to_oracle(d["x"]), *args, top_k=cfg.top_k)
    sub = [3, 17, 0]
    rs = oracle.moe_forward(to_oracle(d["x"]), *args, top_k=cfg.top_k, tokens=sub)
    assert np.array_equal(rs["y"], r["y"][sub])


# --------------------------------------------------------------------------------------
# the pages' shape constants
# --------------------------------------------------------------------------------------
def test_page_shapes_give_the_published_parameter_totals():
    c = json.load(open(os.path.join(GOLDEN, "step35_flash_shapes.json")))
    H, E, I, Is = c["hidden_size"], c["moe_num_experts"], c["moe_intermediate_size"], c["share_expert_dim"]
    n_moe = c["moe_layers_enum_last"] - c["moe_layers_enum_first"] + 1
    assert n_moe == 42
    per_expert = 3 * H * I  # gate, up and down matrices of H x I
    per_layer = E * per_expert + 3 * H * Is + E * H
    total_moe = n_moe * per_layer
    embed = 2 * c["vocab_size"] * H  # untied input and output embeddings
    dense = (c["moe_layers_enum_first"]) * 3 * H * c["intermediate_size"]
    # the routed experts are most of the 196 B; attention and norms make up the rest
    assert 0.9 * 196e9 < total_moe + embed + dense < 196e9
    # active: top-8 routed + shared + router per MoE layer, plus the dense layers and embeddings
    active = n_moe * ((c["moe_top_k"] + 1) * per_expert + E * H) + dense + embed
    assert 0.6 * 11e9 < active < 11e9
    # two-matrix experts would be inconsistent with the published total
    assert n_moe * E * 2 * H * I < 0.7 * 196e9


def test_workload_table_matches_the_pages():
    c = json.load(open(os.path.join(GOLDEN, "step35_flash_shapes.json")))
    for name in ("decode_t4", "decode_t128", "prefill_t4096", "prefill_t16384_skew"):
        cfg = inputs.CONFIGS[name]
        assert (cfg.H, cfg.E, cfg.top_k, cfg.I, cfg.I_shared) == (
            c["hidden_size"], c["moe_num_experts"], c["moe_top_k"], c["moe_intermediate_size"],
            c["share_expert_dim"])


# --------------------------------------------------------------------------------------
# the router as configured: sigmoid scores, selection-only bias, renormalised and scaled
# weights (llm-atlas page "Step-3.5-Flash", table "Champs bruts du config.json":
# moe_router_activation, use_moe_router_bias, moe_router_scaling_factor)
# --------------------------------------------------------------------------------------
def _sigma32_reference(s):
    """fp32 rounding of 1/(1+e^-s) evaluated with 40-digit decimal arithmetic."""
    from decimal import Decimal, getcontext
    getcontext().prec = 40
    out = []
    for v in np.asarray(s, np.float32).tolist():
        out.append(float(1 / (1 + (-Decimal(v)).exp())))
    return np.array(out, np.float64).astype(np.float32)


def test_sigmoid32_against_high_precision_values():
    rng = np.random.default_rng(7)
    s = np.concatenate([rng.uniform(-110, 40, 400), rng.normal(0, 3, 400), [0.0, 1e-8, -1e-8, 17.0, -87.5]])
    s = s.astype(np.float32)
    p = oracle.sigmoid32(s)
    want = _sigma32_reference(s)
    # fp32 results equal the correctly rounded value (a near-tie could differ by one ulp)
    ulps = np.abs(p.view(np.int32).astype(np.int64) - want.view(np.int32).astype(np.int64))
    assert ulps.max() <= 1 and (ulps == 0).mean() >= 0.995, (ulps.max(), (ulps == 0).mean())


def test_sigmoid32_special_values_and_monotonicity():
    p = oracle.sigmoid32(np.array([0.0, 40.5, 1e30, -110.5, -1e30], np.float32))
    assert p.tolist() == [0.5, 1.0, 1.0, 0.0, 0.0]
    grid = np.sort(np.concatenate([np.linspace(-110, 40, 200001), np.linspace(-1, 1, 100001)])).astype(np.float32)
    pg = oracle.sigmoid32(grid)
    assert np.all(np.diff(pg.astype(np.float64)) >= 0)
    s = np.linspace(-30, 30, 1001).astype(np.float32)
    assert np.abs(oracle.sigmoid32(s).astype(np.float64) + oracle.sigmoid32(-s) - 1).max() < 2e-7


@pytest.mark.parametrize("E", [5, 8])
def test_sigmoid_router_selection_brute_force(E):
    rng = np.random.default_rng(E)
    for trial in range(40):
        k = int(rng.integers(1, E + 1))
        s = rng.normal(0, 2, (1, E)).astype(np.float32)
        bias = rng.normal(0, 0.3, E).astype(np.float32) if trial % 2 else None
        if trial % 5 == 0:  # saturated scores: equal p, ties toward the lower index
            s[0, : E // 2] = 50.0
        idx, _, _ = oracle.route(s, k, bias, router="sigmoid", scale=3.0)
        p = oracle.sigmoid32(s[0])
        key = p + (bias if bias is not None else np.float32(0))
        key = key.astype(np.float32)
        valid = []
        for S in itertools.combinations(range(E), k):
            rest = [f for f in range(E) if f not in S]
            if all((key[e] > key[f]) or (key[e] == key[f] and e < f) for e in S for f in rest):
                valid.append(S)
        assert len(valid) == 1 and tuple(idx[0]) == valid[0]


def test_sigmoid_router_weights_use_scores_not_keys():
    """w_j = 3 p_j / sum_S p with p = sigma32(s); the bias steers the choice only."""
    E, k = 8, 3
    s = np.array([[-6.0, 2.0, 1.0, 0.5, 0.0, -1.0, 3.0, -2.0]], np.float32)
    bias = np.zeros(E, np.float32)
    bias[0] = 100.0  # expert 0 (a tiny score) is always chosen
    idx, w, w64 = oracle.route(s, k, bias, router="sigmoid", scale=3.0)
    p = oracle.sigmoid32(s[0]).astype(np.float64)
    assert idx[0].tolist() == [0, 1, 6]
    want = 3.0 * p[[0, 1, 6]] / p[[0, 1, 6]].sum()
    assert np.allclose(w64[0], want, rtol=1e-15, atol=0)
    assert abs(w64[0].sum() - 3.0) < 1e-14 and w64[0][0] < 0.01
    # without the bias the same scores pick the three best p
    idx2, _, w2 = oracle.route(s, k, None, router="sigmoid", scale=3.0)
    assert idx2[0].tolist() == [1, 2, 6] and abs(w2[0].sum() - 3.0) < 1e-14


# --------------------------------------------------------------------------------------
# blockwise FP8 expert weights: E4M3 codes, one E8M0 scale per 128 x 128 block
# --------------------------------------------------------------------------------------
def torch_e4m3(codes: np.ndarray) -> np.ndarray:
    """Library decoding of E4M3 codes (torch.float8_e4m3fn) to fp64."""
    return torch.from_numpy(np.ascontiguousarray(codes, np.uint8)).view(torch.float8_e4m3fn).double().numpy()


def torch_e8m0(codes: np.ndarray) -> np.ndarray:
    """Library decoding of E8M0 scale codes (torch.float8_e8m0fnu) to fp64."""
    return torch.from_numpy(np.ascontiguousarray(codes, np.uint8)).view(torch.float8_e8m0fnu).double().numpy()


def test_e4m3_decoding_of_all_codes_matches_the_library():
    q = np.arange(256, dtype=np.uint8).reshape(2, 128)
    got = oracle.dequant_e4m3(q, np.full((1, 1), 127, np.uint8))  # scale 2^0
    ref = torch_e4m3(q)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan) and nan.sum() == 2  # S.1111.111 only
    assert np.array_equal(got[~nan], ref[~nan])
    # landmarks of the format: 1.0, the largest finite value, the smallest subnormal, -0
    assert got[0, 0x38] == 1.0 and got[0, 0x7E] == 448.0 and got[0, 0x01] == 2.0 ** -9
    assert got[1, 0] == 0.0 and math.copysign(1.0, got[1, 0]) == -1.0


def test_e8m0_scales_match_the_library():
    v = np.arange(255, dtype=np.uint8)
    q = np.full((1, 255 * 128), 0x38, np.uint8)  # every weight 1.0, one block per scale
    got = oracle.dequant_e4m3(q, v.reshape(1, 255))[0, ::128]
    assert np.array_equal(got, torch_e8m0(v))
    assert got[127] == 1.0 and got[0] == 2.0 ** -127


def test_fp8_block_scales_index_row_and_column_blocks():
    """Ragged 3 x 4 block grid, a different scale per block: the decoded matrix must equal the
    library decoding of each code times its own block's scale, built by block expansion."""
    rng = np.random.default_rng(7)
    R, K = 320, 448
    q = rng.integers(0, 256, size=(R, K), dtype=np.uint8)
    q[(q & 0x7F) == 0x7F] = 0x3C  # no NaN codes
    s = rng.integers(100, 150, size=oracle.fp8_scale_shape(R, K), dtype=np.uint8)
    assert s.shape == (3, 4)
    expanded = np.kron(torch_e8m0(s), np.ones((128, 128)))[:R, :K]
    ref = torch_e4m3(q) * expanded
    assert np.array_equal(oracle.dequant_e4m3(q, s), ref)


def _fp8_layer(rng, E, H, I, Is):
    def mat(*shape):
        q = rng.integers(0, 256, size=shape, dtype=np.uint8)
        q[(q & 0x7F) == 0x7F] = 0xB8  # no NaN codes
        s = rng.integers(118, 128, size=shape[:-2] + oracle.fp8_scale_shape(*shape[-2:]), dtype=np.uint8)
        return q, s
    return mat(E, 2 * I, H), mat(E, H, I), mat(2 * Is, H), mat(H, Is)


def _as_bf16_bits(w: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(w).to(torch.bfloat16)
    assert np.array_equal(t.double().numpy(), w), "FP8 weights must be exact in bf16"
    return t.view(torch.int16).numpy().view(np.uint16)


def test_fp8_layer_equals_the_bf16_layer_on_the_decoded_weights():
    """Every E4M3 value times a power of two in the test's range is exact in bf16, so the FP8
    layer must give the bf16 layer's output bit for bit once the weights are decoded by the
    library (per expert, with per-expert scale tables and gate rows before up rows)."""
    rng = np.random.default_rng(11)
    E, H, I, Is, T, k = 4, 256, 256, 128, 5, 2
    gu, dn, sgu, sdn = _fp8_layer(rng, E, H, I, Is)

    def decode(q, s):  # library decoding, block expansion per matrix
        if q.ndim == 3:
            return np.stack([decode(q[e], s[e]) for e in range(q.shape[0])])
        return torch_e4m3(q) * np.kron(torch_e8m0(s), np.ones((128, 128)))[: q.shape[0], : q.shape[1]]

    x = torch.randn(T, H, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    idx = np.array([[0, 3], [1, 2], [2, 3], [0, 1], [3, 0]], np.int32)
    w64 = rng.random((T, k))
    y8 = oracle.moe_tokens_fp8(xb, idx, w64, gu, dn, sgu, sdn, swiglu_limit=7.0)
    yb = oracle.moe_tokens(xb, idx, w64, _as_bf16_bits(decode(*gu)), _as_bf16_bits(decode(*dn)),
                           _as_bf16_bits(decode(*sgu)), _as_bf16_bits(decode(*sdn)), swiglu_limit=7.0)
    assert np.array_equal(y8, yb)
    # the shared expert alone: routed down-projections of zero give the shared output
    zq = np.zeros_like(dn[0])
    y_sh = oracle.moe_tokens_fp8(xb, idx, w64, gu, (zq, dn[1]), sgu, sdn)
    y_ref = oracle.moe_tokens(xb, idx, w64, _as_bf16_bits(decode(*gu)), _as_bf16_bits(np.zeros((E, H, I))),
                              _as_bf16_bits(decode(*sgu)), _as_bf16_bits(decode(*sdn)))
    assert np.array_equal(y_sh, y_ref)


def test_e8m0_nan_code_and_negative_zero_codes():
    """E8M0 255 is NaN (like the library's float8_e8m0fnu); a -0 code times any scale is -0."""
    q = np.full((1, 256), 0x80, np.uint8)
    got = oracle.dequant_e4m3(q, np.array([[255, 3]], np.uint8))
    assert np.isnan(got[0, :128]).all() and np.isnan(torch_e8m0(np.array([255], np.uint8))).all()
    assert (got[0, 128:] == 0).all() and (np.signbit(got[0, 128:])).all()


def test_fp8_layer_token_subset_and_permutation():
    """Invariants of the FP8 layer: a token subset gives the same rows as the full batch, and
    permuting the tokens (with their routing) permutes the outputs."""
    rng = np.random.default_rng(12)
    E, H, I, Is, T, k = 3, 256, 128, 128, 6, 2
    gu, dn, sgu, sdn = _fp8_layer(rng, E, H, I, Is)
    x = torch.randn(T, H, generator=torch.Generator().manual_seed(4)).to(torch.bfloat16)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    idx = np.array([[0, 1], [1, 2], [0, 2], [2, 0], [1, 0], [0, 1]], np.int32)
    w64 = rng.random((T, k))
    full = oracle.moe_tokens_fp8(xb, idx, w64, gu, dn, sgu, sdn)
    sub = oracle.moe_tokens_fp8(xb, idx, w64, gu, dn, sgu, sdn, tokens=[4, 1])
    assert np.array_equal(sub, full[[4, 1]])
    perm = rng.permutation(T)
    permuted = oracle.moe_tokens_fp8(np.ascontiguousarray(xb[perm]), idx[perm], w64[perm], gu, dn, sgu, sdn)
    assert np.array_equal(permuted, full[perm])


# --------------------------------------------------------------------------------------
# the routed-expert gather and the weighted combine, restated with numpy
# --------------------------------------------------------------------------------------
def _numpy_layer(x, idx, w, Wgu, Wd, Wsgu=None, Wsd=None):
    """y_t = sum_j w[t, j] * FFN_{idx[t, j]}(x_t) + shared(x_t), written independently of the
    oracle with numpy fp64 matmuls: for each expert, the (token, slot) pairs routed to it
    are found with numpy and their weighted FFN rows are scattered back with np.add.at
    (the definition of the layer on the llm-atlas page "Step-3.5-Flash", "Champs bruts du
    config.json": moe_top_k, norm_expert_weight; the weights are inputs here)."""
    T, H = x.shape
    y = np.zeros((T, H))
    for e in np.unique(idx):
        tok, slot = np.nonzero(idx == e)
        np.add.at(y, tok, w[tok, slot][:, None] * _numpy_ffn(x[tok], Wgu[e], Wd[e]))
    if Wsgu is not None:
        y += _numpy_ffn(x, Wsgu, Wsd)
    return y


def _hand_routing(T, E, k, rng):
    """Distinct experts per token in a scrambled order (no slot j holds expert j) with
    deliberately unequal weights."""
    idx = np.empty((T, k), np.int32)
    for t in range(T):
        while True:
            c = rng.choice(E, size=k, replace=False)
            if not np.any(c == np.arange(k)):
                break
        idx[t] = np.sort(c)[::-1]  # descending, unlike the oracle's own ascending routing
    w = rng.dirichlet(np.linspace(0.5, 4.0, k), size=T)
    return idx, w


@pytest.mark.parametrize("case", ["tiny_f32_t64", "bf16_k3_of_8", "decode_shaped_bf16"])
@pytest.mark.parametrize("routing", ["oracle", "hand"])
def test_routed_gather_matches_a_numpy_restatement(case, routing):
    """The routed experts' gather (expert idx[t, j] with weight w[t, j]) and the combine of
    oracle.moe_tokens against an independent numpy restatement, with top_k < E and distinct
    experts, so that reading the slot index j as the expert, or pairing weights with the
    wrong slot, fails.  Cases: the tiny fp32 workload (top-2 of 16); bf16 top-3 of 8;
    decode-shaped routing (H = 4096, top-8 of 288) with narrow experts."""
    rng = np.random.default_rng(21)
    if case == "tiny_f32_t64":
        cfg = inputs.CONFIGS["tiny_f32_t64"]
    elif case == "bf16_k3_of_8":
        cfg = _small("bf16", T=40, H=128, E=8, top_k=3, I=64, I_shared=32, w_std=0.1)
    else:
        cfg = inputs.small_config(T=4, H=4096, E=288, top_k=8, I=32, I_shared=32, seed=1, w_std=0.05)
    d = inputs.make_inputs(cfg)
    xo = to_oracle(d["x"])
    if routing == "oracle":
        s = oracle.router_scores(xo, to_oracle(d["W_router"]))
        idx, _, w64 = oracle.route(s, cfg.top_k)
    else:
        idx, w64 = _hand_routing(cfg.T, cfg.E, cfg.top_k, rng)
    assert cfg.top_k < cfg.E
    assert len(np.unique(idx.ravel())) > cfg.top_k  # tokens use different experts
    args = [to_oracle(d[k]) for k in ("W_gate_up", "W_down", "Ws_gate_up", "Ws_down")]
    got = oracle.moe_tokens(xo, idx, w64, *args)
    want = _numpy_layer(_f64(d["x"]), idx, w64, _f64(d["W_gate_up"]), _f64(d["W_down"]),
                        _f64(d["Ws_gate_up"]), _f64(d["Ws_down"]))
    rel = np.abs(got - want).max() / np.abs(want).max()
    assert rel <= 1e-5, rel
    # the pin separates the experts: treating slot j as expert j, or reversing the weights'
    # pairing with the slots, moves the output far outside the tolerance
    wrong_e = _numpy_layer(_f64(d["x"]), np.tile(np.arange(cfg.top_k, dtype=np.int32), (cfg.T, 1)), w64,
                           _f64(d["W_gate_up"]), _f64(d["W_down"]), _f64(d["Ws_gate_up"]), _f64(d["Ws_down"]))
    wrong_w = _numpy_layer(_f64(d["x"]), idx, w64[:, ::-1], _f64(d["W_gate_up"]), _f64(d["W_down"]),
                           _f64(d["Ws_gate_up"]), _f64(d["Ws_down"]))
    for wrong in (wrong_e, wrong_w):
        assert np.abs(wrong - want).max() / np.abs(want).max() > 1e-3


def test_fp8_routed_gather_matches_a_numpy_restatement():
    """oracle.moe_tokens_fp8 against the numpy restatement on weights decoded by the library's
    E4M3 / E8M0 decoders (block expansion per matrix), with a hand routing of distinct
    experts in scrambled slots and unequal weights."""
    rng = np.random.default_rng(22)
    E, H, I, Is, T, k = 6, 256, 128, 128, 7, 3
    gu, dn, sgu, sdn = _fp8_layer(rng, E, H, I, Is)

    def decode(q, s):
        if q.ndim == 3:
            return np.stack([decode(q[e], s[e]) for e in range(q.shape[0])])
        return torch_e4m3(q) * np.kron(torch_e8m0(s), np.ones((128, 128)))[: q.shape[0], : q.shape[1]]

    x = torch.randn(T, H, generator=torch.Generator().manual_seed(6)).to(torch.bfloat16)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    idx, w64 = _hand_routing(T, E, k, rng)
    got = oracle.moe_tokens_fp8(xb, idx, w64, gu, dn, sgu, sdn)
    want = _numpy_layer(x.double().numpy(), idx, w64, decode(*gu), decode(*dn), decode(*sgu), decode(*sdn))
    assert np.abs(got - want).max() / np.abs(want).max() <= 1e-5
