"""The Python binding's argument checks (CPU only).  The C ABI receives bare pointers and
cannot see buffer sizes, so shape, dtype and device mismatches must be caught in the
binding, before anything is launched: each case here raises ValueError on CPU tensors."""
import pytest
import torch

import sparse_mixture_experts_ffn_b200 as moe

T, H, E, I, Is, K = 6, 128, 8, 256, 128, 2


def layer(dtype=torch.bfloat16, **over):
    d = dict(x=torch.zeros(T, H, dtype=dtype), W_router=torch.zeros(E, H, dtype=dtype),
             W_gate_up=torch.zeros(E, 2 * I, H, dtype=dtype), W_down=torch.zeros(E, H, I, dtype=dtype),
             Ws_gate_up=torch.zeros(2 * Is, H, dtype=dtype), Ws_down=torch.zeros(H, Is, dtype=dtype))
    d.update(over)
    return d


def call(d, **kw):
    return moe.moe_layer_forward(d["x"], d["W_router"], d["W_gate_up"], d["W_down"], d["Ws_gate_up"],
                                 d["Ws_down"], top_k=K, **kw)


def test_consistent_arguments_fail_only_for_want_of_a_gpu():
    with pytest.raises(ValueError, match="CUDA"):
        call(layer())
    with pytest.raises(ValueError, match="CUDA"):  # fp32 router weights with bf16 tokens are allowed
        call(layer(W_router=torch.zeros(E, H)))


@pytest.mark.parametrize("name,bad,match", [
    ("W_gate_up", torch.zeros(E, 2 * I, H), "W_gate_up"),                       # fp32 experts, bf16 tokens
    ("W_gate_up", torch.zeros(E - 1, 2 * I, H, dtype=torch.bfloat16), "W_gate_up"),  # fewer experts than the router
    ("W_down", torch.zeros(E, I, H, dtype=torch.bfloat16), "W_down"),           # transposed
    ("Ws_gate_up", torch.zeros(Is, H, dtype=torch.bfloat16), "Ws_gate_up|Ws_down"),
    ("Ws_down", torch.zeros(H, 2 * Is, dtype=torch.bfloat16), "Ws_down"),
    ("W_router", torch.zeros(E, H + 8, dtype=torch.bfloat16), "W_router"),
    ("x", torch.zeros(T, H, 1, dtype=torch.bfloat16), r"x must be \[T, H\]"),
    ("x", torch.zeros(T, H, dtype=torch.float16), "bf16 or fp32"),
    ("W_gate_up", torch.zeros(2 * I, H, dtype=torch.bfloat16), "W_gate_up"),
])
def test_mismatched_tensors_are_rejected(name, bad, match):
    with pytest.raises(ValueError, match=match):
        call(layer(**{name: bad}))


def test_fp32_tokens_need_fp32_router_weights():
    with pytest.raises(ValueError, match="W_router"):
        call(layer(torch.float32, W_router=torch.zeros(E, H, dtype=torch.bfloat16)))


def test_router_bias_and_y_are_checked():
    with pytest.raises(ValueError, match="router_bias"):
        call(layer(), router_bias=torch.zeros(E + 1))
    with pytest.raises(ValueError, match="router_bias"):
        call(layer(), router_bias=torch.zeros(E, dtype=torch.float64))
    with pytest.raises(ValueError, match="y must be"):
        call(layer(), y=torch.zeros(T, H))
    with pytest.raises(ValueError, match="y must be"):
        call(layer(), y=torch.zeros(T + 1, H, dtype=torch.bfloat16))


def test_one_shared_matrix_without_the_other_is_rejected():
    d = layer()
    with pytest.raises(ValueError, match="shared"):
        moe.moe_layer_forward(d["x"], d["W_router"], d["W_gate_up"], d["W_down"], d["Ws_gate_up"], None, top_k=K)


def test_layout_and_device_are_checked():
    with pytest.raises(ValueError, match="contiguous"):
        call(layer(W_down=torch.zeros(E, I, H, dtype=torch.bfloat16).transpose(1, 2)))
    with pytest.raises(ValueError, match="meta"):
        call(layer(W_down=torch.zeros(E, H, I, dtype=torch.bfloat16, device="meta")))


def fp8_pair(rows, cols, lead=()):
    return (torch.zeros(*lead, rows, cols, dtype=torch.uint8),
            torch.zeros(*lead, -(-rows // 128), -(-cols // 128), dtype=torch.uint8))


def fp8_weights(**over):
    w = dict(W_gate_up=fp8_pair(2 * I, H, (E,)), W_down=fp8_pair(H, I, (E,)), Ws_gate_up=fp8_pair(2 * Is, H),
             Ws_down=fp8_pair(H, Is))
    w.update(over)
    return w


def call_fp8(w, dtype=torch.bfloat16):
    x = torch.zeros(T, H, dtype=dtype)
    return moe.moe_layer_forward_fp8(x, torch.zeros(E, H, dtype=dtype), w, top_k=K)


def test_fp8_weights_are_checked():
    with pytest.raises(ValueError, match="CUDA"):
        call_fp8(fp8_weights())
    with pytest.raises(ValueError, match="W_down scales"):
        call_fp8(fp8_weights(W_down=(fp8_pair(H, I, (E,))[0], torch.zeros(E, 2, 2, dtype=torch.uint8))))
    with pytest.raises(ValueError, match="W_gate_up codes"):
        call_fp8(fp8_weights(W_gate_up=fp8_pair(2 * I, H, (E - 1,))))
    with pytest.raises(ValueError, match="Ws_down codes"):
        call_fp8(fp8_weights(Ws_down=fp8_pair(H, 2 * Is)))
    with pytest.raises(ValueError, match="bf16 tokens"):
        call_fp8(fp8_weights(), dtype=torch.float32)
