"""The C-ABI library loads, exports every entry point its header declares, and validates
its arguments on the host (no device work is enqueued for any of these calls)."""
import ctypes
import os
import re

import pytest

import sparse_mixture_experts_ffn_b200 as moe
from sparse_mixture_experts_ffn_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return moe.load_library()


def declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"^MOE_API\s+[\w\s\*]+?\b(\w+)\s*\(", text, flags=re.M)
    return names


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert set(names) >= set(moe.EXPORTED)
    for n in names:
        assert hasattr(lib, n), n


def shape(**kw):
    base = dict(T=4096, H=4096, E=288, I=1280, I_shared=1280, top_k=8, dtype=moe.MOE_BF16)
    base.update(kw)
    return moe.MoEShape(base["T"], base["H"], base["E"], base["I"], base["I_shared"], base["top_k"], base["dtype"])


def test_workspace_bytes(lib):
    s = shape()
    n = moe.workspace_bytes(s)
    T, H, E, k, I = 4096, 4096, 288, 8, 1280
    P = T * k
    # x_perm, h, o (bf16) dominate; everything else is small
    assert n >= 2 * (P * H + P * I + P * H + T * I + T * H)
    assert n < 2 * (P * H + P * I + P * H + T * I + T * H) + 64 * 1024 * 1024
    # 16-token tiles (decode) gather token rows from x: no permuted copy of x
    d = moe.workspace_bytes(shape(T=4))
    assert d < 2 * (4 * k * H) + 2 * (4 * k * I + 4 * k * H + 4 * I + 4 * H) + 64 * 1024 * 1024
    assert moe.workspace_bytes(shape(T=0)) > 0
    for bad in (shape(top_k=0), shape(top_k=289), shape(E=0), shape(H=4000), shape(I=1000),
                shape(I_shared=100), shape(E=1025, top_k=8), shape(dtype=7), shape(T=-1)):
        assert moe.workspace_bytes(bad) == 0
    # fp32 accepts any H multiple of 8 and any widths
    assert moe.workspace_bytes(shape(dtype=moe.MOE_F32, H=72, I=40, I_shared=24)) > 0


def test_workspace_layout_is_inside_the_workspace(lib):
    s = shape(T=100)
    lay = moe.workspace_layout(s)
    n = moe.workspace_bytes(s)
    for off in (lay.x_perm, lay.h, lay.h_shared, lay.o, lay.o_shared, lay.row_w):
        assert off % 256 == 0 and off < n


def call_forward(lib, s, x=16, wr=16, bias=None, wgu=16, wd=16, wsgu=16, wsd=16, y=16, ws=256,
                 ws_bytes=None):
    if ws_bytes is None:
        ws_bytes = moe.workspace_bytes(s) if moe.workspace_bytes(s) else 1 << 40
    P = ctypes.c_void_p
    return lib.moe_layer_forward(ctypes.byref(s), P(x), P(wr), P(bias), P(wgu), P(wd), P(wsgu), P(wsd),
                                 P(y), None, P(ws), ws_bytes, None)


def test_forward_rejects_bad_arguments_before_any_launch(lib):
    s = shape()
    # fake, aligned, never dereferenced addresses: every call below fails validation first
    assert call_forward(lib, s, x=None) == 1
    assert call_forward(lib, s, y=None) == 1
    assert call_forward(lib, s, ws=None) == 1
    assert call_forward(lib, s, x=24) == 1            # misaligned
    assert call_forward(lib, s, ws=512 + 16) == 1     # workspace not 256-byte aligned
    assert call_forward(lib, s, bias=18) == 1         # misaligned bias
    assert call_forward(lib, s, wsgu=None) == 1       # shared expert half given
    assert call_forward(lib, shape(I_shared=0)) == 1  # shared weights given without width
    assert call_forward(lib, shape(top_k=0)) == 1
    assert call_forward(lib, shape(top_k=300)) == 1
    assert call_forward(lib, shape(H=4000)) == 2
    assert call_forward(lib, shape(E=2000)) == 2
    assert call_forward(lib, s, ws_bytes=moe.workspace_bytes(s) - 1) == 3
    assert call_forward(lib, shape(T=0)) == 0         # empty batch: nothing to do
    assert call_forward(lib, None if False else shape(dtype=5)) == 1


def test_status_strings(lib):
    for code, name in moe.STATUS_NAMES.items():
        assert moe.status_string(code).startswith(name)
    assert moe.status_string(99) == "unknown moe_status"


def test_forward_ex_rejects_bad_swiglu_limits_before_any_launch(lib):
    s = shape()
    P = ctypes.c_void_p
    n = moe.workspace_bytes(s)

    def call(limit, limit_shared, router=0, scale=0.0):
        opts = moe.MoEOptions(limit, limit_shared, router, scale)
        return lib.moe_layer_forward_ex(ctypes.byref(s), P(16), P(16), None, P(16), P(16), P(16), P(16),
                                        P(16), None, ctypes.byref(opts), P(256), n, None)

    for bad in ((-1.0, 0.0), (0.0, -0.5), (float("nan"), 0.0), (0.0, float("inf")), (0.0, 0.0, 2),
                (0.0, 0.0, 1, -3.0), (0.0, 0.0, 1, float("nan"))):
        assert call(*bad) == 1, bad
    # NULL options is the plain forward (validation of the other arguments still runs)
    assert lib.moe_layer_forward_ex(ctypes.byref(s), None, P(16), None, P(16), P(16), P(16), P(16),
                                    P(16), None, None, P(256), n, None) == 1


def test_forward_fp8_rejects_bad_arguments_before_any_launch(lib):
    P = ctypes.c_void_p

    def call(s, scales=(1, 1, 1, 1), codes=(16, 16, 16, 16), weights=True, ws_bytes=None):
        n = moe.workspace_bytes(s) if ws_bytes is None else ws_bytes
        fw = moe.MoEFp8Weights(codes[0], scales[0], codes[1], scales[1], codes[2], scales[2], codes[3],
                               scales[3])
        return lib.moe_layer_forward_fp8(ctypes.byref(s), P(16), P(16), None,
                                         ctypes.byref(fw) if weights else None, P(16), None, None, P(256),
                                         n or 1, None)

    assert call(shape(), weights=False) == 1
    assert call(shape(dtype=moe.MOE_F32)) == 2        # FP8 weights go with bf16 tokens only
    assert call(shape(H=4160)) == 2                   # not a multiple of 128
    assert call(shape(I=1344)) == 2
    assert call(shape(H=8320)) == 2                   # more than 64 scale blocks per reduction
    assert call(shape(), scales=(None, 1, 1, 1)) == 1  # a scale table missing
    assert call(shape(), scales=(1, 1, 1, None)) == 1
    assert call(shape(), codes=(24, 16, 16, 16)) == 1  # codes misaligned
    assert call(shape(), ws_bytes=moe.workspace_bytes(shape()) - 1) == 3
    assert call(shape(T=0)) == 0                      # empty batch: nothing to do


C_TYPES = {"int64_t": ctypes.c_int64, "int32_t": ctypes.c_int32, "float": ctypes.c_float,
           "size_t": ctypes.c_size_t}


def header_structs():
    """{struct name: [(field, C type), ...]} parsed from the typedef'd structs of the header."""
    text = open(os.path.join(ROOT, "include", "moe_layer.h")).read()
    out = {}
    for body, name in re.findall(r"typedef struct \{(.*?)\}\s*(\w+);", text, flags=re.S):
        fields = []
        for decl in re.sub(r"/\*.*?\*/", "", body, flags=re.S).split(";"):
            decl = decl.strip()
            if not decl:
                continue
            m = re.match(r"(const\s+)?(\w+)\s*(\*?)\s*(.*)", decl)
            ctype = "pointer" if m.group(3) else m.group(2)
            for f in m.group(4).split(","):
                fields.append((f.strip().lstrip("*"), ctype))
        out[name] = fields
    return out


@pytest.mark.parametrize("c_name, py_struct", [
    ("moe_layer_shape", moe.MoEShape), ("moe_routing_out", moe.MoERoutingOut),
    ("moe_layer_options", moe.MoEOptions), ("moe_fp8_weights", moe.MoEFp8Weights),
    ("moe_route_stats", moe.MoERouteStats), ("moe_workspace_layout", moe.MoEWorkspaceLayout),
    ("moe_ep_range", moe.MoEEpRange)])
def test_binding_structs_match_the_header(c_name, py_struct):
    """Every ctypes structure of the binding has the header's fields, in order, with the same
    C types (pointers as pointers), so that the marshalled bytes are what the library reads."""
    fields = header_structs()[c_name]
    py = py_struct._fields_
    assert [f for f, _ in fields] == [f for f, _ in py], c_name
    for (f, ctype), (_, pytype) in zip(fields, py):
        if ctype == "pointer":
            assert pytype is ctypes.c_void_p, (c_name, f)
        else:
            assert ctypes.sizeof(pytype) == ctypes.sizeof(C_TYPES[ctype]), (c_name, f)
            assert (pytype is ctypes.c_float) == (ctype == "float"), (c_name, f)


def test_forward_ep_and_sum_partials_reject_bad_arguments_before_any_launch(lib):
    P = ctypes.c_void_p

    def ep(s, rng, yp=16, ws_bytes=None):
        nb = moe.workspace_bytes(s) if ws_bytes is None else ws_bytes
        r = None if rng is None else ctypes.byref(moe.MoEEpRange(*rng))
        return lib.moe_layer_forward_ep(ctypes.byref(s), P(16), P(16), None, P(16), P(16), P(16), P(16), r,
                                        P(yp), None, None, P(256), nb if nb else 1 << 40, None)
    s = shape(T=64)
    assert ep(s, None) == 1                           # no range
    assert ep(s, (0, 0, 0, 64)) == 1                  # empty expert range
    assert ep(s, (10, 289, 0, 64)) == 1               # past E
    assert ep(s, (-1, 8, 0, 64)) == 1
    assert ep(s, (0, 36, 10, 5)) == 1                 # shared rows reversed
    assert ep(s, (0, 36, 0, 65)) == 1                 # shared rows past T
    assert ep(s, (0, 36, 0, 64), yp=None) == 1        # no partial output
    assert ep(s, (0, 36, 0, 64), yp=24) == 1          # misaligned partial output
    assert ep(shape(T=64, dtype=moe.MOE_F32, H=72, I=40, I_shared=24), (0, 36, 0, 64)) == 2  # bf16 only
    assert ep(s, (0, 36, 0, 64), ws_bytes=moe.workspace_bytes(s) - 1) == 3
    assert ep(shape(T=0), (0, 36, 0, 0)) == 0          # empty batch

    def sp(T, H, dtype, ptrs, y=16):
        arr = (ctypes.c_void_p * max(len(ptrs), 1))(*ptrs)
        return lib.moe_layer_sum_partials(T, H, dtype, len(ptrs), arr, P(y), None)
    assert sp(4, 64, moe.MOE_BF16, []) == 1
    assert sp(4, 64, moe.MOE_BF16, [16] * 17) == 1    # more than 16 parts
    assert sp(4, 60, moe.MOE_BF16, [16]) == 1         # H not a multiple of 8
    assert sp(4, 64, 9, [16]) == 1
    assert sp(4, 64, moe.MOE_BF16, [16, 24]) == 1     # misaligned part
    assert sp(4, 64, moe.MOE_BF16, [16], y=None) == 1
    assert sp(0, 64, moe.MOE_BF16, [16]) == 0
