"""The seeded input generators (CPU): the FP8 expert weights stand for the bf16 draws they
were cast from, within E4M3's rounding, and are reproducible."""
import numpy as np
import torch

import oracle
from sparse_mixture_experts_ffn_b200 import inputs


def test_fp8_weights_round_the_bf16_draws():
    cfg = inputs.small_config(T=4, H=384, E=3, top_k=2, I=256, I_shared=128)
    w8 = inputs.make_fp8_expert_weights(cfg)
    wb = dict(zip(("W_gate_up", "W_down", "Ws_gate_up", "Ws_down"), inputs.make_expert_weights(cfg)))
    for name, (q, s) in w8.items():
        ref = wb[name].double().numpy()
        qn, sn = q.numpy(), s.numpy()
        mats = [(qn[e], sn[e], ref[e]) for e in range(qn.shape[0])] if qn.ndim == 3 else [(qn, sn, ref)]
        for qm, sm, rm in mats:
            d = oracle.dequant_e4m3(qm, sm)
            assert not np.isnan(d).any(), name
            # each block: scale = 2^ceil(log2(amax / 448)), so amax / scale lies in (224, 448]
            scale = 2.0 ** (sm.astype(np.float64) - 127)
            blocks = np.abs(rm).reshape(sm.shape[0], 128, sm.shape[1], 128).max(axis=(1, 3))
            assert np.all(blocks / scale <= 448) and np.all(blocks / scale > 224), name
            # E4M3 keeps 4 significant bits: nearest rounding is within 2^-4 relative above
            # its normal range (2^-6 of the scale) and within half its subnormal step below
            big = np.abs(rm) >= np.kron(scale, np.ones((128, 128))) * 2.0 ** -6
            err = np.abs(d - rm)
            assert np.all(err[big] <= np.abs(rm[big]) * 2.0 ** -4), name
            assert np.all(err[~big] <= np.kron(scale, np.ones((128, 128)))[~big] * 2.0 ** -10), name


def test_fp8_weights_are_reproducible():
    cfg = inputs.small_config(T=4, H=256, E=2, top_k=1, I=128, I_shared=128)
    a, b = inputs.make_fp8_expert_weights(cfg), inputs.make_fp8_expert_weights(cfg)
    for k in a:
        for u, v in zip(a[k], b[k]):
            assert torch.equal(u, v), k


def test_bench_algorithmic_bytes_closed_form():
    """The benchmark's algorithmic byte and FLOP counts, against their closed forms for a
    decode batch: bf16 weights at 2 bytes, FP8 at 1 byte plus one scale byte per 128x128 block."""
    import bench
    cfg = inputs.CONFIGS["decode_t4"]
    counts = np.zeros(cfg.E, np.int64)
    counts[:32] = 1
    H, I, Is, E, T, k = cfg.H, cfg.I, cfg.I_shared, cfg.E, cfg.T, cfg.top_k
    b = bench.algorithmic(cfg, counts)
    f = bench.algorithmic(cfg, counts, fp8=True)
    weights = 32 * 3 * H * I + 3 * H * Is
    assert b["layer_bytes"] == 2 * weights + 2 * (E * H + 2 * T * H)
    assert f["layer_bytes"] == weights + weights // (128 * 128) + 2 * (E * H + 2 * T * H)
    assert b["layer_flops"] == f["layer_flops"] == 2 * T * E * H + T * k * 6 * H * I + T * 6 * H * Is
    assert b["gate_up_bytes"] == 2 * (32 * 2 * I * H + 2 * Is * H) + 2 * (T * k * H + T * H + T * k * I + T * Is)


def test_bench_roofline_of_the_one_gemm_launch():
    """With 16-token tiles (decode) the dominant kernel is the one launch of both GEMMs: its
    roofline counts both GEMMs' bytes and FLOPs; the long prefill's is the gate/up GEMM's."""
    import bench
    peaks = dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")
    d4, p16 = inputs.CONFIGS["decode_t4"], inputs.CONFIGS["prefill_t16384_skew"]
    assert bench.gemms_in_one_launch(d4, False) and bench.gemms_in_one_launch(inputs.CONFIGS["decode_t128"], False)
    assert not bench.gemms_in_one_launch(d4, True)  # FP8 weights: two launches
    assert not bench.gemms_in_one_launch(p16, False) and not bench.gemms_in_one_launch(inputs.CONFIGS["prefill_t4096"], False)
    counts = np.zeros(d4.E, np.int64)
    counts[:32] = 1
    alg = bench.algorithmic(d4, counts)
    r = bench.roofline(alg, peaks, 0.16, False, "decode_t4", fused=True)
    assert r["bound"] == "hbm" and r["algorithmic_bytes"] == alg["gate_up_bytes"] + alg["down_bytes"]
    assert abs(r["achieved"] - (alg["gate_up_bytes"] + alg["down_bytes"]) / 0.16e-3 / 1e9) < 1e-6
    r2 = bench.roofline(alg, peaks, 0.12, False, "decode_t4", fused=False)
    assert r2["algorithmic_bytes"] == alg["gate_up_bytes"]


def test_bench_traffic_ratio_follows_its_source(tmp_path, monkeypatch):
    """roofline.traffic comes from a `traffic-ratio` line of a committed ncu summary, scaled
    to the launch's algorithmic bytes, and is null once the kernel's code no longer matches
    the digest recorded with the capture; edits to comments and layout keep it."""
    import bench
    src = tmp_path / "kernel.cu"
    src.write_bytes(b'int k(int a) { return a + 1; }  // as captured\nconst char* s = "x//y";\n')
    digest = bench.code_digest(src.read_bytes())
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "gemm.md").write_text(
        "# capture\n\n    traffic-ratio gate_up decode_t4 1.25 kernel.cu %s\n" % digest)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.ncu_traffic("gate_up", "decode_t4", 1000.0) == 1250.0
    assert bench.ncu_traffic("gate_up", "decode_t128", 1000.0) is None  # no capture
    # comments reworded, a block comment added, lines re-indented: same code, same digest
    src.write_bytes(b'/* kernel */\nint k(int a) {\n    return a + 1;  // reworded\n}\n'
                    b'const char* s = "x//y";\n')
    assert bench.ncu_traffic("gate_up", "decode_t4", 1000.0) == 1250.0
    # a change inside a string literal is a change of the code
    src.write_bytes(b'int k(int a) { return a + 1; }\nconst char* s = "x/y";\n')
    assert bench.ncu_traffic("gate_up", "decode_t4", 1000.0) is None
    src.write_bytes(b'int k(int a) { return a + 2; }\nconst char* s = "x//y";\n')
    assert bench.ncu_traffic("gate_up", "decode_t4", 1000.0) is None
