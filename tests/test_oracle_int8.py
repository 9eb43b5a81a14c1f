"""Pins for the oracle's INT8 tensorwise (+ optional ConvRot) functions (CPU only).

Format: symmetric 8-bit codes with scale amax / 127, the fallback format of the
pages ("Qwen-Image-Edit-2511 — INT4 tensorwise W4A4 (+ConvRot, mixed int8
fallback)", introduction; "Qwen Image 2.1 — Hybrid W4A8 / INT8 ConvRot",
layer list).
"""

import json
import os

import numpy as np

import oracle
from w4a8_rotated_quantized_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_int8_scale_special_values():
    # amax values whose quotient by 127 is exact, and the all-zero tensor
    assert oracle.scale8_from_amax(127.0) == np.float32(1.0)
    assert oracle.scale8_from_amax(63.5) == np.float32(0.5)
    assert oracle.scale8_from_amax(254.0) == np.float32(2.0)
    assert oracle.scale8_from_amax(0.0) == np.float32(1.0)
    assert oracle.tensor_scale8(np.zeros((3, 4))) == np.float32(1.0)
    # the largest magnitude always lands on +-127
    rng = np.random.default_rng(3)
    y = rng.standard_normal((16, 256)) * 5
    q = oracle.quantize8(y, oracle.tensor_scale8(y))
    assert np.max(np.abs(q)) == 127


def test_int8_round_half_even_and_clamp():
    t = np.array([0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 126.5, -126.5, 127.4, 128.0, -128.0, -129.0, 300.0])
    q = oracle.quantize8(t, np.float32(1.0))
    assert q.tolist() == [0, 2, 2, 0, -2, -2, 126, -126, 127, 127, -128, -128, 127]


def test_int8_worked_example_by_construction():
    doc = json.load(open(os.path.join(GOLDEN, "worked_int8_example.json")))
    K = doc["K"]
    y = np.zeros((1, K))
    g0, g1 = doc["y_group0_nonzero"], doc["y_group1_nonzero"]
    y[0, :len(g0)] = g0
    y[0, 256:256 + len(g1)] = g1
    H = oracle.regular_hadamard(256)
    x = np.concatenate([y[:, g * 256:(g + 1) * 256] @ H for g in range(K // 256)], axis=1)
    x_bits = workloads.bf16_bits_from_f32(x.astype(np.float32))
    assert np.array_equal(oracle.bf16_bits_to_f64(x_bits), x)  # exact in bfloat16
    q, s_a, yrot = oracle.quant_act8(x_bits)
    assert np.array_equal(yrot, y)
    assert s_a == np.float32(doc["expected_scale"])
    p0, p1 = doc["expected_codes_group0_prefix"], doc["expected_codes_group1_prefix"]
    assert q[0, :len(p0)].tolist() == p0
    assert q[0, 256:256 + len(p1)].tolist() == p1
    assert np.count_nonzero(q) == np.count_nonzero(p0) + np.count_nonzero(p1)


def test_int8_without_rotation_quantises_x_itself():
    # stock int8_tensorwise: no rotation; X = [127, -63.5, 1.25, 0] -> scale 1, codes rne(X)
    x = np.zeros((2, 256))
    x[0, :3] = [127.0, -63.5, 1.25]
    x[1, 5] = -2.5
    q, s_a, y = oracle.quant_act8(workloads.bf16_bits_from_f32(x.astype(np.float32)), rotate_groups=False)
    assert s_a == np.float32(1.0)
    assert q[0, :3].tolist() == [127, -64, 1] and q[1, 5] == -2
    assert np.count_nonzero(q) == 4


def test_int8_gemm_brute_force_full_code_range():
    rng = np.random.default_rng(11)
    qa = rng.integers(-128, 128, size=(5, 256)).astype(np.int8)
    qw = rng.integers(-128, 128, size=(6, 256)).astype(np.int8)
    want = np.zeros((5, 6), dtype=np.int64)
    for m in range(5):
        for n in range(6):
            want[m, n] = sum(int(qa[m, k]) * int(qw[n, k]) for k in range(256))
    assert np.array_equal(oracle.int_gemm(qa, qw), want)
    # the extreme accumulator of K = 256 codes -128 * -128
    ext = oracle.int_gemm(np.full((1, 256), -128, np.int8), np.full((1, 256), -128, np.int8))
    assert ext[0, 0] == 256 * 16384


def test_int8_layer_zero_input_gives_bias_and_rotation_helps_on_outliers():
    d = workloads.make_inputs("tiny")
    qw, s_w, _ = oracle.pack_weight8(d["W"])
    zero = np.zeros_like(d["X"])
    out = oracle.int8_linear(zero, qw, s_w, d["bias"])
    assert np.array_equal(out["Y"], np.broadcast_to(d["bias"], out["Y"].shape))
    # with outlier channels, the rotated INT8 layer is closer to the float layer than the plain one
    ref = oracle.reference_linear(d["X"], d["W"], d["bias"])
    y_rot = oracle.bf16_bits_to_f64(oracle.int8_linear(d["X"], qw, s_w, d["bias"])["Y"])
    qw0, s_w0, _ = oracle.pack_weight8(d["W"], rotate_groups=False)
    y_plain = oracle.bf16_bits_to_f64(oracle.int8_linear(d["X"], qw0, s_w0, d["bias"], rotate_groups=False)["Y"])
    assert oracle.relative_error(y_rot, ref) < oracle.relative_error(y_plain, ref)
    assert oracle.relative_error(y_rot, ref) < 0.02


def test_a8w4_layer_brute_force_and_composition():
    # INT8 activation codes against packed INT4 weights: explicit loops on a tiny case, and the
    # same integer product as the INT8 layer fed the INT4 weight codes
    rng = np.random.default_rng(41)
    M, N, K = 3, 5, 256
    x = workloads.bf16_bits_from_f32(rng.standard_normal((M, K)).astype(np.float32))
    w = workloads.bf16_bits_from_f32((rng.standard_normal((N, K)) * 0.02).astype(np.float32))
    b = workloads.bf16_bits_from_f32((rng.standard_normal(N) * 0.01).astype(np.float32))
    wq, s_w, qw, _ = oracle.pack_weight(w)
    r = oracle.a8w4_linear(x, wq, s_w, b)
    for m in range(M):
        for n in range(N):
            assert r["acc"][m, n] == sum(int(r["qa"][m, k]) * int(qw[n, k]) for k in range(K))
    r8 = oracle.int8_linear(x, qw, s_w, b)
    assert np.array_equal(r8["acc"], r["acc"]) and np.array_equal(r8["Y"], r["Y"])
    # INT8 activation codes carry more of X than INT4 ones: the INT8-branch error is lower
    ref = oracle.reference_linear(x, w, b)
    err8 = oracle.relative_error(oracle.bf16_bits_to_f64(r["Y"]), ref)
    err4 = oracle.relative_error(oracle.bf16_bits_to_f64(oracle.w4a4_linear(x, wq, s_w, b)["Y"]), ref)
    assert err8 < err4
