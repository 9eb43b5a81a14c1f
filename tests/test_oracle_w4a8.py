"""Pins for the oracle's W4A8 functions (CPU only): asymmetric 4-bit weights,
group 16 along K, fp16 scale and 4-bit zero point per group ("Qwen-Image-Edit-2511
— W4A8 ConvRot", build table and file layout; "Qwen Image 2.1 — Hybrid W4A8 /
INT8 ConvRot", recipe), INT8 tensorwise activations, both rotated."""

import json
import os

import numpy as np

import oracle
from w4a8_rotated_quantized_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_worked_groups():
    doc = json.load(open(os.path.join(GOLDEN, "worked_w4a8_example.json")))
    for g in doc["groups"]:
        w = np.array([g["w"]])
        s, z = oracle.asym_params16(w)
        if "scale" in g:
            assert s[0, 0] == np.float16(g["scale"]), g["comment"]
        else:
            assert s[0, 0].view(np.uint16) == int(g["scale_fp16_bits"], 16), g["comment"]
        assert z[0, 0] == g["zero"], g["comment"]
        q = oracle.quantize_asym16(w, s, z)
        assert q[0].tolist() == g["q"], g["comment"]
        if "w_hat" in g:
            assert oracle.dequant_asym16(q, s, z)[0].tolist() == g["w_hat"], g["comment"]


def test_reconstruction_error_is_half_a_step():
    # where the zero point is not clamped (every group of normal data holds both signs),
    # |w - w^| <= s / 2 plus the overshoot the float16 rounding of the step allows: with
    # s = (hi - lo) / 15 * (1 + d), |d| <= 2**-11, the group spans 15 / (1 + d) steps, so the
    # code of an extreme value may clamp by up to 15 |d| of a step
    rng = np.random.default_rng(11)
    y = rng.standard_normal((64, 512)) * 0.02
    s, z = oracle.asym_params16(y)
    q = oracle.quantize_asym16(y, s, z)
    err = np.abs(y - oracle.dequant_asym16(q, s, z))
    half = np.repeat(s.astype(np.float64), 16, axis=1) / 2
    g = y.reshape(64, 32, 16)
    both_signs = np.repeat((g.min(axis=2) < 0) & (g.max(axis=2) > 0), 16, axis=1)
    assert both_signs.mean() > 0.99
    assert np.all(err[both_signs] <= half[both_signs] * (1 + 2 * (15 * 2.0 ** -11 + 1e-6)))
    assert np.mean(err[both_signs] <= half[both_signs] * (1 + 1e-6)) > 0.999
    # the group's extremes are represented to within half a step too, and codes span 0..15
    assert q.min() == 0 and q.max() == 15


def test_scale_is_the_fp16_rounding_of_the_float32_step():
    rng = np.random.default_rng(12)
    y = rng.standard_normal((8, 256))
    s, _ = oracle.asym_params16(y)
    g = y.astype(np.float32).reshape(8, 16, 16)
    step = (g.max(axis=2) - g.min(axis=2)) / np.float32(15)
    assert np.array_equal(s, step.astype(np.float16))


def test_pack_u4_round_trip_and_nibble_order():
    q = np.array([[1, 2, 15, 0, 7, 8]], dtype=np.uint8)
    p = oracle.pack_u4(q)
    assert p.tolist() == [[0x21, 0x0F, 0x87]]
    assert np.array_equal(oracle.unpack_u4(p), q)


def test_layer_brute_force_tiny():
    # explicit per-element loops over k (groups of 16 looked up one element at a time)
    rng = np.random.default_rng(13)
    M, N, K = 3, 4, 256
    x = workloads.bf16_bits_from_f32(rng.standard_normal((M, K)).astype(np.float32))
    w = workloads.bf16_bits_from_f32((rng.standard_normal((N, K)) * 0.02).astype(np.float32))
    b = workloads.bf16_bits_from_f32((rng.standard_normal(N) * 0.01).astype(np.float32))
    pw = oracle.pack_weight_w4a8(w)
    r = oracle.w4a8_linear(x, pw["q"], pw["s"], pw["z"], b)
    for m in range(M):
        for n in range(N):
            tot = 0.0
            for k in range(K):
                tot += float(r["qa"][m, k]) * float(pw["s"][n, k // 16]) * (int(pw["q"][n, k]) - int(pw["z"][n, k // 16]))
            assert abs(tot - r["acc"][m, n]) <= 1e-12 * max(1.0, abs(tot))
    y = oracle.w4a8_epilogue(r["acc"], r["s_a"], b)
    assert np.array_equal(y, r["Y"])


def test_unit_scales_and_zero_eight_reduce_to_the_integer_product():
    # s = 1 and z = 8 make w^ = q - 8, a symmetric integer weight: the layer is then
    # the textbook integer matmul with the INT8 activation codes
    rng = np.random.default_rng(14)
    M, N, K = 5, 8, 512
    x = workloads.bf16_bits_from_f32(rng.standard_normal((M, K)).astype(np.float32))
    q = rng.integers(0, 16, (N, K)).astype(np.uint8)
    s = np.ones((N, K // 16), dtype=np.float16)
    z = np.full((N, K // 16), 8, dtype=np.uint8)
    b = workloads.bf16_bits_from_f32(rng.standard_normal(N).astype(np.float32))
    r = oracle.w4a8_linear(x, q, s, z, b)
    acc_int = oracle.int_gemm(r["qa"], q.astype(np.int64) - 8)
    assert np.array_equal(r["acc"], acc_int.astype(np.float64))
    assert np.array_equal(r["Y"], oracle.epilogue(acc_int, r["s_a"], np.ones(N, np.float32), b))


def test_rotation_is_applied_to_weights_and_activations():
    # with rotation on both sides, the layer approximates x . w^T: the product of the
    # rotated operands equals the unrotated product (H orthogonal), so the error against the
    # float64 reference is the quantisation error alone and is small for smooth data
    rng = np.random.default_rng(15)
    M, N, K = 16, 32, 512
    x = workloads.bf16_bits_from_f32(rng.standard_normal((M, K)).astype(np.float32))
    w = workloads.bf16_bits_from_f32((rng.standard_normal((N, K)) * 0.02).astype(np.float32))
    pw = oracle.pack_weight_w4a8(w, rotate_groups=True)
    r = oracle.w4a8_linear(x, pw["q"], pw["s"], pw["z"], None, rotate_groups=True)
    ref = oracle.bf16_bits_to_f64(x) @ oracle.bf16_bits_to_f64(w).T
    got = oracle.bf16_bits_to_f64(r["Y"])
    # 4-bit codes over a group of 16 normal values: a step of about range / 15 ~ 0.25 sigma,
    # so about 7% relative error; a rotation applied to one side only scrambles the product
    assert oracle.relative_error(got, ref) < 0.1
    r1 = oracle.w4a8_linear(x, pw["q"], pw["s"], pw["z"], None, rotate_groups=False)
    assert oracle.relative_error(oracle.bf16_bits_to_f64(r1["Y"]), ref) > 0.5
    # a zero weight group dequantises to exactly zero
    w0 = np.zeros((2, 256), np.uint16)
    p0 = oracle.pack_weight_w4a8(w0)
    assert not p0["q"].any() and np.all(p0["s"] == 1) and not p0["z"].any()
