"""Pins for the oracle's integer product, epilogue and bfloat16 rounding (CPU only)."""

import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from w4a8_rotated_quantized_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.mark.parametrize("K", [256, 512])
def test_int_gemm_brute_force(K):
    rng = np.random.default_rng(K)
    qa = rng.integers(-8, 8, size=(5, K)).astype(np.int8)
    qw = rng.integers(-8, 8, size=(7, K)).astype(np.int8)
    got = oracle.int_gemm(qa, qw)
    for m in range(5):
        for n in range(7):
            s = 0
            for k in range(K):
                s += int(qa[m, k]) * int(qw[n, k])
            assert got[m, n] == s


def test_int_gemm_extreme_values_exact():
    K = 12288
    qa = np.full((2, K), -8, np.int8)
    qw = np.full((3, K), -8, np.int8)
    assert np.all(oracle.int_gemm(qa, qw) == 64 * K)


def _exact_bf16_bits(fr: Fraction) -> int:
    """Round an exact rational to bfloat16 (ties to even) by exact comparisons."""
    if fr == 0:
        return 0
    sign = 0x8000 if fr < 0 else 0
    a = abs(fr)
    e = 0
    while a >= 2:
        a /= 2
        e += 1
    while a < 1:
        a *= 2
        e -= 1
    # a in [1, 2): value = a * 2**e; spacing 2**(e-7) (normal range only here)
    assert -126 <= e <= 127
    scaled = a * 128  # in [128, 256)
    r = int(scaled)
    rem = scaled - r
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and r % 2 == 1):
        r += 1
    if r == 256:
        r = 128
        e += 1
    exp_field = e + 127
    return sign | (exp_field << 7) | (r - 128)


def test_epilogue_matches_exact_rational_arithmetic():
    rng = np.random.default_rng(21)
    M, N = 6, 9
    acc = rng.integers(-600000, 600000, size=(M, N))
    s_a = np.float32(rng.uniform(0.01, 3.0))
    s_w = rng.uniform(1e-4, 1e-2, size=N).astype(np.float32)
    bias = workloads.bf16_bits_from_f32(rng.standard_normal(N).astype(np.float32) * 0.01)
    got = oracle.epilogue(acc, s_a, s_w, bias)
    bias_f = oracle.bf16_bits_to_f64(bias)
    for m in range(M):
        for n in range(N):
            exact = Fraction(int(acc[m, n])) * Fraction(float(s_a)) * Fraction(float(s_w[n])) + Fraction(float(bias_f[n]))
            assert got[m, n] == _exact_bf16_bits(exact), (m, n)


def test_bf16_rounding_golden():
    for ln in open(os.path.join(GOLDEN, "bf16_rounding.txt")):
        if not ln.strip() or ln.startswith("#"):
            continue
        v, h = ln.split()
        got = oracle.bf16_rne_bits(np.array([float.fromhex(v)]))[0]
        assert got == int(h, 16), ln


def test_bf16_rounding_agrees_with_torch_on_float32_inputs():
    # For values already in float32 there is no double rounding, so torch's
    # float32 -> bfloat16 conversion (round to nearest even) is a reference.
    rng = np.random.default_rng(5)
    v = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(1e3),
        (rng.standard_normal(2000) * 1e-39).astype(np.float32),  # subnormals
        np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 65504.0, 1e-45], dtype=np.float32),
    ])
    want = workloads.bf16_bits_from_f32(v)
    got = oracle.bf16_rne_bits(v.astype(np.float64))
    assert np.array_equal(got, want)


def _sparse_code_inputs(rng, R, K):
    """Rows whose rotation is an exact integer code row with a +-7 present.

    Each 256-group carries at most one nonzero code c at position i, so the
    bfloat16 input is c * H[i, :] = +-c/16: exact.  Rotating gives back c e_i.
    """
    H = oracle.regular_hadamard(256)
    codes = np.zeros((R, K), dtype=np.int64)
    x = np.zeros((R, K))
    for r in range(R):
        for g in range(K // 256):
            i = rng.integers(0, 256)
            c = rng.integers(-7, 8)
            codes[r, g * 256 + i] = c
            x[r, g * 256:(g + 1) * 256] = c * H[i]
    codes[0, 0] = 7  # make amax exactly 7 somewhere
    x[0, :256] = 0.0
    x[0, :256] = 7 * H[0] + sum(codes[0, j] * H[j] for j in range(1, 256) if codes[0, j])
    return codes, x


def test_layer_reduces_to_textbook_integer_matmul():
    # With exact integer rotated codes and amax = 7 on both sides, scales are 1
    # and the layer is  bf16(C_a C_w^T + b): an integer matrix product.
    rng = np.random.default_rng(8)
    M, N, K = 9, 12, 768
    ca, x = _sparse_code_inputs(rng, M, K)
    cw, w = _sparse_code_inputs(rng, N, K)
    x_bits = workloads.bf16_bits_from_f32(x.astype(np.float32))
    w_bits = workloads.bf16_bits_from_f32(w.astype(np.float32))
    assert np.array_equal(oracle.bf16_bits_to_f64(x_bits), x)
    bias = workloads.bf16_bits_from_f32(rng.standard_normal(N).astype(np.float32))
    wq, s_w, qw, _ = oracle.pack_weight(w_bits)
    assert np.all(s_w == 1.0) and np.array_equal(qw, cw)
    out = oracle.w4a4_linear(x_bits, wq, s_w, bias)
    assert out["s_a"] == 1.0 and np.array_equal(out["qa"], ca)
    want = np.matmul(ca, cw.T).astype(np.float64) + oracle.bf16_bits_to_f64(bias)[None, :]
    assert np.array_equal(out["Y"], workloads.bf16_bits_from_f32(want.astype(np.float32)))


def test_zero_activation_or_weight_gives_bias():
    d = workloads.make_inputs("tiny")
    wq, s_w, _, _ = oracle.pack_weight(d["W"])
    out = oracle.w4a4_linear(np.zeros_like(d["X"]), wq, s_w, d["bias"])
    assert np.array_equal(out["Y"], np.broadcast_to(d["bias"], out["Y"].shape))
    wq0, s_w0, _, _ = oracle.pack_weight(np.zeros_like(d["W"]))
    out0 = oracle.w4a4_linear(d["X"], wq0, s_w0, d["bias"])
    assert np.array_equal(out0["Y"], np.broadcast_to(d["bias"], out0["Y"].shape))


def test_rotation_lowers_w4a4_error_on_outlier_inputs():
    # Side report of the per-layer error (format vs unquantised reference):
    # with outlier channels, rotating before INT4 must help, and the error
    # stays in the range INT4 activations give.
    d = workloads.make_inputs("tiny")
    ref = oracle.reference_linear(d["X"], d["W"], d["bias"])
    wq, s_w, _, _ = oracle.pack_weight(d["W"])
    rot = oracle.bf16_bits_to_f64(oracle.w4a4_linear(d["X"], wq, s_w, d["bias"])["Y"])
    # same quantiser without the rotation
    X = oracle.bf16_bits_to_f64(d["X"])
    W = oracle.bf16_bits_to_f64(d["W"])
    sa, sw = oracle.tensor_scale(X), oracle.tensor_scale(W)
    acc = oracle.int_gemm(oracle.quantize(X, sa), oracle.quantize(W, sw))
    norot = oracle.bf16_bits_to_f64(oracle.epilogue(acc, sa, np.full(W.shape[0], sw, np.float32), d["bias"]))
    e_rot, e_norot = oracle.relative_error(rot, ref), oracle.relative_error(norot, ref)
    assert e_rot < e_norot
    assert e_rot < 0.35
