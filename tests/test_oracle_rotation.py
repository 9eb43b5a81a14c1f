"""Pins for the oracle's rotation (CPU only).

Each test checks the oracle against something other than its own formula: an
explicit Kronecker construction, an independent fast transform written here,
the golden H4 factor, and identities that hold for any regular Hadamard
rotation (orthogonality, involution, constant row sums, rotation invariance of
the exact product).
"""

import os

import numpy as np
import pytest

import oracle
from w4a8_rotated_quantized_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _h4_golden():
    rows = [ln.split() for ln in open(os.path.join(GOLDEN, "h4_regular.txt")) if ln.strip() and not ln.startswith("#")]
    return np.array(rows, dtype=np.float64)


def test_h4_factor_matches_golden():
    # order 4: one factor, normalised by 1/2
    assert np.array_equal(oracle.regular_hadamard(4) * 2.0, _h4_golden())


@pytest.mark.parametrize("n", [4, 16, 64, 256, 1024])
def test_closed_form_equals_kronecker_power(n):
    h4 = _h4_golden()
    H = np.array([[1.0]])
    p = 0
    while H.shape[0] < n:
        H = np.kron(H, h4)
        p += 1
    H = H / 2.0 ** p
    assert np.array_equal(oracle.regular_hadamard(n), H)


def test_h256_identities():
    H = oracle.regular_hadamard(256)
    assert np.all(np.abs(H) == 1.0 / 16.0)
    assert np.array_equal(H, H.T)
    assert np.array_equal(H @ H.T, np.eye(256))  # entries are +-1/256 sums: exact
    assert np.array_equal(H @ H, np.eye(256))  # symmetric + orthogonal => involution
    assert np.array_equal(H.sum(axis=1), np.ones(256))  # regular: constant row sum 16/16
    assert np.array_equal(H.sum(axis=0), np.ones(256))


def test_non_power_of_four_rejected():
    with pytest.raises(ValueError):
        oracle.regular_hadamard(128)


def _fwht_radix4(x):
    """Independent fast transform: one radix-4 pass per base-4 digit.

    For H4 = J - 2I, each pass replaces the four values that differ only in
    one digit by (their sum) - 2 * (own value); after 4 passes divide by 16.
    """
    x = np.array(x, dtype=np.float64)
    R, G = x.shape
    y = x.copy()
    stride = 1
    while stride < G:
        z = y.reshape(R, G // (4 * stride), 4, stride)
        s = z.sum(axis=2, keepdims=True)
        y = (s - 2.0 * z).reshape(R, G)
        stride *= 4
    return y / np.sqrt(G)


def test_rotate_matches_independent_fast_transform():
    rng = np.random.default_rng(11)
    x = rng.standard_normal((5, 3 * 256))
    got = oracle.rotate(x)
    want = np.concatenate([_fwht_radix4(x[:, g * 256:(g + 1) * 256]) for g in range(3)], axis=1)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-13)


def test_rotate_groups_are_independent_and_contiguous():
    rng = np.random.default_rng(12)
    x = rng.standard_normal((3, 1024))
    y0 = oracle.rotate(x)
    x2 = x.copy()
    x2[:, 256:512] += rng.standard_normal((3, 256))
    y1 = oracle.rotate(x2)
    changed = np.any(y0 != y1, axis=0)
    assert not changed[:256].any() and not changed[512:].any() and changed[256:512].all()


def test_rotation_maps_hadamard_rows_to_unit_vectors():
    H = oracle.regular_hadamard(256)
    for i in (0, 1, 77, 255):
        e = np.zeros(256)
        e[i] = 1.0
        np.testing.assert_array_equal(oracle.rotate(H[i:i + 1]), e[None, :])


def test_shift_invariance_constant_row_sum():
    # 1^T H = 1^T (regular, row sum 1): a constant shift passes through unchanged
    rng = np.random.default_rng(13)
    x = rng.standard_normal((4, 512))
    np.testing.assert_allclose(oracle.rotate(x + 3.25), oracle.rotate(x) + 3.25, rtol=0, atol=1e-12)


def test_exact_product_is_rotation_invariant():
    # (X H)(W H)^T = X W^T in float64, on the tiny workload's inputs
    d = workloads.make_inputs("tiny")
    X = oracle.bf16_bits_to_f64(d["X"])
    W = oracle.bf16_bits_to_f64(d["W"])
    lhs = oracle.rotate(X) @ oracle.rotate(W).T
    rhs = X @ W.T
    assert np.linalg.norm(lhs - rhs) / np.linalg.norm(rhs) <= 1e-12


def test_rotation_spreads_an_outlier_channel():
    # An outlier confined to one channel is spread evenly over its group:
    # a unit spike becomes +-1/16 on all 256 entries.
    x = np.zeros((1, 256))
    x[0, 37] = 1.0
    y = oracle.rotate(x)
    assert np.all(np.abs(y) == 1.0 / 16.0)


def test_other_groups_match_independent_fast_transform():
    # groups of 16, 64 and 1024 ("W4A4 also accepts 16 / 64 / 1024", "Qwen-Image-Edit-2511 — W4A8 ConvRot"):
    # block-diagonal Kronecker powers of H4 over sqrt(group) on contiguous slices
    rng = np.random.default_rng(17)
    x = rng.standard_normal((4, 2048))
    for g in (16, 64, 1024):
        got = oracle.rotate(x, g)
        want = np.concatenate([_fwht_radix4(x[:, i * g:(i + 1) * g]) for i in range(2048 // g)], axis=1)
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-13)
        # the product stays exact
        w = rng.standard_normal((3, 2048))
        np.testing.assert_allclose(oracle.rotate(x, g) @ oracle.rotate(w, g).T, x @ w.T, rtol=1e-12, atol=1e-10)


def test_group16_worked_codes():
    # y = (7, 2.5, -3.5, 0.5, ...) in the first group of 16, X = y H16 (entries multiples of 1/32,
    # exact in bf16): the rotation gives y back, amax 7, scale 1, codes rne(y)
    y = np.zeros((1, 256))
    y[0, :4] = [7.0, 2.5, -3.5, 0.5]
    H16 = oracle.regular_hadamard(16)
    x = np.concatenate([y[:, i * 16:(i + 1) * 16] @ H16 for i in range(16)], axis=1)
    x_bits = workloads.bf16_bits_from_f32(x.astype(np.float32))
    assert np.array_equal(oracle.bf16_bits_to_f64(x_bits), x)
    packed, s, q, yr = oracle.rotate_quant_act(x_bits, group=16)
    np.testing.assert_allclose(yr, y, rtol=0, atol=1e-15)
    assert s == np.float32(1.0)
    assert q[0, :4].tolist() == [7, 2, -4, 0] and not q[0, 4:].any()


def test_group1024_worked_codes():
    # y with a 7 in the second 256-block of a 1024-group (so the worked value crosses units), X = y H1024
    # (entries multiples of 2**-5 times small integers, exact in bf16): codes rne(y), scale 1
    y = np.zeros((1, 1024))
    y[0, [0, 300, 700, 1023]] = [7.0, -2.5, 1.5, 3.5]
    H = oracle.regular_hadamard(1024)
    x = y @ H
    x_bits = workloads.bf16_bits_from_f32(x.astype(np.float32))
    assert np.array_equal(oracle.bf16_bits_to_f64(x_bits), x)
    _, s, q, yr = oracle.rotate_quant_act(x_bits, group=1024)
    np.testing.assert_allclose(yr, y, rtol=0, atol=1e-14)
    assert s == np.float32(1.0)
    assert q[0, [0, 300, 700, 1023]].tolist() == [7, -2, 2, 4] and np.count_nonzero(q) == 4
