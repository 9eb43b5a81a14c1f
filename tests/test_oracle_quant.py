"""Pins for the oracle's scales, codes and packing (CPU only)."""

import json
import os

import numpy as np
import pytest

import oracle
from w4a8_rotated_quantized_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_worked_example_by_construction():
    doc = json.load(open(os.path.join(GOLDEN, "worked_quant_example.json")))
    K = doc["K"]
    y = np.zeros((1, K))
    y[0, :7] = doc["y_first_group_nonzero"]
    H = oracle.regular_hadamard(256)
    x = np.concatenate([y[:, g * 256:(g + 1) * 256] @ H for g in range(K // 256)], axis=1)
    x_bits = workloads.bf16_bits_from_f32(x.astype(np.float32))
    # the construction is exact in bfloat16
    assert np.array_equal(oracle.bf16_bits_to_f64(x_bits), x)
    packed, s_a, q, yrot = oracle.rotate_quant_act(x_bits)
    assert np.array_equal(yrot, y)
    assert s_a == np.float32(doc["expected_scale"])
    pre = doc["expected_codes_prefix"]
    assert q[0, :len(pre)].tolist() == pre
    assert not q[0, len(pre):].any()
    hexes = [f"{b:02X}" for b in packed[0, :len(doc["expected_packed_prefix_hex"])]]
    assert hexes == doc["expected_packed_prefix_hex"]


def test_round_half_even_on_exact_half_integers():
    t = np.arange(-7.5, 8.0, 1.0)  # -7.5 .. 7.5
    q = oracle.quantize(t, np.float32(1.0))
    want = [-8, -6, -6, -4, -4, -2, -2, 0, 0, 2, 2, 4, 4, 6, 6, 8]
    want = np.clip(want, -8, 7)
    assert q.tolist() == list(want)


def test_clamp_range():
    q = oracle.quantize(np.array([-100.0, -8.4, 7.4, 100.0]), np.float32(1.0))
    assert q.tolist() == [-8, -8, 7, 7]


def test_zero_tensor_has_unit_scale_and_zero_codes():
    packed, s_a, q, _ = oracle.rotate_quant_act(np.zeros((3, 512), dtype=np.uint16))
    assert s_a == np.float32(1.0)
    assert not q.any() and not packed.any()


def test_scale_is_float32_amax_over_7():
    assert oracle.scale_from_amax(7.0) == np.float32(1.0)
    assert oracle.scale_from_amax(14.0) == np.float32(2.0)
    # amax is rounded to float32 first, then divided in float32
    a = 1.0 + 2.0 ** -40
    assert oracle.scale_from_amax(a) == np.float32(1.0) / np.float32(7.0)


def test_tensorwise_codes_reach_7_and_never_minus_8():
    for name in ("tiny", "text_enc_up_21"):
        d = workloads.make_inputs(name, with_weight=False, M=16)
        _, s_a, q, _ = oracle.rotate_quant_act(d["X"])
        assert q.min() >= -7 and q.max() <= 7
        assert np.abs(q).max() == 7


def test_codes_dequantise_within_half_a_step():
    d = workloads.make_inputs("tiny")
    _, s_a, q, y = oracle.rotate_quant_act(d["X"])
    err = np.abs(q.astype(np.float64) * np.float64(s_a) - y)
    assert err.max() <= 0.5 * np.float64(s_a) * (1 + 1e-6)


def test_pack_matches_golden_bytes():
    for ln in open(os.path.join(GOLDEN, "pack_nibbles.txt")):
        if not ln.strip() or ln.startswith("#"):
            continue
        a, b, h = ln.split()
        got = oracle.pack_int4(np.array([[int(a), int(b)]]))
        assert got[0, 0] == int(h, 16), ln
        assert oracle.unpack_int4(got).tolist() == [[int(a), int(b)]]


def test_pack_unpack_round_trip():
    rng = np.random.default_rng(3)
    q = rng.integers(-8, 8, size=(7, 64)).astype(np.int8)
    assert np.array_equal(oracle.unpack_int4(oracle.pack_int4(q)), q)


def test_row_scales_are_per_row_and_scale_invariant():
    rng = np.random.default_rng(4)
    base = rng.standard_normal((1, 512)).astype(np.float32)
    w = np.concatenate([base, base * np.float32(4.0)], axis=0)  # power-of-2 multiple: exact
    bits = workloads.bf16_bits_from_f32(w)
    _, s_row, q_row, _ = oracle.pack_weight(bits, scale_mode="row")
    assert s_row[1] == s_row[0] * np.float32(4.0)
    assert np.array_equal(q_row[0], q_row[1])
    _, s_t, q_t, _ = oracle.pack_weight(bits, scale_mode="tensor")
    assert s_t[0] == s_t[1] == s_row[1]
    assert not np.array_equal(q_t[0], q_t[1])


def test_near_tie_mask():
    m = oracle.near_tie_mask(np.array([2.5, 2.4, -3.5, 2.5 * (1 + 2e-6), 0.0]), 1.0)
    assert m.tolist() == [True, False, True, True, False]


@pytest.mark.parametrize("mode", ["tensor", "row"])
def test_weight_codes_bounded(mode):
    d = workloads.make_inputs("tiny")
    _, s_w, q, _ = oracle.pack_weight(d["W"], scale_mode=mode)
    assert s_w.dtype == np.float32 and s_w.shape == (256,)
    assert q.min() >= -7 and q.max() <= 7
