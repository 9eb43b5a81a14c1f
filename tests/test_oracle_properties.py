"""Property pins for the oracle over random shapes and values (hypothesis):
invariants that a dropped term, a wrong sign or a transposed operand would
break, checked far beyond the fixed-seed cases."""

import numpy as np
from hypothesis import given, settings, strategies as st

import oracle

GROUPS = st.sampled_from([16, 64, 256, 1024])


@settings(max_examples=40, deadline=None)
@given(st.integers(1, 6), st.integers(1, 3), GROUPS, st.integers(0, 2**31 - 1))
def test_rotation_preserves_norms_and_inner_products(rows, groups, g, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, g * groups)) * rng.uniform(0.01, 100)
    w = rng.standard_normal((3, g * groups))
    y = oracle.rotate(x, g)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-12)
    np.testing.assert_allclose(y @ oracle.rotate(w, g).T, x @ w.T, rtol=1e-10, atol=1e-9 * np.abs(x).max())
    # the rotation is an involution (H = H^T = H^-1)
    np.testing.assert_allclose(oracle.rotate(y, g), x, rtol=0, atol=1e-12 * max(1.0, np.abs(x).max()))


@settings(max_examples=60, deadline=None)
@given(st.integers(1, 8), st.integers(1, 64), st.floats(1e-6, 1e6), st.integers(0, 2**31 - 1))
def test_symmetric_codes_stay_within_half_a_step(rows, cols, scale, seed):
    rng = np.random.default_rng(seed)
    y = rng.standard_normal((rows, cols)) * scale
    for s, q, qmax in ((oracle.tensor_scale(y), oracle.quantize(y, oracle.tensor_scale(y)), 7),
                       (oracle.tensor_scale8(y), oracle.quantize8(y, oracle.tensor_scale8(y)), 127)):
        assert q.min() >= -qmax and q.max() <= qmax  # amax maps to +-qmax, so -qmax-1 never occurs
        assert np.abs(q).max() == qmax
        err = np.abs(y - np.float64(s) * q)
        assert np.all(err <= 0.5 * np.float64(s) * (1 + 1e-6) + 1e-300)


@settings(max_examples=60, deadline=None)
@given(st.integers(1, 6), st.integers(1, 40), st.integers(0, 2**31 - 1))
def test_int4_packing_round_trips(rows, half_cols, seed):
    rng = np.random.default_rng(seed)
    q = rng.integers(-8, 8, (rows, 2 * half_cols)).astype(np.int8)
    p = oracle.pack_int4(q)
    assert p.shape == (rows, half_cols) and p.dtype == np.uint8
    assert np.array_equal(oracle.unpack_int4(p), q)
    u = rng.integers(0, 16, (rows, 2 * half_cols)).astype(np.uint8)
    assert np.array_equal(oracle.unpack_u4(oracle.pack_u4(u)), u)


@settings(max_examples=40, deadline=None)
@given(st.integers(1, 4), st.integers(1, 8), st.floats(1e-3, 1e3), st.integers(0, 2**31 - 1))
def test_asymmetric_group16_codes_and_reconstruction(rows, groups, scale, seed):
    rng = np.random.default_rng(seed)
    y = rng.standard_normal((rows, 16 * groups)) * scale
    s, z = oracle.asym_params16(y)
    q = oracle.quantize_asym16(y, s, z)
    assert q.min() >= 0 and q.max() <= 15 and z.max() <= 15
    w = oracle.dequant_asym16(q, s, z)
    g = y.reshape(rows, groups, 16)
    both = np.repeat((g.min(axis=2) < 0) & (g.max(axis=2) > 0), 16, axis=1)
    step = np.repeat(s.astype(np.float64), 16, axis=1)
    err = np.abs(y - w)
    assert np.all(err[both] <= step[both] * (0.5 + 16 * 2.0 ** -11) + 1e-12)


@settings(max_examples=30, deadline=None)
@given(st.integers(1, 5), st.integers(1, 5), st.integers(1, 3), st.integers(0, 2**31 - 1))
def test_integer_product_and_epilogue_against_loops(M, N, kb, seed):
    rng = np.random.default_rng(seed)
    K = 32 * kb
    qa = rng.integers(-128, 128, (M, K))
    qw = rng.integers(-8, 8, (N, K))
    acc = oracle.int_gemm(qa, qw)
    for m in range(M):
        for n in range(N):
            assert acc[m, n] == sum(int(qa[m, k]) * int(qw[n, k]) for k in range(K))
    s_a = np.float32(rng.uniform(1e-3, 1))
    s_w = rng.uniform(1e-3, 1, N).astype(np.float32)
    y = oracle.bf16_bits_to_f64(oracle.epilogue(acc, s_a, s_w, None))
    exact = acc * np.float64(s_a) * s_w.astype(np.float64)[None, :]
    # one round-to-nearest to bfloat16 (8 significant bits): within half an ulp, at most 2^-8 relative
    assert np.all(np.abs(y - exact) <= np.abs(exact) * 2.0 ** -8 * (1 + 1e-12) + 1e-300)
    # and y is the nearest bfloat16: the neighbours one ulp away are no closer
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(y), 1e-300))) - 7)
    assert np.all(np.abs(y - exact) <= np.minimum(np.abs(y + ulp - exact), np.abs(y - ulp - exact)) + 1e-300)
