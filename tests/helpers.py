"""Comparison helpers shared by the GPU parity tests (no arithmetic of the layer here)."""

import numpy as np

import oracle

# Codes: the GPU rotates in float32 and the oracle in float64, so a code may
# differ by one where the scaled value sits within 1e-5 (relative) of a
# rounding boundary, on at most 0.1% of the elements.
TIE_REL = 1e-5
MAX_FLIP_FRAC = 1e-3


def bf16_ord(bits: np.ndarray) -> np.ndarray:
    """Map bfloat16 bit patterns to integers ordered like the values (+0 and -0 coincide)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.int64)
    mag = b & 0x7FFF
    return np.where(b & 0x8000, -mag, mag)


def assert_bf16_within_1ulp(got_bits: np.ndarray, want_bits: np.ndarray, what: str = "Y"):
    d = np.abs(bf16_ord(got_bits) - bf16_ord(want_bits))
    bad = np.argwhere(d > 1)
    assert bad.size == 0, f"{what}: {len(bad)} outputs differ by more than 1 bf16 ulp, first at {bad[:5].tolist()}, max {d.max()}"
    return int((d == 1).sum())


def assert_codes_match(q_gpu: np.ndarray, q_ref: np.ndarray, y_ref: np.ndarray, s_ref, what: str = "codes"):
    """Codes equal, except +-1 flips at oracle-flagged near-ties on <= 0.1% of elements."""
    diff = q_gpu.astype(np.int16) - q_ref.astype(np.int16)
    idx = np.nonzero(diff)
    n = len(idx[0])
    if n == 0:
        return 0
    assert np.all(np.abs(diff[idx]) == 1), f"{what}: a code differs by more than 1"
    s = np.asarray(s_ref, dtype=np.float64)
    s_at = s if s.ndim == 0 else np.broadcast_to(s.reshape(-1, 1), q_ref.shape)[idx]
    tie = oracle.near_tie_mask(y_ref[idx], s_at, TIE_REL)
    assert tie.all(), f"{what}: {int((~tie).sum())} flips are not near a rounding boundary"
    assert n <= MAX_FLIP_FRAC * q_ref.size, f"{what}: {n} flips out of {q_ref.size}"
    return n


def rotation_error_bound(x_bits: np.ndarray, group: int = 256) -> float:
    """Largest absolute error of a float32 radix-4 rotation of one group, over all groups.

    Each of the p = log4(group) radix-4 passes rounds 3 times on the way to any
    output, and every intermediate value is a +-1 combination of disjoint input
    subsets, so the unnormalised output error is at most 3p * 2**-24 * sum(|x|)
    over the group; the 1/2**p normalisation divides it by 2**p.
    """
    x = np.abs(oracle.bf16_bits_to_f64(x_bits))
    if x.size == 0:
        return 0.0
    R, K = x.shape
    p = {16: 2, 64: 3, 256: 4, 1024: 5}[group]
    sums = x.reshape(R, K // group, group).sum(axis=2)
    return float(3 * p * 2.0 ** -24 * sums.max() / 2.0 ** p)


def assert_scale_close(s_gpu: float, s_ref: float, x_bits: np.ndarray = None, what: str = "scale",
                       qpos: float = 7.0, group: int = 256):
    """The scale is the float32 max of the rotated values over qpos (7 for INT4,
    127 for INT8): it may differ from the oracle's by the float32 rotation error
    of the max element (divided by qpos) plus one ulp for the division.  Without
    ``x_bits`` (no rotation) only the one ulp is allowed."""
    a, b = np.float32(s_gpu), np.float32(s_ref)
    tol = float(np.spacing(np.abs(b)))
    if x_bits is not None:
        tol += rotation_error_bound(x_bits, group) / qpos
    assert abs(np.float64(a) - np.float64(b)) <= tol, f"{what}: {a!r} vs {b!r} (tolerance {tol:.3g})"
