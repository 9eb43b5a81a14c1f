"""Plain CPU oracle for the ConvRot W4A4 linear layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this module:
only the test suite, the smoke check in ``__graft_entry__`` and the CPU-baseline
arm of ``bench.py`` use it.  It shares no code with the CUDA library.

What it computes (the model cards describe the method; the formulas below are
the plainest reading of them):

* "Qwen-Image-Edit-2511 — INT4 tensorwise W4A4 (+ConvRot, mixed int8 fallback)",
  introduction: weights are packed signed INT4, two per byte, after a
  group-256 regular-Hadamard ("ConvRot") rotation; activations are rotated
  online and quantised dynamically to INT4; no calibration.  Section
  "Measurements": the product kernel is a "rank-one" s4 MMA, i.e. an integer
  product scaled by (activation scale) x (weight scale).
* "Qwen3-4B — ConvRot W4A4 (ComfyUI text encoder)", section "Format": a
  quantised layer stores ``weight`` as I8 [rows, cols/2] holding signed INT4
  and ``weight_scale`` as F32 [rows]; convrot_groupsize is 256.

The regular Hadamard matrix of order 256 is not printed on any page.  Reading
used here: H4 = J - 2I (the order-4 regular Hadamard matrix, every row sums
to 2) and H256 = H4 (x) H4 (x) H4 (x) H4 / 16, which is symmetric, orthogonal
and has every row sum equal to 1.  Other readings this oracle fixes, each
listed with its reason in the design notes:

* groups are contiguous 256-wide slices of K, rotated independently;
* scale = amax / 7 (symmetric INT4 range; the clamp range is [-8, 7]);
* codes are taken with round-half-to-even.  The pages do not say in what
  precision the quotient y / s is formed before rounding; reading used here:
  single precision, t = fl32(fl32(y) / s), with s itself a float32.  A code
  is an integer decided by floating point, so the side being checked must
  take the same decision in the same precision; the stated tolerance (codes
  may flip by one only where y / s lies within 1e-5 relative of a half
  integer) covers any difference in how the rotated value y was summed;
* nibble order: the low nibble of byte j holds element 2j, two's complement;
* epilogue: y = acc * s_a * s_w[n] + bias[n] in float64, rounded once to
  bfloat16 (round-to-nearest-even).

The INT8 tensorwise format (with or without the ConvRot rotation) is the
fallback format of the same pages: "Qwen-Image-Edit-2511 — INT4 tensorwise
W4A4 (+ConvRot, mixed int8 fallback)", introduction (sensitive layers kept as
stock ``int8_tensorwise``), and "Qwen Image 2.1 — Hybrid W4A8 / INT8 ConvRot",
layer list ("INT8 tensorwise + ConvRot").  Reading used here: the same
symmetric recipe with 8 bits, scale = amax / 127, codes clamped to
[-128, 127], weights and activations alike, the rotation optional.

The W4A8 format (4-bit asymmetric weights, group 16 along K, fp16 scale and
4-bit zero point per group, INT8 tensorwise activations, both rotated) comes
from "Qwen-Image-Edit-2511 — W4A8 ConvRot" (build table, file layout) and
"Qwen Image 2.1 — Hybrid W4A8 / INT8 ConvRot" (recipe); its reading is stated
above the functions that implement it.

Parity pins for every function live in the CPU test suite (closed forms,
brute force on tiny inputs, worked examples built so the answer is known).
"""

from __future__ import annotations

from typing import Tuple

import numpy as np

GROUP = 256
QMIN, QMAX = -8, 7
QPOS = 7.0  # scale divisor: amax maps to +7
Q8MIN, Q8MAX = -128, 127
Q8POS = 127.0  # INT8: amax maps to +127

__all__ = [
    "GROUP", "QMIN", "QMAX",
    "regular_hadamard", "rotate", "scale_from_amax", "tensor_scale", "row_scales",
    "quantize", "pack_int4", "unpack_int4", "int_gemm", "bf16_bits_to_f64",
    "bf16_rne_bits", "epilogue", "rotate_quant_act", "pack_weight", "w4a4_linear",
    "near_tie_mask", "reference_linear", "relative_error",
    "Q8MIN", "Q8MAX", "scale8_from_amax", "tensor_scale8", "row_scales8", "quantize8",
    "quant_act8", "pack_weight8", "int8_linear", "a8w4_linear",
    "QG16", "U4MAX", "asym_params16", "quantize_asym16", "dequant_asym16", "pack_u4", "unpack_u4",
    "pack_weight_w4a8", "w4a8_linear", "w4a8_acc", "w4a8_epilogue",
]


# ---------------------------------------------------------------------------
# Rotation
# ---------------------------------------------------------------------------

def regular_hadamard(n: int = GROUP) -> np.ndarray:
    """Regular Hadamard matrix of order n = 4**p, normalised to be orthogonal.

    Closed form of H4 (x) ... (x) H4 (p factors) / 2**p with H4 = J - 2I:
    H4[a][b] is -1 when a == b and +1 otherwise, so the Kronecker product's
    entry (i, j) is (-1) ** (number of base-4 digits where i and j agree).

    Cites "Qwen-Image-Edit-2511 — INT4 tensorwise W4A4 (+ConvRot, mixed int8
    fallback)", introduction ("group-256 regular-Hadamard ConvRot rotation").
    """
    p = 0
    while 4 ** p < n:
        p += 1
    if 4 ** p != n:
        raise ValueError(f"regular Hadamard order must be a power of 4, got {n}")
    i = np.arange(n)
    agree = np.zeros((n, n), dtype=np.int64)
    for d in range(p):
        di = (i >> (2 * d)) & 3
        agree += (di[:, None] == di[None, :])
    return np.where(agree % 2 == 0, 1.0, -1.0) / float(2 ** p)


def rotate(x: np.ndarray, group: int = GROUP) -> np.ndarray:
    """Rotate each row by H, one contiguous K-slice of width ``group`` at a time.

    y[r, g*G + j] = sum_i x[r, g*G + i] * H[i][j]   (float64).

    The same transform rotates activation rows online and weight rows offline,
    which is what keeps the layer's exact product unchanged:
    (X H)(W H)^T = X W^T because H H^T = I.
    Cites the introduction of "Qwen-Image-Edit-2511 — INT4 tensorwise W4A4
    (+ConvRot, mixed int8 fallback)" (weights rotated, activations rotated
    online) and "Qwen3-4B — ConvRot W4A4 (ComfyUI text encoder)", section
    "Format" (convrot_groupsize 256).
    """
    x = np.asarray(x, dtype=np.float64)
    R, K = x.shape
    if K % group:
        raise ValueError(f"K={K} is not a multiple of the rotation group {group}")
    H = regular_hadamard(group)
    return (x.reshape(R, K // group, group) @ H).reshape(R, K)


# ---------------------------------------------------------------------------
# Scales and codes
# ---------------------------------------------------------------------------

def scale_from_amax(amax) -> np.ndarray:
    """INT4 scale for a given absolute maximum: fl32(fl32(amax) / 7); 1 if amax is 0.

    The symmetric INT4 grid maps amax to +7 ("packed signed INT4",
    introduction of "Qwen-Image-Edit-2511 — INT4 tensorwise W4A4 (+ConvRot,
    mixed int8 fallback)"); an all-zero tensor gets scale 1 and all-zero codes.
    """
    a32 = np.asarray(amax, dtype=np.float64).astype(np.float32)
    s = a32 / np.float32(QPOS)
    return np.where(a32 == 0, np.float32(1.0), s).astype(np.float32)


def tensor_scale(y: np.ndarray) -> np.float32:
    """One scale for the whole tensor ("tensorwise", dynamic, calibration-free).

    Cites "Qwen-Image-Edit-2511 — INT4 tensorwise W4A4 (+ConvRot, mixed int8
    fallback)", title and introduction.
    """
    y = np.asarray(y, dtype=np.float64)
    amax = np.max(np.abs(y)) if y.size else 0.0
    return np.float32(scale_from_amax(amax))


def row_scales(y: np.ndarray) -> np.ndarray:
    """One scale per row, the granularity of ``weight_scale`` F32 [rows].

    Cites "Qwen3-4B — ConvRot W4A4 (ComfyUI text encoder)", section "Format".
    """
    y = np.asarray(y, dtype=np.float64)
    return scale_from_amax(np.max(np.abs(y), axis=1)).astype(np.float32)


def quantize(y: np.ndarray, s) -> np.ndarray:
    """Signed INT4 codes: q = clamp(round_half_even(fl32(fl32(y) / s)), -8, 7).

    ``s`` is a float32 scalar or a float32 column (one scale per row).  The
    pages leave the precision of the quotient open; it is formed in single
    precision here (module docstring), and rounded half to even.
    """
    t = np.asarray(y, dtype=np.float64).astype(np.float32) / np.asarray(s, dtype=np.float32)
    q = np.rint(t)  # numpy rint rounds half to even
    return np.clip(q, QMIN, QMAX).astype(np.int8)


def pack_int4(q: np.ndarray) -> np.ndarray:
    """Pack signed INT4 codes two per byte: byte j = (q[2j] & 0xF) | (q[2j+1] & 0xF) << 4.

    Cites "Qwen3-4B — ConvRot W4A4 (ComfyUI text encoder)", section "Format":
    an I8 container of shape [rows, cols/2] holding signed INT4.
    """
    q = np.asarray(q, dtype=np.int64)
    if q.shape[-1] % 2:
        raise ValueError("pack_int4 needs an even number of columns")
    lo = q[..., 0::2] & 0xF
    hi = q[..., 1::2] & 0xF
    return (lo | (hi << 4)).astype(np.uint8)


def unpack_int4(p: np.ndarray) -> np.ndarray:
    """Inverse of :func:`pack_int4` (two's-complement nibbles to int8)."""
    p = np.asarray(p, dtype=np.uint8).astype(np.int64)
    lo = p & 0xF
    hi = p >> 4
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.int8)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


# ---------------------------------------------------------------------------
# Integer product and epilogue
# ---------------------------------------------------------------------------

def int_gemm(qa: np.ndarray, qw: np.ndarray) -> np.ndarray:
    """acc[m, n] = sum_k qa[m, k] * qw[n, k], exactly, as int64.

    Uses a float64 matrix product: every term is an integer of magnitude at
    most 128 * 128 (INT8 codes; 64 for INT4) and every partial sum stays far
    below 2**53, so the float64 product is exact whatever order the library
    sums in.
    Cites "Qwen-Image-Edit-2511 — INT4 tensorwise W4A4 (+ConvRot, mixed int8
    fallback)", section "Measurements" (s4 MMA: integer products).
    """
    qa = np.asarray(qa)
    qw = np.asarray(qw)
    K = qa.shape[1]
    if qw.shape[1] != K:
        raise ValueError("inner dimensions differ")
    if 16384 * K >= 2 ** 53:
        raise ValueError("K too large for an exact float64 product")
    acc = qa.astype(np.float64) @ qw.astype(np.float64).T
    out = acc.astype(np.int64)
    if out.size and np.max(np.abs(out)) >= 2 ** 31:
        raise OverflowError("accumulator does not fit int32")
    return out


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) to float64 (exact)."""
    u = np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def bf16_rne_bits(v: np.ndarray) -> np.ndarray:
    """Round float64 values to bfloat16 with one round-to-nearest-even step.

    bfloat16 keeps 8 significant bits and float32's exponent range; below
    2**-126 the spacing is 2**-133 (subnormals).  The value is scaled by the
    spacing of its binade, rounded half-to-even to an integer, scaled back
    (all exact in float64), and the result is returned as uint16 bits.
    """
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    with np.errstate(invalid="ignore", over="ignore"):
        _, e = np.frexp(a)  # a = m * 2**e with m in [0.5, 1)
        q_exp = np.maximum(e.astype(np.int64) - 8, -133)
        r = np.rint(np.ldexp(a, -q_exp))
        res = np.ldexp(r, q_exp)
        res = np.where(np.isfinite(a), res, a)
        bits = (res.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)  # exact in float32, or inf
    bits = np.where(np.signbit(v), bits | np.uint16(0x8000), bits)
    bits = np.where(np.isnan(v), np.uint16(0x7FC0), bits)
    return bits.astype(np.uint16)


def epilogue(acc: np.ndarray, s_a, s_w: np.ndarray, bias_bits: np.ndarray | None) -> np.ndarray:
    """y[m, n] = bf16_rne(acc[m, n] * s_a * s_w[n] + bias[n]), float64 inside.

    The scale is rank one (activation scale times per-row weight scale),
    "Qwen-Image-Edit-2511 — INT4 tensorwise W4A4 (+ConvRot, mixed int8
    fallback)", section "Measurements"; the bias and bfloat16 output are the
    layer's own.  ``s_a`` is a float32 scalar, ``s_w`` float32 [N], ``bias``
    bfloat16 bits [N] or None.  Returns bfloat16 bits [M, N].
    """
    acc = np.asarray(acc, dtype=np.float64)
    scale = np.float64(np.float32(s_a)) * np.asarray(s_w, dtype=np.float32).astype(np.float64)
    y = acc * scale[None, :]
    if bias_bits is not None:
        y = y + bf16_bits_to_f64(bias_bits)[None, :]
    return bf16_rne_bits(y)


# ---------------------------------------------------------------------------
# The three calls of the layer
# ---------------------------------------------------------------------------

def rotate_quant_act(x_bits: np.ndarray, group: int = GROUP) -> Tuple[np.ndarray, np.float32, np.ndarray, np.ndarray]:
    """Online activation path: rotate, one dynamic tensorwise scale, INT4 codes, pack.

    Returns (packed uint8 [M, K/2], s_a float32, codes int8 [M, K], rotated float64 [M, K]).
    Cites the introduction of "Qwen-Image-Edit-2511 — INT4 tensorwise W4A4
    (+ConvRot, mixed int8 fallback)": activations rotated online and
    dynamically quantised to INT4, calibration-free.
    """
    y = rotate(bf16_bits_to_f64(x_bits), group)
    s_a = tensor_scale(y)
    q = quantize(y, s_a)
    return pack_int4(q), s_a, q, y


def pack_weight(w_bits: np.ndarray, group: int = GROUP, scale_mode: str = "tensor") -> Tuple[np.ndarray, np.ndarray, np.ndarray, np.ndarray]:
    """Offline weight path: rotate rows, scale (one for the tensor or one per row), INT4 codes, pack.

    Returns (packed uint8 [N, K/2], s_w float32 [N], codes int8 [N, K], rotated float64 [N, K]).
    A tensorwise scale is stored repeated in every row of the [N] vector.
    Cites "Qwen3-4B — ConvRot W4A4 (ComfyUI text encoder)", section "Format"
    (I8 [rows, cols/2] + F32 [rows]), and the tensorwise naming of
    "Qwen-Image-Edit-2511 — INT4 tensorwise W4A4 (+ConvRot, mixed int8 fallback)".
    """
    y = rotate(bf16_bits_to_f64(w_bits), group)
    N = y.shape[0]
    if scale_mode == "tensor":
        s_w = np.full((N,), tensor_scale(y), dtype=np.float32)
    elif scale_mode == "row":
        s_w = row_scales(y)
    else:
        raise ValueError(f"unknown scale_mode {scale_mode!r}")
    q = quantize(y, s_w[:, None])
    return pack_int4(q), s_w, q, y


def w4a4_linear(x_bits: np.ndarray, wq_packed: np.ndarray, s_w: np.ndarray,
                bias_bits: np.ndarray | None, group: int = GROUP) -> dict:
    """The whole layer: rotate + quantise X, integer product with packed W, epilogue.

    Returns a dict with ``Y`` (bfloat16 bits [M, N]) and the intermediates
    ``Xq``, ``s_a``, ``qa``, ``acc``.
    """
    xq, s_a, qa, _ = rotate_quant_act(x_bits, group)
    qw = unpack_int4(wq_packed)
    acc = int_gemm(qa, qw)
    y = epilogue(acc, s_a, s_w, bias_bits)
    return {"Y": y, "Xq": xq, "s_a": s_a, "qa": qa, "acc": acc}


# ---------------------------------------------------------------------------
# INT8 tensorwise (+ optional ConvRot rotation): the fallback format
# ---------------------------------------------------------------------------

def scale8_from_amax(amax) -> np.ndarray:
    """INT8 scale: fl32(fl32(amax) / 127); 1 if amax is 0.

    Symmetric 8-bit grid, amax maps to +127 (stock ``int8_tensorwise`` of
    "Qwen-Image-Edit-2511 — INT4 tensorwise W4A4 (+ConvRot, mixed int8
    fallback)", introduction).
    """
    a32 = np.asarray(amax, dtype=np.float64).astype(np.float32)
    s = a32 / np.float32(Q8POS)
    return np.where(a32 == 0, np.float32(1.0), s).astype(np.float32)


def tensor_scale8(y: np.ndarray) -> np.float32:
    """One INT8 scale for the whole tensor (tensorwise, dynamic for activations)."""
    y = np.asarray(y, dtype=np.float64)
    amax = np.max(np.abs(y)) if y.size else 0.0
    return np.float32(scale8_from_amax(amax))


def row_scales8(y: np.ndarray) -> np.ndarray:
    """One INT8 scale per row (the F32 [rows] ``weight_scale`` granularity)."""
    y = np.asarray(y, dtype=np.float64)
    return scale8_from_amax(np.max(np.abs(y), axis=1)).astype(np.float32)


def quantize8(y: np.ndarray, s) -> np.ndarray:
    """Signed INT8 codes: q = clamp(round_half_even(fl32(fl32(y) / s)), -128, 127).

    The decision is taken in float32, like :func:`quantize`.
    """
    t = np.asarray(y, dtype=np.float64).astype(np.float32) / np.asarray(s, dtype=np.float32)
    return np.clip(np.rint(t), Q8MIN, Q8MAX).astype(np.int8)


def quant_act8(x_bits: np.ndarray, rotate_groups: bool = True, group: int = GROUP) -> Tuple[np.ndarray, np.float32, np.ndarray]:
    """INT8 activation path: (optional ConvRot rotation), one dynamic tensorwise scale, codes.

    Returns (codes int8 [M, K], s_a float32, the quantised values float64 [M, K]).
    With ``rotate_groups=False`` this is the stock int8_tensorwise activation path.
    """
    y = bf16_bits_to_f64(x_bits)
    if rotate_groups:
        y = rotate(y, group)
    s_a = tensor_scale8(y)
    return quantize8(y, s_a), s_a, y


def pack_weight8(w_bits: np.ndarray, rotate_groups: bool = True, scale_mode: str = "tensor",
                 group: int = GROUP) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """INT8 weight path: (optional rotation of the rows), tensorwise or per-row scale, codes.

    Returns (codes int8 [N, K], s_w float32 [N], the quantised values float64 [N, K]).
    """
    y = bf16_bits_to_f64(w_bits)
    if rotate_groups:
        y = rotate(y, group)
    N = y.shape[0]
    if scale_mode == "tensor":
        s_w = np.full((N,), tensor_scale8(y), dtype=np.float32)
    elif scale_mode == "row":
        s_w = row_scales8(y)
    else:
        raise ValueError(f"unknown scale_mode {scale_mode!r}")
    return quantize8(y, s_w[:, None]), s_w, y


def int8_linear(x_bits: np.ndarray, qw: np.ndarray, s_w: np.ndarray, bias_bits: np.ndarray | None,
                rotate_groups: bool = True, group: int = GROUP) -> dict:
    """The INT8 layer: (rotate +) quantise X to INT8, exact integer product, the same epilogue.

    Returns a dict with ``Y`` (bfloat16 bits [M, N]), ``qa``, ``s_a`` and ``acc``.
    """
    qa, s_a, _ = quant_act8(x_bits, rotate_groups, group)
    acc = int_gemm(qa, qw)
    return {"Y": epilogue(acc, s_a, s_w, bias_bits), "qa": qa, "s_a": s_a, "acc": acc}


def a8w4_linear(x_bits: np.ndarray, wq_packed: np.ndarray, s_w: np.ndarray, bias_bits: np.ndarray | None,
                rotate_groups: bool = True, group: int = GROUP) -> dict:
    """The "INT8 branch" of the W4A4 format: INT8 tensorwise activation codes (after the rotation)
    against the format's packed INT4 weights, exact integer product, the same epilogue.

    "Qwen3-4B — ConvRot W4A4 (ComfyUI text encoder)", section "Hardware": on newer GPUs the W4A4
    format runs an INT8 activation branch.  Returns a dict with ``Y``, ``qa``, ``s_a`` and ``acc``.
    """
    qa, s_a, _ = quant_act8(x_bits, rotate_groups, group)
    acc = int_gemm(qa, unpack_int4(wq_packed))
    return {"Y": epilogue(acc, s_a, s_w, bias_bits), "qa": qa, "s_a": s_a, "acc": acc}


# ---------------------------------------------------------------------------
# W4A8 asymmetric, group 16 (+ ConvRot rotation): 4-bit weights, 8-bit activations
# ---------------------------------------------------------------------------
#
# "Qwen-Image-Edit-2511 — W4A8 ConvRot", build table and file layout: weights
# 4-bit asymmetric ("asym_w4a8_int8"), group_size 16, convrot_groupsize 256,
# activations 8-bit; "Qwen Image 2.1 — Hybrid W4A8 / INT8 ConvRot", recipe:
# asymmetric W4A8 for most linear layers.  The pages name the format but not
# its formulas.  Reading used here (the common asymmetric min/max recipe, with
# an fp16 scale and a 4-bit zero point per group of 16 consecutive K elements
# of a rotated weight row):
#   lo, hi = min, max of the group;  s = fp16(fl32(hi - lo) / 15), 1 if that is 0
#   z = clamp(rne(-lo / s), 0, 15);  q = clamp(rne(w / s) + z, 0, 15)
#   dequantised weight  w^ = s * (q - z)
# with every rounding decision taken in float32: the pages leave the precision
# open, and an integer decided by floating point must be decided the same way
# on both sides of a comparison (the stated tolerances cover the rest).
# Activations: the INT8 tensorwise path with rotation (quant_act8).
# Layer: y = bf16_rne(s_a * sum_k qa[m, k] * w^[n, k] + bias[n]), float64 inside.

QG16 = 16
U4MAX = 15


def asym_params16(y: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Scale (float16) and zero point (uint8, 0..15) of every group of 16 along the last axis.

    ``y`` is [N, K] (float64 values, rounded to float32 first: decisions are taken in float32).
    """
    y32 = np.asarray(y, dtype=np.float64).astype(np.float32)
    N, K = y32.shape
    if K % QG16:
        raise ValueError("K must be a multiple of 16")
    g = y32.reshape(N, K // QG16, QG16)
    lo = g.min(axis=2)
    hi = g.max(axis=2)
    s32 = (hi - lo) / np.float32(U4MAX)          # float32 subtraction and division, each rounded once
    s16 = s32.astype(np.float16)                 # round to nearest even
    s16 = np.where(s16 == 0, np.float16(1.0), s16)
    z = np.clip(np.rint(-lo / s16.astype(np.float32)), 0, U4MAX)
    return s16.astype(np.float16), z.astype(np.uint8)


def quantize_asym16(y: np.ndarray, s16: np.ndarray, z: np.ndarray) -> np.ndarray:
    """Unsigned 4-bit codes q = clamp(rne(fl32(fl32(w) / s)) + z, 0, 15) with the group's s and z."""
    y32 = np.asarray(y, dtype=np.float64).astype(np.float32)
    N, K = y32.shape
    sf = np.repeat(np.asarray(s16, dtype=np.float16).astype(np.float32), QG16, axis=1)
    zf = np.repeat(np.asarray(z, dtype=np.int64), QG16, axis=1)
    q = np.rint(y32 / sf).astype(np.int64) + zf
    return np.clip(q, 0, U4MAX).astype(np.uint8)


def dequant_asym16(q: np.ndarray, s16: np.ndarray, z: np.ndarray) -> np.ndarray:
    """w^ = s * (q - z), exact in float64."""
    sf = np.repeat(np.asarray(s16, dtype=np.float16).astype(np.float64), QG16, axis=1)
    zf = np.repeat(np.asarray(z, dtype=np.int64), QG16, axis=1)
    return sf * (np.asarray(q, dtype=np.int64) - zf).astype(np.float64)


def pack_u4(q: np.ndarray) -> np.ndarray:
    """Pack unsigned 4-bit values two per byte, element 2j in the low nibble of byte j."""
    q = np.asarray(q, dtype=np.int64)
    if q.shape[-1] % 2:
        raise ValueError("pack_u4 needs an even number of columns")
    return ((q[..., 0::2] & 0xF) | ((q[..., 1::2] & 0xF) << 4)).astype(np.uint8)


def unpack_u4(p: np.ndarray) -> np.ndarray:
    """Inverse of :func:`pack_u4`."""
    p = np.asarray(p, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


def pack_weight_w4a8(w_bits: np.ndarray, rotate_groups: bool = True, group: int = GROUP) -> dict:
    """W4A8 weight path: (rotation of the rows), per-group-16 asymmetric 4-bit codes.

    Returns a dict: ``q`` uint8 [N, K] (0..15), ``Wq`` packed [N, K/2], ``s`` float16
    [N, K/16], ``z`` uint8 [N, K/16], ``Z`` packed zero points [N, K/32], ``y`` the
    (rotated) float64 weights.
    """
    y = bf16_bits_to_f64(w_bits)
    if rotate_groups:
        y = rotate(y, group)
    s16, z = asym_params16(y)
    q = quantize_asym16(y, s16, z)
    return {"q": q, "Wq": pack_u4(q), "s": s16, "z": z, "Z": pack_u4(z), "y": y}


def w4a8_linear(x_bits: np.ndarray, q: np.ndarray, s16: np.ndarray, z: np.ndarray,
                bias_bits: np.ndarray | None, rotate_groups: bool = True, group: int = GROUP) -> dict:
    """The W4A8 layer: INT8 tensorwise activation codes (after rotation) against
    dequantised asymmetric 4-bit weights, float64 sum, one rounding to bfloat16.

    Returns a dict with ``Y`` (bfloat16 bits [M, N]), ``qa``, ``s_a`` and ``acc``
    (sum_k qa * w^, float64, before the activation scale and bias).
    """
    qa, s_a, _ = quant_act8(x_bits, rotate_groups, group)
    acc = w4a8_acc(qa, q, s16, z)
    return {"Y": w4a8_epilogue(acc, s_a, bias_bits), "qa": qa, "s_a": s_a, "acc": acc}


def w4a8_acc(qa: np.ndarray, q: np.ndarray, s16: np.ndarray, z: np.ndarray) -> np.ndarray:
    """acc[m, n] = sum_k qa[m, k] * s[n, k/16] * (q[n, k] - z[n, k/16]) in float64.

    Every term has at most 8 + 11 + 5 significant bits, so the float64 sum
    carries a relative error of at most K * 2**-53 of sum |terms|.
    """
    return np.asarray(qa, dtype=np.float64) @ dequant_asym16(q, s16, z).T


def w4a8_epilogue(acc: np.ndarray, s_a, bias_bits: np.ndarray | None) -> np.ndarray:
    """y = bf16_rne(acc * s_a + bias), float64 inside."""
    y = np.asarray(acc, dtype=np.float64) * np.float64(np.float32(s_a))
    if bias_bits is not None:
        y = y + bf16_bits_to_f64(bias_bits)[None, :]
    return bf16_rne_bits(y)


# ---------------------------------------------------------------------------
# Helpers for comparing against other implementations
# ---------------------------------------------------------------------------

def near_tie_mask(y: np.ndarray, s, rel: float = 1e-5) -> np.ndarray:
    """True where y / s lies within ``rel`` (relative) of a half-integer rounding boundary.

    A code may legitimately differ by one at such points between two
    implementations that round the rotation differently.
    """
    t = np.asarray(y, dtype=np.float64) / np.asarray(s, dtype=np.float64)
    frac = np.abs(t - np.floor(t) - 0.5)
    return frac <= rel * np.maximum(np.abs(t), 1e-30)


def reference_linear(x_bits: np.ndarray, w_bits: np.ndarray, bias_bits: np.ndarray | None) -> np.ndarray:
    """Unquantised float64 layer X W^T + b, for the relative-error side report.

    The per-layer error metric of "Qwen-Image-Edit-2511-W4A8-ConvRot" (per-layer
    error table: error of a format against a float32 reference) is measured
    against this.
    """
    y = bf16_bits_to_f64(x_bits) @ bf16_bits_to_f64(w_bits).T
    if bias_bits is not None:
        y = y + bf16_bits_to_f64(bias_bits)[None, :]
    return y


def relative_error(y: np.ndarray, y_ref: np.ndarray) -> float:
    """||y - y_ref||_F / ||y_ref||_F."""
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    return float(np.linalg.norm(y - y_ref) / np.linalg.norm(y_ref))
