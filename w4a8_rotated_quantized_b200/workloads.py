"""Seeded synthetic workloads for the ConvRot W4A4 linear layer.

This module only draws random inputs.  It holds none of the layer's
arithmetic (no rotation, no scales, no quantisation), so both the CPU oracle
and the CUDA path can be fed from it without sharing any of the method.

Shapes and value ranges follow the model cards' layers:

* "Qwen-Image-Edit-2511-W4A8-ConvRot", per-family error table: the DiT
  linears are [3072, 3072], [12288, 3072] and [3072, 12288].
* "Qwen3-4B — ConvRot W4A4 (ComfyUI text encoder)", section "What it costs in
  fidelity": prompts of 21-23 tokens, hidden size 2560, conditioning values
  with an absolute maximum near 1.4e4; section "What it costs in speed":
  prompt lengths around 22 and 130 tokens.  The Qwen3-4B MLP is
  2560 -> 9728 -> 2560.

The real weights and activations behind those cards are not available, so
these seeded draws stand in for them.

Recipe (every config): ``numpy.random.default_rng(seed)`` (PCG64); draw the
outlier channel indices first, then X, then W, then the bias; values are
produced in float32 and rounded to bfloat16 round-to-nearest-even.  The
bfloat16 tensors are returned as uint16 bit patterns.
"""

from __future__ import annotations

import dataclasses
from typing import Dict

import numpy as np

__all__ = ["Workload", "CONFIGS", "make_inputs", "bf16_bits_from_f32", "f32_from_bf16_bits"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    M: int
    K: int
    N: int
    seed: int
    x_dist: str  # "normal" | "gelu_normal" | "student_t3"
    n_outliers: int  # number of outlier channels (columns of X)
    outlier_scale: float
    x_peak: float = 0.0  # if nonzero, X[0, first outlier channel] is set to this value
    w_std: float = 0.02
    bias_std: float = 0.01
    description: str = ""

    @property
    def ops(self) -> int:
        """Integer multiply-adds counted as 2 operations: 2*M*N*K."""
        return 2 * self.M * self.N * self.K


def _pct(K: int, frac: float) -> int:
    return int(round(frac * K))


CONFIGS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("tiny", 64, 512, 256, 0, "normal", 2, 20.0,
                 description="tiny parity case: X [64,512] N(0,1), 2 channels x20; W [256,512] N(0,0.02)"),
        Workload("dit_attn", 4096, 3072, 3072, 1, "normal", _pct(3072, 0.01), 50.0,
                 description="DiT attention projection: X [4096,3072] N(0,1), 1% channels x50; W [3072,3072]"),
        Workload("dit_mlp_up", 8192, 3072, 12288, 2, "normal", _pct(3072, 0.01), 50.0,
                 description="DiT MLP up, two-image edit: X [8192,3072] -> W [12288,3072]"),
        Workload("dit_mlp_down", 8192, 12288, 3072, 5, "gelu_normal", _pct(12288, 0.01), 50.0,
                 description="DiT MLP down: X [8192,12288] = GELU(N(0,1)), 1% channels x50 -> W [3072,12288]"),
        Workload("w4a8_up", 4096, 3072, 12288, 3, "student_t3", 0, 1.0,
                 description="W4A8 case: X [4096,3072] Student-t nu=3 -> W [12288,3072]"),
        Workload("text_enc_up_21", 21, 2560, 9728, 4, "normal", 2, 1000.0, x_peak=14000.0,
                 description="text encoder MLP up, 21 tokens: X [21,2560] -> W [9728,2560]"),
        Workload("text_enc_up_130", 130, 2560, 9728, 4, "normal", 2, 1000.0, x_peak=14000.0,
                 description="text encoder MLP up, 130 tokens: X [130,2560] -> W [9728,2560]"),
        Workload("text_enc_down_21", 21, 9728, 2560, 4, "normal", 9, 1000.0, x_peak=14000.0,
                 description="text encoder MLP down, 21 tokens: X [21,9728] -> W [2560,9728]"),
        Workload("text_enc_down_130", 130, 9728, 2560, 4, "normal", 9, 1000.0, x_peak=14000.0,
                 description="text encoder MLP down, 130 tokens: X [130,9728] -> W [2560,9728]"),
    ]
}


def bf16_bits_from_f32(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round-to-nearest-even), as uint16 bits.

    Uses torch's float32 -> bfloat16 conversion (a library rounding routine).
    """
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def f32_from_bf16_bits(b: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns to float32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _draw_x(rng: np.random.Generator, w: Workload, M: int, K: int) -> np.ndarray:
    import torch

    if w.x_dist == "normal":
        x = rng.standard_normal((M, K), dtype=np.float32)
    elif w.x_dist == "gelu_normal":
        z = rng.standard_normal((M, K), dtype=np.float32)
        x = torch.nn.functional.gelu(torch.from_numpy(z)).numpy()  # exact erf form
    elif w.x_dist == "student_t3":
        x = rng.standard_t(3.0, size=(M, K)).astype(np.float32)
    else:
        raise ValueError(f"unknown x_dist {w.x_dist!r}")
    return x


def make_inputs(w: Workload | str, *, M: int | None = None, with_weight: bool = True,
                seed: int | None = None) -> dict:
    """Draw X, W and bias for a workload.

    ``M`` overrides the token count (the weight and bias draws do not depend on
    it, but the X draw does).  ``seed`` overrides the workload's seed.

    Returns a dict of uint16 bfloat16 bit patterns: ``X`` [M,K], ``W`` [N,K]
    and ``bias`` [N], plus ``outlier_channels`` (int64 indices).
    """
    if isinstance(w, str):
        w = CONFIGS[w]
    M = w.M if M is None else int(M)
    rng = np.random.default_rng(w.seed if seed is None else seed)
    K, N = w.K, w.N
    ch = np.sort(rng.choice(K, size=w.n_outliers, replace=False)) if w.n_outliers else np.zeros(0, np.int64)
    x = _draw_x(rng, w, M, K)
    if len(ch):
        x[:, ch] *= np.float32(w.outlier_scale)
        if w.x_peak and M > 0:
            x[0, ch[0]] = np.float32(w.x_peak)
    out = {"X": bf16_bits_from_f32(x), "outlier_channels": ch.astype(np.int64)}
    if with_weight:
        wt = rng.standard_normal((N, K), dtype=np.float32) * np.float32(w.w_std)
        b = rng.standard_normal((N,), dtype=np.float32) * np.float32(w.bias_std)
        out["W"] = bf16_bits_from_f32(wt)
        out["bias"] = bf16_bits_from_f32(b)
    return out
