"""Thin ctypes binding over the C ABI in include/convrot.h.

Every function here only marshals arguments: it allocates outputs with
torch, passes raw device pointers, sizes and the current CUDA stream to the
library, and raises ``ConvRotError`` on a non-zero status.  All arithmetic of
the layer runs in the library's CUDA kernels; there is no CPU fallback and
importing this module fails loudly when the library has not been built.
"""

from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Tuple

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libconvrot_b200.so")

CR_OK = 0
CR_SCALE_TENSOR = 0
CR_SCALE_ROW = 1
GROUP = 256

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"ConvRot CUDA library not found at {LIB_PATH}; build it with "
        "`python -m w4a8_rotated_quantized_b200.build` (or __graft_entry__.build())")

_lib = ctypes.CDLL(LIB_PATH)

_vp, _i, _i64, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
_SIGS = {
    "cr_status_string": (ctypes.c_char_p, [_i]),
    "cr_api_version": (_i, []),
    "cr_rotate_quant_act_workspace_size": (_sz, [_i, _i, _i]),
    "cr_pack_weight_workspace_size": (_sz, [_i, _i, _i, _i]),
    "cr_w4a4_gemm_workspace_size": (_sz, [_i, _i, _i]),
    "cr_w4a4_linear_workspace_size": (_sz, [_i, _i, _i, _i]),
    "cr_pack_weight": (_i, [_vp, _i, _i, _i64, _i, _i, _vp, _vp, _vp, _sz, _vp]),
    "cr_rotate_quant_act": (_i, [_vp, _i, _i, _i64, _i, _vp, _vp, _vp, _sz, _vp]),
    "cr_w4a4_gemm": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i, _i, _i, _vp, _sz, _vp]),
    "cr_w4a4_gemm_s32": (_i, [_vp, _vp, _vp, _i64, _i, _i, _i, _vp, _sz, _vp]),
    "cr_w4a4_linear": (_i, [_vp, _i64, _vp, _vp, _vp, _vp, _i64, _i, _i, _i, _i, _vp, _sz, _vp]),
    "cr_read_device_status": (_i, [_vp, ctypes.POINTER(_i), _vp]),
    "cr_w4a4_linear_noalloc": (_i, [_vp, _i64, _vp, _vp, _vp, _vp, _i64, _i, _i, _i, _i, _vp]),
    "cr_int8_gemm_workspace_size": (_sz, [_i, _i, _i]),
    "cr_int8_linear_workspace_size": (_sz, [_i, _i, _i, _i]),
    "cr_pack_weight_ex": (_i, [_vp, _i, _i, _i64, _i, _i, _i, _i, _vp, _vp, _vp, _sz, _vp]),
    "cr_rotate_quant_act_ex": (_i, [_vp, _i, _i, _i64, _i, _i, _i, _vp, _vp, _vp, _sz, _vp]),
    "cr_int8_gemm": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i, _i, _i, _vp, _sz, _vp]),
    "cr_int8_gemm_s32": (_i, [_vp, _vp, _vp, _i64, _i, _i, _i, _vp, _sz, _vp]),
    "cr_int8_linear": (_i, [_vp, _i64, _i, _vp, _vp, _vp, _vp, _i64, _i, _i, _i, _i, _vp, _sz, _vp]),
    "cr_w4a8_gemm_workspace_size": (_sz, [_i, _i, _i]),
    "cr_w4a8_linear_workspace_size": (_sz, [_i, _i, _i, _i]),
    "cr_pack_weight_w4a8": (_i, [_vp, _i, _i, _i64, _i, _i, _vp, _vp, _vp, _vp, _sz, _vp]),
    "cr_w4a8_gemm": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i, _i, _i, _vp, _sz, _vp]),
    "cr_w4a8_gemm_f32": (_i, [_vp, _vp, _vp, _vp, _vp, _i64, _i, _i, _i, _vp, _sz, _vp]),
    "cr_w4a8_linear": (_i, [_vp, _i64, _vp, _vp, _vp, _vp, _vp, _i64, _i, _i, _i, _i, _vp, _sz, _vp]),
    "cr_a8w4_gemm_workspace_size": (_sz, [_i, _i, _i]),
    "cr_a8w4_linear_workspace_size": (_sz, [_i, _i, _i, _i]),
    "cr_a8w4_gemm": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i, _i, _i, _vp, _sz, _vp]),
    "cr_a8w4_gemm_s32": (_i, [_vp, _vp, _vp, _i64, _i, _i, _i, _vp, _sz, _vp]),
    "cr_a8w4_linear": (_i, [_vp, _i64, _vp, _vp, _vp, _vp, _i64, _i, _i, _i, _i, _vp, _sz, _vp]),
    "cr_selftest_wait_timeout": (_i, [_vp, _sz, _vp]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class ConvRotError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {cr_status_string(status)}")


def cr_status_string(status: int) -> str:
    return _lib.cr_status_string(int(status)).decode()


def cr_api_version() -> int:
    return int(_lib.cr_api_version())


def _check(fn: str, status: int) -> None:
    if status != CR_OK:
        raise ConvRotError(fn, status)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


# One zero-initialised workspace per device, grown on demand.  Its first bytes
# hold the device status word, which the kernels only ever set to an error.
_ws_lock = threading.Lock()
_ws: dict = {}


def workspace(device: torch.device, nbytes: int) -> torch.Tensor:
    key = torch.device(device).index if torch.device(device).index is not None else torch.cuda.current_device()
    with _ws_lock:
        buf = _ws.get(key)
        if buf is None or buf.numel() < nbytes:
            buf = torch.zeros(max(nbytes, 1 << 20), dtype=torch.uint8, device=torch.device("cuda", key))
            _ws[key] = buf
        return buf


def _rows(t: torch.Tensor, name: str) -> Tuple[int, int, int]:
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{name} must be 2-D with unit stride along the last dimension")
    return t.shape[0], t.shape[1], t.stride(0)


def _bf16_cuda(t: torch.Tensor, name: str) -> None:
    if t.dtype != torch.bfloat16 or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA bfloat16 tensor")


def cr_pack_weight(W: torch.Tensor, group: int = GROUP, scale_mode: str = "tensor") -> Tuple[torch.Tensor, torch.Tensor]:
    """Offline: rotate, quantise and pack a bf16 weight [N, K] -> (Wq uint8 [N, K/2], w_scale float32 [N])."""
    _bf16_cuda(W, "W")
    N, K, ldw = _rows(W, "W")
    mode = {"tensor": CR_SCALE_TENSOR, "row": CR_SCALE_ROW}[scale_mode]
    Wq = torch.empty((N, K // 2), dtype=torch.uint8, device=W.device)
    w_scale = torch.empty((N,), dtype=torch.float32, device=W.device)
    nbytes = _lib.cr_pack_weight_workspace_size(N, K, group, mode)
    ws = workspace(W.device, nbytes)
    _check("cr_pack_weight", _lib.cr_pack_weight(_ptr(W), N, K, ldw, group, mode, _ptr(Wq), _ptr(w_scale),
                                                 _ptr(ws), ws.numel(), _stream(W.device)))
    return Wq, w_scale


def cr_rotate_quant_act(X: torch.Tensor, group: int = GROUP) -> Tuple[torch.Tensor, torch.Tensor]:
    """Online: rotate + dynamic tensorwise INT4 quantisation of bf16 X [M, K] -> (Xq uint8 [M, K/2], a_scale float32 [1])."""
    _bf16_cuda(X, "X")
    M, K, ldx = _rows(X, "X")
    Xq = torch.empty((M, K // 2), dtype=torch.uint8, device=X.device)
    a_scale = torch.empty((1,), dtype=torch.float32, device=X.device)
    ws = workspace(X.device, _lib.cr_rotate_quant_act_workspace_size(M, K, group))
    _check("cr_rotate_quant_act", _lib.cr_rotate_quant_act(_ptr(X), M, K, ldx, group, _ptr(Xq), _ptr(a_scale),
                                                           _ptr(ws), ws.numel(), _stream(X.device)))
    return Xq, a_scale


def cr_w4a4_gemm(Xq: torch.Tensor, a_scale: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor,
                 bias: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Y bf16 [M, N] = (Xq . Wq^T) * a_scale * w_scale[n] + bias[n]."""
    M, Kh = Xq.shape
    N = Wq.shape[0]
    K = 2 * Kh
    if Wq.shape[1] != Kh:
        raise ValueError("Xq and Wq disagree on K")
    for t, name in ((Xq, "Xq"), (Wq, "Wq")):
        if t.dtype != torch.uint8 or not t.is_contiguous():
            raise TypeError(f"{name} must be a contiguous uint8 tensor")
    if bias is not None:
        _bf16_cuda(bias, "bias")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=Xq.device)
    _, _, ldy = _rows(out, "out")
    ws = workspace(Xq.device, _lib.cr_w4a4_gemm_workspace_size(M, N, K))
    _check("cr_w4a4_gemm", _lib.cr_w4a4_gemm(_ptr(Xq), _ptr(a_scale), _ptr(Wq), _ptr(w_scale), _ptr(bias),
                                             _ptr(out), ldy, M, N, K, _ptr(ws), ws.numel(), _stream(Xq.device)))
    return out


def cr_w4a4_gemm_s32(Xq: torch.Tensor, Wq: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Raw int32 product C [M, N] = sum_k qa[m, k] * qw[n, k] of packed INT4 codes."""
    M, Kh = Xq.shape
    N = Wq.shape[0]
    if Wq.shape[1] != Kh:
        raise ValueError("Xq and Wq disagree on K")
    if out is None:
        out = torch.empty((M, N), dtype=torch.int32, device=Xq.device)
    _, _, ldc = _rows(out, "out")
    ws = workspace(Xq.device, _lib.cr_w4a4_gemm_workspace_size(M, N, 2 * Kh))
    _check("cr_w4a4_gemm_s32", _lib.cr_w4a4_gemm_s32(_ptr(Xq), _ptr(Wq), _ptr(out), ldc, M, N, 2 * Kh, _ptr(ws),
                                                     ws.numel(), _stream(Xq.device)))
    return out


def cr_w4a4_linear(X: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor, bias: Optional[torch.Tensor] = None,
                   out: Optional[torch.Tensor] = None, group: int = GROUP) -> torch.Tensor:
    """The whole online layer: Y = linear(rotate_quant(X), Wq) with one call into the library."""
    _bf16_cuda(X, "X")
    M, K, ldx = _rows(X, "X")
    N = Wq.shape[0]
    if bias is not None:
        _bf16_cuda(bias, "bias")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    _, _, ldy = _rows(out, "out")
    ws = workspace(X.device, _lib.cr_w4a4_linear_workspace_size(M, N, K, group))
    _check("cr_w4a4_linear", _lib.cr_w4a4_linear(_ptr(X), ldx, _ptr(Wq), _ptr(w_scale), _ptr(bias), _ptr(out), ldy,
                                                 M, N, K, group, _ptr(ws), ws.numel(), _stream(X.device)))
    return out


def cr_read_device_status(device: Optional[torch.device] = None) -> int:
    """Device status word of this device's shared workspace (synchronises the current stream)."""
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    ws = workspace(device, 256)
    st = ctypes.c_int(0)
    _check("cr_read_device_status", _lib.cr_read_device_status(_ptr(ws), ctypes.byref(st), _stream(device)))
    return st.value


def cr_w4a4_linear_noalloc(X: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor,
                           bias: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                           group: int = GROUP) -> torch.Tensor:
    """The one-call layer for callers that cannot allocate device scratch.

    The library keeps this call's scratch in a fixed device array (M * K / 2 <= 8 MiB);
    calls whose GPU work overlaps race on it.  ``out`` may be passed to avoid the
    output allocation this wrapper otherwise makes.
    """
    _bf16_cuda(X, "X")
    M, K, ldx = _rows(X, "X")
    N = Wq.shape[0]
    if bias is not None:
        _bf16_cuda(bias, "bias")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    _, _, ldy = _rows(out, "out")
    _check("cr_w4a4_linear_noalloc", _lib.cr_w4a4_linear_noalloc(
        _ptr(X), ldx, _ptr(Wq), _ptr(w_scale), _ptr(bias), _ptr(out), ldy, M, N, K, group, _stream(X.device)))
    return out


# ---------------------------------------------------------------------------
# Code formats other than packed INT4 of rotated values (bits 4 or 8, rotation on or off)
# ---------------------------------------------------------------------------

def _code_cols(K: int, bits: int) -> int:
    if bits not in (4, 8):
        raise ValueError("bits must be 4 or 8")
    return K // 2 if bits == 4 else K


def cr_pack_weight_ex(W: torch.Tensor, bits: int = 8, rotate: bool = True, scale_mode: str = "tensor",
                      group: int = GROUP) -> Tuple[torch.Tensor, torch.Tensor]:
    """Offline weight codes in any format: (Wq [N, K/2] uint8 for bits 4 | int8 [N, K] for bits 8, w_scale [N])."""
    _bf16_cuda(W, "W")
    N, K, ldw = _rows(W, "W")
    mode = {"tensor": CR_SCALE_TENSOR, "row": CR_SCALE_ROW}[scale_mode]
    Wq = torch.empty((N, _code_cols(K, bits)), dtype=torch.uint8 if bits == 4 else torch.int8, device=W.device)
    w_scale = torch.empty((N,), dtype=torch.float32, device=W.device)
    ws = workspace(W.device, _lib.cr_pack_weight_workspace_size(N, K, group, mode))
    _check("cr_pack_weight_ex", _lib.cr_pack_weight_ex(_ptr(W), N, K, ldw, group, bits, int(bool(rotate)), mode,
                                                       _ptr(Wq), _ptr(w_scale), _ptr(ws), ws.numel(),
                                                       _stream(W.device)))
    return Wq, w_scale


def cr_rotate_quant_act_ex(X: torch.Tensor, bits: int = 8, rotate: bool = True,
                           group: int = GROUP) -> Tuple[torch.Tensor, torch.Tensor]:
    """Online activation codes in any format: (Xq, a_scale float32 [1]); layout as cr_pack_weight_ex."""
    _bf16_cuda(X, "X")
    M, K, ldx = _rows(X, "X")
    Xq = torch.empty((M, _code_cols(K, bits)), dtype=torch.uint8 if bits == 4 else torch.int8, device=X.device)
    a_scale = torch.empty((1,), dtype=torch.float32, device=X.device)
    ws = workspace(X.device, _lib.cr_rotate_quant_act_workspace_size(M, K, group))
    _check("cr_rotate_quant_act_ex", _lib.cr_rotate_quant_act_ex(_ptr(X), M, K, ldx, group, bits, int(bool(rotate)),
                                                                 _ptr(Xq), _ptr(a_scale), _ptr(ws), ws.numel(),
                                                                 _stream(X.device)))
    return Xq, a_scale


def _int8_operands(Xq: torch.Tensor, Wq: torch.Tensor) -> Tuple[int, int, int]:
    for t, name in ((Xq, "Xq"), (Wq, "Wq")):
        if t.dtype != torch.int8 or not t.is_contiguous() or t.dim() != 2:
            raise TypeError(f"{name} must be a contiguous 2-D int8 tensor")
    if Wq.shape[1] != Xq.shape[1]:
        raise ValueError("Xq and Wq disagree on K")
    return Xq.shape[0], Wq.shape[0], Xq.shape[1]


def cr_int8_gemm(Xq: torch.Tensor, a_scale: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor,
                 bias: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Y bf16 [M, N] = (Xq . Wq^T) * a_scale * w_scale[n] + bias[n] over INT8 codes."""
    M, N, K = _int8_operands(Xq, Wq)
    if bias is not None:
        _bf16_cuda(bias, "bias")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=Xq.device)
    _, _, ldy = _rows(out, "out")
    ws = workspace(Xq.device, _lib.cr_int8_gemm_workspace_size(M, N, K))
    _check("cr_int8_gemm", _lib.cr_int8_gemm(_ptr(Xq), _ptr(a_scale), _ptr(Wq), _ptr(w_scale), _ptr(bias),
                                             _ptr(out), ldy, M, N, K, _ptr(ws), ws.numel(), _stream(Xq.device)))
    return out


def cr_int8_gemm_s32(Xq: torch.Tensor, Wq: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Raw int32 product C [M, N] = sum_k qa[m, k] * qw[n, k] of INT8 codes."""
    M, N, K = _int8_operands(Xq, Wq)
    if out is None:
        out = torch.empty((M, N), dtype=torch.int32, device=Xq.device)
    _, _, ldc = _rows(out, "out")
    ws = workspace(Xq.device, _lib.cr_int8_gemm_workspace_size(M, N, K))
    _check("cr_int8_gemm_s32", _lib.cr_int8_gemm_s32(_ptr(Xq), _ptr(Wq), _ptr(out), ldc, M, N, K, _ptr(ws),
                                                     ws.numel(), _stream(Xq.device)))
    return out


def cr_int8_linear(X: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor, bias: Optional[torch.Tensor] = None,
                   rotate: bool = True, out: Optional[torch.Tensor] = None, group: int = GROUP) -> torch.Tensor:
    """The whole INT8 layer in one call: (rotate +) quantise X to INT8, product, epilogue."""
    _bf16_cuda(X, "X")
    M, K, ldx = _rows(X, "X")
    N = Wq.shape[0]
    if Wq.dtype != torch.int8 or Wq.shape[1] != K:
        raise TypeError("Wq must be int8 [N, K] (cr_pack_weight_ex with bits=8)")
    if bias is not None:
        _bf16_cuda(bias, "bias")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    _, _, ldy = _rows(out, "out")
    ws = workspace(X.device, _lib.cr_int8_linear_workspace_size(M, N, K, group))
    _check("cr_int8_linear", _lib.cr_int8_linear(_ptr(X), ldx, int(bool(rotate)), _ptr(Wq), _ptr(w_scale),
                                                 _ptr(bias), _ptr(out), ldy, M, N, K, group, _ptr(ws), ws.numel(),
                                                 _stream(X.device)))
    return out


# ---------------------------------------------------------------------------
# W4A8: asymmetric 4-bit weights (group 16, fp16 scale, 4-bit zero), INT8 activations
# ---------------------------------------------------------------------------

def cr_pack_weight_w4a8(W: torch.Tensor, rotate: bool = True,
                        group: int = GROUP) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Offline W4A8 weights: (Wq uint8 [N, K/2], gscale float16 [N, K/16], gzero uint8 [N, K/32])."""
    _bf16_cuda(W, "W")
    N, K, ldw = _rows(W, "W")
    Wq = torch.empty((N, K // 2), dtype=torch.uint8, device=W.device)
    gs = torch.empty((N, K // 16), dtype=torch.float16, device=W.device)
    gz = torch.empty((N, K // 32), dtype=torch.uint8, device=W.device)
    ws = workspace(W.device, _lib.cr_pack_weight_workspace_size(N, K, group, CR_SCALE_TENSOR))
    _check("cr_pack_weight_w4a8", _lib.cr_pack_weight_w4a8(_ptr(W), N, K, ldw, group, int(bool(rotate)), _ptr(Wq),
                                                           _ptr(gs), _ptr(gz), _ptr(ws), ws.numel(),
                                                           _stream(W.device)))
    return Wq, gs, gz


def _w4a8_operands(Xq, Wq, gs, gz) -> Tuple[int, int, int]:
    if Xq.dtype != torch.int8 or not Xq.is_contiguous() or Xq.dim() != 2:
        raise TypeError("Xq must be a contiguous 2-D int8 tensor")
    M, K = Xq.shape
    N = Wq.shape[0]
    if Wq.dtype != torch.uint8 or tuple(Wq.shape) != (N, K // 2) or not Wq.is_contiguous():
        raise TypeError("Wq must be contiguous uint8 [N, K/2]")
    if gs.dtype != torch.float16 or tuple(gs.shape) != (N, K // 16) or not gs.is_contiguous():
        raise TypeError("gscale must be contiguous float16 [N, K/16]")
    if gz.dtype != torch.uint8 or tuple(gz.shape) != (N, K // 32) or not gz.is_contiguous():
        raise TypeError("gzero must be contiguous uint8 [N, K/32]")
    return M, N, K


def cr_w4a8_gemm(Xq: torch.Tensor, a_scale: torch.Tensor, Wq: torch.Tensor, gscale: torch.Tensor,
                 gzero: torch.Tensor, bias: Optional[torch.Tensor] = None,
                 out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Y bf16 [M, N] = a_scale * sum_k Xq * s * (q - z) + bias."""
    M, N, K = _w4a8_operands(Xq, Wq, gscale, gzero)
    if bias is not None:
        _bf16_cuda(bias, "bias")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=Xq.device)
    _, _, ldy = _rows(out, "out")
    ws = workspace(Xq.device, _lib.cr_w4a8_gemm_workspace_size(M, N, K))
    _check("cr_w4a8_gemm", _lib.cr_w4a8_gemm(_ptr(Xq), _ptr(a_scale), _ptr(Wq), _ptr(gscale), _ptr(gzero),
                                             _ptr(bias), _ptr(out), ldy, M, N, K, _ptr(ws), ws.numel(),
                                             _stream(Xq.device)))
    return out


def cr_w4a8_gemm_f32(Xq: torch.Tensor, Wq: torch.Tensor, gscale: torch.Tensor, gzero: torch.Tensor,
                     out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The float32 sums C [M, N] = sum_k Xq * fp16(s * (q - z)) (no activation scale, no bias)."""
    M, N, K = _w4a8_operands(Xq, Wq, gscale, gzero)
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32, device=Xq.device)
    _, _, ldc = _rows(out, "out")
    ws = workspace(Xq.device, _lib.cr_w4a8_gemm_workspace_size(M, N, K))
    _check("cr_w4a8_gemm_f32", _lib.cr_w4a8_gemm_f32(_ptr(Xq), _ptr(Wq), _ptr(gscale), _ptr(gzero), _ptr(out), ldc,
                                                     M, N, K, _ptr(ws), ws.numel(), _stream(Xq.device)))
    return out


def cr_w4a8_linear(X: torch.Tensor, Wq: torch.Tensor, gscale: torch.Tensor, gzero: torch.Tensor,
                   bias: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                   group: int = GROUP) -> torch.Tensor:
    """The whole W4A8 layer in one call: rotation + INT8 activation codes, then the W4A8 product."""
    _bf16_cuda(X, "X")
    M, K, ldx = _rows(X, "X")
    N = Wq.shape[0]
    if bias is not None:
        _bf16_cuda(bias, "bias")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    _, _, ldy = _rows(out, "out")
    ws = workspace(X.device, _lib.cr_w4a8_linear_workspace_size(M, N, K, group))
    _check("cr_w4a8_linear", _lib.cr_w4a8_linear(_ptr(X), ldx, _ptr(Wq), _ptr(gscale), _ptr(gzero), _ptr(bias),
                                                 _ptr(out), ldy, M, N, K, group, _ptr(ws), ws.numel(),
                                                 _stream(X.device)))
    return out


# ---------------------------------------------------------------------------
# INT8 activation codes against the W4A4 format's packed INT4 weights ("INT8 branch")
# ---------------------------------------------------------------------------

def _a8w4_operands(Xq: torch.Tensor, Wq: torch.Tensor) -> Tuple[int, int, int]:
    if Xq.dtype != torch.int8 or not Xq.is_contiguous() or Xq.dim() != 2:
        raise TypeError("Xq must be a contiguous 2-D int8 tensor")
    if Wq.dtype != torch.uint8 or not Wq.is_contiguous() or Wq.dim() != 2 or Wq.shape[1] * 2 != Xq.shape[1]:
        raise TypeError("Wq must be contiguous uint8 [N, K/2] (packed INT4)")
    return Xq.shape[0], Wq.shape[0], Xq.shape[1]


def cr_a8w4_gemm(Xq: torch.Tensor, a_scale: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor,
                 bias: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Y bf16 [M, N] = (Xq . Wq^T) * a_scale * w_scale[n] + bias[n], INT8 codes against packed INT4 weights."""
    M, N, K = _a8w4_operands(Xq, Wq)
    if bias is not None:
        _bf16_cuda(bias, "bias")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=Xq.device)
    _, _, ldy = _rows(out, "out")
    ws = workspace(Xq.device, _lib.cr_a8w4_gemm_workspace_size(M, N, K))
    _check("cr_a8w4_gemm", _lib.cr_a8w4_gemm(_ptr(Xq), _ptr(a_scale), _ptr(Wq), _ptr(w_scale), _ptr(bias),
                                             _ptr(out), ldy, M, N, K, _ptr(ws), ws.numel(), _stream(Xq.device)))
    return out


def cr_a8w4_gemm_s32(Xq: torch.Tensor, Wq: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Raw int32 product C [M, N] = sum_k qa[m, k] * qw[n, k] (INT8 codes, packed INT4 weights)."""
    M, N, K = _a8w4_operands(Xq, Wq)
    if out is None:
        out = torch.empty((M, N), dtype=torch.int32, device=Xq.device)
    _, _, ldc = _rows(out, "out")
    ws = workspace(Xq.device, _lib.cr_a8w4_gemm_workspace_size(M, N, K))
    _check("cr_a8w4_gemm_s32", _lib.cr_a8w4_gemm_s32(_ptr(Xq), _ptr(Wq), _ptr(out), ldc, M, N, K, _ptr(ws),
                                                     ws.numel(), _stream(Xq.device)))
    return out


def cr_a8w4_linear(X: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor, bias: Optional[torch.Tensor] = None,
                   out: Optional[torch.Tensor] = None, group: int = GROUP) -> torch.Tensor:
    """The whole layer with INT8 activations against the packed INT4 weights of cr_pack_weight."""
    _bf16_cuda(X, "X")
    M, K, ldx = _rows(X, "X")
    N = Wq.shape[0]
    if bias is not None:
        _bf16_cuda(bias, "bias")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    _, _, ldy = _rows(out, "out")
    ws = workspace(X.device, _lib.cr_a8w4_linear_workspace_size(M, N, K, group))
    _check("cr_a8w4_linear", _lib.cr_a8w4_linear(_ptr(X), ldx, _ptr(Wq), _ptr(w_scale), _ptr(bias), _ptr(out), ldy,
                                                 M, N, K, group, _ptr(ws), ws.numel(), _stream(X.device)))
    return out


def cr_selftest_wait_timeout(ws: torch.Tensor) -> None:
    """Enqueue the bounded-wait self-test on ``ws`` (a zeroed uint8 CUDA workspace of >= 256 bytes)."""
    _check("cr_selftest_wait_timeout", _lib.cr_selftest_wait_timeout(_ptr(ws), ws.numel(), _stream(ws.device)))
