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
    "cr_w4a4_linear_ex": (_i, [_vp, _i64, _vp, _vp, _vp, _vp, _i64, _i, _i, _i, _i, _i, _vp, _sz, _vp]),
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
    "cr_selftest_act_fallback": (_i, [_vp, _i, _i, _i64, _i, _i, _i, _vp, _vp, _vp, _sz, _vp]),
    "cr_w4a4_gemm_multi": (_i, [_vp, _vp, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "cr_w4a4_gemm_multi_s32": (_i, [_vp, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "cr_w4a4_linear_multi": (_i, [_vp, _i64, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
}
CR_MAX_PROJ = 4
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
    if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA bfloat16 tensor")


# Every tensor handed to the library is checked here before its pointer is taken: the library sees
# only raw addresses and sizes, so a tensor of the wrong shape, dtype or device would make a kernel
# read or write outside it.

def _dev(t: torch.Tensor, name: str, dtype: torch.dtype, device: torch.device) -> None:
    """dtype and device of an operand.  ``device`` is the first input's, which the wrappers check to be
    a CUDA device before anything else, so every operand ends up on that one GPU."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.device != device:
        raise TypeError(f"{name} must be on {device}, got {t.device}")


def _dense(t: torch.Tensor, name: str, dtype: torch.dtype, device: torch.device, shape: Tuple[int, ...]) -> None:
    """A contiguous tensor of exactly this shape, dtype and device."""
    _dev(t, name, dtype, device)
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _vec(t: Optional[torch.Tensor], name: str, dtype: torch.dtype, device: torch.device, n: int,
         optional: bool = False) -> None:
    """A contiguous 1-D tensor of n elements (a per-output-column scale or bias)."""
    if t is None and optional:
        return
    _dense(t, name, dtype, device, (n,))


def _scalar(t: torch.Tensor, name: str, device: torch.device) -> None:
    """The tensorwise activation scale: at least one float32 on the device."""
    _dev(t, name, torch.float32, device)
    if t.numel() < 1:
        raise ValueError(f"{name} must hold one float32")


def _out(out: Optional[torch.Tensor], M: int, N: int, dtype: torch.dtype, device: torch.device) -> Tuple[torch.Tensor, int]:
    """The caller's output (rows may be strided, columns dense) or a new one; returns it and its row stride."""
    if out is None:
        out = torch.empty((M, N), dtype=dtype, device=device)
    _dev(out, "out", dtype, device)
    if tuple(out.shape) != (M, N):
        raise ValueError(f"out must have shape {(M, N)}, got {tuple(out.shape)}")
    if out.numel() == 0:  # nothing is written; torch gives empty tensors arbitrary strides
        return out, N
    return out, _rows(out, "out")[2]


def _codes(t: torch.Tensor, name: str, dtype: torch.dtype) -> Tuple[int, int]:
    """Contiguous 2-D code matrix; its device is checked by :func:`_cuda` once the shapes agree."""
    if not isinstance(t, torch.Tensor) or t.dtype != dtype or t.dim() != 2 or not t.is_contiguous():
        raise TypeError(f"{name} must be a contiguous 2-D {dtype} tensor")
    return t.shape[0], t.shape[1]


def _cuda(t: torch.Tensor, name: str) -> None:
    """The first input must live on a CUDA device; every other operand must share that device."""
    if not t.is_cuda:
        raise TypeError(f"{name} must be on a CUDA device, got {t.device}")


def _w4a4_weights(Wq: torch.Tensor, w_scale: torch.Tensor, bias: Optional[torch.Tensor], K: int,
                  device: torch.device) -> int:
    """Packed INT4 weights [N, K/2] uint8, w_scale float32 [N], bias bfloat16 [N] or None; returns N."""
    _dev(Wq, "Wq", torch.uint8, device)
    if Wq.dim() != 2:
        raise ValueError("Wq must be 2-D [N, K/2]")
    N = Wq.shape[0]
    _dense(Wq, "Wq", torch.uint8, device, (N, K // 2))
    _vec(w_scale, "w_scale", torch.float32, device, N)
    _vec(bias, "bias", torch.bfloat16, device, N, optional=True)
    return N


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
    M, Kh = _codes(Xq, "Xq", torch.uint8)
    K = 2 * Kh
    _scalar(a_scale, "a_scale", Xq.device)
    N = _w4a4_weights(Wq, w_scale, bias, K, Xq.device)
    _cuda(Xq, "Xq")
    out, ldy = _out(out, M, N, torch.bfloat16, Xq.device)
    ws = workspace(Xq.device, _lib.cr_w4a4_gemm_workspace_size(M, N, K))
    _check("cr_w4a4_gemm", _lib.cr_w4a4_gemm(_ptr(Xq), _ptr(a_scale), _ptr(Wq), _ptr(w_scale), _ptr(bias),
                                             _ptr(out), ldy, M, N, K, _ptr(ws), ws.numel(), _stream(Xq.device)))
    return out


def cr_w4a4_gemm_s32(Xq: torch.Tensor, Wq: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Raw int32 product C [M, N] = sum_k qa[m, k] * qw[n, k] of packed INT4 codes."""
    M, Kh = _codes(Xq, "Xq", torch.uint8)
    _dev(Wq, "Wq", torch.uint8, Xq.device)
    if Wq.dim() != 2 or Wq.shape[1] != Kh:
        raise ValueError("Xq and Wq disagree on K")
    N = Wq.shape[0]
    _dense(Wq, "Wq", torch.uint8, Xq.device, (N, Kh))
    _cuda(Xq, "Xq")
    out, ldc = _out(out, M, N, torch.int32, Xq.device)
    ws = workspace(Xq.device, _lib.cr_w4a4_gemm_workspace_size(M, N, 2 * Kh))
    _check("cr_w4a4_gemm_s32", _lib.cr_w4a4_gemm_s32(_ptr(Xq), _ptr(Wq), _ptr(out), ldc, M, N, 2 * Kh, _ptr(ws),
                                                     ws.numel(), _stream(Xq.device)))
    return out


LINEAR_AUTO, LINEAR_ONE_LAUNCH, LINEAR_TWO_LAUNCHES = 0, 1, 2


def cr_w4a4_linear(X: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor, bias: Optional[torch.Tensor] = None,
                   out: Optional[torch.Tensor] = None, group: int = GROUP, mode: int = LINEAR_AUTO) -> torch.Tensor:
    """The whole online layer: Y = linear(rotate_quant(X), Wq) with one call into the library.

    ``mode`` picks the launch arrangement (``cr_w4a4_linear_ex``): LINEAR_AUTO (the library's choice),
    LINEAR_ONE_LAUNCH (rotation, codes and GEMM fused; at most 256 tokens) or LINEAR_TWO_LAUNCHES.
    The outputs are the same bit for bit.
    """
    if mode not in (LINEAR_AUTO, LINEAR_ONE_LAUNCH, LINEAR_TWO_LAUNCHES):
        raise ValueError(f"mode must be 0, 1 or 2, got {mode}")
    _bf16_cuda(X, "X")
    M, K, ldx = _rows(X, "X")
    N = _w4a4_weights(Wq, w_scale, bias, K, X.device)
    out, ldy = _out(out, M, N, torch.bfloat16, X.device)
    ws = workspace(X.device, _lib.cr_w4a4_linear_workspace_size(M, N, K, group))
    _check("cr_w4a4_linear_ex",
           _lib.cr_w4a4_linear_ex(_ptr(X), ldx, _ptr(Wq), _ptr(w_scale), _ptr(bias), _ptr(out), ldy, M, N, K, group,
                                  mode, _ptr(ws), ws.numel(), _stream(X.device)))
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
    N = _w4a4_weights(Wq, w_scale, bias, K, X.device)
    out, ldy = _out(out, M, N, torch.bfloat16, X.device)
    _check("cr_w4a4_linear_noalloc", _lib.cr_w4a4_linear_noalloc(
        _ptr(X), ldx, _ptr(Wq), _ptr(w_scale), _ptr(bias), _ptr(out), ldy, M, N, K, group, _stream(X.device)))
    return out


# ---------------------------------------------------------------------------
# Shared activation quantisation for split projections (one set of codes, several weights)
# ---------------------------------------------------------------------------

def _proj_lists(Wqs, w_scales, biases, K: int, device: torch.device):
    if not isinstance(Wqs, (list, tuple)) or not 1 <= len(Wqs) <= CR_MAX_PROJ:
        raise ValueError(f"give 1 to {CR_MAX_PROJ} projections")
    n = len(Wqs)
    if w_scales is None or len(w_scales) != n:
        raise ValueError("one w_scale per projection")
    biases = [None] * n if biases is None else list(biases)
    if len(biases) != n:
        raise ValueError("one bias (or None) per projection")
    Ns = [_w4a4_weights(Wqs[j], w_scales[j], biases[j], K, device) for j in range(n)]
    return Ns, biases


def _ptr_array(ts):
    return (ctypes.c_void_p * len(ts))(*[None if t is None else t.data_ptr() for t in ts])


def _outs(outs, M: int, Ns, dtype: torch.dtype, device: torch.device):
    outs = [None] * len(Ns) if outs is None else list(outs)
    if len(outs) != len(Ns):
        raise ValueError("one output (or None) per projection")
    res = [_out(o, M, n, dtype, device) for o, n in zip(outs, Ns)]
    return [r[0] for r in res], (ctypes.c_int64 * len(res))(*[r[1] for r in res])


def cr_w4a4_gemm_multi(Xq: torch.Tensor, a_scale: torch.Tensor, Wqs, w_scales, biases=None, outs=None):
    """One set of activation codes against several packed weights: [Y_j bf16 [M, N_j]] (one launch for M > 128)."""
    M, Kh = _codes(Xq, "Xq", torch.uint8)
    K = 2 * Kh
    _scalar(a_scale, "a_scale", Xq.device)
    Ns, biases = _proj_lists(Wqs, w_scales, biases, K, Xq.device)
    _cuda(Xq, "Xq")
    outs, ldy = _outs(outs, M, Ns, torch.bfloat16, Xq.device)
    n = len(Ns)
    ws = workspace(Xq.device, _lib.cr_w4a4_gemm_workspace_size(M, 0, K))
    _check("cr_w4a4_gemm_multi", _lib.cr_w4a4_gemm_multi(
        _ptr(Xq), _ptr(a_scale), M, K, n, _ptr_array(Wqs), _ptr_array(w_scales),
        None if all(b is None for b in biases) else _ptr_array(biases), _ptr_array(outs), ldy,
        (ctypes.c_int * n)(*Ns), _ptr(ws), ws.numel(), _stream(Xq.device)))
    return outs


def cr_w4a4_gemm_multi_s32(Xq: torch.Tensor, Wqs, outs=None):
    """Raw int32 products of one set of activation codes with several packed weights."""
    M, Kh = _codes(Xq, "Xq", torch.uint8)
    K = 2 * Kh
    if not isinstance(Wqs, (list, tuple)) or not 1 <= len(Wqs) <= CR_MAX_PROJ:
        raise ValueError(f"give 1 to {CR_MAX_PROJ} projections")
    Ns = []
    for j, W in enumerate(Wqs):
        _dev(W, f"Wq[{j}]", torch.uint8, Xq.device)
        if W.dim() != 2:
            raise ValueError("Wq must be 2-D [N, K/2]")
        _dense(W, f"Wq[{j}]", torch.uint8, Xq.device, (W.shape[0], Kh))
        Ns.append(W.shape[0])
    _cuda(Xq, "Xq")
    outs, ldc = _outs(outs, M, Ns, torch.int32, Xq.device)
    n = len(Ns)
    ws = workspace(Xq.device, _lib.cr_w4a4_gemm_workspace_size(M, 0, K))
    _check("cr_w4a4_gemm_multi_s32", _lib.cr_w4a4_gemm_multi_s32(
        _ptr(Xq), M, K, n, _ptr_array(Wqs), _ptr_array(outs), ldc, (ctypes.c_int * n)(*Ns), _ptr(ws), ws.numel(),
        _stream(Xq.device)))
    return outs


def cr_w4a4_linear_multi(X: torch.Tensor, Wqs, w_scales, biases=None, outs=None, group: int = GROUP):
    """Rotate and quantise X once, then every projection: [Y_j bf16 [M, N_j]] (two launches for M > 128)."""
    _bf16_cuda(X, "X")
    M, K, ldx = _rows(X, "X")
    Ns, biases = _proj_lists(Wqs, w_scales, biases, K, X.device)
    outs, ldy = _outs(outs, M, Ns, torch.bfloat16, X.device)
    n = len(Ns)
    ws = workspace(X.device, _lib.cr_w4a4_linear_workspace_size(M, 0, K, group))
    _check("cr_w4a4_linear_multi", _lib.cr_w4a4_linear_multi(
        _ptr(X), ldx, M, K, group, n, _ptr_array(Wqs), _ptr_array(w_scales),
        None if all(b is None for b in biases) else _ptr_array(biases), _ptr_array(outs), ldy,
        (ctypes.c_int * n)(*Ns), _ptr(ws), ws.numel(), _stream(X.device)))
    return outs


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


def cr_selftest_act_fallback(X: torch.Tensor, bits: int = 4, rotate: bool = True,
                             group: int = GROUP) -> Tuple[torch.Tensor, torch.Tensor]:
    """Diagnostic: cr_rotate_quant_act_ex on the fallback kernels (the two streaming passes that run when the
    device refuses the one-launch pass's cooperative launch); the same (Xq, a_scale) bit for bit."""
    _bf16_cuda(X, "X")
    M, K, ldx = _rows(X, "X")
    Xq = torch.empty((M, _code_cols(K, bits)), dtype=torch.uint8 if bits == 4 else torch.int8, device=X.device)
    a_scale = torch.empty((1,), dtype=torch.float32, device=X.device)
    ws = workspace(X.device, _lib.cr_rotate_quant_act_workspace_size(M, K, group))
    _check("cr_selftest_act_fallback",
           _lib.cr_selftest_act_fallback(_ptr(X), M, K, ldx, group, bits, int(bool(rotate)), _ptr(Xq), _ptr(a_scale),
                                         _ptr(ws), ws.numel(), _stream(X.device)))
    return Xq, a_scale


def _int8_operands(Xq: torch.Tensor, Wq: torch.Tensor) -> Tuple[int, int, int]:
    M, K = _codes(Xq, "Xq", torch.int8)
    if not isinstance(Wq, torch.Tensor) or Wq.dtype != torch.int8 or Wq.dim() != 2 or not Wq.is_contiguous():
        raise TypeError("Wq must be a contiguous 2-D int8 tensor")
    if Wq.shape[1] != K:
        raise ValueError("Xq and Wq disagree on K")
    _dev(Wq, "Wq", torch.int8, Xq.device)
    _cuda(Xq, "Xq")
    return M, Wq.shape[0], K


def cr_int8_gemm(Xq: torch.Tensor, a_scale: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor,
                 bias: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Y bf16 [M, N] = (Xq . Wq^T) * a_scale * w_scale[n] + bias[n] over INT8 codes."""
    M, N, K = _int8_operands(Xq, Wq)
    _scalar(a_scale, "a_scale", Xq.device)
    _vec(w_scale, "w_scale", torch.float32, Xq.device, N)
    _vec(bias, "bias", torch.bfloat16, Xq.device, N, optional=True)
    out, ldy = _out(out, M, N, torch.bfloat16, Xq.device)
    ws = workspace(Xq.device, _lib.cr_int8_gemm_workspace_size(M, N, K))
    _check("cr_int8_gemm", _lib.cr_int8_gemm(_ptr(Xq), _ptr(a_scale), _ptr(Wq), _ptr(w_scale), _ptr(bias),
                                             _ptr(out), ldy, M, N, K, _ptr(ws), ws.numel(), _stream(Xq.device)))
    return out


def cr_int8_gemm_s32(Xq: torch.Tensor, Wq: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Raw int32 product C [M, N] = sum_k qa[m, k] * qw[n, k] of INT8 codes."""
    M, N, K = _int8_operands(Xq, Wq)
    out, ldc = _out(out, M, N, torch.int32, Xq.device)
    ws = workspace(Xq.device, _lib.cr_int8_gemm_workspace_size(M, N, K))
    _check("cr_int8_gemm_s32", _lib.cr_int8_gemm_s32(_ptr(Xq), _ptr(Wq), _ptr(out), ldc, M, N, K, _ptr(ws),
                                                     ws.numel(), _stream(Xq.device)))
    return out


def cr_int8_linear(X: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor, bias: Optional[torch.Tensor] = None,
                   rotate: bool = True, out: Optional[torch.Tensor] = None, group: int = GROUP) -> torch.Tensor:
    """The whole INT8 layer in one call: (rotate +) quantise X to INT8, product, epilogue."""
    _bf16_cuda(X, "X")
    M, K, ldx = _rows(X, "X")
    if not isinstance(Wq, torch.Tensor) or Wq.dtype != torch.int8 or Wq.dim() != 2 or Wq.shape[1] != K:
        raise TypeError("Wq must be int8 [N, K] (cr_pack_weight_ex with bits=8)")
    N = Wq.shape[0]
    _dense(Wq, "Wq", torch.int8, X.device, (N, K))
    _vec(w_scale, "w_scale", torch.float32, X.device, N)
    _vec(bias, "bias", torch.bfloat16, X.device, N, optional=True)
    out, ldy = _out(out, M, N, torch.bfloat16, X.device)
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


def _w4a8_weights(Wq, gs, gz, K: int, device: torch.device) -> int:
    """W4A8 weights: codes uint8 [N, K/2], group scales float16 [N, K/16], zero points uint8 [N, K/32]."""
    if not isinstance(Wq, torch.Tensor) or Wq.dtype != torch.uint8 or Wq.dim() != 2 or Wq.shape[1] != K // 2 \
            or not Wq.is_contiguous():
        raise TypeError("Wq must be contiguous uint8 [N, K/2]")
    N = Wq.shape[0]
    if not isinstance(gs, torch.Tensor) or gs.dtype != torch.float16 or tuple(gs.shape) != (N, K // 16) \
            or not gs.is_contiguous():
        raise TypeError("gscale must be contiguous float16 [N, K/16]")
    if not isinstance(gz, torch.Tensor) or gz.dtype != torch.uint8 or tuple(gz.shape) != (N, K // 32) \
            or not gz.is_contiguous():
        raise TypeError("gzero must be contiguous uint8 [N, K/32]")
    for t, name, dt in ((Wq, "Wq", torch.uint8), (gs, "gscale", torch.float16), (gz, "gzero", torch.uint8)):
        _dev(t, name, dt, device)
    return N


def _w4a8_operands(Xq, Wq, gs, gz) -> Tuple[int, int, int]:
    M, K = _codes(Xq, "Xq", torch.int8)
    N = _w4a8_weights(Wq, gs, gz, K, Xq.device)
    _cuda(Xq, "Xq")
    return M, N, K


def cr_w4a8_gemm(Xq: torch.Tensor, a_scale: torch.Tensor, Wq: torch.Tensor, gscale: torch.Tensor,
                 gzero: torch.Tensor, bias: Optional[torch.Tensor] = None,
                 out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Y bf16 [M, N] = a_scale * sum_k Xq * s * (q - z) + bias."""
    M, N, K = _w4a8_operands(Xq, Wq, gscale, gzero)
    _scalar(a_scale, "a_scale", Xq.device)
    _vec(bias, "bias", torch.bfloat16, Xq.device, N, optional=True)
    out, ldy = _out(out, M, N, torch.bfloat16, Xq.device)
    ws = workspace(Xq.device, _lib.cr_w4a8_gemm_workspace_size(M, N, K))
    _check("cr_w4a8_gemm", _lib.cr_w4a8_gemm(_ptr(Xq), _ptr(a_scale), _ptr(Wq), _ptr(gscale), _ptr(gzero),
                                             _ptr(bias), _ptr(out), ldy, M, N, K, _ptr(ws), ws.numel(),
                                             _stream(Xq.device)))
    return out


def cr_w4a8_gemm_f32(Xq: torch.Tensor, Wq: torch.Tensor, gscale: torch.Tensor, gzero: torch.Tensor,
                     out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The float32 sums C [M, N] = sum_k Xq * fp16(s * (q - z)) (no activation scale, no bias)."""
    M, N, K = _w4a8_operands(Xq, Wq, gscale, gzero)
    out, ldc = _out(out, M, N, torch.float32, Xq.device)
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
    N = _w4a8_weights(Wq, gscale, gzero, K, X.device)
    _vec(bias, "bias", torch.bfloat16, X.device, N, optional=True)
    out, ldy = _out(out, M, N, torch.bfloat16, X.device)
    ws = workspace(X.device, _lib.cr_w4a8_linear_workspace_size(M, N, K, group))
    _check("cr_w4a8_linear", _lib.cr_w4a8_linear(_ptr(X), ldx, _ptr(Wq), _ptr(gscale), _ptr(gzero), _ptr(bias),
                                                 _ptr(out), ldy, M, N, K, group, _ptr(ws), ws.numel(),
                                                 _stream(X.device)))
    return out


# ---------------------------------------------------------------------------
# INT8 activation codes against the W4A4 format's packed INT4 weights ("INT8 branch")
# ---------------------------------------------------------------------------

def _a8w4_operands(Xq: torch.Tensor, Wq: torch.Tensor) -> Tuple[int, int, int]:
    M, K = _codes(Xq, "Xq", torch.int8)
    if not isinstance(Wq, torch.Tensor) or Wq.dtype != torch.uint8 or Wq.dim() != 2 or Wq.shape[1] * 2 != K \
            or not Wq.is_contiguous():
        raise TypeError("Wq must be contiguous uint8 [N, K/2] (packed INT4)")
    _dev(Wq, "Wq", torch.uint8, Xq.device)
    _cuda(Xq, "Xq")
    return M, Wq.shape[0], K


def cr_a8w4_gemm(Xq: torch.Tensor, a_scale: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor,
                 bias: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Y bf16 [M, N] = (Xq . Wq^T) * a_scale * w_scale[n] + bias[n], INT8 codes against packed INT4 weights."""
    M, N, K = _a8w4_operands(Xq, Wq)
    _scalar(a_scale, "a_scale", Xq.device)
    _vec(w_scale, "w_scale", torch.float32, Xq.device, N)
    _vec(bias, "bias", torch.bfloat16, Xq.device, N, optional=True)
    out, ldy = _out(out, M, N, torch.bfloat16, Xq.device)
    ws = workspace(Xq.device, _lib.cr_a8w4_gemm_workspace_size(M, N, K))
    _check("cr_a8w4_gemm", _lib.cr_a8w4_gemm(_ptr(Xq), _ptr(a_scale), _ptr(Wq), _ptr(w_scale), _ptr(bias),
                                             _ptr(out), ldy, M, N, K, _ptr(ws), ws.numel(), _stream(Xq.device)))
    return out


def cr_a8w4_gemm_s32(Xq: torch.Tensor, Wq: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Raw int32 product C [M, N] = sum_k qa[m, k] * qw[n, k] (INT8 codes, packed INT4 weights)."""
    M, N, K = _a8w4_operands(Xq, Wq)
    out, ldc = _out(out, M, N, torch.int32, Xq.device)
    ws = workspace(Xq.device, _lib.cr_a8w4_gemm_workspace_size(M, N, K))
    _check("cr_a8w4_gemm_s32", _lib.cr_a8w4_gemm_s32(_ptr(Xq), _ptr(Wq), _ptr(out), ldc, M, N, K, _ptr(ws),
                                                     ws.numel(), _stream(Xq.device)))
    return out


def cr_a8w4_linear(X: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor, bias: Optional[torch.Tensor] = None,
                   out: Optional[torch.Tensor] = None, group: int = GROUP) -> torch.Tensor:
    """The whole layer with INT8 activations against the packed INT4 weights of cr_pack_weight."""
    _bf16_cuda(X, "X")
    M, K, ldx = _rows(X, "X")
    N = _w4a4_weights(Wq, w_scale, bias, K, X.device)
    out, ldy = _out(out, M, N, torch.bfloat16, X.device)
    ws = workspace(X.device, _lib.cr_a8w4_linear_workspace_size(M, N, K, group))
    _check("cr_a8w4_linear", _lib.cr_a8w4_linear(_ptr(X), ldx, _ptr(Wq), _ptr(w_scale), _ptr(bias), _ptr(out), ldy,
                                                 M, N, K, group, _ptr(ws), ws.numel(), _stream(X.device)))
    return out


def cr_selftest_wait_timeout(ws: torch.Tensor) -> None:
    """Enqueue the bounded-wait self-test on ``ws`` (a zeroed uint8 CUDA workspace of >= 256 bytes)."""
    _check("cr_selftest_wait_timeout", _lib.cr_selftest_wait_timeout(_ptr(ws), ws.numel(), _stream(ws.device)))
