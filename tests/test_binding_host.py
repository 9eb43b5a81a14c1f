"""Argument checks of the Python binding that run before any CUDA call (CPU
only): wrong dtypes, devices, shapes and layouts raise instead of reaching
the library."""

import pytest
import torch

from w4a8_rotated_quantized_b200 import binding as b


def test_bf16_cuda_inputs_required():
    with pytest.raises(TypeError):
        b.cr_pack_weight(torch.zeros((8, 256), dtype=torch.float32))
    with pytest.raises(TypeError):
        b.cr_rotate_quant_act(torch.zeros((8, 256), dtype=torch.bfloat16))  # not on a CUDA device
    with pytest.raises(TypeError):
        b.cr_w4a8_linear(torch.zeros((8, 256), dtype=torch.float16), None, None, None)


def test_int8_operand_checks():
    xq = torch.zeros((4, 256), dtype=torch.int8)
    with pytest.raises(TypeError):
        b.cr_int8_gemm_s32(xq.to(torch.uint8), torch.zeros((8, 256), dtype=torch.int8))
    with pytest.raises(ValueError):
        b.cr_int8_gemm_s32(xq, torch.zeros((8, 512), dtype=torch.int8))  # K disagrees
    with pytest.raises(TypeError):
        b.cr_a8w4_gemm_s32(xq, torch.zeros((8, 256), dtype=torch.uint8))  # W must be packed [N, K/2]


def test_w4a8_operand_checks():
    xq = torch.zeros((4, 256), dtype=torch.int8)
    wq = torch.zeros((8, 128), dtype=torch.uint8)
    gs = torch.zeros((8, 16), dtype=torch.float16)
    gz = torch.zeros((8, 8), dtype=torch.uint8)
    with pytest.raises(TypeError):
        b.cr_w4a8_gemm_f32(xq, wq, gs.to(torch.float32), gz)
    with pytest.raises(TypeError):
        b.cr_w4a8_gemm_f32(xq, wq, gs, torch.zeros((8, 16), dtype=torch.uint8))  # zero points [N, K/32]
    with pytest.raises(TypeError):
        b.cr_w4a8_gemm_f32(xq, torch.zeros((8, 256), dtype=torch.uint8), gs, gz)


def test_code_width_must_be_4_or_8():
    with pytest.raises(ValueError):
        b._code_cols(256, 6)
    assert b._code_cols(256, 4) == 128 and b._code_cols(256, 8) == 256


def test_rows_helper_rejects_strided_last_dimension():
    t = torch.zeros((4, 8))
    with pytest.raises(ValueError):
        b._rows(t.t(), "t")
    assert b._rows(t[:, :4], "t") == (4, 4, 8)


def test_w4a4_wrappers_need_cuda_inputs():
    # the first operand decides the device; a host tensor is refused before any library call
    xq = torch.zeros((4, 128), dtype=torch.uint8)
    wq = torch.zeros((8, 128), dtype=torch.uint8)
    s = torch.ones((8,), dtype=torch.float32)
    with pytest.raises(TypeError):
        b.cr_w4a4_gemm(xq, torch.ones(1), wq, s)
    with pytest.raises(TypeError):
        b.cr_w4a4_gemm_s32(xq, wq)
    x = torch.zeros((4, 256), dtype=torch.bfloat16)
    for fn in (b.cr_w4a4_linear, b.cr_w4a4_linear_noalloc, b.cr_a8w4_linear):
        with pytest.raises(TypeError):
            fn(x, wq, s)


def test_w4a4_weight_operand_checks():
    cpu = torch.device("cpu")
    K, N = 256, 8
    wq = torch.zeros((N, K // 2), dtype=torch.uint8)
    s = torch.ones((N,), dtype=torch.float32)
    bias = torch.zeros((N,), dtype=torch.bfloat16)
    assert b._w4a4_weights(wq, s, bias, K, cpu) == N
    assert b._w4a4_weights(wq, s, None, K, cpu) == N
    with pytest.raises(ValueError):
        b._w4a4_weights(torch.zeros((N, K), dtype=torch.uint8), s, bias, K, cpu)  # not packed [N, K/2]
    with pytest.raises(TypeError):
        b._w4a4_weights(wq.to(torch.int8), s, bias, K, cpu)
    with pytest.raises(TypeError):
        b._w4a4_weights(wq, s.to(torch.float16), bias, K, cpu)  # w_scale must be float32
    with pytest.raises(ValueError):
        b._w4a4_weights(wq, torch.ones((N - 1,), dtype=torch.float32), bias, K, cpu)  # one scale per row
    with pytest.raises(ValueError):
        b._w4a4_weights(wq, s, torch.zeros((2 * N,), dtype=torch.bfloat16), K, cpu)  # bias length N
    with pytest.raises(TypeError):
        b._w4a4_weights(wq, s, bias.float(), K, cpu)
    with pytest.raises(ValueError):
        b._w4a4_weights(torch.zeros((N, K), dtype=torch.uint8)[:, ::2], s, bias, K, cpu)  # not contiguous
    # an operand on another device than the first input's
    with pytest.raises(TypeError):
        b._w4a4_weights(wq, s, bias, K, torch.device("meta"))


def test_output_checks():
    cpu = torch.device("cpu")
    y = torch.empty((4, 8), dtype=torch.bfloat16)
    assert b._out(y, 4, 8, torch.bfloat16, cpu)[1] == 8
    big = torch.empty((4, 16), dtype=torch.bfloat16)
    assert b._out(big[:, :8], 4, 8, torch.bfloat16, cpu)[1] == 16  # strided rows are fine
    with pytest.raises(ValueError):
        b._out(torch.empty((1, 8), dtype=torch.bfloat16), 4, 8, torch.bfloat16, cpu)  # too few rows
    with pytest.raises(ValueError):
        b._out(torch.empty((4, 4), dtype=torch.bfloat16), 4, 8, torch.bfloat16, cpu)
    with pytest.raises(TypeError):
        b._out(torch.empty((4, 8), dtype=torch.float32), 4, 8, torch.bfloat16, cpu)
    with pytest.raises(ValueError):
        b._out(torch.empty((8, 4), dtype=torch.bfloat16).t(), 4, 8, torch.bfloat16, cpu)  # columns strided
    with pytest.raises(TypeError):
        b._out(y, 4, 8, torch.bfloat16, torch.device("meta"))
    with pytest.raises(ValueError):
        b._scalar(torch.ones((0,), dtype=torch.float32), "a_scale", cpu)


def test_linear_mode_checked_before_anything_else():
    x = torch.zeros((4, 256), dtype=torch.bfloat16)
    wq = torch.zeros((8, 128), dtype=torch.uint8)
    s = torch.ones((8,), dtype=torch.float32)
    with pytest.raises(ValueError):
        b.cr_w4a4_linear(x, wq, s, mode=3)
