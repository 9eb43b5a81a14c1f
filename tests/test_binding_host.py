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
