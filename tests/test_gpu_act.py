"""GPU parity of the activation path and the weight packer against the oracle."""

import numpy as np
import pytest
import torch

import oracle
from helpers import assert_codes_match, assert_scale_close
from w4a8_rotated_quantized_b200 import workloads

pytestmark = pytest.mark.gpu


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def cr():
    import w4a8_rotated_quantized_b200 as m

    return m


@pytest.mark.parametrize("name,M", [
    ("tiny", None), ("tiny", 1), ("tiny", 3), ("tiny", 129),
    ("text_enc_up_21", None), ("text_enc_up_130", None),      # every text-encoder shape
    ("text_enc_down_21", None), ("text_enc_down_130", None),
    ("dit_attn", None),          # full-size DiT attention input (4096 x 3072)
    ("dit_mlp_down", None),      # full-size post-GELU input (8192 x 12288), larger than L2
])
def test_act_codes_and_scale_match_oracle(name, M):
    d = workloads.make_inputs(name, M=M, with_weight=False)
    Xq, s = cr().cr_rotate_quant_act(dev_bf16(d["X"]))
    torch.cuda.synchronize()
    _, s_o, q_o, y_o = oracle.rotate_quant_act(d["X"])
    assert_scale_close(s.item(), s_o, d["X"])
    q_gpu = oracle.unpack_int4(Xq.cpu().numpy())
    assert_codes_match(q_gpu, q_o, y_o, s_o)


def test_act_strided_rows():
    d = workloads.make_inputs("tiny", with_weight=False)
    M, K = d["X"].shape
    big = np.zeros((M, K + 64), dtype=np.uint16)
    big[:, :K] = d["X"]
    Xbig = dev_bf16(big)
    Xq, s = cr().cr_rotate_quant_act(Xbig[:, :K])
    Xq2, s2 = cr().cr_rotate_quant_act(dev_bf16(d["X"]))
    assert torch.equal(Xq, Xq2) and torch.equal(s, s2)


def test_act_zero_and_empty():
    Xq, s = cr().cr_rotate_quant_act(torch.zeros((5, 512), dtype=torch.bfloat16, device="cuda"))
    assert s.item() == 1.0 and not Xq.any()
    Xq0, s0 = cr().cr_rotate_quant_act(torch.zeros((0, 512), dtype=torch.bfloat16, device="cuda"))
    assert Xq0.shape == (0, 256) and s0.item() == 1.0


def test_act_worked_example_bit_exact():
    # X = y H with y = (7, 2.5, 3.5, -2.5, 0.5, -0.5, 1.5, 0, ...): the rotation is exact
    # in float32 too, scale 1, codes by round-half-even.
    y = np.zeros((1, 512))
    y[0, :7] = [7.0, 2.5, 3.5, -2.5, 0.5, -0.5, 1.5]
    H = oracle.regular_hadamard(256)
    x = np.concatenate([y[:, :256] @ H, y[:, 256:] @ H], axis=1)
    Xq, s = cr().cr_rotate_quant_act(dev_bf16(workloads.bf16_bits_from_f32(x.astype(np.float32))))
    assert s.item() == 1.0
    assert [f"{b:02X}" for b in Xq.cpu().numpy()[0, :5]] == ["27", "E4", "00", "02", "00"]


@pytest.mark.parametrize("name,mode", [("tiny", "tensor"), ("tiny", "row"), ("text_enc_up_21", "tensor"),
                                       ("text_enc_down_21", "row"), ("dit_attn", "tensor")])
def test_pack_weight_matches_oracle(name, mode):
    d = workloads.make_inputs(name, M=1)
    Wq, s_w = cr().cr_pack_weight(dev_bf16(d["W"]), scale_mode=mode)
    torch.cuda.synchronize()
    _, s_o, q_o, y_o = oracle.pack_weight(d["W"], scale_mode=mode)
    s_g = s_w.cpu().numpy()
    step = max(1, len(s_g) // 64)
    for i in range(0, len(s_g), step):
        assert_scale_close(s_g[i], s_o[i], d["W"] if mode == "tensor" else d["W"][i:i + 1])
    if mode == "tensor":
        assert np.all(s_g == s_g[0])
    q_gpu = oracle.unpack_int4(Wq.cpu().numpy())
    assert_codes_match(q_gpu, q_o, y_o, s_o if mode == "row" else s_o[0])


@pytest.mark.parametrize("name,bits,group", [("tiny", 4, 256), ("text_enc_up_130", 4, 256), ("dit_attn", 4, 256),
                                             ("dit_attn", 8, 256), ("text_enc_down_21", 4, 64),
                                             ("dit_attn", 4, 1024)])
def test_act_fallback_kernels_match_the_one_launch_pass(name, bits, group):
    # the two streaming kernels (run when the cooperative launch is refused) give the same codes and scale
    import w4a8_rotated_quantized_b200 as cr
    from w4a8_rotated_quantized_b200 import workloads

    d = workloads.make_inputs(name, with_weight=False)
    X = torch.from_numpy(np.ascontiguousarray(d["X"]).view(np.int16)).cuda().view(torch.bfloat16)
    q1, s1 = cr.cr_rotate_quant_act_ex(X, bits=bits, group=group)
    q2, s2 = cr.cr_selftest_act_fallback(X, bits=bits, group=group)
    torch.cuda.synchronize()
    assert cr.cr_read_device_status() == 0
    assert torch.equal(s1, s2) and torch.equal(q1, q2)


# Shapes that exercise the one-launch pass's tiling (units numbered row by row, tiles of 8, rounds of 16
# tiles per CTA, the last two rounds kept in TMEM and the one before in shared memory) against the oracle
# and, bit for bit, against the fallback kernels.
@pytest.mark.parametrize("M,K,ldx_pad", [
    (1, 256, 0),      # one unit: one tile, one CTA
    (3, 768, 0),      # 9 units: a full tile and one with a single unit
    (37, 1280, 64),   # ragged last tile, strided rows
    (2368, 2048, 0),  # exactly one full round on each of 148 CTAs
    (2369, 2048, 0),  # one tile more: a second round on one CTA
    (9000, 1024, 0),  # two rounds per CTA: both kept in TMEM
    (4736, 2560, 0),  # three rounds: two in TMEM, one in shared memory
    (16576, 1024, 0), # four rounds: one rotated again in the second pass
])
def test_act_tiling_edge_shapes(M, K, ldx_pad):
    rng = np.random.default_rng(M * 7 + K)
    x = (rng.standard_normal((M, K)) * 0.7).astype(np.float32)
    bits = workloads.bf16_bits_from_f32(x)
    if ldx_pad:
        big = np.zeros((M, K + ldx_pad), dtype=np.uint16)
        big[:, :K] = bits
        X = dev_bf16(big)[:, :K]
    else:
        X = dev_bf16(bits)
    Xq, s = cr().cr_rotate_quant_act(X)
    Xq_f, s_f = cr().cr_selftest_act_fallback(X)
    torch.cuda.synchronize()
    assert cr().cr_read_device_status() == 0
    assert torch.equal(s, s_f) and torch.equal(Xq, Xq_f)
    _, s_o, q_o, y_o = oracle.rotate_quant_act(bits)
    assert_scale_close(s.item(), s_o, bits)
    assert_codes_match(oracle.unpack_int4(Xq.cpu().numpy()), q_o, y_o, s_o)


@pytest.mark.parametrize("M,K,bits,group", [(37, 1280, 8, 256), (37, 1280, 4, 64), (37, 1280, 8, 16),
                                            (3, 1024, 4, 1024), (37, 2048, 8, 1024), (4736, 2560, 8, 256)])
def test_act_formats_and_groups_on_edge_shapes(M, K, bits, group):
    # other code widths and rotation groups through the same tiling: the one-launch pass equals the fallback
    # kernels bit for bit (the format and group paths are checked against the oracle elsewhere)
    rng = np.random.default_rng(M + K + bits + group)
    X = dev_bf16(workloads.bf16_bits_from_f32((rng.standard_normal((M, K)) * 0.7).astype(np.float32)))
    q1, s1 = cr().cr_rotate_quant_act_ex(X, bits=bits, group=group)
    q2, s2 = cr().cr_selftest_act_fallback(X, bits=bits, group=group)
    torch.cuda.synchronize()
    assert cr().cr_read_device_status() == 0
    assert torch.equal(s1, s2) and torch.equal(q1, q2)
