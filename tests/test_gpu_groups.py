"""GPU parity of the rotation with groups of 16, 64 and 1024 (the W4A4 format accepts
16 / 64 / 1024 besides 256: "Qwen-Image-Edit-2511 — W4A8 ConvRot", notes on
convrot_groupsize).  Codes and scales against the oracle's rotation with the
same group (near-tie tolerance as for 256, with the float32 error bound of the
shorter transform), integer products bit-exact, one-call layers equal to the
separate calls."""

import numpy as np
import pytest
import torch

import oracle
from helpers import assert_bf16_within_1ulp, assert_codes_match, assert_scale_close
from w4a8_rotated_quantized_b200 import workloads

pytestmark = pytest.mark.gpu


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def host_bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def cr():
    import w4a8_rotated_quantized_b200 as m

    return m


# tiny, text_enc_down_130 and dit_attn: the fused pass; dit_mlp_down (8192 x 12288): the two streaming passes
@pytest.mark.parametrize("group", [16, 64])
@pytest.mark.parametrize("name", ["tiny", "text_enc_down_130", "dit_attn", "dit_mlp_down"])
def test_act4_groups_match_oracle(name, group):
    d = workloads.make_inputs(name, with_weight=False)
    Xq, s = cr().cr_rotate_quant_act(dev_bf16(d["X"]), group=group)
    torch.cuda.synchronize()
    _, s_o, q_o, y_o = oracle.rotate_quant_act(d["X"], group)
    assert_scale_close(s.item(), s_o, d["X"], group=group)
    assert_codes_match(oracle.unpack_int4(Xq.cpu().numpy()), q_o, y_o, s_o)


@pytest.mark.parametrize("group", [16, 64])
def test_act8_groups_match_oracle(group):
    d = workloads.make_inputs("text_enc_up_130", with_weight=False)
    Xq, s = cr().cr_rotate_quant_act_ex(dev_bf16(d["X"]), bits=8, rotate=True, group=group)
    torch.cuda.synchronize()
    q_o, s_o, y_o = oracle.quant_act8(d["X"], True, group)
    assert_scale_close(s.item(), s_o, d["X"], qpos=127.0, group=group)
    assert_codes_match(Xq.cpu().numpy(), q_o, y_o, s_o)


@pytest.mark.parametrize("group,mode", [(16, "tensor"), (64, "row")])
def test_pack_weight_groups_match_oracle(group, mode):
    d = workloads.make_inputs("text_enc_down_21", M=1)
    Wq, s_w = cr().cr_pack_weight(dev_bf16(d["W"]), group=group, scale_mode=mode)
    torch.cuda.synchronize()
    _, s_o, q_o, y_o = oracle.pack_weight(d["W"], group, mode)
    s_g = s_w.cpu().numpy()
    for i in range(0, len(s_g), 97):
        assert_scale_close(s_g[i], s_o[i], d["W"] if mode == "tensor" else d["W"][i:i + 1], group=group)
    assert_codes_match(oracle.unpack_int4(Wq.cpu().numpy()), q_o, y_o, s_o if mode == "row" else s_o[0])


def test_group16_worked_example_bit_exact():
    y = np.zeros((1, 256))
    y[0, :4] = [7.0, 2.5, -3.5, 0.5]
    H16 = oracle.regular_hadamard(16)
    x = np.concatenate([y[:, i * 16:(i + 1) * 16] @ H16 for i in range(16)], axis=1)
    Xq, s = cr().cr_rotate_quant_act(dev_bf16(workloads.bf16_bits_from_f32(x.astype(np.float32))), group=16)
    assert s.item() == 1.0
    q = oracle.unpack_int4(Xq.cpu().numpy())
    assert q[0, :4].tolist() == [7, 2, -4, 0] and not q[0, 4:].any()


@pytest.mark.parametrize("group", [16, 64])
def test_layer_with_group_matches_oracle(group):
    d = workloads.make_inputs("tiny")
    X, W, b = dev_bf16(d["X"]), dev_bf16(d["W"]), dev_bf16(d["bias"])
    Wq, s_w = cr().cr_pack_weight(W, group=group)
    Xq, s_a = cr().cr_rotate_quant_act(X, group=group)
    acc = cr().cr_w4a4_gemm_s32(Xq, Wq)
    Y = cr().cr_w4a4_gemm(Xq, s_a, Wq, s_w, b)
    Y1 = cr().cr_w4a4_linear(X, Wq, s_w, b, group=group)
    Y2 = cr().cr_w4a4_linear_noalloc(X, Wq, s_w, b, group=group)
    torch.cuda.synchronize()
    assert cr().cr_read_device_status() == 0
    assert torch.equal(Y, Y1) and torch.equal(Y, Y2)
    qa = oracle.unpack_int4(Xq.cpu().numpy())
    qw = oracle.unpack_int4(Wq.cpu().numpy())
    acc_o = oracle.int_gemm(qa, qw)
    assert np.array_equal(acc.cpu().numpy(), acc_o)
    assert_bf16_within_1ulp(host_bits(Y), oracle.epilogue(acc_o, np.float32(s_a.item()), s_w.cpu().numpy(), d["bias"]))
    # the INT8 branch and the INT8 layer take the group too
    Y8 = cr().cr_a8w4_linear(X, Wq, s_w, b, group=group)
    Xq8, s8 = cr().cr_rotate_quant_act_ex(X, bits=8, rotate=True, group=group)
    assert torch.equal(Y8, cr().cr_a8w4_gemm(Xq8, s8, Wq, s_w, b))


def test_w4a8_rejects_other_groups():
    W = torch.zeros((8, 256), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(cr().ConvRotError):
        cr().cr_pack_weight_w4a8(W, group=64)


# groups of 1024 combine four consecutive 256-element units across lanes; K must be a multiple of 1024
@pytest.mark.parametrize("name,M", [("dit_attn", None), ("dit_attn", 3), ("dit_mlp_down", None)])
def test_act4_group1024_matches_oracle(name, M):
    d = workloads.make_inputs(name, M=M, with_weight=False)
    Xq, s = cr().cr_rotate_quant_act(dev_bf16(d["X"]), group=1024)
    torch.cuda.synchronize()
    _, s_o, q_o, y_o = oracle.rotate_quant_act(d["X"], 1024)
    assert_scale_close(s.item(), s_o, d["X"], group=1024)
    assert_codes_match(oracle.unpack_int4(Xq.cpu().numpy()), q_o, y_o, s_o)


def test_group1024_worked_example_bit_exact():
    y = np.zeros((2, 2048))
    y[0, [0, 300, 700, 1023]] = [7.0, -2.5, 1.5, 3.5]
    y[1, [1024, 1500]] = [-6.5, 0.5]
    H = oracle.regular_hadamard(1024)
    x = np.concatenate([y[:, :1024] @ H, y[:, 1024:] @ H], axis=1)
    Xq, s = cr().cr_rotate_quant_act(dev_bf16(workloads.bf16_bits_from_f32(x.astype(np.float32))), group=1024)
    assert s.item() == 1.0
    q = oracle.unpack_int4(Xq.cpu().numpy())
    want = np.zeros((2, 2048), np.int8)
    want[0, [0, 300, 700, 1023]] = [7, -2, 2, 4]
    want[1, [1024, 1500]] = [-6, 0]
    assert np.array_equal(q, want)


@pytest.mark.parametrize("mode", ["tensor", "row"])
def test_layer_group1024(mode):
    rng = np.random.default_rng(53)
    M, N, K = 200, 264, 2048
    d = {"X": workloads.bf16_bits_from_f32(rng.standard_normal((M, K)).astype(np.float32)),
         "W": workloads.bf16_bits_from_f32((rng.standard_normal((N, K)) * 0.02).astype(np.float32))}
    X, W = dev_bf16(d["X"]), dev_bf16(d["W"])
    Wq, s_w = cr().cr_pack_weight(W, group=1024, scale_mode=mode)
    Xq, s_a = cr().cr_rotate_quant_act(X, group=1024)
    Y = cr().cr_w4a4_gemm(Xq, s_a, Wq, s_w, None)
    Y1 = cr().cr_w4a4_linear(X, Wq, s_w, None, group=1024)
    Xq8, s8 = cr().cr_rotate_quant_act_ex(X, bits=8, rotate=True, group=1024)
    torch.cuda.synchronize()
    assert cr().cr_read_device_status() == 0
    assert torch.equal(Y, Y1)
    _, s_o, q_o, y_o = oracle.pack_weight(d["W"], 1024, mode)
    assert_codes_match(oracle.unpack_int4(Wq.cpu().numpy()), q_o, y_o, s_o if mode == "row" else s_o[0])
    q8_o, s8_o, y8_o = oracle.quant_act8(d["X"], True, 1024)
    assert_codes_match(Xq8.cpu().numpy(), q8_o, y8_o, s8_o)
    qa = oracle.unpack_int4(Xq.cpu().numpy())
    acc_o = oracle.int_gemm(qa, oracle.unpack_int4(Wq.cpu().numpy()))
    assert_bf16_within_1ulp(host_bits(Y), oracle.epilogue(acc_o, np.float32(s_a.item()), s_w.cpu().numpy(), None))
