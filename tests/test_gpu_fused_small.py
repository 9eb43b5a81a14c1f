"""The one-launch layer for few tokens: cr_w4a4_linear in mode LINEAR_ONE_LAUNCH
(M <= 256) rotates and quantises X inside the few-token GEMM (two bounded grid barriers between the
activation phases and the weight stream).  Its codes and scale are those of
cr_rotate_quant_act bit for bit (same lane mapping, transform, division and
max), so its output must equal cr_rotate_quant_act + cr_w4a4_gemm bit for bit,
and match the oracle like every other path (codes near-ties only, outputs
within one bf16 ulp of the oracle's epilogue on the GPU's codes)."""

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


def check_layer(X_bits, W_bits, bias_bits, group=256, scale_mode="tensor"):
    X, W = dev_bf16(X_bits), dev_bf16(W_bits)
    b = None if bias_bits is None else dev_bf16(bias_bits)
    Wq, s_w = cr().cr_pack_weight(W, group=group, scale_mode=scale_mode)
    Y1 = cr().cr_w4a4_linear(X, Wq, s_w, b, group=group, mode=cr().LINEAR_ONE_LAUNCH)  # one launch
    Xq, s_a = cr().cr_rotate_quant_act(X, group=group)               # two launches
    Y2 = cr().cr_w4a4_gemm(Xq, s_a, Wq, s_w, b)
    torch.cuda.synchronize()
    assert cr().cr_read_device_status() == 0
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16)), "fused layer vs separate calls"
    # the library's own choice and the forced two-launch arrangement give the same bits
    for mode in (cr().LINEAR_AUTO, cr().LINEAR_TWO_LAUNCHES):
        Ym = cr().cr_w4a4_linear(X, Wq, s_w, b, group=group, mode=mode)
        assert torch.equal(Ym.view(torch.int16), Y2.view(torch.int16)), f"mode {mode}"
    # oracle: scale within the float32 rotation bound, codes up to near-ties, outputs to one ulp
    _, s_o, q_o, y_o = oracle.rotate_quant_act(X_bits, group)
    assert_scale_close(s_a.item(), s_o, X_bits, group=group)
    q_g = oracle.unpack_int4(Xq.cpu().numpy())
    s_g = np.float32(s_a.item())
    assert_codes_match(q_g, oracle.quantize(y_o, s_g), y_o, s_g)
    acc = oracle.int_gemm(q_g, oracle.unpack_int4(Wq.cpu().numpy()))
    assert_bf16_within_1ulp(host_bits(Y1), oracle.epilogue(acc, s_g, s_w.cpu().numpy(), bias_bits))
    return Y1


@pytest.mark.parametrize("name", ["text_enc_up_21", "text_enc_down_21"])
def test_fused_text_encoder_layers(name):
    d = workloads.make_inputs(name)
    check_layer(d["X"], d["W"], d["bias"])


@pytest.mark.parametrize("M", [1, 2, 17, 64, 100, 127, 128, 129, 200, 256])
def test_fused_token_counts(M):
    # one token up to the largest few-token count (the padded token count is 16 .. 256; above 128
    # tokens the one-CTA-per-SM configuration with a 256-column accumulator)
    d = workloads.make_inputs("text_enc_up_21", M=M)
    check_layer(d["X"], d["W"][:1024], d["bias"][:1024])


@pytest.mark.parametrize("name", ["text_enc_up_130", "text_enc_down_130"])
def test_fused_text_encoder_layers_130_tokens(name):
    d = workloads.make_inputs(name)
    check_layer(d["X"], d["W"], d["bias"])


@pytest.mark.parametrize("group", [16, 64])
def test_fused_groups(group):
    d = workloads.make_inputs("text_enc_down_21")
    check_layer(d["X"], d["W"], d["bias"], group=group)


def test_fused_ragged_n_row_scales_no_bias():
    rng = np.random.default_rng(3)
    M, N, K = 37, 264, 1280  # N: two weight tiles, the second ragged; K: 5 units per row
    X = workloads.bf16_bits_from_f32(rng.standard_normal((M, K)).astype(np.float32))
    W = workloads.bf16_bits_from_f32((rng.standard_normal((N, K)) * 0.02).astype(np.float32))
    check_layer(X, W, None, scale_mode="row")


def test_fused_zero_input_gives_bias():
    d = workloads.make_inputs("tiny")
    X = torch.zeros((9, 512), dtype=torch.bfloat16, device="cuda")
    Wq, s_w = cr().cr_pack_weight(dev_bf16(d["W"]))
    b = dev_bf16(d["bias"])
    Y = cr().cr_w4a4_linear(X, Wq, s_w, b, mode=cr().LINEAR_ONE_LAUNCH)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(Y), np.broadcast_to(d["bias"], (9, 256)))


def test_fused_repeated_launches_identical():
    # the grid barriers' words are reused by every launch; run many in a row on changing inputs
    d = workloads.make_inputs("text_enc_down_21")
    Wq, s_w = cr().cr_pack_weight(dev_bf16(d["W"]))
    b = dev_bf16(d["bias"])
    Xs = [dev_bf16(workloads.make_inputs("text_enc_down_21", with_weight=False, seed=50 + i)["X"]) for i in range(3)]
    refs = []
    for X in Xs:
        Xq, s_a = cr().cr_rotate_quant_act(X)
        refs.append(cr().cr_w4a4_gemm(Xq, s_a, Wq, s_w, b))
    for it in range(20):
        j = it % 3
        Y = cr().cr_w4a4_linear(Xs[j], Wq, s_w, b, mode=cr().LINEAR_ONE_LAUNCH)
        torch.cuda.synchronize()
        assert torch.equal(Y.view(torch.int16), refs[j].view(torch.int16)), f"launch {it}"
    assert cr().cr_read_device_status() == 0


def test_one_launch_refused_above_256_tokens():
    # more tokens than the few-token kernel holds: the forced one-launch mode is refused, nothing runs
    d = workloads.make_inputs("tiny", M=300)
    X = dev_bf16(d["X"])
    Wq, s_w = cr().cr_pack_weight(dev_bf16(d["W"]))
    with pytest.raises(cr().ConvRotError) as e:
        cr().cr_w4a4_linear(X, Wq, s_w, mode=cr().LINEAR_ONE_LAUNCH)
    assert e.value.status == 2  # CR_ERR_UNSUPPORTED_SHAPE
