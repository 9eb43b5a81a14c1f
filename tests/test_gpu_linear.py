"""The one-call layer (cr_w4a4_linear) against the separate calls and the oracle end to end."""

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


# every text-encoder shape (21 and 130 tokens, both directions), the tiny case and the DiT attention
# projection; M <= 128 runs the few-token GEMM, M = 130 the CTA-pair kernel with one ragged M tile
@pytest.mark.parametrize("name", ["tiny", "text_enc_up_21", "text_enc_up_130", "text_enc_down_21",
                                  "text_enc_down_130", "dit_attn"])
def test_linear_equals_separate_calls_and_oracle(name):
    import w4a8_rotated_quantized_b200 as cr

    d = workloads.make_inputs(name)
    X, W, bias = dev_bf16(d["X"]), dev_bf16(d["W"]), dev_bf16(d["bias"])
    Wq, s_w = cr.cr_pack_weight(W)
    Y1 = cr.cr_w4a4_linear(X, Wq, s_w, bias)
    Xq, s_a = cr.cr_rotate_quant_act(X)
    Y2 = cr.cr_w4a4_gemm(Xq, s_a, Wq, s_w, bias)
    torch.cuda.synchronize()
    assert cr.cr_read_device_status() == 0
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))

    wq, sw = Wq.cpu().numpy(), s_w.cpu().numpy()
    qw = oracle.unpack_int4(wq)
    q_g = oracle.unpack_int4(Xq.cpu().numpy())
    s_g = np.float32(s_a.item())
    yg = host_bits(Y1)
    _, s_o, q_o, y_o = oracle.rotate_quant_act(d["X"])
    assert_scale_close(s_g, s_o, d["X"])

    # (1) the oracle's layer from the oracle's own rotated values, quantised with the scale the GPU
    #     found (equal to the oracle's, or within the float32 rotation bound of it): codes may differ
    #     only at near-ties, and every row without a flipped code matches the oracle output to 1 ulp
    q_ref = oracle.quantize(y_o, s_g)
    assert_codes_match(q_g, q_ref, y_o, s_g)
    clean = ~np.any(q_g != q_ref, axis=1)
    assert clean.sum() >= 1
    y_ref = oracle.epilogue(oracle.int_gemm(q_ref[clean], qw), s_g, sw, d["bias"])
    assert_bf16_within_1ulp(yg[clean], y_ref, f"{name}: rows with no flipped code")

    # (2) every row: the oracle's product and epilogue on the GPU's codes and scale
    assert_bf16_within_1ulp(yg, oracle.epilogue(oracle.int_gemm(q_g, qw), s_g, sw, d["bias"]), f"{name}: all rows")

    # (3) where the scales agree bit for bit, the oracle's own end-to-end layer, no GPU value fed back
    if s_g == s_o:
        out = oracle.w4a4_linear(d["X"], wq, sw, d["bias"])
        clean_o = ~np.any(q_g != out["qa"], axis=1)
        assert_bf16_within_1ulp(yg[clean_o], out["Y"][clean_o], f"{name}: oracle layer")
