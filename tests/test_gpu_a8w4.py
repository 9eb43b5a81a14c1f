"""GPU parity of the INT8 branch of the W4A4 format: INT8 activation codes
(after the rotation) against the format's packed INT4 weights on the kind::i8
tensor cores.  int32 accumulators bit-exact against the oracle's integer
product of the GPU's own codes, bf16 outputs within one ulp of the oracle's
epilogue on those accumulators."""

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


def run_a8w4(d, scale_mode="tensor", with_bias=True):
    X, W = dev_bf16(d["X"]), dev_bf16(d["W"])
    bias = dev_bf16(d["bias"]) if with_bias else None
    Wq, s_w = cr().cr_pack_weight(W, scale_mode=scale_mode)
    Xq, s_a = cr().cr_rotate_quant_act_ex(X, bits=8, rotate=True)
    acc = cr().cr_a8w4_gemm_s32(Xq, Wq)
    Y = cr().cr_a8w4_gemm(Xq, s_a, Wq, s_w, bias)
    Y1 = cr().cr_a8w4_linear(X, Wq, s_w, bias)
    torch.cuda.synchronize()
    assert cr().cr_read_device_status() == 0
    assert torch.equal(Y, Y1), "the one-call layer differs from the separate calls"
    return dict(Xq=Xq.cpu().numpy(), s_a=np.float32(s_a.item()), Wq=Wq.cpu().numpy(), s_w=s_w.cpu().numpy(),
                acc=acc.cpu().numpy(), Y=host_bits(Y), bias=d["bias"] if with_bias else None,
                dev=(Xq, Wq))


def check(r, rows=None, cols=None):
    qa = r["Xq"] if rows is None else r["Xq"][rows]
    qw = oracle.unpack_int4(r["Wq"] if cols is None else r["Wq"][cols])
    acc_o = oracle.int_gemm(qa, qw)
    acc_g = r["acc"] if rows is None else r["acc"][np.ix_(rows, cols)]
    y_g = r["Y"] if rows is None else r["Y"][np.ix_(rows, cols)]
    assert np.array_equal(acc_g, acc_o), f"accumulators differ at {np.argwhere(acc_g != acc_o)[:5].tolist()}"
    s_w = r["s_w"] if cols is None else r["s_w"][cols]
    bias = None if r["bias"] is None else (r["bias"] if cols is None else r["bias"][cols])
    assert_bf16_within_1ulp(y_g, oracle.epilogue(acc_o, r["s_a"], s_w, bias))


@pytest.mark.parametrize("name,M", [("tiny", None), ("tiny", 1), ("tiny", 255), ("tiny", 257),
                                    ("text_enc_up_21", None), ("text_enc_down_130", None)])
def test_a8w4_full_compare(name, M):
    check(run_a8w4(workloads.make_inputs(name, M=M)))


def test_a8w4_layer_end_to_end_against_oracle():
    d = workloads.make_inputs("tiny")
    r = run_a8w4(d)
    wq, s_w, _, _ = oracle.pack_weight(d["W"])
    want = oracle.a8w4_linear(d["X"], wq, s_w, d["bias"])
    assert_scale_close(r["s_a"], want["s_a"], d["X"], qpos=127.0)
    assert_codes_match(r["Xq"], want["qa"], oracle.rotate(oracle.bf16_bits_to_f64(d["X"])), want["s_a"])
    same = np.all(r["Xq"] == want["qa"], axis=1) & (r["s_a"] == want["s_a"])
    if np.array_equal(r["Wq"], wq) and same.any():
        assert_bf16_within_1ulp(r["Y"][same], want["Y"][same])


def test_a8w4_ragged_row_scales_no_bias():
    rng = np.random.default_rng(43)
    M, N, K = 300, 392, 768
    d = {"X": workloads.bf16_bits_from_f32(rng.standard_normal((M, K)).astype(np.float32)),
         "W": workloads.bf16_bits_from_f32((rng.standard_normal((N, K)) * 0.02).astype(np.float32)),
         "bias": None}
    check(run_a8w4(d, scale_mode="row", with_bias=False))


def test_a8w4_minimum_sizes():
    rng = np.random.default_rng(47)
    M, N, K = 1, 8, 256
    d = {"X": workloads.bf16_bits_from_f32(rng.standard_normal((M, K)).astype(np.float32)),
         "W": workloads.bf16_bits_from_f32(rng.standard_normal((N, K)).astype(np.float32)),
         "bias": workloads.bf16_bits_from_f32(rng.standard_normal(N).astype(np.float32))}
    check(run_a8w4(d))


def test_a8w4_extreme_codes_exact():
    # K = 65536 with activation codes -128 and weights -8 / 7: |acc| up to 2^26
    K, M, N = 65536, 300, 16
    xq = np.full((M, K), -128, np.int8)
    wq = np.full((N, K // 2), 0x77, np.uint8)  # every code 7
    wq[1::2] = 0x88                            # every code -8
    acc = cr().cr_a8w4_gemm_s32(torch.from_numpy(xq).cuda(), torch.from_numpy(wq).cuda()).cpu().numpy()
    want = np.where(np.arange(N) % 2 == 0, -128 * 7 * K, 128 * 8 * K)
    assert np.array_equal(acc, np.broadcast_to(want, (M, N)))


def test_a8w4_full_size_matches_library_int_mm():
    # DiT MLP up shape: accumulators against torch._int_mm on the unpacked weight codes, repeated
    d = workloads.make_inputs("dit_mlp_up")
    r = run_a8w4(d)
    Xq, Wq = r["dev"]
    qw = torch.from_numpy(oracle.unpack_int4(r["Wq"])).cuda()
    ref = torch._int_mm(Xq, qw.t())
    assert np.array_equal(r["acc"], ref.cpu().numpy())
    for _ in range(4):
        assert torch.equal(cr().cr_a8w4_gemm_s32(Xq, Wq), ref)
    rng = np.random.default_rng(4)
    M, N = r["acc"].shape
    check(r, np.sort(rng.choice(M, 192, replace=False)), np.sort(rng.choice(N, 192, replace=False)))


def test_a8w4_strided_output_rows_and_zero_activation():
    d = workloads.make_inputs("tiny")
    M, N = d["X"].shape[0], d["W"].shape[0]
    Wq, s_w = cr().cr_pack_weight(dev_bf16(d["W"]))
    Xq, s_a = cr().cr_rotate_quant_act_ex(dev_bf16(d["X"]), bits=8)
    b = dev_bf16(d["bias"])
    Y = cr().cr_a8w4_gemm(Xq, s_a, Wq, s_w, b)
    Ybig = torch.zeros((M, N + 8), dtype=torch.bfloat16, device="cuda")
    cr().cr_a8w4_gemm(Xq, s_a, Wq, s_w, b, out=Ybig[:, :N])
    Xz, sz = cr().cr_rotate_quant_act_ex(torch.zeros((M, 512), dtype=torch.bfloat16, device="cuda"), bits=8)
    Yz = cr().cr_a8w4_gemm(Xz, sz, Wq, s_w, b)
    torch.cuda.synchronize()
    assert torch.equal(Ybig[:, :N], Y) and not Ybig[:, N:].any()
    assert np.array_equal(host_bits(Yz), np.broadcast_to(d["bias"], (M, N)))
