"""GPU parity of the INT8 tensorwise format, with and without the ConvRot
rotation: activation and weight codes against the oracle's INT8 functions,
int32 accumulators bit-exact against the oracle's integer product of the GPU's
own codes, bf16 outputs within one ulp of the oracle's epilogue.

Without the rotation the values are the bf16 inputs themselves (exact in
float32), so the scale and every code must match the oracle bit for bit."""

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


def check_codes(q_gpu, s_gpu, q_o, s_o, y_o, x_bits, rotate):
    if rotate:
        assert_scale_close(s_gpu, s_o, x_bits, qpos=127.0)
        assert_codes_match(q_gpu, q_o, y_o, s_o)
    else:
        assert np.float32(s_gpu) == np.float32(s_o)
        assert np.array_equal(q_gpu, q_o)


# tiny and text_enc shapes: the fused single pass; dit_mlp_down (8192 x 12288) the two streaming passes
@pytest.mark.parametrize("rotate", [True, False])
@pytest.mark.parametrize("name,M", [("tiny", None), ("tiny", 1), ("tiny", 129), ("text_enc_down_130", None),
                                    ("dit_attn", None), ("dit_mlp_down", None)])
def test_act8_codes_and_scale_match_oracle(name, M, rotate):
    d = workloads.make_inputs(name, M=M, with_weight=False)
    Xq, s = cr().cr_rotate_quant_act_ex(dev_bf16(d["X"]), bits=8, rotate=rotate)
    torch.cuda.synchronize()
    q_o, s_o, y_o = oracle.quant_act8(d["X"], rotate_groups=rotate)
    check_codes(Xq.cpu().numpy(), s.item(), q_o, s_o, y_o, d["X"], rotate)


@pytest.mark.parametrize("rotate", [True, False])
def test_act4_without_rotation_is_exact(rotate):
    # bits 4 through the any-format call: with rotation it equals the INT4 call; without, the plain
    # tensorwise INT4 codes of X (scale amax / 7) are exact
    d = workloads.make_inputs("tiny", with_weight=False)
    Xq, s = cr().cr_rotate_quant_act_ex(dev_bf16(d["X"]), bits=4, rotate=rotate)
    if rotate:
        Xq1, s1 = cr().cr_rotate_quant_act(dev_bf16(d["X"]))
        assert torch.equal(Xq, Xq1) and torch.equal(s, s1)
    else:
        y = oracle.bf16_bits_to_f64(d["X"])
        s_o = oracle.tensor_scale(y)
        assert np.float32(s.item()) == s_o
        assert np.array_equal(oracle.unpack_int4(Xq.cpu().numpy()), oracle.quantize(y, s_o))


@pytest.mark.parametrize("rotate", [True, False])
@pytest.mark.parametrize("name,mode", [("tiny", "tensor"), ("tiny", "row"), ("text_enc_down_21", "row"),
                                       ("dit_attn", "tensor")])
def test_pack_weight8_matches_oracle(name, mode, rotate):
    d = workloads.make_inputs(name, M=1)
    Wq, s_w = cr().cr_pack_weight_ex(dev_bf16(d["W"]), bits=8, rotate=rotate, scale_mode=mode)
    torch.cuda.synchronize()
    q_o, s_o, y_o = oracle.pack_weight8(d["W"], rotate_groups=rotate, scale_mode=mode)
    s_g = s_w.cpu().numpy()
    q_g = Wq.cpu().numpy()
    if mode == "tensor":
        assert np.all(s_g == s_g[0])
        check_codes(q_g, s_g[0], q_o, s_o[0], y_o, d["W"], rotate)
    elif not rotate:
        assert np.array_equal(s_g, s_o) and np.array_equal(q_g, q_o)
    else:
        step = max(1, len(s_g) // 64)
        for i in range(0, len(s_g), step):
            assert_scale_close(s_g[i], s_o[i], d["W"][i:i + 1], qpos=127.0)
        assert_codes_match(q_g, q_o, y_o, s_o)


def run_layer8(d, rotate=True, scale_mode="tensor", with_bias=True):
    X, W = dev_bf16(d["X"]), dev_bf16(d["W"])
    bias = dev_bf16(d["bias"]) if with_bias else None
    Wq, s_w = cr().cr_pack_weight_ex(W, bits=8, rotate=rotate, scale_mode=scale_mode)
    Xq, s_a = cr().cr_rotate_quant_act_ex(X, bits=8, rotate=rotate)
    acc = cr().cr_int8_gemm_s32(Xq, Wq)
    Y = cr().cr_int8_gemm(Xq, s_a, Wq, s_w, bias)
    Y1 = cr().cr_int8_linear(X, Wq, s_w, bias, rotate=rotate)
    torch.cuda.synchronize()
    assert cr().cr_read_device_status() == 0
    assert torch.equal(Y, Y1), "the one-call layer differs from the separate calls"
    return dict(Xq=Xq.cpu().numpy(), s_a=np.float32(s_a.item()), Wq=Wq.cpu().numpy(), s_w=s_w.cpu().numpy(),
                acc=acc.cpu().numpy(), Y=host_bits(Y), bias=d["bias"] if with_bias else None)


def check8(r, rows=None, cols=None):
    qa = r["Xq"] if rows is None else r["Xq"][rows]
    qw = r["Wq"] if cols is None else r["Wq"][cols]
    acc_o = oracle.int_gemm(qa, qw)
    acc_g = r["acc"] if rows is None else r["acc"][np.ix_(rows, cols)]
    y_g = r["Y"] if rows is None else r["Y"][np.ix_(rows, cols)]
    assert np.array_equal(acc_g, acc_o), f"accumulators differ at {np.argwhere(acc_g != acc_o)[:5].tolist()}"
    s_w = r["s_w"] if cols is None else r["s_w"][cols]
    bias = None if r["bias"] is None else (r["bias"] if cols is None else r["bias"][cols])
    assert_bf16_within_1ulp(y_g, oracle.epilogue(acc_o, r["s_a"], s_w, bias))


@pytest.mark.parametrize("rotate", [True, False])
@pytest.mark.parametrize("name,M", [("tiny", None), ("tiny", 1), ("tiny", 255), ("tiny", 257),
                                    ("text_enc_up_21", None), ("text_enc_down_130", None)])
def test_int8_gemm_full_compare(name, M, rotate):
    check8(run_layer8(workloads.make_inputs(name, M=M), rotate=rotate))


def test_int8_layer_matches_oracle_end_to_end():
    # the oracle's whole INT8 layer on its own codes; GPU codes may flip at near-ties, so the
    # comparison of Y is made where the GPU's activation codes equal the oracle's
    d = workloads.make_inputs("tiny")
    r = run_layer8(d, rotate=True)
    q_w, s_w, _ = oracle.pack_weight8(d["W"], rotate_groups=True)
    want = oracle.int8_linear(d["X"], q_w, s_w, d["bias"], rotate_groups=True)
    same_rows = np.all(r["Xq"] == want["qa"], axis=1) & np.all(r["Wq"] == q_w)
    assert same_rows.mean() > 0.9
    assert_bf16_within_1ulp(r["Y"][same_rows], want["Y"][same_rows])


def test_int8_gemm_ragged_tiles_row_scales_no_bias():
    rng = np.random.default_rng(17)
    M, N, K = 300, 392, 768
    d = {"X": workloads.bf16_bits_from_f32(rng.standard_normal((M, K)).astype(np.float32)),
         "W": workloads.bf16_bits_from_f32((rng.standard_normal((N, K)) * 0.02).astype(np.float32)),
         "bias": None}
    check8(run_layer8(d, rotate=True, scale_mode="row", with_bias=False))


def test_int8_gemm_minimum_sizes():
    rng = np.random.default_rng(19)
    M, N, K = 1, 8, 256
    d = {"X": workloads.bf16_bits_from_f32(rng.standard_normal((M, K)).astype(np.float32)),
         "W": workloads.bf16_bits_from_f32(rng.standard_normal((N, K)).astype(np.float32)),
         "bias": workloads.bf16_bits_from_f32(rng.standard_normal(N).astype(np.float32))}
    check8(run_layer8(d, rotate=False))


def test_int8_gemm_extreme_codes_exact():
    # K = 65536 with codes -128 and 127: |acc| up to 2^30, the largest the call accepts
    K, M, N = 65536, 300, 16
    xq = np.full((M, K), -128, np.int8)
    wq = np.full((N, K), 127, np.int8)
    wq[1::2] = -128
    acc = cr().cr_int8_gemm_s32(torch.from_numpy(xq).cuda(), torch.from_numpy(wq).cuda()).cpu().numpy()
    want = np.where(np.arange(N) % 2 == 0, -128 * 127 * K, 128 * 128 * K)
    assert np.array_equal(acc, np.broadcast_to(want, (M, N)))


def test_int8_zero_activation_gives_bias():
    d = workloads.make_inputs("tiny")
    Wq, s_w = cr().cr_pack_weight_ex(dev_bf16(d["W"]), bits=8)
    Xq, s_a = cr().cr_rotate_quant_act_ex(torch.zeros((64, 512), dtype=torch.bfloat16, device="cuda"), bits=8)
    assert s_a.item() == 1.0 and not Xq.any()
    Y = cr().cr_int8_gemm(Xq, s_a, Wq, s_w, dev_bf16(d["bias"]))
    assert np.array_equal(host_bits(Y), np.broadcast_to(d["bias"], (64, 256)))


def test_int8_gemm_full_size_matches_library_int_mm():
    # DiT attention shape: accumulators against torch._int_mm (an independent library product), and
    # the epilogue on sampled outputs against the oracle; repeated to catch pipeline-ordering slips
    d = workloads.make_inputs("dit_attn")
    r = run_layer8(d, rotate=True)
    ref = torch._int_mm(torch.from_numpy(r["Xq"]).cuda(), torch.from_numpy(r["Wq"]).cuda().t())
    assert np.array_equal(r["acc"], ref.cpu().numpy())
    Xq, Wq = torch.from_numpy(r["Xq"]).cuda(), torch.from_numpy(r["Wq"]).cuda()
    for _ in range(4):
        assert torch.equal(cr().cr_int8_gemm_s32(Xq, Wq), ref)
    rng = np.random.default_rng(2)
    check8(r, np.sort(rng.choice(4096, 256, replace=False)), np.sort(rng.choice(3072, 256, replace=False)))


def test_int8_gemm_large_k_sampled():
    # DiT MLP down projection (K = 12288, inputs larger than L2)
    d = workloads.make_inputs("dit_mlp_down")
    r = run_layer8(d, rotate=True)
    rng = np.random.default_rng(3)
    M, N = r["acc"].shape
    check8(r, np.sort(rng.choice(M, 128, replace=False)), np.sort(rng.choice(N, 128, replace=False)))


def test_int8_strided_input_and_output_rows():
    # X rows ldx = K + 64 apart and Y rows ldy = N + 8 apart give the same codes and outputs as dense ones
    d = workloads.make_inputs("tiny")
    M, K = d["X"].shape
    N = d["W"].shape[0]
    big = np.zeros((M, K + 64), dtype=np.uint16)
    big[:, :K] = d["X"]
    Xs = dev_bf16(big)[:, :K]
    Xq_s, s_s = cr().cr_rotate_quant_act_ex(Xs, bits=8, rotate=True)
    Xq, s = cr().cr_rotate_quant_act_ex(dev_bf16(d["X"]), bits=8, rotate=True)
    assert torch.equal(Xq_s, Xq) and torch.equal(s_s, s)
    Wq, s_w = cr().cr_pack_weight_ex(dev_bf16(d["W"]), bits=8)
    b = dev_bf16(d["bias"])
    Y = cr().cr_int8_gemm(Xq, s, Wq, s_w, b)
    Ybig = torch.zeros((M, N + 8), dtype=torch.bfloat16, device="cuda")
    cr().cr_int8_gemm(Xq, s, Wq, s_w, b, out=Ybig[:, :N])
    torch.cuda.synchronize()
    assert torch.equal(Ybig[:, :N], Y) and not Ybig[:, N:].any()
