"""GPU parity of the W4A8 path (asymmetric 4-bit weights, group 16, fp16
scale and 4-bit zero point; INT8 tensorwise activations; both rotated).

* Weight packing: without the rotation every scale, zero point and code equals
  the oracle's bit for bit.  With it, the float32 rotation may move a group's
  min / max by its rounding error, so a scale may differ by one fp16 ulp (on
  few groups) and a zero point or code by one at a near-tie; codes are compared
  against the oracle's codes for the GPU's own scales and zero points.
* Product: the tensor cores multiply fp16(s * (q - z)) by the exact activation
  codes and sum in float32.  Against the exact float64 sum of those operands
  the float32 sums are within K * 2**-23 * sum |terms|; against the oracle's
  exact dequantised weights the outputs are within one bf16 ulp plus
  s_a * (2**-11 * sum |qa w^| + K * 2**-23 * sum |terms|) (fp16 rounding of
  the weight, float32 sum).
"""

import numpy as np
import pytest
import torch

import oracle
from helpers import rotation_error_bound
from w4a8_rotated_quantized_b200 import workloads

pytestmark = pytest.mark.gpu


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def host_bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def cr():
    import w4a8_rotated_quantized_b200 as m

    return m


def pack_gpu(w_bits, rotate=True):
    Wq, gs, gz = cr().cr_pack_weight_w4a8(dev_bf16(w_bits), rotate=rotate)
    torch.cuda.synchronize()
    return (oracle.unpack_u4(Wq.cpu().numpy()), gs.cpu().numpy(), oracle.unpack_u4(gz.cpu().numpy()),
            (Wq, gs, gz))


@pytest.mark.parametrize("name", ["tiny", "text_enc_down_21", "w4a8_up"])
def test_pack_w4a8_without_rotation_is_exact(name):
    d = workloads.make_inputs(name, M=1)
    q, s, z, _ = pack_gpu(d["W"], rotate=False)
    want = oracle.pack_weight_w4a8(d["W"], rotate_groups=False)
    assert np.array_equal(s.view(np.uint16), want["s"].view(np.uint16))
    assert np.array_equal(z, want["z"])
    assert np.array_equal(q, want["q"])


@pytest.mark.parametrize("name", ["tiny", "text_enc_down_21", "w4a8_up"])
def test_pack_w4a8_with_rotation_matches_oracle(name):
    d = workloads.make_inputs(name, M=1)
    q, s, z, _ = pack_gpu(d["W"], rotate=True)
    want = oracle.pack_weight_w4a8(d["W"], rotate_groups=True)
    y = want["y"]
    s_o, z_o = want["s"], want["z"]
    # scales: at most one fp16 ulp apart, on few groups
    sd = np.abs(s.astype(np.float64) - s_o.astype(np.float64))
    ulp = np.spacing(np.abs(s_o)).astype(np.float64)
    assert np.all(sd <= ulp), "a group scale differs by more than one fp16 ulp"
    assert (sd > 0).mean() <= 0.01
    # codes and zero points: the oracle's, for the GPU's own scales, up to near-ties of the rotation
    err = rotation_error_bound(d["W"])
    s_e = np.repeat(s.astype(np.float64), 16, axis=1)
    q_o = oracle.quantize_asym16(y, s, z)
    diff = q.astype(np.int16) - q_o.astype(np.int16)
    bad = np.nonzero(diff)
    t = y[bad] / s_e[bad]
    near = np.abs(t - np.floor(t) - 0.5) <= err / s_e[bad] + 1e-5 * np.abs(t)
    assert np.all(np.abs(diff[bad]) == 1) and np.all(near), "a code differs away from a rounding boundary"
    assert len(bad[0]) <= 1e-3 * q.size
    # zero points where the scale agrees: equal up to a near-tie of -lo / s
    same = sd == 0
    lo = y.astype(np.float32).reshape(y.shape[0], -1, 16).min(axis=2).astype(np.float64)
    tz = -lo / s.astype(np.float64)
    zdiff = (z.astype(np.int16) - z_o.astype(np.int16))[same]
    near_z = (np.abs(tz - np.floor(tz) - 0.5) <= err / s.astype(np.float64) + 1e-5 * np.abs(tz))[same]
    assert np.all((zdiff == 0) | ((np.abs(zdiff) == 1) & near_z))


def check_w4a8(r, rows=None, cols=None):
    """Parity of the float32 sums and the bf16 outputs, given the GPU's own codes and parameters."""
    rows = np.arange(r["Xq"].shape[0]) if rows is None else rows
    cols = np.arange(r["q"].shape[0]) if cols is None else cols
    qa = r["Xq"][rows].astype(np.float64)
    q, s, z = r["q"][cols], r["s"][cols], r["z"][cols]
    K = qa.shape[1]
    w_exact = oracle.dequant_asym16(q, s, z)
    acc_exact = oracle.w4a8_acc(r["Xq"][rows], q, s, z)
    # the GPU's B operand: s * (q - z) rounded once to fp16 (exact in float32 first, then one rounding)
    zf = np.repeat(z.astype(np.float32), 16, axis=1)
    w16 = (np.repeat(s.astype(np.float32), 16, axis=1) * (q.astype(np.float32) - zf)).astype(np.float16)
    w16 = w16.astype(np.float64)
    acc16 = qa @ w16.T
    sabs = np.abs(qa) @ np.abs(w16).T
    sabs_exact = np.abs(qa) @ np.abs(w_exact).T
    fp32_sum = K * 2.0 ** -23 * sabs + 1e-30
    acc_g = r["acc"][np.ix_(rows, cols)].astype(np.float64)
    dev = np.abs(acc_g - acc16)
    assert np.all(dev <= fp32_sum), f"float32 sums off by {np.max(dev / fp32_sum):.3g} x the bound"
    # outputs against the exact oracle
    s_a = np.float64(np.float32(r["s_a"]))
    bias = np.zeros(len(cols)) if r["bias"] is None else oracle.bf16_bits_to_f64(r["bias"][cols])
    y_exact = acc_exact * s_a + bias[None, :]
    y_g = oracle.bf16_bits_to_f64(r["Y"][np.ix_(rows, cols)])
    y_o = oracle.bf16_bits_to_f64(oracle.w4a8_epilogue(acc_exact, r["s_a"],
                                                       None if r["bias"] is None else r["bias"][cols]))
    ulp = np.spacing(np.abs(y_o).astype(np.float32)).astype(np.float64) * 2.0 ** 16  # bf16 ulp at |y|
    ulp = np.maximum(ulp, 2.0 ** -133)
    tol = ulp + s_a * (2.0 ** -11 * sabs_exact + fp32_sum)
    assert np.all(np.abs(y_g - y_exact) <= tol), "an output is outside the W4A8 error bound"
    # Against the exact sum of the GPU's own fp16 operands only the float32 summation remains (relative
    # ~ sqrt(K) 2**-24 of sum |terms|, far below a bf16 ulp): nearly every output is that value rounded
    # to bf16, or its neighbour.  (Against the exact dequantised weights the fp16 rounding of w^ moves
    # small outputs, where terms cancel, by more than an ulp; the bound above covers them.)
    y16 = oracle.bf16_bits_to_f64(oracle.w4a8_epilogue(acc16, r["s_a"], None if r["bias"] is None else r["bias"][cols]))
    ulp16 = np.maximum(np.spacing(np.abs(y16).astype(np.float32)).astype(np.float64) * 2.0 ** 16, 2.0 ** -133)
    within1 = np.abs(y_g - y16) <= ulp16
    assert within1.mean() >= 0.999, f"only {within1.mean():.5f} of outputs within one ulp of the fp16-operand sum"


def run_w4a8(d, with_bias=True, M=None):
    X, W = dev_bf16(d["X"]), dev_bf16(d["W"])
    bias = dev_bf16(d["bias"]) if with_bias else None
    Wq, gs, gz = cr().cr_pack_weight_w4a8(W)
    Xq, s_a = cr().cr_rotate_quant_act_ex(X, bits=8, rotate=True)
    acc = cr().cr_w4a8_gemm_f32(Xq, Wq, gs, gz)
    Y = cr().cr_w4a8_gemm(Xq, s_a, Wq, gs, gz, bias)
    Y1 = cr().cr_w4a8_linear(X, Wq, gs, gz, bias)
    torch.cuda.synchronize()
    assert cr().cr_read_device_status() == 0
    assert torch.equal(Y, Y1), "the one-call layer differs from the separate calls"
    return dict(Xq=Xq.cpu().numpy(), s_a=np.float32(s_a.item()), q=oracle.unpack_u4(Wq.cpu().numpy()),
                s=gs.cpu().numpy(), z=oracle.unpack_u4(gz.cpu().numpy()), acc=acc.cpu().numpy(), Y=host_bits(Y),
                bias=d["bias"] if with_bias else None, dev=(Xq, Wq, gs, gz))


@pytest.mark.parametrize("name,M", [("tiny", None), ("tiny", 1), ("tiny", 255), ("tiny", 257),
                                    ("text_enc_up_21", None), ("text_enc_down_130", None)])
def test_w4a8_gemm_full_compare(name, M):
    check_w4a8(run_w4a8(workloads.make_inputs(name, M=M)))


def test_w4a8_ragged_tiles_no_bias():
    rng = np.random.default_rng(23)
    M, N, K = 300, 392, 768
    d = {"X": workloads.bf16_bits_from_f32(rng.standard_t(3.0, (M, K)).astype(np.float32)),
         "W": workloads.bf16_bits_from_f32((rng.standard_normal((N, K)) * 0.02).astype(np.float32)),
         "bias": None}
    check_w4a8(run_w4a8(d, with_bias=False))


def test_w4a8_minimum_sizes():
    rng = np.random.default_rng(29)
    M, N, K = 1, 8, 256
    d = {"X": workloads.bf16_bits_from_f32(rng.standard_normal((M, K)).astype(np.float32)),
         "W": workloads.bf16_bits_from_f32(rng.standard_normal((N, K)).astype(np.float32)),
         "bias": workloads.bf16_bits_from_f32(rng.standard_normal(N).astype(np.float32))}
    check_w4a8(run_w4a8(d))


def test_w4a8_unit_scales_zero_eight_is_integer_exact():
    # s = 1, z = 8: w^ = q - 8 exactly in fp16, every partial sum an integer below 2^24: the float32
    # sums must equal the integer product of the codes (torch._int_mm) exactly
    rng = np.random.default_rng(31)
    M, N, K = 256, 192, 1024
    xq = torch.from_numpy(rng.integers(-127, 128, (M, K)).astype(np.int8)).cuda()
    q = rng.integers(0, 16, (N, K)).astype(np.uint8)
    Wq = torch.from_numpy(oracle.pack_u4(q)).cuda()
    gs = torch.ones((N, K // 16), dtype=torch.float16, device="cuda")
    gz = torch.from_numpy(oracle.pack_u4(np.full((N, K // 16), 8, np.uint8))).cuda()
    acc = cr().cr_w4a8_gemm_f32(xq, Wq, gs, gz)
    ref = torch._int_mm(xq, torch.from_numpy(q.astype(np.int8) - 8).cuda().t())
    assert torch.equal(acc, ref.to(torch.float32))


def test_w4a8_zero_activation_gives_bias():
    d = workloads.make_inputs("tiny")
    Wq, gs, gz = cr().cr_pack_weight_w4a8(dev_bf16(d["W"]))
    Xq, s_a = cr().cr_rotate_quant_act_ex(torch.zeros((64, 512), dtype=torch.bfloat16, device="cuda"), bits=8)
    Y = cr().cr_w4a8_gemm(Xq, s_a, Wq, gs, gz, dev_bf16(d["bias"]))
    assert np.array_equal(host_bits(Y), np.broadcast_to(d["bias"], (64, 256)))


def test_w4a8_full_size_against_library_and_oracle():
    # the W4A8 workload (X [4096,3072] Student-t nu=3, W [12288,3072]): the float32 sums against a
    # library fp16 GEMM with float32 accumulation on the same operands, repeated runs identical,
    # and the oracle's bound on sampled outputs
    d = workloads.make_inputs("w4a8_up")
    r = run_w4a8(d)
    Xq, Wq, gs, gz = r["dev"]
    q = torch.from_numpy(r["q"].astype(np.float32)).cuda()
    zf = torch.from_numpy(np.repeat(r["z"].astype(np.float32), 16, axis=1)).cuda()
    sf = torch.from_numpy(np.repeat(r["s"].astype(np.float32), 16, axis=1)).cuda()
    w16 = (sf * (q - zf)).to(torch.float16).to(torch.float32)
    assert not torch.backends.cuda.matmul.allow_tf32  # full float32 products (exact here) and sums
    ref = torch.matmul(Xq.to(torch.float32), w16.t())
    acc = torch.from_numpy(r["acc"]).cuda()
    sabs = torch.matmul(Xq.to(torch.float32).abs(), w16.abs().t())
    assert torch.all((acc - ref).abs() <= 2 * 3072 * 2.0 ** -23 * sabs + 1e-30)
    for _ in range(3):
        assert torch.equal(cr().cr_w4a8_gemm_f32(Xq, Wq, gs, gz), acc)
    rng = np.random.default_rng(5)
    check_w4a8(r, np.sort(rng.choice(4096, 128, replace=False)), np.sort(rng.choice(12288, 128, replace=False)))


def test_w4a8_strided_output_rows():
    d = workloads.make_inputs("tiny")
    M, N = d["X"].shape[0], d["W"].shape[0]
    Wq, gs, gz = cr().cr_pack_weight_w4a8(dev_bf16(d["W"]))
    Xq, s_a = cr().cr_rotate_quant_act_ex(dev_bf16(d["X"]), bits=8)
    b = dev_bf16(d["bias"])
    Y = cr().cr_w4a8_gemm(Xq, s_a, Wq, gs, gz, b)
    Ybig = torch.zeros((M, N + 8), dtype=torch.bfloat16, device="cuda")
    cr().cr_w4a8_gemm(Xq, s_a, Wq, gs, gz, b, out=Ybig[:, :N])
    torch.cuda.synchronize()
    assert torch.equal(Ybig[:, :N], Y) and not Ybig[:, N:].any()
