"""GPU parity of the INT4 GEMM: int32 accumulators bit-exact against the
oracle's integer product of the GPU's own codes, bf16 outputs within one ulp
of the oracle's epilogue on those accumulators."""

import numpy as np
import pytest
import torch

import oracle
from helpers import assert_bf16_within_1ulp
from w4a8_rotated_quantized_b200 import workloads

pytestmark = pytest.mark.gpu


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def host_bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def cr():
    import w4a8_rotated_quantized_b200 as m

    return m


def run_layer(d, scale_mode="tensor", with_bias=True):
    X, W = dev_bf16(d["X"]), dev_bf16(d["W"])
    bias = dev_bf16(d["bias"]) if with_bias else None
    Wq, s_w = cr().cr_pack_weight(W, scale_mode=scale_mode)
    Xq, s_a = cr().cr_rotate_quant_act(X)
    acc = cr().cr_w4a4_gemm_s32(Xq, Wq)
    Y = cr().cr_w4a4_gemm(Xq, s_a, Wq, s_w, bias)
    torch.cuda.synchronize()
    assert cr().cr_read_device_status() == 0
    return dict(Xq=Xq.cpu().numpy(), s_a=np.float32(s_a.item()), Wq=Wq.cpu().numpy(), s_w=s_w.cpu().numpy(),
                acc=acc.cpu().numpy(), Y=host_bits(Y), bias=d["bias"] if with_bias else None)


def check(r, rows=None, cols=None):
    qa = oracle.unpack_int4(r["Xq"] if rows is None else r["Xq"][rows])
    qw = oracle.unpack_int4(r["Wq"] if cols is None else r["Wq"][cols])
    acc_o = oracle.int_gemm(qa, qw)
    acc_g = r["acc"] if rows is None else r["acc"][np.ix_(rows, cols)]
    y_g = r["Y"] if rows is None else r["Y"][np.ix_(rows, cols)]
    assert np.array_equal(acc_g, acc_o), f"accumulators differ at {np.argwhere(acc_g != acc_o)[:5].tolist()}"
    s_w = r["s_w"] if cols is None else r["s_w"][cols]
    bias = None if r["bias"] is None else (r["bias"] if cols is None else r["bias"][cols])
    assert_bf16_within_1ulp(y_g, oracle.epilogue(acc_o, r["s_a"], s_w, bias))


# M <= 128 runs the few-token kernel (K split over a cluster: 2 CTAs for tiny, 7 for text_enc_down_21), 129..256
# its one-CTA-per-SM configuration when the weight tiles leave room for a K split (tiny, text_enc_down_130), else
# and above the CTA-pair kernel; M = 16, 100, 128, 256 cover the smallest, a ragged and the largest paddings;
# the four text-encoder shapes (21 and 130 tokens, K = 2560 <-> 9728) are compared in full
@pytest.mark.parametrize("name,M", [("tiny", None), ("tiny", 1), ("tiny", 16), ("tiny", 100), ("tiny", 128),
                                    ("tiny", 129), ("tiny", 256), ("tiny", 257), ("text_enc_up_21", None),
                                    ("text_enc_down_21", None), ("text_enc_up_130", None),
                                    ("text_enc_down_130", None)])
def test_gemm_small_full_compare(name, M):
    check(run_layer(workloads.make_inputs(name, M=M)))


def test_gemm_ragged_tiles_row_scales_no_bias():
    # M, N not multiples of the 128 x 256 tile; N a multiple of 8 only; per-row weight scales; no bias
    rng = np.random.default_rng(7)
    M, N, K = 200, 264, 768
    d = {"X": workloads.bf16_bits_from_f32(rng.standard_normal((M, K)).astype(np.float32)),
         "W": workloads.bf16_bits_from_f32((rng.standard_normal((N, K)) * 0.02).astype(np.float32)),
         "bias": None}
    check(run_layer(d, scale_mode="row", with_bias=False))


def test_gemm_minimum_sizes():
    rng = np.random.default_rng(9)
    M, N, K = 1, 8, 256
    d = {"X": workloads.bf16_bits_from_f32(rng.standard_normal((M, K)).astype(np.float32)),
         "W": workloads.bf16_bits_from_f32(rng.standard_normal((N, K)).astype(np.float32)),
         "bias": workloads.bf16_bits_from_f32(rng.standard_normal(N).astype(np.float32))}
    check(run_layer(d))


def test_gemm_extreme_codes_exact():
    # all codes -8 or 7 at K = 65536 - the largest accumulators the kernel accepts
    K, M, N = 65536, 130, 16
    xq = np.full((M, K // 2), 0x88, np.uint8)  # every code -8
    wq = np.full((N, K // 2), 0x77, np.uint8)  # every code 7
    wq[1::2] = 0x88
    acc = cr().cr_w4a4_gemm_s32(torch.from_numpy(xq).cuda(), torch.from_numpy(wq).cuda()).cpu().numpy()
    want = np.where(np.arange(N) % 2 == 0, -8 * 7 * K, 64 * K)
    assert np.array_equal(acc, np.broadcast_to(want, (M, N)))


def test_gemm_zero_activation_gives_bias():
    d = workloads.make_inputs("tiny")
    W, bias = dev_bf16(d["W"]), dev_bf16(d["bias"])
    Wq, s_w = cr().cr_pack_weight(W)
    Xq, s_a = cr().cr_rotate_quant_act(torch.zeros((64, 512), dtype=torch.bfloat16, device="cuda"))
    Y = cr().cr_w4a4_gemm(Xq, s_a, Wq, s_w, bias)
    assert np.array_equal(host_bits(Y), np.broadcast_to(d["bias"], (64, 256)))


def test_gemm_empty_m():
    d = workloads.make_inputs("tiny")
    Wq, s_w = cr().cr_pack_weight(dev_bf16(d["W"]))
    Xq, s_a = cr().cr_rotate_quant_act(torch.zeros((0, 512), dtype=torch.bfloat16, device="cuda"))
    Y = cr().cr_w4a4_gemm(Xq, s_a, Wq, s_w, None)
    assert Y.shape == (0, 256)


def test_gemm_matches_library_int_mm():
    # independent library cross-check of the accumulators: torch._int_mm on the unpacked codes
    d = workloads.make_inputs("dit_attn")
    r = run_layer(d)
    qa = torch.from_numpy(oracle.unpack_int4(r["Xq"])).cuda()
    qw = torch.from_numpy(oracle.unpack_int4(r["Wq"])).cuda()
    ref = torch._int_mm(qa, qw.t()).cpu().numpy()
    assert np.array_equal(r["acc"], ref)
    rng = np.random.default_rng(0)
    check(r, np.sort(rng.choice(4096, 256, replace=False)), np.sort(rng.choice(3072, 256, replace=False)))


@pytest.mark.parametrize("name", ["dit_mlp_up", "dit_mlp_down"])
def test_gemm_full_size_sampled(name):
    d = workloads.make_inputs(name)
    r = run_layer(d)
    rng = np.random.default_rng(1)
    M, N = r["acc"].shape
    check(r, np.sort(rng.choice(M, 192, replace=False)), np.sort(rng.choice(N, 192, replace=False)))


def test_gemm_repeated_runs_are_identical_to_library():
    # the pair kernel's pipeline has many hand-offs between warps and CTAs; a
    # missing ordering shows up as rare wrong rows, so run the big shape repeatedly
    d = workloads.make_inputs("dit_mlp_up")
    W, X = dev_bf16(d["W"]), dev_bf16(d["X"])
    Wq, _ = cr().cr_pack_weight(W)
    Xq, _ = cr().cr_rotate_quant_act(X)
    qa = torch.from_numpy(oracle.unpack_int4(Xq.cpu().numpy())).cuda()
    qw = torch.from_numpy(oracle.unpack_int4(Wq.cpu().numpy())).cuda()
    ref = torch._int_mm(qa, qw.t())
    for _ in range(8):
        acc = cr().cr_w4a4_gemm_s32(Xq, Wq)
        torch.cuda.synchronize()
        assert torch.equal(acc, ref)
    assert cr().cr_read_device_status() == 0


def test_gemm_few_tokens_split_k_repeated_runs():
    # the few-token kernel adds the partial sums of 7 CTAs through distributed shared memory;
    # a missing ordering would show up as run-to-run differences
    d = workloads.make_inputs("text_enc_down_21")
    W, X = dev_bf16(d["W"]), dev_bf16(d["X"])
    Wq, _ = cr().cr_pack_weight(W)
    Xq, _ = cr().cr_rotate_quant_act(X)
    qa = torch.from_numpy(oracle.unpack_int4(Xq.cpu().numpy())).cuda()
    qw = torch.from_numpy(oracle.unpack_int4(Wq.cpu().numpy())).cuda()
    # torch._int_mm wants at least 17 rows: pad the 21 tokens to 32 with zero codes
    qa32 = torch.zeros((32, qa.shape[1]), dtype=torch.int8, device="cuda")
    qa32[: qa.shape[0]] = qa
    ref = torch._int_mm(qa32, qw.t())[: qa.shape[0]]
    for _ in range(8):
        acc = cr().cr_w4a4_gemm_s32(Xq, Wq)
        torch.cuda.synchronize()
        assert torch.equal(acc, ref)
    assert cr().cr_read_device_status() == 0
