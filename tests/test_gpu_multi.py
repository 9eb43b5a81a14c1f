"""Shared activation quantisation for split projections (cr_w4a4_gemm_multi,
cr_w4a4_gemm_multi_s32, cr_w4a4_linear_multi): one set of activation codes
feeds several weight matrices.  Every projection's output must be bit-identical
to a separate cr_w4a4_gemm call on the same codes, and its accumulators equal
to the oracle's integer product; outputs within one bf16 ulp of the oracle's
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


def same_bits(a, b):
    return torch.equal(a.view(torch.int16), b.view(torch.int16))


def cr():
    import w4a8_rotated_quantized_b200 as m

    return m


def projections(K, Ns, seed, scale_mode="tensor", bias_mask=None):
    """Packed weights of several projections (distinct seeded draws) and their bf16 biases."""
    rng = np.random.default_rng(seed)
    out = []
    for j, N in enumerate(Ns):
        if N == 0:  # an empty projection: no weights to pack
            out.append((torch.empty((0, K // 2), dtype=torch.uint8, device="cuda"),
                        torch.empty((0,), dtype=torch.float32, device="cuda"), None, None))
            continue
        W = workloads.bf16_bits_from_f32((rng.standard_normal((N, K)) * 0.02).astype(np.float32))
        b = workloads.bf16_bits_from_f32((rng.standard_normal(N) * 0.01).astype(np.float32))
        Wq, s_w = cr().cr_pack_weight(dev_bf16(W), scale_mode=scale_mode)
        keep_bias = bias_mask is None or bias_mask[j]
        out.append((Wq, s_w, dev_bf16(b) if keep_bias else None, b if keep_bias else None))
    return out


def check_against_oracle(y, Xq, s_a, Wq, s_w, bias_bits, rows=None):
    qa = oracle.unpack_int4(Xq.cpu().numpy())
    qw = oracle.unpack_int4(Wq.cpu().numpy())
    yg = host_bits(y)
    if rows is not None:
        qa, yg = qa[rows], yg[rows]
    acc = oracle.int_gemm(qa, qw)
    assert_bf16_within_1ulp(yg, oracle.epilogue(acc, np.float32(s_a.item()), s_w.cpu().numpy(), bias_bits))


def test_qkv_dit_attention_shared_codes():
    # the DiT attention input X [4096, 3072] feeding three [3072, 3072] projections: one rotation and
    # quantisation of X, one GEMM launch over the 3 x 256 tiles (last round split into half tiles)
    d = workloads.make_inputs("dit_attn", with_weight=False)
    X = dev_bf16(d["X"])
    proj = projections(3072, [3072, 3072, 3072], seed=31)
    Wqs, sws, bs = [p[0] for p in proj], [p[1] for p in proj], [p[2] for p in proj]
    Ys = cr().cr_w4a4_linear_multi(X, Wqs, sws, bs)
    Xq, s_a = cr().cr_rotate_quant_act(X)
    Ym = cr().cr_w4a4_gemm_multi(Xq, s_a, Wqs, sws, bs)
    sep = [cr().cr_w4a4_gemm(Xq, s_a, Wq, sw, b) for Wq, sw, b in zip(Wqs, sws, bs)]
    torch.cuda.synchronize()
    assert cr().cr_read_device_status() == 0
    for j in range(3):
        assert same_bits(Ys[j], sep[j]) and same_bits(Ym[j], sep[j]), f"projection {j}"
    # the shared codes against the oracle, then every projection's product and epilogue on sampled rows
    _, s_o, q_o, y_o = oracle.rotate_quant_act(d["X"])
    assert_scale_close(s_a.item(), s_o, d["X"])
    assert_codes_match(oracle.unpack_int4(Xq.cpu().numpy()), q_o, y_o, s_o)
    rows = np.sort(np.random.default_rng(5).choice(4096, 384, replace=False))
    for j, (Wq, sw, _, b_bits) in enumerate(proj):
        check_against_oracle(Ym[j], Xq, s_a, Wq, sw, b_bits, rows)


def test_multi_ragged_projections_exact_accumulators():
    # unequal widths (one tile, a ragged tile, an empty projection, the minimum width), per-row weight
    # scales, biases on some projections only, M not a multiple of the 256-row tile
    rng = np.random.default_rng(8)
    M, K = 300, 768
    Ns = [264, 0, 520, 8]
    X = dev_bf16(workloads.bf16_bits_from_f32(rng.standard_normal((M, K)).astype(np.float32)))
    proj = projections(K, Ns, seed=9, scale_mode="row", bias_mask=[True, True, False, True])
    Wqs, sws, bs = [p[0] for p in proj], [p[1] for p in proj], [p[2] for p in proj]
    Xq, s_a = cr().cr_rotate_quant_act(X)
    accs = cr().cr_w4a4_gemm_multi_s32(Xq, Wqs)
    Ys = cr().cr_w4a4_gemm_multi(Xq, s_a, Wqs, sws, bs)
    torch.cuda.synchronize()
    assert cr().cr_read_device_status() == 0
    qa = oracle.unpack_int4(Xq.cpu().numpy())
    for j, (Wq, sw, b, b_bits) in enumerate(proj):
        assert Ys[j].shape == (M, Ns[j]) and accs[j].shape == (M, Ns[j])
        acc_o = oracle.int_gemm(qa, oracle.unpack_int4(Wq.cpu().numpy()))
        assert np.array_equal(accs[j].cpu().numpy(), acc_o), f"projection {j}"
        if Ns[j]:
            assert_bf16_within_1ulp(host_bits(Ys[j]), oracle.epilogue(acc_o, np.float32(s_a.item()),
                                                                       sw.cpu().numpy(), b_bits))
            assert same_bits(Ys[j], cr().cr_w4a4_gemm(Xq, s_a, Wq, sw, b))


@pytest.mark.parametrize("M", [21, 130])
def test_multi_text_encoder_projections(M):
    # few tokens (one few-token launch per projection) and 130 tokens (one CTA-pair launch)
    d = workloads.make_inputs("text_enc_up_21", M=M, with_weight=False)
    X = dev_bf16(d["X"])
    proj = projections(2560, [2560, 1024, 1024], seed=12)
    Wqs, sws, bs = [p[0] for p in proj], [p[1] for p in proj], [p[2] for p in proj]
    Ys = cr().cr_w4a4_linear_multi(X, Wqs, sws, bs)
    Xq, s_a = cr().cr_rotate_quant_act(X)
    torch.cuda.synchronize()
    for j, (Wq, sw, b, b_bits) in enumerate(proj):
        assert same_bits(Ys[j], cr().cr_w4a4_gemm(Xq, s_a, Wq, sw, b))
        check_against_oracle(Ys[j], Xq, s_a, Wq, sw, b_bits)


def test_multi_repeated_runs_are_identical():
    # many tiles over three projections with half tiles in the last round, run repeatedly
    d = workloads.make_inputs("dit_attn", with_weight=False)
    X = dev_bf16(d["X"])
    proj = projections(3072, [3072, 3072, 3072], seed=44)
    Wqs = [p[0] for p in proj]
    Xq, _ = cr().cr_rotate_quant_act(X)
    qa = torch.from_numpy(oracle.unpack_int4(Xq.cpu().numpy())).cuda()
    refs = [torch._int_mm(qa, torch.from_numpy(oracle.unpack_int4(W.cpu().numpy())).cuda().t()) for W in Wqs]
    for _ in range(4):
        accs = cr().cr_w4a4_gemm_multi_s32(Xq, Wqs)
        torch.cuda.synchronize()
        for a, r in zip(accs, refs):
            assert torch.equal(a, r)
    assert cr().cr_read_device_status() == 0
