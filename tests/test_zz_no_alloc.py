"""The no-allocation entry point (cr_w4a4_linear_noalloc) against cr_w4a4_linear.

cr_w4a4_linear_noalloc is for callers that cannot allocate device memory
(no workspace argument; its scratch is a fixed device array inside the
library).  It launches the same kernels as the workspace entry point on the
same inputs, so its output must be bit-identical, also on the second of two
calls in a row with different inputs (the fixed scratch keeps the previous
call's contents).  It must accept problems whose packed activation codes
fill its scratch exactly and reject the next size up.

This file is collected last on purpose, and passes alone in a fresh process
as well as after the rest of the suite.
"""

import numpy as np
import pytest
import torch

from w4a8_rotated_quantized_b200 import workloads

pytestmark = pytest.mark.gpu

SCRATCH_XQ_BYTES = 8 << 20  # the entry point's limit on M * K / 2
CR_ERR_WORKSPACE = 5


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def same_bits(a, b):
    return torch.equal(a.view(torch.int16), b.view(torch.int16))


def make_case(name, seed, M=None):
    import w4a8_rotated_quantized_b200 as cr

    d = workloads.make_inputs(name, seed=seed, M=M)
    Wq, s_w = cr.cr_pack_weight(dev_bf16(d["W"]))
    return dev_bf16(d["X"]), Wq, s_w, dev_bf16(d["bias"])


def random_case(M, K, N, seed):
    import w4a8_rotated_quantized_b200 as cr

    g = torch.Generator(device="cuda").manual_seed(seed)
    X = torch.randn((M, K), generator=g, device="cuda").to(torch.bfloat16)
    W = (torch.randn((N, K), generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    b = (torch.randn((N,), generator=g, device="cuda") * 0.01).to(torch.bfloat16)
    Wq, s_w = cr.cr_pack_weight(W)
    return X, Wq, s_w, b


def test_noalloc_matches_linear_on_two_calls_in_a_row():
    import w4a8_rotated_quantized_b200 as cr

    # the DiT attention projection (fused single-pass activation kernel, CTA-pair GEMM) and the
    # 130-token text-encoder down projection (few rows, K = 9728)
    cases = [make_case("dit_attn", 11), make_case("text_enc_down_130", 12)]
    # two calls in a row through the C ABI, different shapes and data, then compare each
    outs = [cr.cr_w4a4_linear_noalloc(X, Wq, s_w, b) for (X, Wq, s_w, b) in cases]
    torch.cuda.synchronize()
    for (X, Wq, s_w, b), y in zip(cases, outs):
        ref = cr.cr_w4a4_linear(X, Wq, s_w, b)
        torch.cuda.synchronize()
        assert same_bits(y, ref), "noalloc vs linear"
    # and once more on the first case, after the second case left its contents in the scratch
    again = cr.cr_w4a4_linear_noalloc(*cases[0])
    ref0 = cr.cr_w4a4_linear(*cases[0])
    torch.cuda.synchronize()
    assert same_bits(again, ref0), "noalloc repeat"


def test_noalloc_two_pass_activation_path_and_exact_limit():
    import w4a8_rotated_quantized_b200 as cr

    # M * K too large for the single-pass activation kernel (more than 384 units of 256 per SM),
    # so the two streaming passes run and read per-block maxima back from the fixed scratch:
    # 1344 x 12288 (codes 7.9 MiB), then 4096 x 4096 whose codes fill the 8 MiB exactly
    big = [random_case(1344, 12288, 256, 21), random_case(4096, 4096, 256, 22)]
    assert big[1][0].numel() // 2 == SCRATCH_XQ_BYTES
    for _ in range(2):  # two rounds in a row: each call follows one that left other contents behind
        for (X, Wq, s_w, b) in big:
            y = cr.cr_w4a4_linear_noalloc(X, Wq, s_w, b)
            ref = cr.cr_w4a4_linear(X, Wq, s_w, b)
            torch.cuda.synchronize()
            assert same_bits(y, ref), f"noalloc vs linear at {tuple(X.shape)}"
    assert cr.cr_read_device_status() == 0


@pytest.mark.parametrize("M,K", [(4097, 4096), (8192, 3072)])
def test_noalloc_rejects_problems_beyond_its_scratch(M, K):
    import w4a8_rotated_quantized_b200 as cr
    from w4a8_rotated_quantized_b200 import binding

    N = 256
    assert M * K // 2 > SCRATCH_XQ_BYTES
    X = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    Wq = torch.zeros((N, K // 2), dtype=torch.uint8, device="cuda")
    s_w = torch.ones((N,), dtype=torch.float32, device="cuda")
    Y = torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(binding.ConvRotError) as e:
        cr.cr_w4a4_linear_noalloc(X, Wq, s_w, None, out=Y)
    assert e.value.status == CR_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((Y == 7.0).all())  # nothing was launched
