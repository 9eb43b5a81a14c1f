"""The no-allocation entry point (cr_w4a4_linear_noalloc) against cr_w4a4_linear.

cr_w4a4_linear_noalloc is for callers that cannot allocate device memory
(no workspace argument; its scratch is a fixed device array inside the
library).  It must give the same layer output as the workspace entry point,
also on the second of two calls in a row with different inputs (the fixed
scratch keeps the previous call's contents), and it must reject problems
whose packed activation codes do not fit its scratch.

This file is collected last on purpose, and passes alone in a fresh process
as well as after the rest of the suite.
"""

import numpy as np
import pytest
import torch

from helpers import assert_bf16_within_1ulp
from w4a8_rotated_quantized_b200 import workloads

pytestmark = pytest.mark.gpu


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def host_bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def test_noalloc_matches_linear_on_two_calls_in_a_row():
    import w4a8_rotated_quantized_b200 as cr

    cases = []
    for name, seed in (("dit_attn", 11), ("text_enc_down_130", 12)):
        d = workloads.make_inputs(name, seed=seed)
        W = dev_bf16(d["W"])
        Wq, s_w = cr.cr_pack_weight(W)
        cases.append((dev_bf16(d["X"]), Wq, s_w, dev_bf16(d["bias"])))
    # two calls in a row through the C ABI, different shapes and data, then compare each
    outs = [cr.cr_w4a4_linear_noalloc(X, Wq, s_w, b) for (X, Wq, s_w, b) in cases]
    torch.cuda.synchronize()
    for (X, Wq, s_w, b), y in zip(cases, outs):
        ref = cr.cr_w4a4_linear(X, Wq, s_w, b)
        torch.cuda.synchronize()
        assert_bf16_within_1ulp(host_bits(y), host_bits(ref), "noalloc vs linear")
    # and once more on the first case, after the second case left its contents in the scratch
    again = cr.cr_w4a4_linear_noalloc(*cases[0])
    ref0 = cr.cr_w4a4_linear(*cases[0])
    torch.cuda.synchronize()
    assert_bf16_within_1ulp(host_bits(again), host_bits(ref0), "noalloc repeat")


def test_noalloc_rejects_problems_beyond_its_scratch():
    import w4a8_rotated_quantized_b200 as cr
    from w4a8_rotated_quantized_b200 import binding

    M, K, N = 8192, 3072, 256  # packed codes 12 MiB > 8 MiB
    X = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    Wq = torch.zeros((N, K // 2), dtype=torch.uint8, device="cuda")
    s_w = torch.ones((N,), dtype=torch.float32, device="cuda")
    Y = torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(binding.ConvRotError) as e:
        cr.cr_w4a4_linear_noalloc(X, Wq, s_w, None, out=Y)
    assert e.value.status == 5  # CR_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((Y == 7.0).all())  # nothing was launched
