"""The C ABI library loads, exports every declared symbol and validates
arguments on the host (CPU only: no compute call runs here)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "convrot.h")


def _lib_path():
    from w4a8_rotated_quantized_b200 import build

    return build.build()


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"^(?:const char\*|int|size_t|cr_status)\s+(cr_\w+)\s*\(", text, re.M)


def test_header_declares_the_boundary():
    names = set(declared_functions())
    for n in ("cr_pack_weight", "cr_rotate_quant_act", "cr_w4a4_gemm", "cr_w4a4_gemm_s32", "cr_w4a4_linear",
              "cr_read_device_status", "cr_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(_lib_path())
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings_and_version():
    import w4a8_rotated_quantized_b200 as cr

    assert cr.cr_api_version() == 1
    for code in range(8):
        assert cr.cr_status_string(code).startswith("CR_")
    assert "UNKNOWN" in cr.cr_status_string(99)


def test_workspace_sizes():
    from w4a8_rotated_quantized_b200 import binding

    lib = binding._lib
    assert lib.cr_rotate_quant_act_workspace_size(4096, 3072, 256) >= 256
    assert lib.cr_w4a4_gemm_workspace_size(4096, 3072, 3072) >= 16
    lin = lib.cr_w4a4_linear_workspace_size(4096, 3072, 3072, 256)
    assert lin >= 4096 * 3072 // 2 and lin % 256 == 0
    lin8 = lib.cr_int8_linear_workspace_size(4096, 3072, 3072, 256)
    assert lin8 >= 4096 * 3072 and lin8 % 256 == 0
    assert lib.cr_int8_gemm_workspace_size(4096, 3072, 3072) >= 16
    assert lib.cr_w4a8_linear_workspace_size(4096, 12288, 3072, 256) >= 4096 * 3072


def _no_gpu():
    import torch

    return not torch.cuda.is_available()


@pytest.mark.skipif(not _no_gpu(), reason="fake device pointers are only safe where no GPU can be reached")
def test_validation_codes_without_a_device():
    from w4a8_rotated_quantized_b200 import binding

    lib = binding._lib
    P = ctypes.c_void_p
    A = P(1 << 20)  # aligned stand-in address, never dereferenced: validation or the device check fails first
    ws, wsn = P(1 << 21), 1 << 20
    # rotate_quant_act
    assert lib.cr_rotate_quant_act(None, 4, 512, 512, 256, A, A, ws, wsn, None) == 1
    assert lib.cr_rotate_quant_act(A, -1, 512, 512, 256, A, A, ws, wsn, None) == 1
    assert lib.cr_rotate_quant_act(A, 4, 300, 512, 256, A, A, ws, wsn, None) == 2
    assert lib.cr_rotate_quant_act(A, 4, 512, 512, 32, A, A, ws, wsn, None) == 2  # group 32: no such size
    assert lib.cr_rotate_quant_act(A, 4, 512, 512, 1024, A, A, ws, wsn, None) == 2  # group 1024 needs K % 1024
    assert lib.cr_rotate_quant_act(A, 4, 1024, 1024, 1024, A, A, ws, wsn, None) in (4, 6)
    assert lib.cr_rotate_quant_act(A, 4, 512, 512, 64, A, A, ws, wsn, None) in (4, 6)
    assert lib.cr_rotate_quant_act(A, 4, 512, 512, 16, A, A, ws, wsn, None) in (4, 6)
    assert lib.cr_pack_weight_w4a8(A, 8, 512, 512, 64, 1, A, A, A, ws, wsn, None) == 2  # W4A8: 256 only
    assert lib.cr_rotate_quant_act(A, 4, 65536 + 256, 65536 + 256, 256, A, A, ws, wsn, None) == 2
    assert lib.cr_rotate_quant_act(A, 4, 512, 256, 256, A, A, ws, wsn, None) == 1  # ldx < K
    assert lib.cr_rotate_quant_act(P((1 << 20) + 8), 4, 512, 512, 256, A, A, ws, wsn, None) == 3
    assert lib.cr_rotate_quant_act(A, 4, 512, 516, 256, A, A, ws, wsn, None) == 3  # ldx % 8
    assert lib.cr_rotate_quant_act(A, 4, 512, 512, 256, A, A, None, wsn, None) == 5
    assert lib.cr_rotate_quant_act(A, 4, 512, 512, 256, A, A, ws, 16, None) == 5
    # valid arguments: the device check is the first thing that fails on a machine without a GPU
    assert lib.cr_rotate_quant_act(A, 4, 512, 512, 256, A, A, ws, wsn, None) in (4, 6)
    # an empty X may be NULL: validation passes and only the device check fails here
    assert lib.cr_rotate_quant_act(None, 0, 512, 512, 256, None, A, ws, wsn, None) in (4, 6)
    # pack_weight
    assert lib.cr_pack_weight(A, 8, 512, 512, 256, 7, A, A, ws, wsn, None) == 1
    assert lib.cr_pack_weight(A, 8, 520, 520, 256, 0, A, A, ws, wsn, None) == 2
    # gemm
    assert lib.cr_w4a4_gemm(A, A, A, A, None, A, 12, 4, 12, 512, ws, wsn, None) == 2  # N % 8
    assert lib.cr_w4a4_gemm(A, A, A, A, None, A, 8, 4, 16, 512, ws, wsn, None) == 1  # ldy < N
    assert lib.cr_w4a4_gemm(A, A, A, A, None, P((1 << 20) + 2), 16, 4, 16, 512, ws, wsn, None) == 3
    assert lib.cr_w4a4_gemm(A, None, A, A, None, A, 16, 4, 16, 512, ws, wsn, None) == 1
    assert lib.cr_w4a4_gemm(A, A, A, A, None, A, 16, 4, 16, 512, ws, 0, None) == 5
    assert lib.cr_w4a4_gemm(A, A, A, A, None, A, 16, 4, 16, 512, ws, wsn, None) in (4, 6)
    assert lib.cr_w4a4_gemm_s32(A, A, A, 12, 4, 16, 512, ws, wsn, None) == 1  # ldc < N
    # linear
    assert lib.cr_w4a4_linear(A, 512, A, A, None, A, 16, 4, 16, 512, 32, ws, wsn, None) == 2  # group
    assert lib.cr_w4a4_linear(A, 512, A, A, None, A, 16, 4, 16, 512, 256, ws, 64, None) == 5
    # the launch-arrangement form: an unknown mode is refused first; the modes validate like the plain call
    assert lib.cr_w4a4_linear_ex(A, 512, A, A, None, A, 16, 4, 16, 512, 256, 3, ws, wsn, None) == 1
    assert lib.cr_w4a4_linear_ex(A, 512, A, A, None, A, 16, 4, 16, 512, 256, -1, ws, wsn, None) == 1
    for mode in (0, 1, 2):
        assert lib.cr_w4a4_linear_ex(A, 512, A, A, None, A, 16, 4, 16, 512, 32, mode, ws, wsn, None) == 2
        assert lib.cr_w4a4_linear_ex(A, 512, A, A, None, A, 16, 4, 16, 512, 256, mode, ws, 64, None) == 5
        assert lib.cr_w4a4_linear_ex(A, 512, A, A, None, A, 16, 4, 16, 512, 256, mode, ws, wsn, None) in (4, 6)
    assert lib.cr_read_device_status(None, None, None) == 1
    # the fallback diagnostic validates like cr_rotate_quant_act_ex
    assert lib.cr_selftest_act_fallback(A, 4, 512, 512, 256, 5, 1, A, A, ws, wsn, None) == 1  # bits
    assert lib.cr_selftest_act_fallback(A, 4, 300, 512, 256, 4, 1, A, A, ws, wsn, None) == 2
    assert lib.cr_selftest_act_fallback(A, 4, 512, 512, 256, 4, 1, A, A, ws, wsn, None) in (4, 6)
    # any-format calls: bits and rotate are checked before anything else about the format
    assert lib.cr_rotate_quant_act_ex(A, 4, 512, 512, 256, 6, 1, A, A, ws, wsn, None) == 1
    assert lib.cr_rotate_quant_act_ex(A, 4, 512, 512, 256, 8, 2, A, A, ws, wsn, None) == 1
    assert lib.cr_rotate_quant_act_ex(A, 4, 300, 512, 256, 8, 0, A, A, ws, wsn, None) == 2
    assert lib.cr_rotate_quant_act_ex(A, 4, 512, 512, 256, 8, 0, A, A, ws, wsn, None) in (4, 6)
    assert lib.cr_pack_weight_ex(A, 8, 512, 512, 256, 8, 1, 7, A, A, ws, wsn, None) == 1
    assert lib.cr_pack_weight_ex(A, 8, 512, 512, 256, 2, 1, 0, A, A, ws, wsn, None) == 1
    assert lib.cr_pack_weight_ex(A, 8, 512, 512, 256, 8, 1, 1, A, A, ws, wsn, None) in (4, 6)
    # INT8 GEMM and layer: the W4A4 call's rules
    assert lib.cr_int8_gemm(A, A, A, A, None, A, 12, 4, 12, 512, ws, wsn, None) == 2  # N % 8
    assert lib.cr_int8_gemm(A, A, A, A, None, A, 16, 4, 16, 384, ws, wsn, None) == 2  # K % 256
    assert lib.cr_int8_gemm(A, A, A, A, None, A, 16, 4, 16, 512, ws, 0, None) == 5
    assert lib.cr_int8_gemm(A, A, A, A, None, A, 16, 4, 16, 512, ws, wsn, None) in (4, 6)
    assert lib.cr_int8_gemm_s32(A, A, A, 12, 4, 16, 512, ws, wsn, None) == 1  # ldc < N
    assert lib.cr_int8_linear(A, 512, 3, A, A, None, A, 16, 4, 16, 512, 256, ws, wsn, None) == 1  # rotate
    assert lib.cr_int8_linear(A, 512, 1, A, A, None, A, 16, 4, 16, 512, 256, ws, 64, None) == 5
    # W4A8
    assert lib.cr_pack_weight_w4a8(A, 8, 512, 512, 256, 2, A, A, A, ws, wsn, None) == 1  # rotate
    assert lib.cr_pack_weight_w4a8(A, 8, 512, 512, 256, 1, A, None, A, ws, wsn, None) == 1
    assert lib.cr_pack_weight_w4a8(A, 8, 512, 512, 256, 1, A, P((1 << 20) + 2), A, ws, wsn, None) == 3
    assert lib.cr_pack_weight_w4a8(A, 8, 512, 512, 256, 1, A, A, A, ws, wsn, None) in (4, 6)
    assert lib.cr_w4a8_gemm(A, A, A, A, A, None, A, 12, 4, 12, 512, ws, wsn, None) == 2  # N % 8
    assert lib.cr_w4a8_gemm(A, A, A, A, None, None, A, 16, 4, 16, 512, ws, wsn, None) == 1  # no zero points
    assert lib.cr_w4a8_gemm(A, A, A, A, A, None, A, 16, 4, 16, 512, ws, 0, None) == 5
    assert lib.cr_w4a8_gemm(A, A, A, A, A, None, A, 16, 4, 16, 512, ws, wsn, None) in (4, 6)
    assert lib.cr_w4a8_gemm_f32(A, A, A, A, A, 18, 4, 16, 512, ws, wsn, None) == 3  # ldc % 4
    assert lib.cr_w4a8_linear(A, 512, A, A, A, None, A, 16, 4, 16, 512, 64, ws, wsn, None) == 2  # group
    # INT8 activations x packed INT4 weights
    assert lib.cr_a8w4_gemm(A, A, A, A, None, A, 12, 4, 12, 512, ws, wsn, None) == 2  # N % 8
    assert lib.cr_a8w4_gemm(A, A, A, A, None, A, 16, 4, 16, 512, ws, 0, None) == 5
    assert lib.cr_a8w4_gemm(A, A, A, A, None, A, 16, 4, 16, 512, ws, wsn, None) in (4, 6)
    assert lib.cr_a8w4_gemm_s32(A, A, A, 12, 4, 16, 512, ws, wsn, None) == 1  # ldc < N
    assert lib.cr_a8w4_linear(A, 512, A, A, None, A, 16, 4, 16, 512, 1024, ws, wsn, None) == 2  # K % group
    # several projections of one set of activation codes: host arrays of per-projection arguments
    ptrs = lambda n, v=A: (ctypes.c_void_p * n)(*([v.value] * n))
    ld = lambda *v: (ctypes.c_int64 * len(v))(*v)
    ns = lambda *v: (ctypes.c_int * len(v))(*v)
    three = (ptrs(3), ptrs(3), None, ptrs(3), ld(16, 16, 16), ns(16, 16, 16))
    assert lib.cr_w4a4_gemm_multi(A, A, 4, 512, 3, *three, ws, wsn, None) in (4, 6)
    assert lib.cr_w4a4_gemm_multi(A, A, 4, 512, 0, *three, ws, wsn, None) == 1  # no projection
    assert lib.cr_w4a4_gemm_multi(A, A, 4, 512, 5, ptrs(5), ptrs(5), None, ptrs(5), ld(*[16] * 5),
                                  ns(*[16] * 5), ws, wsn, None) == 1  # more than CR_MAX_PROJ
    assert lib.cr_w4a4_gemm_multi(A, A, 4, 512, 3, ptrs(3), ptrs(3), None, ptrs(3), ld(16, 16, 16),
                                  ns(16, 12, 16), ws, wsn, None) == 2  # a projection with N % 8 != 0
    assert lib.cr_w4a4_gemm_multi(A, A, 4, 512, 3, ptrs(3), ptrs(3), None, ptrs(3), ld(16, 8, 16),
                                  ns(16, 16, 16), ws, wsn, None) == 1  # ldy < N
    assert lib.cr_w4a4_gemm_multi(A, A, 4, 512, 2, ptrs(2), None, None, ptrs(2), ld(16, 16), ns(16, 16),
                                  ws, wsn, None) == 1  # no scale array
    assert lib.cr_w4a4_gemm_multi(A, A, 4, 512, 3, *three, ws, 0, None) == 5
    assert lib.cr_w4a4_gemm_multi_s32(A, 4, 512, 2, ptrs(2), ptrs(2), ld(16, 12), ns(16, 16), ws, wsn,
                                      None) == 1  # ldc < N
    assert lib.cr_w4a4_gemm_multi_s32(A, 4, 512, 2, ptrs(2), ptrs(2), ld(16, 16), ns(16, 16), ws, wsn,
                                      None) in (4, 6)
    assert lib.cr_w4a4_linear_multi(A, 512, 4, 512, 32, 3, *three, ws, wsn, None) == 2  # group
    assert lib.cr_w4a4_linear_multi(A, 512, 4, 512, 256, 3, *three, ws, 64, None) == 5
    assert lib.cr_w4a4_linear_multi(A, 512, 4, 512, 256, 3, *three, ws, wsn, None) in (4, 6)


def test_product_path_has_no_oracle_dependency():
    # the package and its CUDA sources never reach into the oracle
    pkg = os.path.join(ROOT, "w4a8_rotated_quantized_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f


def test_header_is_plain_c_and_a_c_program_links(tmp_path):
    # the boundary is a C ABI: the header compiles as C99 and a C program links against the library
    import shutil
    import subprocess

    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    lib = _lib_path()
    src = tmp_path / "probe.c"
    src.write_text(
        '#include "convrot.h"\n'
        "#include <stdio.h>\n"
        "int main(void) {\n"
        "  size_t ws = cr_w4a4_linear_workspace_size(4096, 3072, 3072, CR_GROUP_256);\n"
        "  cr_status st = cr_w4a4_gemm(0, 0, 0, 0, 0, 0, 8, 4, 12, 512, 0, 0, 0);\n"
        '  printf("%d %zu %d %s\\n", cr_api_version(), ws, (int)st, cr_status_string(st));\n'
        "  return 0;\n"
        "}\n")
    exe = tmp_path / "probe"
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                        str(src), "-o", str(exe), lib, f"-Wl,-rpath,{os.path.dirname(lib)}"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stderr
    ver, ws, st, name = out.stdout.split()[:4]
    assert ver == "1" and int(ws) >= 4096 * 3072 // 2 and st == "1" and name.startswith("CR_ERR_INVALID_ARG")
