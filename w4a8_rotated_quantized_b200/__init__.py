"""ConvRot W4A4 linear layer for NVIDIA B200 (sm_100a).

The public functions mirror the C ABI in ``include/convrot.h``:
``cr_pack_weight``, ``cr_rotate_quant_act``, ``cr_w4a4_gemm``,
``cr_w4a4_gemm_s32``, ``cr_w4a4_linear`` (with the launch arrangement of
``cr_w4a4_linear_ex`` as its ``mode``), ``cr_read_device_status``, and the
INT8 / any-format calls ``cr_pack_weight_ex``, ``cr_rotate_quant_act_ex``,
``cr_int8_gemm``, ``cr_int8_gemm_s32``, ``cr_int8_linear``, and the W4A8 calls
``cr_pack_weight_w4a8``, ``cr_w4a8_gemm``, ``cr_w4a8_gemm_f32``, ``cr_w4a8_linear``,
and the INT8-activation branch of the W4A4 weights ``cr_a8w4_gemm``, ``cr_a8w4_gemm_s32``,
``cr_a8w4_linear``, and shared activation quantisation for several projections
``cr_w4a4_gemm_multi``, ``cr_w4a4_gemm_multi_s32``, ``cr_w4a4_linear_multi``.  They are loaded lazily from
the in-tree CUDA library, so that ``workloads`` and ``build`` can be imported
on a machine where the library is not built yet; touching any of them without
the library raises ImportError.  There is no CPU fallback.
"""

_BINDING_NAMES = {
    "cr_pack_weight", "cr_rotate_quant_act", "cr_w4a4_gemm", "cr_w4a4_gemm_s32", "cr_w4a4_linear", "cr_w4a4_linear_noalloc", "cr_read_device_status",
    "cr_pack_weight_ex", "cr_rotate_quant_act_ex", "cr_int8_gemm", "cr_int8_gemm_s32", "cr_int8_linear",
    "cr_pack_weight_w4a8", "cr_w4a8_gemm", "cr_w4a8_gemm_f32", "cr_w4a8_linear",
    "cr_a8w4_gemm", "cr_a8w4_gemm_s32", "cr_a8w4_linear", "cr_selftest_wait_timeout", "cr_selftest_act_fallback",
    "cr_w4a4_gemm_multi", "cr_w4a4_gemm_multi_s32", "cr_w4a4_linear_multi",
    "cr_status_string", "cr_api_version", "ConvRotError", "workspace", "LIB_PATH",
    "LINEAR_AUTO", "LINEAR_ONE_LAUNCH", "LINEAR_TWO_LAUNCHES",
}


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import binding

        return getattr(binding, name)
    raise AttributeError(name)
