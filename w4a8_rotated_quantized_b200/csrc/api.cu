// api.cu -- the extern "C" entry points declared in include/convrot.h:
// argument validation on the host, device check (sm_100 only, no fallback),
// workspace carving and kernel launches on the caller's stream.
//
// The two-call interface (offline weight preparation, online linear) follows
// "Qwen3-4B -- ConvRot W4A4 (ComfyUI text encoder)", section "Hardware": the
// converter quantises weights with one op and runs the layer with another,
// and refuses to run when those ops would resolve to a non-CUDA backend.
// Here there is no other backend: a device that is not sm_100 is an error.

#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "../../include/convrot.h"
#include "cr_internal.h"

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  int state = 0;  // 0 unknown, 1 supported, 2 unsupported
  int num_sms = 0;
};
DeviceInfo g_dev[kMaxDevices];

// Supported device = compute capability 10.0 (B200).  Fills *num_sms.
cr_status check_device(int* num_sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return CR_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return CR_ERR_UNSUPPORTED_ARCH;
  DeviceInfo& d = g_dev[dev];
  if (d.state == 0) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return CR_ERR_CUDA;
    }
    d.num_sms = sms;
    d.state = (major == 10 && minor == 0) ? 1 : 2;
  }
  if (d.state != 1) return CR_ERR_UNSUPPORTED_ARCH;
  *num_sms = d.num_sms;
  return CR_OK;
}

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

inline cr_status cuda_status(cudaError_t e) { return e == cudaSuccess ? CR_OK : CR_ERR_CUDA; }

// Shared shape rule for everything that rotates or multiplies along K.  The kernels work on
// 256-element units of a row, so K is a multiple of 256 for every group size.
inline cr_status check_k(int K, int group) {
  if (group != CR_GROUP_256 && group != CR_GROUP_64 && group != CR_GROUP_16 && group != CR_GROUP_1024)
    return CR_ERR_UNSUPPORTED_SHAPE;
  if (K < 256 || (K % 256) != 0 || K > CR_MAX_K || (K % group) != 0) return CR_ERR_UNSUPPORTED_SHAPE;
  return CR_OK;
}

constexpr size_t kLinScaleOff = cr::kActWsBytes;           // float a_scale (own 256-byte slot)
constexpr size_t kLinXqOff = cr::kActWsBytes + 256;        // packed activation codes

size_t act_ws_bytes() { return cr::kActWsBytes; }

inline int* ws_status(void* workspace) {
  return reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) + cr::kWsStatusOff);
}

}  // namespace

extern "C" {

const char* cr_status_string(int status) {
  switch (status) {
    case CR_OK: return "CR_OK";
    case CR_ERR_INVALID_ARG: return "CR_ERR_INVALID_ARG: null pointer, negative size or unknown enum value";
    case CR_ERR_UNSUPPORTED_SHAPE: return "CR_ERR_UNSUPPORTED_SHAPE: size breaks a shape rule (K % 256, N % 8, group, K limit)";
    case CR_ERR_MISALIGNED: return "CR_ERR_MISALIGNED: pointer or leading dimension not 16-byte aligned";
    case CR_ERR_UNSUPPORTED_ARCH: return "CR_ERR_UNSUPPORTED_ARCH: current device is not sm_100 (B200)";
    case CR_ERR_WORKSPACE: return "CR_ERR_WORKSPACE: workspace missing or too small";
    case CR_ERR_CUDA: return "CR_ERR_CUDA: a CUDA runtime or driver call failed";
    case CR_ERR_TIMEOUT: return "CR_ERR_TIMEOUT: a bounded device-side wait expired";
    default: return "CR_ERR_UNKNOWN";
  }
}

int cr_api_version(void) { return CR_API_VERSION; }

size_t cr_rotate_quant_act_workspace_size(int M, int K, int group) {
  (void)M; (void)K; (void)group;
  return act_ws_bytes();
}

size_t cr_pack_weight_workspace_size(int N, int K, int group, int scale_mode) {
  (void)N; (void)K; (void)group; (void)scale_mode;
  return act_ws_bytes();
}

size_t cr_w4a4_gemm_workspace_size(int M, int N, int K) {
  (void)M; (void)N; (void)K;
  return 256;
}

size_t cr_w4a4_linear_workspace_size(int M, int N, int K, int group) {
  (void)N; (void)group;
  if (M < 0 || K < 0) return kLinXqOff;
  return kLinXqOff + cr::round_up(static_cast<size_t>(M) * static_cast<size_t>(K) / 2, 256);
}

static cr_status rotate_quant_act_impl(const void* X, int M, int K, int64_t ldx, int group, int bits, int rotate,
                                       void* Xq, float* a_scale, void* workspace, size_t workspace_bytes,
                                       void* stream, int path = cr::kActAuto) {
  // an empty X (M == 0) may come with NULL data pointers; only a_scale is written
  if (!a_scale || M < 0 || K < 0 || ldx < 0 || (M > 0 && (!X || !Xq))) return CR_ERR_INVALID_ARG;
  if ((bits != 4 && bits != 8) || (rotate != 0 && rotate != 1)) return CR_ERR_INVALID_ARG;
  cr_status st = check_k(K, group);
  if (st != CR_OK) return st;
  if (ldx < K) return CR_ERR_INVALID_ARG;
  if (!aligned(X, 16) || !aligned(Xq, 16) || (ldx % 8) != 0 || !aligned(a_scale, 4)) return CR_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < act_ws_bytes() || !aligned(workspace, 256)) return CR_ERR_WORKSPACE;
  int nsm = 0;
  if ((st = check_device(&nsm)) != CR_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return cuda_status(cr::launch_act_fmt(static_cast<const uint16_t*>(X), M, K, ldx, static_cast<uint8_t*>(Xq), a_scale,
                                        1, bits == 4 ? cr::kFmtPacked4 : cr::kFmtByte8, rotate != 0, group,
                                        static_cast<uint8_t*>(workspace), nsm, path, s));
}

cr_status cr_selftest_act_fallback(const void* X, int M, int K, int64_t ldx, int group, int bits, int rotate,
                                   void* Xq, float* a_scale, void* workspace, size_t workspace_bytes, void* stream) {
  return rotate_quant_act_impl(X, M, K, ldx, group, bits, rotate, Xq, a_scale, workspace, workspace_bytes, stream,
                               cr::kActTwoPass);
}

cr_status cr_rotate_quant_act(const void* X, int M, int K, int64_t ldx, int group, void* Xq, float* a_scale,
                              void* workspace, size_t workspace_bytes, void* stream) {
  return rotate_quant_act_impl(X, M, K, ldx, group, 4, 1, Xq, a_scale, workspace, workspace_bytes, stream);
}

cr_status cr_rotate_quant_act_ex(const void* X, int M, int K, int64_t ldx, int group, int bits, int rotate, void* Xq,
                                 float* a_scale, void* workspace, size_t workspace_bytes, void* stream) {
  return rotate_quant_act_impl(X, M, K, ldx, group, bits, rotate, Xq, a_scale, workspace, workspace_bytes, stream);
}

static cr_status pack_weight_impl(const void* W, int N, int K, int64_t ldw, int group, int bits, int rotate,
                                  int scale_mode, void* Wq, float* w_scale, void* workspace, size_t workspace_bytes,
                                  void* stream) {
  if (N < 0 || K < 0 || ldw < 0 || (N > 0 && (!W || !Wq || !w_scale))) return CR_ERR_INVALID_ARG;
  if ((bits != 4 && bits != 8) || (rotate != 0 && rotate != 1)) return CR_ERR_INVALID_ARG;
  if (scale_mode != CR_SCALE_TENSOR && scale_mode != CR_SCALE_ROW) return CR_ERR_INVALID_ARG;
  cr_status st = check_k(K, group);
  if (st != CR_OK) return st;
  if (ldw < K) return CR_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(Wq, 16) || (ldw % 8) != 0 || !aligned(w_scale, 4)) return CR_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < act_ws_bytes() || !aligned(workspace, 256)) return CR_ERR_WORKSPACE;
  if (N == 0) return CR_OK;
  int nsm = 0;
  if ((st = check_device(&nsm)) != CR_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const uint16_t* w = static_cast<const uint16_t*>(W);
  if (scale_mode == CR_SCALE_ROW)
    return cuda_status(
        cr::launch_pack_rows_fmt(w, N, K, ldw, static_cast<uint8_t*>(Wq), w_scale,
                                 bits == 4 ? cr::kFmtPacked4 : cr::kFmtByte8, rotate != 0, group, s));
  // tensorwise: the activation path's kernels with the scale broadcast to all N entries
  return cuda_status(cr::launch_act_fmt(w, N, K, ldw, static_cast<uint8_t*>(Wq), w_scale, N,
                                        bits == 4 ? cr::kFmtPacked4 : cr::kFmtByte8, rotate != 0, group,
                                        static_cast<uint8_t*>(workspace), nsm, cr::kActAuto, s));
}

cr_status cr_pack_weight(const void* W, int N, int K, int64_t ldw, int group, int scale_mode, void* Wq,
                         float* w_scale, void* workspace, size_t workspace_bytes, void* stream) {
  return pack_weight_impl(W, N, K, ldw, group, 4, 1, scale_mode, Wq, w_scale, workspace, workspace_bytes, stream);
}

cr_status cr_pack_weight_ex(const void* W, int N, int K, int64_t ldw, int group, int bits, int rotate,
                            int scale_mode, void* Wq, float* w_scale, void* workspace, size_t workspace_bytes,
                            void* stream) {
  return pack_weight_impl(W, N, K, ldw, group, bits, rotate, scale_mode, Wq, w_scale, workspace, workspace_bytes,
                          stream);
}

static cr_status validate_gemm(const void* Xq, const float* a_scale, const void* Wq, const float* w_scale,
                               const void* bias, const void* Y, int64_t ldy, int M, int N, int K) {
  if (M < 0 || N < 0 || K < 0 || ldy < 0) return CR_ERR_INVALID_ARG;
  // empty products (M == 0 or N == 0) launch nothing and may pass NULL data pointers
  if (M > 0 && N > 0 && (!Xq || !a_scale || !Wq || !w_scale || !Y)) return CR_ERR_INVALID_ARG;
  cr_status st = check_k(K, CR_GROUP_256);
  if (st != CR_OK) return st;
  if (N % 8 != 0) return CR_ERR_UNSUPPORTED_SHAPE;
  if (ldy < N) return CR_ERR_INVALID_ARG;
  if (!aligned(Xq, 16) || !aligned(Wq, 16) || !aligned(Y, 16) || (ldy % 8) != 0 || !aligned(a_scale, 4) ||
      !aligned(w_scale, 4) || (bias && !aligned(bias, 2)))
    return CR_ERR_MISALIGNED;
  return CR_OK;
}

cr_status cr_w4a4_gemm(const void* Xq, const float* a_scale, const void* Wq, const float* w_scale, const void* bias,
                       void* Y, int64_t ldy, int M, int N, int K, void* workspace, size_t workspace_bytes,
                       void* stream) {
  cr_status st = validate_gemm(Xq, a_scale, Wq, w_scale, bias, Y, ldy, M, N, K);
  if (st != CR_OK) return st;
  if (!workspace || workspace_bytes < cr_w4a4_gemm_workspace_size(M, N, K) || !aligned(workspace, 256))
    return CR_ERR_WORKSPACE;
  int nsm = 0;
  if ((st = check_device(&nsm)) != CR_OK) return st;
  int* status = reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) + cr::kWsStatusOff);
  return static_cast<cr_status>(cr::launch_w4a4_gemm(Xq, a_scale, Wq, w_scale, bias, Y, ldy, M, N, K, status, nsm,
                                                     static_cast<cudaStream_t>(stream)));
}

cr_status cr_w4a4_gemm_s32(const void* Xq, const void* Wq, int32_t* C, int64_t ldc, int M, int N, int K,
                           void* workspace, size_t workspace_bytes, void* stream) {
  if (M < 0 || N < 0 || K < 0 || ldc < 0 || (M > 0 && N > 0 && (!Xq || !Wq || !C))) return CR_ERR_INVALID_ARG;
  cr_status st = check_k(K, CR_GROUP_256);
  if (st != CR_OK) return st;
  if (N % 8 != 0) return CR_ERR_UNSUPPORTED_SHAPE;
  if (ldc < N) return CR_ERR_INVALID_ARG;
  if (!aligned(Xq, 16) || !aligned(Wq, 16) || !aligned(C, 16) || (ldc % 4) != 0) return CR_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < cr_w4a4_gemm_workspace_size(M, N, K) || !aligned(workspace, 256))
    return CR_ERR_WORKSPACE;
  int nsm = 0;
  if ((st = check_device(&nsm)) != CR_OK) return st;
  int* status = reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) + cr::kWsStatusOff);
  return static_cast<cr_status>(
      cr::launch_w4a4_gemm_s32(Xq, Wq, C, ldc, M, N, K, status, nsm, static_cast<cudaStream_t>(stream)));
}

cr_status cr_w4a4_linear(const void* X, int64_t ldx, const void* Wq, const float* w_scale, const void* bias, void* Y,
                         int64_t ldy, int M, int N, int K, int group, void* workspace, size_t workspace_bytes,
                         void* stream) {
  return cr_w4a4_linear_ex(X, ldx, Wq, w_scale, bias, Y, ldy, M, N, K, group, CR_LINEAR_AUTO, workspace,
                           workspace_bytes, stream);
}

cr_status cr_w4a4_linear_ex(const void* X, int64_t ldx, const void* Wq, const float* w_scale, const void* bias,
                            void* Y, int64_t ldy, int M, int N, int K, int group, int mode, void* workspace,
                            size_t workspace_bytes, void* stream) {
  if (mode != CR_LINEAR_AUTO && mode != CR_LINEAR_ONE_LAUNCH && mode != CR_LINEAR_TWO_LAUNCHES)
    return CR_ERR_INVALID_ARG;
  if (ldx < 0 || (M > 0 && !X)) return CR_ERR_INVALID_ARG;
  // the GEMM's operand checks, with stand-in (aligned, non-null) pointers for the workspace-resident Xq/a_scale
  const void* stand_in = workspace ? workspace : reinterpret_cast<const void*>(uintptr_t(256));
  cr_status st = validate_gemm(stand_in, static_cast<const float*>(stand_in), Wq, w_scale, bias, Y, ldy, M, N, K);
  if (st != CR_OK) return st;
  if ((st = check_k(K, group)) != CR_OK) return st;
  if (ldx < K) return CR_ERR_INVALID_ARG;
  if (!aligned(X, 16) || (ldx % 8) != 0) return CR_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < cr_w4a4_linear_workspace_size(M, N, K, group) || !aligned(workspace, 256))
    return CR_ERR_WORKSPACE;
  int nsm = 0;
  if ((st = check_device(&nsm)) != CR_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* a_scale = reinterpret_cast<float*>(ws + kLinScaleOff);
  uint8_t* xq = ws + kLinXqOff;
  int* status = reinterpret_cast<int*>(ws + cr::kWsStatusOff);
  const uint16_t* x = static_cast<const uint16_t*>(X);
  // AUTO is the two-launch arrangement: with the few-token GEMM started as a programmatic dependent of the
  // activation pass it matches or beats the fused launch on every measured shape
  if (mode == CR_LINEAR_ONE_LAUNCH) {
    if (M == 0 || N == 0) return CR_OK;  // nothing to launch
    // few tokens: the whole layer in one launch (activation phases fused into the few-token GEMM)
    const int r = M <= cr::kSmallBigMaxM ? cr::launch_w4a4_linear_small(x, ldx, Wq, w_scale, bias, Y, ldy, M, N, K,
                                                                       group, ws, xq, a_scale, nsm, s)
                                         : cr::kNotFused;
    return r != cr::kNotFused ? static_cast<cr_status>(r) : CR_ERR_UNSUPPORTED_SHAPE;
  }
  if ((st = cuda_status(cr::launch_act_fmt(x, M, K, ldx, xq, a_scale, 1, cr::kFmtPacked4, true, group, ws, nsm,
                                           cr::kActAuto, s))) != CR_OK)
    return st;
  return static_cast<cr_status>(
      cr::launch_w4a4_gemm(xq, a_scale, Wq, w_scale, bias, Y, ldy, M, N, K, status, nsm, s, /*after_act=*/true));
}

static cr_status validate_multi(int num_proj, const void* const* Wq, const float* const* w_scale,
                                const void* const* bias, void* const* Y, const int64_t* ldy, const int* N,
                                const void* Xq, const float* a_scale, int M, int K, bool s32) {
  if (num_proj < 1 || num_proj > CR_MAX_PROJ || !Wq || !Y || !ldy || !N || (!s32 && !w_scale)) return CR_ERR_INVALID_ARG;
  for (int j = 0; j < num_proj; ++j) {
    cr_status st;
    if (s32) {
      if (M < 0 || N[j] < 0 || K < 0 || ldy[j] < 0 || (M > 0 && N[j] > 0 && (!Xq || !Wq[j] || !Y[j])))
        return CR_ERR_INVALID_ARG;
      if ((st = check_k(K, CR_GROUP_256)) != CR_OK) return st;
      if (N[j] % 8 != 0) return CR_ERR_UNSUPPORTED_SHAPE;
      if (ldy[j] < N[j]) return CR_ERR_INVALID_ARG;
      if (!aligned(Xq, 16) || !aligned(Wq[j], 16) || !aligned(Y[j], 16) || (ldy[j] % 4) != 0) return CR_ERR_MISALIGNED;
    } else {
      if ((st = validate_gemm(Xq, a_scale, Wq[j], w_scale[j], bias ? bias[j] : nullptr, Y[j], ldy[j], M, N[j], K)) !=
          CR_OK)
        return st;
    }
  }
  return CR_OK;
}

cr_status cr_w4a4_gemm_multi(const void* Xq, const float* a_scale, int M, int K, int num_proj, const void* const* Wq,
                             const float* const* w_scale, const void* const* bias, void* const* Y, const int64_t* ldy,
                             const int* N, void* workspace, size_t workspace_bytes, void* stream) {
  cr_status st = validate_multi(num_proj, Wq, w_scale, bias, Y, ldy, N, Xq, a_scale, M, K, false);
  if (st != CR_OK) return st;
  if (!workspace || workspace_bytes < cr_w4a4_gemm_workspace_size(M, 0, K) || !aligned(workspace, 256))
    return CR_ERR_WORKSPACE;
  int nsm = 0;
  if ((st = check_device(&nsm)) != CR_OK) return st;
  if (M == 0) return CR_OK;
  return static_cast<cr_status>(cr::launch_w4a4_gemm_multi(Xq, a_scale, num_proj, Wq, w_scale, bias, Y, ldy, N, M, K,
                                                           ws_status(workspace), nsm,
                                                           static_cast<cudaStream_t>(stream)));
}

cr_status cr_w4a4_gemm_multi_s32(const void* Xq, int M, int K, int num_proj, const void* const* Wq, int32_t* const* C,
                                 const int64_t* ldc, const int* N, void* workspace, size_t workspace_bytes,
                                 void* stream) {
  void* const* Cv = reinterpret_cast<void* const*>(C);
  cr_status st = validate_multi(num_proj, Wq, nullptr, nullptr, Cv, ldc, N, Xq, nullptr, M, K, true);
  if (st != CR_OK) return st;
  if (!workspace || workspace_bytes < cr_w4a4_gemm_workspace_size(M, 0, K) || !aligned(workspace, 256))
    return CR_ERR_WORKSPACE;
  int nsm = 0;
  if ((st = check_device(&nsm)) != CR_OK) return st;
  if (M == 0) return CR_OK;
  return static_cast<cr_status>(cr::launch_w4a4_gemm_multi_s32(Xq, num_proj, Wq, Cv, ldc, N, M, K,
                                                               ws_status(workspace), nsm,
                                                               static_cast<cudaStream_t>(stream)));
}

cr_status cr_w4a4_linear_multi(const void* X, int64_t ldx, int M, int K, int group, int num_proj,
                               const void* const* Wq, const float* const* w_scale, const void* const* bias,
                               void* const* Y, const int64_t* ldy, const int* N, void* workspace,
                               size_t workspace_bytes, void* stream) {
  if (ldx < 0 || M < 0 || (M > 0 && !X)) return CR_ERR_INVALID_ARG;
  const void* stand_in = workspace ? workspace : reinterpret_cast<const void*>(uintptr_t(256));
  cr_status st = validate_multi(num_proj, Wq, w_scale, bias, Y, ldy, N, stand_in,
                                static_cast<const float*>(stand_in), M, K, false);
  if (st != CR_OK) return st;
  if ((st = check_k(K, group)) != CR_OK) return st;
  if (ldx < K) return CR_ERR_INVALID_ARG;
  if (!aligned(X, 16) || (ldx % 8) != 0) return CR_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < cr_w4a4_linear_workspace_size(M, 0, K, group) || !aligned(workspace, 256))
    return CR_ERR_WORKSPACE;
  int nsm = 0;
  if ((st = check_device(&nsm)) != CR_OK) return st;
  if (M == 0) return CR_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* a_scale = reinterpret_cast<float*>(ws + kLinScaleOff);
  uint8_t* xq = ws + kLinXqOff;
  if ((st = cuda_status(cr::launch_act_fmt(static_cast<const uint16_t*>(X), M, K, ldx, xq, a_scale, 1,
                                           cr::kFmtPacked4, true, group, ws, nsm, cr::kActAuto, s))) != CR_OK)
    return st;
  return static_cast<cr_status>(
      cr::launch_w4a4_gemm_multi(xq, a_scale, num_proj, Wq, w_scale, bias, Y, ldy, N, M, K, ws_status(ws), nsm, s));
}

size_t cr_int8_gemm_workspace_size(int M, int N, int K) {
  (void)M; (void)N; (void)K;
  return 256;
}

size_t cr_int8_linear_workspace_size(int M, int N, int K, int group) {
  (void)N; (void)group;
  if (M < 0 || K < 0) return kLinXqOff;
  return kLinXqOff + cr::round_up(static_cast<size_t>(M) * static_cast<size_t>(K), 256);
}

cr_status cr_int8_gemm(const void* Xq, const float* a_scale, const void* Wq, const float* w_scale, const void* bias,
                       void* Y, int64_t ldy, int M, int N, int K, void* workspace, size_t workspace_bytes,
                       void* stream) {
  cr_status st = validate_gemm(Xq, a_scale, Wq, w_scale, bias, Y, ldy, M, N, K);
  if (st != CR_OK) return st;
  if (!workspace || workspace_bytes < cr_int8_gemm_workspace_size(M, N, K) || !aligned(workspace, 256))
    return CR_ERR_WORKSPACE;
  int nsm = 0;
  if ((st = check_device(&nsm)) != CR_OK) return st;
  return static_cast<cr_status>(cr::launch_i8_gemm(Xq, a_scale, Wq, w_scale, bias, Y, ldy, M, N, K,
                                                   ws_status(workspace), nsm, static_cast<cudaStream_t>(stream)));
}

cr_status cr_int8_gemm_s32(const void* Xq, const void* Wq, int32_t* C, int64_t ldc, int M, int N, int K,
                           void* workspace, size_t workspace_bytes, void* stream) {
  if (M < 0 || N < 0 || K < 0 || ldc < 0 || (M > 0 && N > 0 && (!Xq || !Wq || !C))) return CR_ERR_INVALID_ARG;
  cr_status st = check_k(K, CR_GROUP_256);
  if (st != CR_OK) return st;
  if (N % 8 != 0) return CR_ERR_UNSUPPORTED_SHAPE;
  if (ldc < N) return CR_ERR_INVALID_ARG;
  if (!aligned(Xq, 16) || !aligned(Wq, 16) || !aligned(C, 16) || (ldc % 4) != 0) return CR_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < cr_int8_gemm_workspace_size(M, N, K) || !aligned(workspace, 256))
    return CR_ERR_WORKSPACE;
  int nsm = 0;
  if ((st = check_device(&nsm)) != CR_OK) return st;
  return static_cast<cr_status>(
      cr::launch_i8_gemm_s32(Xq, Wq, C, ldc, M, N, K, ws_status(workspace), nsm, static_cast<cudaStream_t>(stream)));
}

cr_status cr_int8_linear(const void* X, int64_t ldx, int rotate, const void* Wq, const float* w_scale,
                         const void* bias, void* Y, int64_t ldy, int M, int N, int K, int group, void* workspace,
                         size_t workspace_bytes, void* stream) {
  if (ldx < 0 || (M > 0 && !X) || (rotate != 0 && rotate != 1)) return CR_ERR_INVALID_ARG;
  const void* stand_in = workspace ? workspace : reinterpret_cast<const void*>(uintptr_t(256));
  cr_status st = validate_gemm(stand_in, static_cast<const float*>(stand_in), Wq, w_scale, bias, Y, ldy, M, N, K);
  if (st != CR_OK) return st;
  if ((st = check_k(K, group)) != CR_OK) return st;
  if (ldx < K) return CR_ERR_INVALID_ARG;
  if (!aligned(X, 16) || (ldx % 8) != 0) return CR_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < cr_int8_linear_workspace_size(M, N, K, group) || !aligned(workspace, 256))
    return CR_ERR_WORKSPACE;
  int nsm = 0;
  if ((st = check_device(&nsm)) != CR_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* a_scale = reinterpret_cast<float*>(ws + kLinScaleOff);
  uint8_t* xq = ws + kLinXqOff;
  const uint16_t* x = static_cast<const uint16_t*>(X);
  if ((st = cuda_status(
           cr::launch_act_fmt(x, M, K, ldx, xq, a_scale, 1, cr::kFmtByte8, rotate != 0, group, ws, nsm, cr::kActAuto,
                              s))) !=
      CR_OK)
    return st;
  return static_cast<cr_status>(
      cr::launch_i8_gemm(xq, a_scale, Wq, w_scale, bias, Y, ldy, M, N, K, ws_status(ws), nsm, s));
}

size_t cr_w4a8_gemm_workspace_size(int M, int N, int K) {
  (void)M; (void)N; (void)K;
  return 256;
}

size_t cr_w4a8_linear_workspace_size(int M, int N, int K, int group) {
  return cr_int8_linear_workspace_size(M, N, K, group);
}

cr_status cr_pack_weight_w4a8(const void* W, int N, int K, int64_t ldw, int group, int rotate, void* Wq,
                              void* w_gscale, void* w_zero, void* workspace, size_t workspace_bytes, void* stream) {
  if (N < 0 || K < 0 || ldw < 0 || (N > 0 && (!W || !Wq || !w_gscale || !w_zero))) return CR_ERR_INVALID_ARG;
  if (rotate != 0 && rotate != 1) return CR_ERR_INVALID_ARG;
  cr_status st = check_k(K, group);
  if (st != CR_OK) return st;
  if (group != CR_GROUP_256) return CR_ERR_UNSUPPORTED_SHAPE;  // the W4A8 format rotates by groups of 256
  if (ldw < K) return CR_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(Wq, 16) || (ldw % 8) != 0 || !aligned(w_gscale, 4)) return CR_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < act_ws_bytes() || !aligned(workspace, 256)) return CR_ERR_WORKSPACE;
  if (N == 0) return CR_OK;
  int nsm = 0;
  if ((st = check_device(&nsm)) != CR_OK) return st;
  return cuda_status(cr::launch_pack_w4a8(static_cast<const uint16_t*>(W), N, K, ldw, rotate != 0,
                                          static_cast<uint8_t*>(Wq), w_gscale, static_cast<uint8_t*>(w_zero), nsm,
                                          static_cast<cudaStream_t>(stream)));
}

static cr_status validate_w4a8(const void* Xq, const void* Wq, const void* gscale, const void* gzero, const void* Y,
                               int64_t ldy, int M, int N, int K) {
  if (M < 0 || N < 0 || K < 0 || ldy < 0) return CR_ERR_INVALID_ARG;
  if (M > 0 && N > 0 && (!Xq || !Wq || !gscale || !gzero || !Y)) return CR_ERR_INVALID_ARG;
  cr_status st = check_k(K, CR_GROUP_256);
  if (st != CR_OK) return st;
  if (N % 8 != 0) return CR_ERR_UNSUPPORTED_SHAPE;
  if (ldy < N) return CR_ERR_INVALID_ARG;
  if (!aligned(Xq, 16) || !aligned(Wq, 16) || !aligned(Y, 16) || !aligned(gscale, 4)) return CR_ERR_MISALIGNED;
  return CR_OK;
}

cr_status cr_w4a8_gemm(const void* Xq, const float* a_scale, const void* Wq, const void* w_gscale,
                       const void* w_zero, const void* bias, void* Y, int64_t ldy, int M, int N, int K,
                       void* workspace, size_t workspace_bytes, void* stream) {
  cr_status st = validate_w4a8(Xq, Wq, w_gscale, w_zero, Y, ldy, M, N, K);
  if (st != CR_OK) return st;
  if (M > 0 && N > 0 && !a_scale) return CR_ERR_INVALID_ARG;
  if ((ldy % 8) != 0 || !aligned(a_scale, 4) || (bias && !aligned(bias, 2))) return CR_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < cr_w4a8_gemm_workspace_size(M, N, K) || !aligned(workspace, 256))
    return CR_ERR_WORKSPACE;
  int nsm = 0;
  if ((st = check_device(&nsm)) != CR_OK) return st;
  return static_cast<cr_status>(cr::launch_w4a8_gemm(Xq, a_scale, Wq, w_gscale, w_zero, bias, Y, ldy, M, N, K,
                                                     ws_status(workspace), nsm, static_cast<cudaStream_t>(stream)));
}

cr_status cr_w4a8_gemm_f32(const void* Xq, const void* Wq, const void* w_gscale, const void* w_zero, float* C,
                           int64_t ldc, int M, int N, int K, void* workspace, size_t workspace_bytes, void* stream) {
  cr_status st = validate_w4a8(Xq, Wq, w_gscale, w_zero, C, ldc, M, N, K);
  if (st != CR_OK) return st;
  if ((ldc % 4) != 0) return CR_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < cr_w4a8_gemm_workspace_size(M, N, K) || !aligned(workspace, 256))
    return CR_ERR_WORKSPACE;
  int nsm = 0;
  if ((st = check_device(&nsm)) != CR_OK) return st;
  return static_cast<cr_status>(cr::launch_w4a8_gemm_f32(Xq, Wq, w_gscale, w_zero, C, ldc, M, N, K,
                                                         ws_status(workspace), nsm,
                                                         static_cast<cudaStream_t>(stream)));
}

cr_status cr_w4a8_linear(const void* X, int64_t ldx, const void* Wq, const void* w_gscale, const void* w_zero,
                         const void* bias, void* Y, int64_t ldy, int M, int N, int K, int group, void* workspace,
                         size_t workspace_bytes, void* stream) {
  if (ldx < 0 || (M > 0 && !X)) return CR_ERR_INVALID_ARG;
  const void* stand_in = workspace ? workspace : reinterpret_cast<const void*>(uintptr_t(256));
  cr_status st = validate_w4a8(stand_in, Wq, w_gscale, w_zero, Y, ldy, M, N, K);
  if (st != CR_OK) return st;
  if ((st = check_k(K, group)) != CR_OK) return st;
  if (group != CR_GROUP_256) return CR_ERR_UNSUPPORTED_SHAPE;
  if (ldx < K) return CR_ERR_INVALID_ARG;
  if (!aligned(X, 16) || (ldx % 8) != 0 || (ldy % 8) != 0 || (bias && !aligned(bias, 2))) return CR_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < cr_w4a8_linear_workspace_size(M, N, K, group) || !aligned(workspace, 256))
    return CR_ERR_WORKSPACE;
  int nsm = 0;
  if ((st = check_device(&nsm)) != CR_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* a_scale = reinterpret_cast<float*>(ws + kLinScaleOff);
  uint8_t* xq = ws + kLinXqOff;
  const uint16_t* x = static_cast<const uint16_t*>(X);
  if ((st = cuda_status(cr::launch_act_fmt(x, M, K, ldx, xq, a_scale, 1, cr::kFmtByte8, true, group, ws, nsm, cr::kActAuto,
                                           s))) != CR_OK)
    return st;
  return static_cast<cr_status>(
      cr::launch_w4a8_gemm(xq, a_scale, Wq, w_gscale, w_zero, bias, Y, ldy, M, N, K, ws_status(ws), nsm, s));
}

size_t cr_a8w4_gemm_workspace_size(int M, int N, int K) {
  (void)M; (void)N; (void)K;
  return 256;
}

size_t cr_a8w4_linear_workspace_size(int M, int N, int K, int group) {
  return cr_int8_linear_workspace_size(M, N, K, group);
}

cr_status cr_a8w4_gemm(const void* Xq, const float* a_scale, const void* Wq, const float* w_scale, const void* bias,
                       void* Y, int64_t ldy, int M, int N, int K, void* workspace, size_t workspace_bytes,
                       void* stream) {
  cr_status st = validate_gemm(Xq, a_scale, Wq, w_scale, bias, Y, ldy, M, N, K);
  if (st != CR_OK) return st;
  if (!workspace || workspace_bytes < cr_a8w4_gemm_workspace_size(M, N, K) || !aligned(workspace, 256))
    return CR_ERR_WORKSPACE;
  int nsm = 0;
  if ((st = check_device(&nsm)) != CR_OK) return st;
  return static_cast<cr_status>(cr::launch_a8w4_gemm(Xq, a_scale, Wq, w_scale, bias, Y, ldy, M, N, K,
                                                     ws_status(workspace), nsm, static_cast<cudaStream_t>(stream)));
}

cr_status cr_a8w4_gemm_s32(const void* Xq, const void* Wq, int32_t* C, int64_t ldc, int M, int N, int K,
                           void* workspace, size_t workspace_bytes, void* stream) {
  if (M < 0 || N < 0 || K < 0 || ldc < 0 || (M > 0 && N > 0 && (!Xq || !Wq || !C))) return CR_ERR_INVALID_ARG;
  cr_status st = check_k(K, CR_GROUP_256);
  if (st != CR_OK) return st;
  if (N % 8 != 0) return CR_ERR_UNSUPPORTED_SHAPE;
  if (ldc < N) return CR_ERR_INVALID_ARG;
  if (!aligned(Xq, 16) || !aligned(Wq, 16) || !aligned(C, 16) || (ldc % 4) != 0) return CR_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < cr_a8w4_gemm_workspace_size(M, N, K) || !aligned(workspace, 256))
    return CR_ERR_WORKSPACE;
  int nsm = 0;
  if ((st = check_device(&nsm)) != CR_OK) return st;
  return static_cast<cr_status>(
      cr::launch_a8w4_gemm_s32(Xq, Wq, C, ldc, M, N, K, ws_status(workspace), nsm, static_cast<cudaStream_t>(stream)));
}

cr_status cr_a8w4_linear(const void* X, int64_t ldx, const void* Wq, const float* w_scale, const void* bias, void* Y,
                         int64_t ldy, int M, int N, int K, int group, void* workspace, size_t workspace_bytes,
                         void* stream) {
  if (ldx < 0 || (M > 0 && !X)) return CR_ERR_INVALID_ARG;
  const void* stand_in = workspace ? workspace : reinterpret_cast<const void*>(uintptr_t(256));
  cr_status st = validate_gemm(stand_in, static_cast<const float*>(stand_in), Wq, w_scale, bias, Y, ldy, M, N, K);
  if (st != CR_OK) return st;
  if ((st = check_k(K, group)) != CR_OK) return st;
  if (ldx < K) return CR_ERR_INVALID_ARG;
  if (!aligned(X, 16) || (ldx % 8) != 0) return CR_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < cr_a8w4_linear_workspace_size(M, N, K, group) || !aligned(workspace, 256))
    return CR_ERR_WORKSPACE;
  int nsm = 0;
  if ((st = check_device(&nsm)) != CR_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* a_scale = reinterpret_cast<float*>(ws + kLinScaleOff);
  uint8_t* xq = ws + kLinXqOff;
  const uint16_t* x = static_cast<const uint16_t*>(X);
  if ((st = cuda_status(cr::launch_act_fmt(x, M, K, ldx, xq, a_scale, 1, cr::kFmtByte8, true, group, ws, nsm, cr::kActAuto,
                                           s))) != CR_OK)
    return st;
  return static_cast<cr_status>(
      cr::launch_a8w4_gemm(xq, a_scale, Wq, w_scale, bias, Y, ldy, M, N, K, ws_status(ws), nsm, s));
}

cr_status cr_read_device_status(const void* workspace, int* status, void* stream) {
  if (!workspace || !status) return CR_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int v = 0;
  if (cudaMemcpyAsync(&v, static_cast<const uint8_t*>(workspace) + cr::kWsStatusOff, sizeof(int),
                      cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return CR_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return CR_ERR_CUDA;
  *status = v;
  return CR_OK;
}

}  // extern "C"
