// gemm_w4a4.cu -- dispatch of the INT4 x INT4 GEMM with the rank-one scale + bias
// epilogue ("Qwen-Image-Edit-2511 -- INT4 tensorwise W4A4 (+ConvRot, mixed int8
// fallback)", section "Measurements": an s4 MMA scaled by a rank-one activation
// scale x weight scale factor) between its two sm_100a kernels:
//   * M <= kSmallMaxM tokens: the few-token kernel (gemm_w4a4_small.cu), weights
//     on the MMA's M side, K split over a cluster, bound by the weight stream;
//   * more tokens: the CTA-pair kernel (gemm_w4a4_pair.cu), 256 x 192 tiles.
// Both widen the packed codes to int8 in the kernel and multiply them with the
// exact 8-bit integer MMA (B200 tensor cores have no 4-bit integer MMA).

#include <cuda_runtime.h>

#include <cstdint>

#include "cr_internal.h"

namespace cr {

// Few tokens (M <= kSmallMaxM): the weight stream bounds the layer, the swapped-operand kernel keeps
// every SM streaming; more tokens: the CTA-pair kernel.
int launch_w4a4_gemm(const void* Xq, const float* a_scale, const void* Wq, const float* w_scale, const void* bias,
                     void* Y, int64_t ldy, int M, int N, int K, int* status, int num_sms, cudaStream_t stream,
                     bool after_act) {
  if (use_small_gemm(M, N, num_sms))
    return launch_w4a4_gemm_small(Xq, a_scale, Wq, w_scale, bias, Y, ldy, M, N, K, status, num_sms, stream,
                                  after_act);
  return launch_w4a4_gemm_pair(Xq, a_scale, Wq, w_scale, bias, Y, ldy, M, N, K, status, num_sms, stream);
}

int launch_w4a4_gemm_s32(const void* Xq, const void* Wq, int32_t* C, int64_t ldc, int M, int N, int K, int* status,
                         int num_sms, cudaStream_t stream) {
  if (use_small_gemm(M, N, num_sms))
    return launch_w4a4_gemm_small_s32(Xq, Wq, C, ldc, M, N, K, status, num_sms, stream);
  return launch_w4a4_gemm_pair_s32(Xq, Wq, C, ldc, M, N, K, status, num_sms, stream);
}

int launch_w4a4_gemm_multi(const void* Xq, const float* a_scale, int num_proj, const void* const* Wq,
                           const float* const* w_scale, const void* const* bias, void* const* Y, const int64_t* ldy,
                           const int* N, int M, int K, int* status, int num_sms, cudaStream_t stream) {
  if (M > kSmallMaxM)  // one launch over every projection; per-projection few-token launches below
    return launch_w4a4_gemm_pair_multi(Xq, a_scale, num_proj, Wq, w_scale, bias, Y, ldy, N, M, K, status, num_sms,
                                       stream);
  for (int j = 0; j < num_proj; ++j) {
    const int st = launch_w4a4_gemm_small(Xq, a_scale, Wq[j], w_scale[j], bias ? bias[j] : nullptr, Y[j], ldy[j], M,
                                          N[j], K, status, num_sms, stream);
    if (st != 0) return st;
  }
  return 0;
}

int launch_w4a4_gemm_multi_s32(const void* Xq, int num_proj, const void* const* Wq, void* const* C,
                               const int64_t* ldc, const int* N, int M, int K, int* status, int num_sms,
                               cudaStream_t stream) {
  if (M > kSmallMaxM)
    return launch_w4a4_gemm_pair_multi_s32(Xq, num_proj, Wq, C, ldc, N, M, K, status, num_sms, stream);
  for (int j = 0; j < num_proj; ++j) {
    const int st = launch_w4a4_gemm_small_s32(Xq, Wq[j], static_cast<int32_t*>(C[j]), ldc[j], M, N[j], K, status,
                                              num_sms, stream);
    if (st != 0) return st;
  }
  return 0;
}

}  // namespace cr
