// cr_internal.h -- host-side declarations shared by the library's .cu files
// (kernel launchers and workspace layout).  Not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace cr {

// ---- workspace layout (byte offsets from the workspace base) ----
// [0, 16)             device status word (int32) + padding
// [64, 68), [128, 132) arrival count and generation of the fused activation pass's grid barrier
// [256, 256 + 4*kMaxActBlocks)  per-block partial maxima of the activation pass
constexpr size_t kWsStatusOff = 0;
constexpr size_t kWsBarrierOff = 64;  // count at +0, generation at +64 bytes
constexpr size_t kWsPartialOff = 256;
constexpr int kMaxActBlocks = 1024;
constexpr size_t kActWsBytes = kWsPartialOff + 4 * kMaxActBlocks;  // 4352, a multiple of 256

constexpr size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---- activation path (act_kernels.cu) ----
// Grid used by the two activation kernels for `rows` x K inputs.
int act_grid(int rows, int K, int num_sms);

// Pass 1: per-block maxima of |16 * (x H)| into partial[0 .. grid).
// `status` (device, may be NULL) receives CR_ERR_TIMEOUT if a bounded wait expires.
cudaError_t launch_act_amax(const uint16_t* X, int rows, int K, int64_t ldx, float* partial, int grid, int* status,
                            cudaStream_t stream);

// Pass 2: tensorwise scale from the partial maxima, codes, packing.  Writes
// scale_out[0 .. nscale) = s (the scale of the rotated values).
cudaError_t launch_act_quant(const uint16_t* X, int rows, int K, int64_t ldx, const float* partial, int npartial,
                             uint8_t* Xq, float* scale_out, int nscale, int grid, int* status, cudaStream_t stream);

// The whole tensorwise activation path: the fused single pass when the tensor fits on chip (one CTA
// per SM, cooperative launch, grid barrier words in the workspace), else the two streaming passes.
// `workspace` is the caller's workspace base (status word, barrier words, partial maxima).
cudaError_t launch_act(const uint16_t* X, int rows, int K, int64_t ldx, uint8_t* Xq, float* scale_out, int nscale,
                       uint8_t* workspace, int num_sms, cudaStream_t stream);
bool act_fused_fits(int rows, int K, int num_sms);
cudaError_t launch_act_fused(const uint16_t* X, int rows, int K, int64_t ldx, uint8_t* Xq, float* scale_out, int nscale,
                             float* partial, unsigned int* bar_words, int* status, int num_sms, cudaStream_t stream);

// Per-row scales (weights): one block per row, two passes over the row.
cudaError_t launch_pack_rows(const uint16_t* W, int rows, int K, int64_t ldw, uint8_t* Wq, float* w_scale,
                             cudaStream_t stream);

// ---- GEMM (gemm_w4a4.cu) ----
// Returns CR_* status codes (int) so TMA encoding failures can be reported.
int launch_w4a4_gemm(const void* Xq, const float* a_scale, const void* Wq, const float* w_scale,
                     const void* bias, void* Y, int64_t ldy, int M, int N, int K, int* status, int num_sms,
                     cudaStream_t stream);

// CTA-pair kernels (gemm_w4a4_pair.cu): 256 x 192 tiles on tcgen05 cta_group::2.
int launch_w4a4_gemm_pair(const void* Xq, const float* a_scale, const void* Wq, const float* w_scale,
                          const void* bias, void* Y, int64_t ldy, int M, int N, int K, int* status, int num_sms,
                          cudaStream_t stream);
int launch_w4a4_gemm_pair_s32(const void* Xq, const void* Wq, int32_t* C, int64_t ldc, int M, int N, int K,
                              int* status, int num_sms, cudaStream_t stream);

// Few-token kernels (gemm_w4a4_small.cu): weights on the MMA's M side, K split across a cluster.
constexpr int kSmallMaxM = 128;
int launch_w4a4_gemm_small(const void* Xq, const float* a_scale, const void* Wq, const float* w_scale,
                           const void* bias, void* Y, int64_t ldy, int M, int N, int K, int* status, int num_sms,
                           cudaStream_t stream);
int launch_w4a4_gemm_small_s32(const void* Xq, const void* Wq, int32_t* C, int64_t ldc, int M, int N, int K,
                               int* status, int num_sms, cudaStream_t stream);

// Raw int32 product C[M, N] = sum_k qa*qw (same kernel, integer epilogue).
int launch_w4a4_gemm_s32(const void* Xq, const void* Wq, int32_t* C, int64_t ldc, int M, int N, int K, int* status,
                         int num_sms, cudaStream_t stream);

}  // namespace cr
