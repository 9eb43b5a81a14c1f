// cr_internal.h -- host-side declarations shared by the library's .cu files
// (kernel launchers and workspace layout).  Not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace cr {

// ---- workspace layout (byte offsets from the workspace base) ----
// [0, 16)             device status word (int32) + padding
// [160, 168), [192, 200)  the fused few-token layer's grid barriers: 64-bit weighted arrival counter,
//                     two running-max slots (float bits, used by alternate launches)
// [224, 232), [240, 248)  the one-launch activation pass's grid barrier: the same kind of counter and
//                     max slots
// [256, 256 + 4*kMaxActBlocks)  per-block partial maxima of the activation pass
// The words below 256 start at zero (the caller zeroes the workspace once) and every kernel leaves
// them ready for the next call: counts at zero or advanced by a whole launch's weight, the next
// launch's max slot at zero, generations advanced.
constexpr size_t kWsStatusOff = 0;
constexpr size_t kWsLayerBarOff = 160;  // counter at +0, max slots at +32 and +36 bytes
constexpr size_t kWsActBarOff = 224;    // counter at +0, max slots at +16 and +20 bytes
constexpr size_t kWsPartialOff = 256;
constexpr int kMaxActBlocks = 1024;
constexpr size_t kActWsBytes = kWsPartialOff + 4 * kMaxActBlocks;  // 4352, a multiple of 256

constexpr size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---- activation path (act_kernels.cu) ----
// Grid used by the two activation kernels for `rows` x K inputs.
int act_grid(int rows, int K, int num_sms);

// The whole tensorwise activation path: one persistent launch (one CTA per SM, cooperative, grid
// barrier words in the workspace), or, when that launch cannot be made, two streaming passes
// (per-block maxima, then codes).  INT4 codes of the rotated values, packed two per byte.
// `workspace` is the caller's workspace base (status word, barrier words, partial maxima).
cudaError_t launch_act(const uint16_t* X, int rows, int K, int64_t ldx, uint8_t* Xq, float* scale_out, int nscale,
                       uint8_t* workspace, int num_sms, cudaStream_t stream);

// Same for either code format, with or without the rotation (groups of 16, 64, 256 or 1024):
// kFmtPacked4 (INT4, amax -> 7, packed two per byte) or kFmtByte8 (INT8, amax -> 127, one code
// per byte).  `path` forces a variant (tests).
constexpr int kFmtPacked4 = 4;
constexpr int kFmtByte8 = 8;
enum { kActAuto = 0, kActTwoPass = 1, kActOneLaunch = 2 };
cudaError_t launch_act_fmt(const uint16_t* X, int rows, int K, int64_t ldx, uint8_t* Xq, float* scale_out, int nscale,
                           int fmt, bool rotate, int group, uint8_t* workspace, int num_sms, int path,
                           cudaStream_t stream);

// Per-row scales (weights): one block per row, two passes over the row.
cudaError_t launch_pack_rows(const uint16_t* W, int rows, int K, int64_t ldw, uint8_t* Wq, float* w_scale,
                             cudaStream_t stream);
cudaError_t launch_pack_rows_fmt(const uint16_t* W, int rows, int K, int64_t ldw, uint8_t* Wq, float* w_scale,
                                 int fmt, bool rotate, int group, cudaStream_t stream);

// ---- one-byte activation codes x packed INT4 weights (gemm_a8w4.cu) ----
// Y = bf16(acc * a_scale[0] * w_scale[n] + bias[n]), acc = Xq . Wq^T, Xq one code per byte [M, K],
// Wq packed INT4 [N, K/2].
int launch_a8w4_gemm(const void* Xq, const float* a_scale, const void* Wq, const float* w_scale, const void* bias,
                     void* Y, int64_t ldy, int M, int N, int K, int* status, int num_sms, cudaStream_t stream);
int launch_a8w4_gemm_s32(const void* Xq, const void* Wq, int32_t* C, int64_t ldc, int M, int N, int K, int* status,
                         int num_sms, cudaStream_t stream);

// W4A8 weights: rotation (optional), per-group-16 asymmetric 4-bit codes, fp16 scales, 4-bit zeros.
cudaError_t launch_pack_w4a8(const uint16_t* W, int N, int K, int64_t ldw, bool rotate, uint8_t* Wq, void* gscale,
                             uint8_t* gzero, int num_sms, cudaStream_t stream);

// ---- W4A8 GEMM (gemm_w4a8.cu) ----
// Y = bf16(a_scale[0] * sum_k qa * s * (q - z) + bias[n]); Xq int8 [M, K], Wq packed [N, K/2].
int launch_w4a8_gemm(const void* Xq, const float* a_scale, const void* Wq, const void* gscale, const void* gzero,
                     const void* bias, void* Y, int64_t ldy, int M, int N, int K, int* status, int num_sms,
                     cudaStream_t stream);
// C = sum_k qa * fp16(s * (q - z)) in float32 (no activation scale, no bias).
int launch_w4a8_gemm_f32(const void* Xq, const void* Wq, const void* gscale, const void* gzero, float* C, int64_t ldc,
                         int M, int N, int K, int* status, int num_sms, cudaStream_t stream);

// ---- tensor maps (tmap.cu) ----
// 2-D tensor map over a [rows, cols] matrix whose rows are `row_bytes` apart.
bool make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* ptr, uint64_t rows, uint64_t cols,
                  uint64_t row_bytes, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swizzle,
                  CUtensorMapL2promotion promo);

// ---- INT8 GEMM (gemm_i8.cu) ----
// Y = bf16(acc * a_scale[0] * w_scale[n] + bias[n]), acc = Xq . Wq^T over one-byte codes.
int launch_i8_gemm(const void* Xq, const float* a_scale, const void* Wq, const float* w_scale, const void* bias,
                   void* Y, int64_t ldy, int M, int N, int K, int* status, int num_sms, cudaStream_t stream);
// C = Xq . Wq^T in int32.
int launch_i8_gemm_s32(const void* Xq, const void* Wq, int32_t* C, int64_t ldc, int M, int N, int K, int* status,
                       int num_sms, cudaStream_t stream);

// ---- GEMM (gemm_w4a4.cu) ----
// Returns CR_* status codes (int) so TMA encoding failures can be reported.
// `after_act`: the launch directly follows this library's activation pass on the same stream, whose
// CTAs all start before anything queued after it and which produced Xq and a_scale.  The few-token
// kernel then launches as a programmatic dependent of that pass (it starts while the pass runs, loads the
// weights, and waits for the pass before reading Xq or a_scale); the weights must not be written by the
// pass (they never are: it writes codes and a scale only).
int launch_w4a4_gemm(const void* Xq, const float* a_scale, const void* Wq, const float* w_scale,
                     const void* bias, void* Y, int64_t ldy, int M, int N, int K, int* status, int num_sms,
                     cudaStream_t stream, bool after_act = false);

// CTA-pair kernels (gemm_w4a4_pair.cu): 256 x 192 tiles on tcgen05 cta_group::2.
int launch_w4a4_gemm_pair(const void* Xq, const float* a_scale, const void* Wq, const float* w_scale,
                          const void* bias, void* Y, int64_t ldy, int M, int N, int K, int* status, int num_sms,
                          cudaStream_t stream);
int launch_w4a4_gemm_pair_s32(const void* Xq, const void* Wq, int32_t* C, int64_t ldc, int M, int N, int K,
                              int* status, int num_sms, cudaStream_t stream);
// Up to kMaxProj weight matrices sharing one set of activation codes, in one launch; projection j has
// N[j] output columns (N[j] == 0: left out), its own weights, scales, bias (may be null) and output.
constexpr int kMaxProj = 4;
int launch_w4a4_gemm_pair_multi(const void* Xq, const float* a_scale, int num_proj, const void* const* Wq,
                                const float* const* w_scale, const void* const* bias, void* const* Y,
                                const int64_t* ldy, const int* N, int M, int K, int* status, int num_sms,
                                cudaStream_t stream);
int launch_w4a4_gemm_pair_multi_s32(const void* Xq, int num_proj, const void* const* Wq, void* const* C,
                                    const int64_t* ldc, const int* N, int M, int K, int* status, int num_sms,
                                    cudaStream_t stream);

// Few-token kernels (gemm_w4a4_small.cu): weights on the MMA's M side, K split across a cluster;
// up to kSmallMaxM tokens with two CTAs per SM, up to kSmallBigMaxM with one CTA per SM.
constexpr int kSmallMaxM = 128;
constexpr int kSmallBigMaxM = 256;
// Whether M tokens x N outputs go to the few-token kernels (else the CTA-pair kernel): always up to
// kSmallMaxM; up to kSmallBigMaxM when the 128-row weight tiles leave room for a K split of two or more
// (one CTA per SM).
inline bool use_small_gemm(int M, int N, int num_sms) {
  return M <= kSmallMaxM || (M <= kSmallBigMaxM && 2 * ((N + 127) / 128) <= num_sms);
}
int launch_w4a4_gemm_small(const void* Xq, const float* a_scale, const void* Wq, const float* w_scale,
                           const void* bias, void* Y, int64_t ldy, int M, int N, int K, int* status, int num_sms,
                           cudaStream_t stream, bool after_act = false);
int launch_w4a4_gemm_small_s32(const void* Xq, const void* Wq, int32_t* C, int64_t ldc, int M, int N, int K,
                               int* status, int num_sms, cudaStream_t stream);
// The whole layer for M <= kSmallBigMaxM tokens in one launch: rotation, tensorwise scale and codes of X
// (written to `xq`, [M, K/2] in the workspace; the scale to `a_scale`) fused into the few-token GEMM.
// Uses the workspace's status word, grid barrier words and partial maxima.  Returns kNotFused when
// this call cannot run fused (group 1024, or not every CTA resident): the caller then runs the
// activation kernels and the few-token GEMM.
constexpr int kNotFused = -1;
int launch_w4a4_linear_small(const uint16_t* X, int64_t ldx, const void* Wq, const float* w_scale, const void* bias,
                             void* Y, int64_t ldy, int M, int N, int K, int group, uint8_t* workspace, uint8_t* xq,
                             float* a_scale, int num_sms, cudaStream_t stream);

// Several projections of the same activation codes (CTA-pair kernel: one launch over all of them;
// few tokens: one few-token launch per projection).
int launch_w4a4_gemm_multi(const void* Xq, const float* a_scale, int num_proj, const void* const* Wq,
                           const float* const* w_scale, const void* const* bias, void* const* Y, const int64_t* ldy,
                           const int* N, int M, int K, int* status, int num_sms, cudaStream_t stream);
int launch_w4a4_gemm_multi_s32(const void* Xq, int num_proj, const void* const* Wq, void* const* C,
                               const int64_t* ldc, const int* N, int M, int K, int* status, int num_sms,
                               cudaStream_t stream);

// Raw int32 product C[M, N] = sum_k qa*qw (same kernel, integer epilogue).
int launch_w4a4_gemm_s32(const void* Xq, const void* Wq, int32_t* C, int64_t ldc, int M, int N, int K, int* status,
                         int num_sms, cudaStream_t stream);

}  // namespace cr
