/*
 * convrot.h -- C ABI of the B200 (sm_100a) ConvRot W4A4 linear-layer library.
 *
 * The layer (model cards "Qwen-Image-Edit-2511 -- INT4 tensorwise W4A4
 * (+ConvRot, mixed int8 fallback)", introduction and section "Measurements";
 * "Qwen3-4B -- ConvRot W4A4 (ComfyUI text encoder)", section "Format"):
 *
 *   offline : Wq, s_w = pack(rotate(W))                (cr_pack_weight)
 *   online  : Xq, s_a = quantise(rotate(X))            (cr_rotate_quant_act)
 *             Y = bf16( (Xq . Wq^T) * s_a * s_w[n] + bias[n] )   (cr_w4a4_gemm)
 *
 * rotate() multiplies every contiguous 256-wide slice of a row by the regular
 * Hadamard matrix H256 = (J-2I) (x) (J-2I) (x) (J-2I) (x) (J-2I) / 16 (with
 * `group` 1024, 64 or 16: every slice of that width by the Kronecker power of
 * (J-2I) of that order over sqrt(group), e.g. H16 = (J-2I)^(x)2 / 4).
 * quantise() uses one scale for the whole tensor, s = amax / 7 (float32),
 * codes q = clamp(round_half_even(y / s), -8, 7); packing puts element 2j in
 * the low nibble of byte j and element 2j+1 in the high nibble (two's
 * complement).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every data pointer is a DEVICE pointer owned by the caller.  The library
 *   never allocates or frees device memory and keeps no per-call state.
 * - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *   Calls are asynchronous: CR_OK means the work was enqueued on `stream`.
 * - Arguments are validated on the host before anything is enqueued; on any
 *   error nothing is launched.  Validation order: null pointers and sizes,
 *   shape rules, alignment, workspace, then the device (must be sm_100).
 * - An empty operand (a size of 0) may be passed as NULL.
 * - bfloat16 tensors are passed as raw 16-bit storage.  Row-major layouts;
 *   leading dimensions (`ld*`) are in elements.
 * - `workspace` is caller-owned device scratch of at least the size returned
 *   by the matching *_workspace_size() function, 256-byte aligned.  Its first
 *   256 bytes must be zero before the first use of the workspace: the first
 *   16 hold a device status word (kernels only ever write an error code into
 *   it), the rest the words of the library's grid-wide barriers, which every
 *   call leaves ready for the next.  A call that stopped on a device-side
 *   timeout (status CR_ERR_TIMEOUT) may leave them inconsistent: zero the
 *   256 bytes again before reusing such a workspace.
 *   Calls that share a workspace must be ordered on one stream.
 * - No C++ exception crosses this boundary.  No CPU fallback exists: on a
 *   device other than sm_100 every compute call returns
 *   CR_ERR_UNSUPPORTED_ARCH.
 */
#ifndef CONVROT_H_
#define CONVROT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define CR_API_VERSION 1

typedef enum cr_status {
  CR_OK = 0,
  CR_ERR_INVALID_ARG = 1,       /* null pointer, negative size or unknown enum value */
  CR_ERR_UNSUPPORTED_SHAPE = 2, /* a size breaks a shape rule stated below */
  CR_ERR_MISALIGNED = 3,        /* a pointer or leading dimension breaks an alignment rule */
  CR_ERR_UNSUPPORTED_ARCH = 4,  /* the current device is not compute capability 10.0 */
  CR_ERR_WORKSPACE = 5,         /* workspace is NULL or smaller than required */
  CR_ERR_CUDA = 6,              /* a CUDA runtime or driver call failed */
  CR_ERR_TIMEOUT = 7            /* a bounded device-side wait expired (device status word) */
} cr_status;

/* Weight scale granularity for cr_pack_weight. */
enum { CR_SCALE_TENSOR = 0, CR_SCALE_ROW = 1 };

/* Rotation group sizes: the model cards build with convrot_groupsize 256; the
 * W4A4 format also accepts 16 / 64 / 1024 ("Qwen-Image-Edit-2511 -- W4A8
 * ConvRot", notes on convrot_groupsize).  All four are built for W4A4, INT8
 * and the INT8 branch; W4A8 takes 256 only, as its format does.  K is a
 * multiple of 256 for every group size, and of 1024 for group 1024. */
enum { CR_GROUP_16 = 16, CR_GROUP_64 = 64, CR_GROUP_256 = 256, CR_GROUP_1024 = 1024 };

/* Largest K accepted by the GEMMs: the int32 accumulators stay exact (INT4: the
 * widened 16*q products; INT8: |acc| <= 2^14 K). */
#define CR_MAX_K 65536

/* Human-readable name of a status code (static storage; never NULL). */
const char* cr_status_string(int status);

/* CR_API_VERSION of the loaded library. */
int cr_api_version(void);

/* Workspace sizes in bytes for the calls below (0 is never returned). */
size_t cr_rotate_quant_act_workspace_size(int M, int K, int group);
size_t cr_pack_weight_workspace_size(int N, int K, int group, int scale_mode);
size_t cr_w4a4_gemm_workspace_size(int M, int N, int K);
size_t cr_w4a4_linear_workspace_size(int M, int N, int K, int group);
size_t cr_int8_gemm_workspace_size(int M, int N, int K);
size_t cr_int8_linear_workspace_size(int M, int N, int K, int group);
size_t cr_w4a8_gemm_workspace_size(int M, int N, int K);
size_t cr_a8w4_gemm_workspace_size(int M, int N, int K);
size_t cr_a8w4_linear_workspace_size(int M, int N, int K, int group);
size_t cr_w4a8_linear_workspace_size(int M, int N, int K, int group);

/* Code formats of the *_ex calls: `bits` 4 = signed INT4, amax -> 7, packed two
 * per byte (element 2j in the low nibble of byte j); 8 = signed INT8,
 * amax -> 127, one code per byte.  `rotate` 1 = the ConvRot rotation (slices of
 * `group` elements) is applied first, 0 = the values are quantised as they are. */
enum { CR_BITS_4 = 4, CR_BITS_8 = 8 };

/*
 * cr_pack_weight -- offline weight preparation.
 * Model card "Qwen3-4B -- ConvRot W4A4 (ComfyUI text encoder)", section
 * "Format": weight stored as I8 [rows, cols/2] holding signed INT4 plus
 * weight_scale F32 [rows]; weights rotated with the same group-256 regular
 * Hadamard as the activations ("Qwen-Image-Edit-2511 -- INT4 tensorwise W4A4
 * (+ConvRot, mixed int8 fallback)", introduction).
 *
 *   W        bf16 [N, K], row stride ldw >= K elements (16-byte aligned rows)
 *   group    rotation group: CR_GROUP_256 (the cards' builds), CR_GROUP_1024, _64 or _16
 *   scale_mode CR_SCALE_TENSOR: one scale amax(|W H|)/7 written to all N
 *            entries of w_scale;  CR_SCALE_ROW: one scale per row.
 *   Wq       out: uint8 [N, K/2], dense (row stride K/2 bytes)
 *   w_scale  out: float32 [N]
 * Shape rules: N >= 0, K >= 256, K % 256 == 0, K % group == 0, K <= CR_MAX_K.
 * Alignment: W, Wq 16-byte aligned; ldw % 8 == 0; w_scale 4-byte aligned.
 */
cr_status cr_pack_weight(const void* W, int N, int K, int64_t ldw, int group, int scale_mode,
                         void* Wq, float* w_scale, void* workspace, size_t workspace_bytes,
                         void* stream);

/*
 * cr_rotate_quant_act -- online activation path: rotate every group-slice of
 * every row of X by H_group (float32), take one dynamic tensorwise scale
 * s_a = amax/7 over the whole rotated tensor, write INT4 codes packed two per
 * byte.  ("Qwen-Image-Edit-2511 -- INT4 tensorwise W4A4 (+ConvRot, mixed int8
 * fallback)", introduction: activations rotated online and dynamically
 * quantised to INT4, calibration-free.)
 *
 *   X        bf16 [M, K], row stride ldx >= K elements
 *   Xq       out: uint8 [M, K/2], dense
 *   a_scale  out: one float32 in device memory (s_a; 1.0 if X is all zero)
 * Shape rules: M >= 0 (M == 0 writes only a_scale = 1), K >= 256,
 * K % 256 == 0, K % group == 0, K <= CR_MAX_K.
 * Alignment: X, Xq 16-byte aligned; ldx % 8 == 0.
 * Inputs must be finite.
 */
cr_status cr_rotate_quant_act(const void* X, int M, int K, int64_t ldx, int group,
                              void* Xq, float* a_scale, void* workspace, size_t workspace_bytes,
                              void* stream);

/*
 * cr_pack_weight_ex, cr_rotate_quant_act_ex -- the same two calls for any
 * code format (bits 4 or 8, rotation on or off; see CR_BITS_*).  The INT8
 * tensorwise format, with or without the rotation, is the fallback format of
 * the model cards ("Qwen-Image-Edit-2511 -- INT4 tensorwise W4A4 (+ConvRot,
 * mixed int8 fallback)", introduction: sensitive layers kept as
 * int8_tensorwise; "Qwen Image 2.1 -- Hybrid W4A8 / INT8 ConvRot", layer
 * list: INT8 tensorwise + ConvRot).  Scales: s = amax / 7 (bits 4) or
 * amax / 127 (bits 8) over the (rotated) values, float32; 1.0 for an all-zero
 * tensor; codes round_half_even(y / s).
 *   Wq / Xq  out: uint8 [rows, K/2] for bits 4, int8 [rows, K] for bits 8 (dense)
 * `group` is 16, 64, 256 or 1024 (checked also when rotate is 0).  Other arguments, shape and
 * alignment rules: as cr_pack_weight / cr_rotate_quant_act.  bits outside
 * {4, 8} or rotate outside {0, 1}: CR_ERR_INVALID_ARG.
 * cr_pack_weight(...) == cr_pack_weight_ex(..., 4, 1, ...) and likewise for
 * the activation call.
 */
cr_status cr_pack_weight_ex(const void* W, int N, int K, int64_t ldw, int group, int bits, int rotate,
                            int scale_mode, void* Wq, float* w_scale, void* workspace,
                            size_t workspace_bytes, void* stream);
cr_status cr_rotate_quant_act_ex(const void* X, int M, int K, int64_t ldx, int group, int bits, int rotate,
                                 void* Xq, float* a_scale, void* workspace, size_t workspace_bytes,
                                 void* stream);

/*
 * cr_w4a4_gemm -- integer product of packed INT4 activations and weights with
 * the rank-one scale and bias epilogue ("Qwen-Image-Edit-2511 -- INT4
 * tensorwise W4A4 (+ConvRot, mixed int8 fallback)", section "Measurements":
 * rank-one s4 MMA).
 *
 *   Xq       uint8 [M, K/2] (from cr_rotate_quant_act), dense
 *   a_scale  one float32 (device)
 *   Wq       uint8 [N, K/2] (from cr_pack_weight), dense
 *   w_scale  float32 [N] (device)
 *   bias     bf16 [N] (device) or NULL for no bias
 *   Y        out: bf16 [M, N], row stride ldy >= N elements
 * Y[m,n] = bf16_rn( acc[m,n] * a_scale * w_scale[n] + bias[n] ) with
 * acc = sum_k qa[m,k]*qw[n,k] exact in int32.
 * Shape rules: M >= 0, N >= 0, N % 8 == 0, K >= 256, K % 256 == 0,
 * K <= CR_MAX_K (M == 0 or N == 0: nothing is launched).
 * Alignment: Xq, Wq, Y 16-byte aligned; ldy % 8 == 0.
 */
cr_status cr_w4a4_gemm(const void* Xq, const float* a_scale, const void* Wq, const float* w_scale,
                       const void* bias, void* Y, int64_t ldy, int M, int N, int K,
                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * cr_w4a4_gemm_s32 -- the integer product alone: C[m,n] = sum_k qa[m,k]*qw[n,k]
 * as int32, exact (|C| <= 64*K).  Same main loop as cr_w4a4_gemm with an
 * integer epilogue; for callers that apply their own scales and for checking
 * the accumulators bit for bit.
 *
 *   Xq  uint8 [M, K/2], Wq uint8 [N, K/2] (dense), C out: int32 [M, N] with
 *   row stride ldc >= N elements.
 * Shape rules as cr_w4a4_gemm.  Alignment: Xq, Wq, C 16-byte aligned;
 * ldc % 4 == 0.
 */
cr_status cr_w4a4_gemm_s32(const void* Xq, const void* Wq, int32_t* C, int64_t ldc, int M, int N, int K,
                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * cr_int8_gemm -- the INT8 layer's product: codes one per byte (from the
 * *_ex calls with bits 8), the same rank-one scale and bias epilogue as
 * cr_w4a4_gemm:
 *   Y[m,n] = bf16_rn( acc[m,n] * a_scale * w_scale[n] + bias[n] ),
 *   acc = sum_k qa[m,k]*qw[n,k] exact in int32 (|acc| <= 2^14 K).
 *   Xq  int8 [M, K], Wq int8 [N, K] (dense rows of K bytes)
 * Shape and alignment rules as cr_w4a4_gemm.
 * cr_int8_gemm_s32 -- the integer product alone, C int32 [M, N] (rules as
 * cr_w4a4_gemm_s32).
 */
cr_status cr_int8_gemm(const void* Xq, const float* a_scale, const void* Wq, const float* w_scale,
                       const void* bias, void* Y, int64_t ldy, int M, int N, int K,
                       void* workspace, size_t workspace_bytes, void* stream);
cr_status cr_int8_gemm_s32(const void* Xq, const void* Wq, int32_t* C, int64_t ldc, int M, int N, int K,
                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * cr_int8_linear -- the whole INT8 layer in one call: cr_rotate_quant_act_ex
 * with bits 8 (rotation if `rotate` is 1) followed by cr_int8_gemm, with Xq
 * and a_scale kept in the workspace (cr_int8_linear_workspace_size).  Wq and
 * w_scale come from cr_pack_weight_ex with bits 8 and the same `rotate`.
 */
cr_status cr_int8_linear(const void* X, int64_t ldx, int rotate, const void* Wq, const float* w_scale,
                         const void* bias, void* Y, int64_t ldy, int M, int N, int K, int group,
                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * The "INT8 branch" of the W4A4 format: INT8 activation codes against the W4A4
 * format's packed INT4 weights ("Qwen3-4B -- ConvRot W4A4 (ComfyUI text
 * encoder)", section "Hardware": newer GPUs run the format's INT8 activation
 * branch).
 *
 * cr_a8w4_gemm -- Y[m,n] = bf16_rn( acc[m,n] * a_scale * w_scale[n] + bias[n] ),
 * acc = sum_k qa[m,k]*qw[n,k] exact in int32 (|acc| <= 2^10 K).
 *   Xq int8 [M, K] (cr_rotate_quant_act_ex with bits 8, rotate 1), Wq / w_scale
 *   from cr_pack_weight (INT4, packed), other arguments as cr_w4a4_gemm.
 * Shape and alignment rules as cr_w4a4_gemm.
 * cr_a8w4_gemm_s32 -- the integer product alone (rules as cr_w4a4_gemm_s32).
 * cr_a8w4_linear -- the whole layer: rotation + INT8 activation codes kept in the
 * workspace (cr_a8w4_linear_workspace_size), then cr_a8w4_gemm.
 */
cr_status cr_a8w4_gemm(const void* Xq, const float* a_scale, const void* Wq, const float* w_scale,
                       const void* bias, void* Y, int64_t ldy, int M, int N, int K,
                       void* workspace, size_t workspace_bytes, void* stream);
cr_status cr_a8w4_gemm_s32(const void* Xq, const void* Wq, int32_t* C, int64_t ldc, int M, int N, int K,
                           void* workspace, size_t workspace_bytes, void* stream);
cr_status cr_a8w4_linear(const void* X, int64_t ldx, const void* Wq, const float* w_scale,
                         const void* bias, void* Y, int64_t ldy, int M, int N, int K, int group,
                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * W4A8: asymmetric 4-bit weights with an fp16 scale and a 4-bit zero point
 * per group of 16 consecutive K elements, INT8 tensorwise activations, both
 * rotated by the group-256 ConvRot rotation ("Qwen-Image-Edit-2511 -- W4A8
 * ConvRot", build table and file layout: asym_w4a8_int8, group_size 16,
 * convrot_groupsize 256; "Qwen Image 2.1 -- Hybrid W4A8 / INT8 ConvRot",
 * recipe).
 *
 * cr_pack_weight_w4a8 -- offline: per group of 16 of the (rotated) row, with
 * lo / hi its min / max (float32):
 *   s = fp16(fl(hi - lo) / 15), 1 if that is 0;  z = clamp(rne(-lo / s), 0, 15);
 *   q = clamp(rne(w / s) + z, 0, 15)
 *   Wq       out: uint8 [N, K/2], element 2j in the low nibble of byte j (dense)
 *   w_gscale out: fp16 [N, K/16] (dense, 4-byte aligned)
 *   w_zero   out: uint8 [N, K/32], group 2j in the low nibble of byte j (dense)
 *   rotate   1 = rotate the rows first (the format's definition), 0 = not
 * Workspace: cr_pack_weight_workspace_size.  Other rules as cr_pack_weight.
 *
 * cr_w4a8_gemm -- Y[m,n] = bf16_rn( a_scale * sum_k qa[m,k] * w^[n,k] + bias[n] )
 * with w^ = s * (q - z) rounded once to fp16 and the sum in float32 on the
 * tensor cores (fp16 operands: the INT8 codes are exact in fp16).
 *   Xq int8 [M, K] (cr_rotate_quant_act_ex with bits 8, rotate 1), a_scale one
 *   float32, Wq / w_gscale / w_zero from cr_pack_weight_w4a8, bias bf16 [N] or
 *   NULL, Y bf16 [M, N] with row stride ldy.
 * Shape and alignment rules as cr_w4a4_gemm; w_gscale 4-byte aligned.
 * cr_w4a8_gemm_f32 -- the float32 sums alone (no a_scale, no bias), C float32
 * [M, N] with row stride ldc (ldc % 4 == 0, C 16-byte aligned).
 * cr_w4a8_linear -- the whole layer: rotation + INT8 activation codes kept in
 * the workspace (cr_w4a8_linear_workspace_size), then cr_w4a8_gemm.
 */
cr_status cr_pack_weight_w4a8(const void* W, int N, int K, int64_t ldw, int group, int rotate, void* Wq,
                              void* w_gscale, void* w_zero, void* workspace, size_t workspace_bytes,
                              void* stream);
cr_status cr_w4a8_gemm(const void* Xq, const float* a_scale, const void* Wq, const void* w_gscale,
                       const void* w_zero, const void* bias, void* Y, int64_t ldy, int M, int N, int K,
                       void* workspace, size_t workspace_bytes, void* stream);
cr_status cr_w4a8_gemm_f32(const void* Xq, const void* Wq, const void* w_gscale, const void* w_zero,
                           float* C, int64_t ldc, int M, int N, int K, void* workspace,
                           size_t workspace_bytes, void* stream);
cr_status cr_w4a8_linear(const void* X, int64_t ldx, const void* Wq, const void* w_gscale,
                         const void* w_zero, const void* bias, void* Y, int64_t ldy, int M, int N, int K,
                         int group, void* workspace, size_t workspace_bytes, void* stream);

/*
 * cr_w4a4_linear -- the whole online layer in one call:
 * cr_rotate_quant_act followed by cr_w4a4_gemm, with Xq and a_scale kept in
 * the workspace.  Arguments as above; the shape and alignment rules of both
 * calls apply.
 */
cr_status cr_w4a4_linear(const void* X, int64_t ldx, const void* Wq, const float* w_scale,
                         const void* bias, void* Y, int64_t ldy, int M, int N, int K, int group,
                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * cr_w4a4_linear_ex -- cr_w4a4_linear with the launch arrangement chosen by
 * the caller; the outputs are the same bit for bit in every mode.
 *   CR_LINEAR_AUTO        what cr_w4a4_linear does: two launches (for few
 *                         tokens the GEMM starts beside the activation pass and
 *                         waits for it on the device; measured on B200 this
 *                         matches or beats the one-launch arrangement on every
 *                         shape tried, 1 to 256 tokens)
 *   CR_LINEAR_ONE_LAUNCH  rotation, scale, codes and the few-token GEMM in one
 *                         cooperative launch: M <= 256 and a group of 16, 64
 *                         or 256; CR_ERR_UNSUPPORTED_SHAPE otherwise, or when
 *                         the device cannot hold every CTA of the launch at once
 *   CR_LINEAR_TWO_LAUNCHES  cr_rotate_quant_act, then cr_w4a4_gemm (its few-token
 *                         kernel launched as a programmatic dependent of the
 *                         activation pass)
 * Any other mode: CR_ERR_INVALID_ARG.  Other arguments as cr_w4a4_linear.
 */
#define CR_LINEAR_AUTO 0
#define CR_LINEAR_ONE_LAUNCH 1
#define CR_LINEAR_TWO_LAUNCHES 2
cr_status cr_w4a4_linear_ex(const void* X, int64_t ldx, const void* Wq, const float* w_scale,
                            const void* bias, void* Y, int64_t ldy, int M, int N, int K, int group,
                            int mode, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Shared activation quantisation for split projections: one set of activation
 * codes feeds several weight matrices (e.g. the query, key and value
 * projections of one input), so the rotation and quantisation of X run once.
 * ("qwen-image-edit-2511-int4-comfy", section "Key Technical Optimizations",
 * "Split QKV with Shared Quantization": projections that share an input
 * quantise the activations once and feed separate Q/K/V weight paths; that
 * page's method is SVDQuant, this is the same arrangement for ConvRot W4A4.)
 *
 * cr_w4a4_gemm_multi -- for j < num_proj (1 <= num_proj <= CR_MAX_PROJ):
 *   Y[j][m,n] = bf16_rn( acc_j[m,n] * a_scale * w_scale[j][n] + bias[j][n] ),
 *   acc_j = sum_k qa[m,k] * qw_j[n,k] exact in int32,
 * i.e. cr_w4a4_gemm once per projection, bit for bit, but for M > 128 in ONE
 * launch whose tiles cover every projection (for M <= 128 one few-token launch
 * per projection).
 *   Xq, a_scale  as cr_w4a4_gemm (shared by all projections)
 *   Wq[j]        uint8 [N[j], K/2] (cr_pack_weight), dense
 *   w_scale[j]   float32 [N[j]]
 *   bias         NULL (no bias anywhere) or an array whose entries are bf16 [N[j]] or NULL
 *   Y[j]         out: bf16 [M, N[j]], row stride ldy[j] >= N[j]
 * Wq, w_scale, bias, Y, ldy and N are HOST arrays of num_proj entries, read
 * during the call only; the entries are device pointers.  Each projection
 * obeys cr_w4a4_gemm's shape and alignment rules (N[j] == 0 is allowed and
 * leaves that projection out).  Workspace: cr_w4a4_gemm_workspace_size.
 * cr_w4a4_gemm_multi_s32 -- the integer products alone, C[j] int32 [M, N[j]]
 * with row stride ldc[j] (rules as cr_w4a4_gemm_s32).
 * cr_w4a4_linear_multi -- the whole layer for all projections: one
 * cr_rotate_quant_act of X (codes and scale kept in the workspace,
 * cr_w4a4_linear_workspace_size(M, 0, K, group)) followed by
 * cr_w4a4_gemm_multi: two launches in all for M > 128.
 */
#define CR_MAX_PROJ 4
cr_status cr_w4a4_gemm_multi(const void* Xq, const float* a_scale, int M, int K, int num_proj,
                             const void* const* Wq, const float* const* w_scale, const void* const* bias,
                             void* const* Y, const int64_t* ldy, const int* N,
                             void* workspace, size_t workspace_bytes, void* stream);
cr_status cr_w4a4_gemm_multi_s32(const void* Xq, int M, int K, int num_proj, const void* const* Wq,
                                 int32_t* const* C, const int64_t* ldc, const int* N,
                                 void* workspace, size_t workspace_bytes, void* stream);
cr_status cr_w4a4_linear_multi(const void* X, int64_t ldx, int M, int K, int group, int num_proj,
                               const void* const* Wq, const float* const* w_scale, const void* const* bias,
                               void* const* Y, const int64_t* ldy, const int* N,
                               void* workspace, size_t workspace_bytes, void* stream);

/*
 * cr_w4a4_linear_noalloc -- the whole online layer (as cr_w4a4_linear) for
 * callers that cannot allocate device memory: no workspace argument, and the
 * library allocates nothing either.  The model cards have no counterpart to
 * this entry point; it exists for code that runs where cudaMalloc is
 * forbidden or unavailable (inside another framework's graph-capture region,
 * under a fixed memory pool, or on a host thread that must not synchronise
 * the device by allocating).
 *
 * Its scratch is one file-scope device array inside the library (about 8 MiB
 * plus 5 KiB), created on every GPU that loads the library and held until the
 * process exits.  Limits and rules:
 * - M * K / 2 <= 8 MiB (the packed activation codes must fit); larger calls
 *   return CR_ERR_WORKSPACE and launch nothing;
 * - all calls on a device share that array: calls whose GPU work overlaps
 *   (other streams, other host threads) race and give wrong results;
 * - the array keeps the last call's contents; nothing has to be cleared
 *   between calls (every scratch byte read is written earlier in the call);
 * - the first call on a device looks up the array's device address with that
 *   device current; make the first call before any stream capture;
 * - device-side timeouts are recorded in the array, not reported to the caller.
 * Other arguments, shape and alignment rules: as cr_w4a4_linear.
 */
cr_status cr_w4a4_linear_noalloc(const void* X, int64_t ldx, const void* Wq, const float* w_scale,
                                 const void* bias, void* Y, int64_t ldy, int M, int N, int K, int group,
                                 void* stream);

/*
 * cr_selftest_wait_timeout -- diagnostic: enqueue one small kernel that runs the
 * library's bounded device-side wait on a barrier that is never completed.
 * The wait gives up after its limit (about 2 s) and the kernel writes
 * CR_ERR_TIMEOUT into the status word of `workspace` (read it with
 * cr_read_device_status), exactly as a stalled pipeline inside a compute call
 * would.  Nothing faults and the context stays usable.  For tests of the
 * failure path; never needed in normal use.
 */
cr_status cr_selftest_wait_timeout(void* workspace, size_t workspace_bytes, void* stream);

/*
 * cr_selftest_act_fallback -- diagnostic: cr_rotate_quant_act_ex on the
 * fallback kernels, the two streaming passes (per-block maxima, then codes)
 * that run when the device refuses the one-launch activation pass's
 * cooperative launch (its CTAs cannot all be resident, e.g. while other work
 * holds SMs).  The codes and the scale are the same bit for bit (same lane
 * mapping, transform, division and max).  For tests of that path; never needed
 * in normal use.  Arguments, rules and errors: as cr_rotate_quant_act_ex.
 */
cr_status cr_selftest_act_fallback(const void* X, int M, int K, int64_t ldx, int group, int bits, int rotate,
                                   void* Xq, float* a_scale, void* workspace, size_t workspace_bytes,
                                   void* stream);

/*
 * cr_read_device_status -- copy the device status word of `workspace` into
 * *status (CR_OK or the first device-side error, e.g. CR_ERR_TIMEOUT).
 * Synchronises `stream`.  Clearing the word is the caller's job (write zero).
 */
cr_status cr_read_device_status(const void* workspace, int* status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* CONVROT_H_ */
