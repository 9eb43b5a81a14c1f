// act_kernels.cu -- ConvRot rotation + dynamic INT4 quantisation on sm_100a.
//
// The rotation multiplies every contiguous 256-wide slice of a row by the
// regular Hadamard matrix H256 = (J-2I)^(x4) / 16 ("Qwen-Image-Edit-2511 --
// INT4 tensorwise W4A4 (+ConvRot, mixed int8 fallback)", introduction:
// group-256 regular-Hadamard rotation, activations rotated online and
// quantised dynamically to INT4).  It is computed as a fast transform: one
// radix-4 pass per base-4 digit of the index, each pass replacing the four
// values that differ in that digit by (their sum) - 2 * (own value).
//
// Work split: a 256-slice ("unit") belongs to a pair of adjacent lanes, each
// holding 128 consecutive elements in registers (one 256-byte contiguous
// load per lane).  Digits 0..2 and the low bit of digit 3 are in-thread; the
// high bit of digit 3 is one shuffle with the partner lane.  The 1/16
// normalisation is never applied to the values: codes only depend on the
// ratio y / s, and scaling both by 16 is exact in float32.  The scale written
// out is divided by 16.
//
// Pass 1 (act_amax_kernel) writes one partial max per block; pass 2
// (act_quant_kernel) reduces them, recomputes the rotation (the second read
// of X is served from L2 when X fits there), quantises and packs.

#include <cuda_runtime.h>

#include <cstdint>

#include "cr_device.cuh"
#include "cr_internal.h"

namespace cr {
namespace {

constexpr int kThreads = 256;       // 128 lane pairs = 128 units per block iteration
constexpr int kUnitsPerIter = kThreads / 2;

__device__ __forceinline__ void load_half_unit(const uint16_t* __restrict__ src, float (&v)[128]) {
  const uint4* p = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const uint4 u = __ldg(p + j);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      v[8 * j + 2 * h] = __uint_as_float(w[h] << 16);
      v[8 * j + 2 * h + 1] = __uint_as_float(w[h] & 0xFFFF0000u);
    }
  }
}

// (J - 2I) applied to four values: each becomes (sum of the four) - 2 * itself.
__device__ __forceinline__ void radix4(float& a, float& b, float& c, float& d) {
  const float s = __fadd_rn(__fadd_rn(a, b), __fadd_rn(c, d));
  a = __fmaf_rn(-2.f, a, s);
  b = __fmaf_rn(-2.f, b, s);
  c = __fmaf_rn(-2.f, c, s);
  d = __fmaf_rn(-2.f, d, s);
}

// Unnormalised H256 transform (16 * x H) of the unit split over a lane pair.
// Every lane of the warp must call this (it shuffles with the full mask).
__device__ __forceinline__ void fwht256_pair(float (&v)[128]) {
#pragma unroll
  for (int stride = 1; stride <= 16; stride *= 4) {
#pragma unroll
    for (int base = 0; base < 128; base += 4 * stride) {
#pragma unroll
      for (int j = 0; j < stride; ++j) radix4(v[base + j], v[base + j + stride], v[base + j + 2 * stride], v[base + j + 3 * stride]);
    }
  }
  // digit 3: elements j, j+64 here and j+128, j+192 on the partner lane
#pragma unroll
  for (int j = 0; j < 64; ++j) {
    const float s = __fadd_rn(v[j], v[j + 64]);
    const float S = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, 1));
    v[j] = __fmaf_rn(-2.f, v[j], S);
    v[j + 64] = __fmaf_rn(-2.f, v[j + 64], S);
  }
}

__device__ __forceinline__ float warp_max(float a) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  return a;
}

// Block-wide max of `a` (kThreads threads); result valid in every thread.
__device__ __forceinline__ float block_max(float a, float* red) {
  a = warp_max(a);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = a;
  __syncthreads();
  float b = (lane < kThreads / 32) ? red[lane] : 0.f;
  return warp_max(b);
}

// Correctly rounded y / s given r = RN(1/s): Markstein's correction step
// (P. Markstein, "Computation of elementary functions on the IBM RISC
// System/6000 processor", 1990): the residual y - s*q0 is exact in one fma,
// and one more fma rounds the corrected quotient.
__device__ __forceinline__ float div_rn_by(float y, float s, float r) {
  const float q0 = __fmul_rn(y, r);
  const float e = __fmaf_rn(-q0, s, y);
  return __fmaf_rn(e, r, q0);
}

// Codes for 128 values and their packed 64 bytes (low nibble = even element).
__device__ __forceinline__ void quant_pack_store(const float (&v)[128], float s16, float r16, uint8_t* dst) {
  uint32_t w[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    uint32_t acc = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      int q = __float2int_rn(div_rn_by(v[8 * k + e], s16, r16));
      q = max(-8, min(7, q));
      acc |= (static_cast<uint32_t>(q) & 0xFu) << (4 * e);
    }
    w[k] = acc;
  }
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int j = 0; j < 4; ++j) d[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
}

// Scale of the unnormalised values (16 * s) and its reciprocal, from the max
// of |16 y|.  An all-zero tensor gets s = 1, i.e. 16 here.
__device__ __forceinline__ void scale_from_amax16(float amax16, float& s16, float& r16) {
  s16 = (amax16 > 0.f) ? __fdiv_rn(amax16, 7.f) : 16.f;
  r16 = __frcp_rn(s16);
}

__global__ void __launch_bounds__(kThreads) act_amax_kernel(const uint16_t* __restrict__ X, int rows, int K,
                                                            int64_t ldx, float* __restrict__ partial) {
  __shared__ float red[kThreads / 32];
  const int gpr = K >> 8;  // units per row
  const int64_t units = static_cast<int64_t>(rows) * gpr;
  const int h = threadIdx.x & 1;
  float amax = 0.f;
  for (int64_t base = static_cast<int64_t>(blockIdx.x) * kUnitsPerIter; base < units;
       base += static_cast<int64_t>(gridDim.x) * kUnitsPerIter) {
    const int64_t u = base + (threadIdx.x >> 1);
    float v[128];
    if (u < units) {
      const int64_t r = u / gpr;
      const int g = static_cast<int>(u - r * gpr);
      load_half_unit(X + r * ldx + (g << 8) + (h << 7), v);
    } else {
#pragma unroll
      for (int i = 0; i < 128; ++i) v[i] = 0.f;
    }
    fwht256_pair(v);
#pragma unroll
    for (int i = 0; i < 128; ++i) amax = fmaxf(amax, fabsf(v[i]));
  }
  amax = block_max(amax, red);
  if (threadIdx.x == 0) partial[blockIdx.x] = amax;
}

__global__ void __launch_bounds__(kThreads) act_quant_kernel(const uint16_t* __restrict__ X, int rows, int K,
                                                             int64_t ldx, const float* __restrict__ partial,
                                                             int npartial, uint8_t* __restrict__ Xq,
                                                             float* __restrict__ scale_out, int nscale) {
  __shared__ float red[kThreads / 32];
  float a = 0.f;
  for (int i = threadIdx.x; i < npartial; i += kThreads) a = fmaxf(a, partial[i]);
  const float amax16 = block_max(a, red);
  float s16, r16;
  scale_from_amax16(amax16, s16, r16);
  if (blockIdx.x == 0) {
    const float s = __fmul_rn(s16, 0.0625f);  // exact: power-of-two scaling
    for (int i = threadIdx.x; i < nscale; i += kThreads) scale_out[i] = s;
  }
  const int gpr = K >> 8;
  const int64_t units = static_cast<int64_t>(rows) * gpr;
  const int h = threadIdx.x & 1;
  const int64_t ldq = K >> 1;
  for (int64_t base = static_cast<int64_t>(blockIdx.x) * kUnitsPerIter; base < units;
       base += static_cast<int64_t>(gridDim.x) * kUnitsPerIter) {
    const int64_t u = base + (threadIdx.x >> 1);
    const bool valid = u < units;
    int64_t r = 0;
    int g = 0;
    float v[128];
    if (valid) {
      r = u / gpr;
      g = static_cast<int>(u - r * gpr);
      load_half_unit(X + r * ldx + (g << 8) + (h << 7), v);
    } else {
#pragma unroll
      for (int i = 0; i < 128; ++i) v[i] = 0.f;
    }
    fwht256_pair(v);
    if (valid) quant_pack_store(v, s16, r16, Xq + r * ldq + (g << 7) + (h << 6));
  }
}

// One block per row: pass 1 row max, pass 2 codes with the row's own scale.
__global__ void __launch_bounds__(kThreads) pack_rows_kernel(const uint16_t* __restrict__ W, int K, int64_t ldw,
                                                             uint8_t* __restrict__ Wq,
                                                             float* __restrict__ w_scale) {
  __shared__ float red[kThreads / 32];
  const int row = blockIdx.x;
  const int gpr = K >> 8;
  const int h = threadIdx.x & 1;
  const uint16_t* src = W + static_cast<int64_t>(row) * ldw;
  float amax = 0.f;
  for (int base = 0; base < gpr; base += kUnitsPerIter) {
    const int g = base + (threadIdx.x >> 1);
    float v[128];
    if (g < gpr) {
      load_half_unit(src + (g << 8) + (h << 7), v);
    } else {
#pragma unroll
      for (int i = 0; i < 128; ++i) v[i] = 0.f;
    }
    fwht256_pair(v);
#pragma unroll
    for (int i = 0; i < 128; ++i) amax = fmaxf(amax, fabsf(v[i]));
  }
  const float amax16 = block_max(amax, red);
  float s16, r16;
  scale_from_amax16(amax16, s16, r16);
  if (threadIdx.x == 0) w_scale[row] = __fmul_rn(s16, 0.0625f);
  uint8_t* dst = Wq + static_cast<int64_t>(row) * (K >> 1);
  for (int base = 0; base < gpr; base += kUnitsPerIter) {
    const int g = base + (threadIdx.x >> 1);
    const bool valid = g < gpr;
    float v[128];
    if (valid) {
      load_half_unit(src + (g << 8) + (h << 7), v);
    } else {
#pragma unroll
      for (int i = 0; i < 128; ++i) v[i] = 0.f;
    }
    fwht256_pair(v);
    if (valid) quant_pack_store(v, s16, r16, dst + (g << 7) + (h << 6));
  }
}

}  // namespace

int act_grid(int rows, int K, int num_sms) {
  const int64_t units = static_cast<int64_t>(rows) * (K >> 8);
  int64_t g = (units + kUnitsPerIter - 1) / kUnitsPerIter;
  int64_t cap = static_cast<int64_t>(num_sms) * 4;
  if (cap > kMaxActBlocks) cap = kMaxActBlocks;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return static_cast<int>(g);
}

cudaError_t launch_act_amax(const uint16_t* X, int rows, int K, int64_t ldx, float* partial, int grid,
                            cudaStream_t stream) {
  act_amax_kernel<<<grid, kThreads, 0, stream>>>(X, rows, K, ldx, partial);
  return cudaGetLastError();
}

cudaError_t launch_act_quant(const uint16_t* X, int rows, int K, int64_t ldx, const float* partial, int npartial,
                             uint8_t* Xq, float* scale_out, int nscale, int grid, cudaStream_t stream) {
  act_quant_kernel<<<grid, kThreads, 0, stream>>>(X, rows, K, ldx, partial, npartial, Xq, scale_out, nscale);
  return cudaGetLastError();
}

cudaError_t launch_pack_rows(const uint16_t* W, int rows, int K, int64_t ldw, uint8_t* Wq, float* w_scale,
                             cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  pack_rows_kernel<<<rows, kThreads, 0, stream>>>(W, K, ldw, Wq, w_scale);
  return cudaGetLastError();
}

}  // namespace cr
