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
// Work split: a 256-slice ("unit") belongs to 4 adjacent lanes.  Lane bit 0
// selects element bit 5 and lane bit 1 selects element bit 7, so each lane
// holds two runs of 32 consecutive elements and the local index j covers
// element bits 0-4 and 6.  Digits 0 and 1 are in-thread; digits 2 and 3 each
// have one bit in-thread and one bit across a lane pair, costing one shuffle
// per two values.
//
// Input streaming: each block walks 64-unit chunks (32 KB of bf16) through a
// 3-stage shared-memory ring filled by bulk asynchronous copies (one thread
// issues them, an mbarrier counts the bytes), so the copy engine keeps many
// bytes in flight without spending registers.
//
// The 1/16 normalisation is never applied to the values: codes only depend on
// the ratio y / s, and scaling both by 16 is exact in float32.  The scale
// written out is divided by 16.
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

constexpr int kThreads = 256;
constexpr int kLanesPerUnit = 4;
constexpr int kUnitsPerIter = kThreads / kLanesPerUnit;  // 64

// Raw bf16 data of one lane's share of a unit: 2 runs x 32 elements.
struct Raw {
  uint4 q[8];
};

// Offset (in elements) of this lane's first run inside its unit.
__device__ __forceinline__ int lane_run_offset(int lane) { return ((lane >> 1) & 1) << 7 | (lane & 1) << 5; }

__device__ __forceinline__ void load_raw(const uint16_t* __restrict__ unit, int lane, Raw& r) {
  const uint4* p0 = reinterpret_cast<const uint4*>(unit + lane_run_offset(lane));
  const uint4* p1 = reinterpret_cast<const uint4*>(unit + lane_run_offset(lane) + 64);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    r.q[q] = __ldg(p0 + q);
    r.q[4 + q] = __ldg(p1 + q);
  }
}

__device__ __forceinline__ void zero_raw(Raw& r) {
#pragma unroll
  for (int q = 0; q < 8; ++q) r.q[q] = make_uint4(0, 0, 0, 0);
}

// bf16 -> float32 is a 16-bit shift of the bit pattern.
__device__ __forceinline__ void widen(const Raw& r, float (&v)[64]) {
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const uint32_t w[4] = {r.q[q].x, r.q[q].y, r.q[q].z, r.q[q].w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      v[8 * q + 2 * h] = __uint_as_float(w[h] << 16);
      v[8 * q + 2 * h + 1] = __uint_as_float(w[h] & 0xFFFF0000u);
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

// Radix-4 pass whose digit has one bit in-thread (local stride `st`) and one
// bit across lanes (partner = lane ^ `lane_mask`).
template <int st, int lane_mask>
__device__ __forceinline__ void radix4_split(float (&v)[64]) {
#pragma unroll
  for (int j = 0; j < 64; ++j) {
    if (j & st) continue;
    const float s = __fadd_rn(v[j], v[j + st]);
    const float S = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, lane_mask));
    v[j] = __fmaf_rn(-2.f, v[j], S);
    v[j + st] = __fmaf_rn(-2.f, v[j + st], S);
  }
}

// Unnormalised H256 transform (16 * x H) of the unit spread over 4 lanes.
// Every lane of the warp must call this (it shuffles with the full mask).
__device__ __forceinline__ void fwht256_quad(float (&v)[64]) {
  // digit 0: elements 0-3 of each quad (local stride 1)
#pragma unroll
  for (int b = 0; b < 64; b += 4) radix4(v[b], v[b + 1], v[b + 2], v[b + 3]);
  // digit 1: local stride 4
#pragma unroll
  for (int b = 0; b < 64; b += 16) {
#pragma unroll
    for (int j = 0; j < 4; ++j) radix4(v[b + j], v[b + j + 4], v[b + j + 8], v[b + j + 12]);
  }
  radix4_split<16, 1>(v);  // digit 2: element bit 4 local (stride 16), bit 5 = lane bit 0
  radix4_split<32, 2>(v);  // digit 3: element bit 6 local (stride 32), bit 7 = lane bit 1
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

// Two's-complement nibble of round_half_even(t).  Adding 1.5 * 2^23 puts the
// integer nearest to t (ties to even, by the IEEE add) in the low mantissa
// bits.  No clamp is needed: the scale is fl(amax / 7) with amax the largest
// |value| of the very float32 values being quantised, so |t| <= 7 (1 + 2^-23)
// and round_half_even(t) lies in [-7, 7], inside the code range [-8, 7].
__device__ __forceinline__ uint32_t code_nibble(float t) {
  return __float_as_uint(__fadd_rn(t, 12582912.0f)) & 0xFu;
}

// Codes for the lane's 64 values: two runs of 32 codes, 16 packed bytes each.
__device__ __forceinline__ void quant_pack_store(const float (&v)[64], float s16, float r16, uint8_t* unit_q,
                                                 int lane) {
  uint32_t w[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    uint32_t acc = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc |= code_nibble(div_rn_by(v[8 * k + e], s16, r16)) << (4 * e);
    w[k] = acc;
  }
  const int off = lane_run_offset(lane) >> 1;  // bytes
  *reinterpret_cast<uint4*>(unit_q + off) = make_uint4(w[0], w[1], w[2], w[3]);
  *reinterpret_cast<uint4*>(unit_q + off + 32) = make_uint4(w[4], w[5], w[6], w[7]);
}

// Scale of the unnormalised values (16 * s) and its reciprocal, from the max
// of |16 y|.  An all-zero tensor gets s = 1, i.e. 16 here.
__device__ __forceinline__ void scale_from_amax16(float amax16, float& s16, float& r16) {
  s16 = (amax16 > 0.f) ? __fdiv_rn(amax16, 7.f) : 16.f;
  r16 = __frcp_rn(s16);
}

__device__ __forceinline__ const uint16_t* unit_ptr(const uint16_t* X, int64_t u, int gpr, int64_t ld) {
  const int64_t r = u / gpr;
  return X + r * ld + ((u - r * gpr) << 8);
}

constexpr int kDepth = 3;                          // chunks in flight per block
constexpr int kChunkBytes = kUnitsPerIter * 512;   // 32 KB of bf16 per chunk
constexpr int kStreamSmem = kDepth * kChunkBytes + 64;

struct Stream {
  uint8_t* ring;        // kDepth chunks
  uint64_t* bars;       // kDepth mbarriers
  const uint16_t* X;
  int64_t ldx;
  int gpr;
  int64_t units;

  // Thread 0: bulk-copy chunk `c` (units [64c, 64c+64) clipped) into ring slot `slot`,
  // one copy per row segment (units of one row are contiguous).
  __device__ void issue(int64_t c, int slot) const {
    const int64_t u0 = c * kUnitsPerIter;
    int64_t u1 = u0 + kUnitsPerIter;
    if (u1 > units) u1 = units;
    const uint32_t bar = smem_u32(bars + slot);
    mbar_arrive_expect_tx(bar, static_cast<uint32_t>((u1 - u0) * 512));
    uint8_t* dst = ring + slot * kChunkBytes;
    for (int64_t u = u0; u < u1;) {
      const int64_t r = u / gpr;
      int64_t seg_end = (r + 1) * gpr;
      if (seg_end > u1) seg_end = u1;
      const uint16_t* src = X + r * ldx + ((u - r * gpr) << 8);
      const uint32_t bytes = static_cast<uint32_t>((seg_end - u) * 512);
      asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                       smem_u32(dst + (u - u0) * 512)),
                   "l"(src), "r"(bytes), "r"(bar)
                   : "memory");
      u = seg_end;
    }
  }
};

// Lane's 64 values of its unit, read from a ring slot.
__device__ __forceinline__ void read_slot(const uint8_t* slot, int lane, Raw& r) {
  const uint8_t* unit = slot + (threadIdx.x >> 2) * 512;
  const uint4* p0 = reinterpret_cast<const uint4*>(unit + 2 * lane_run_offset(lane));
  const uint4* p1 = reinterpret_cast<const uint4*>(unit + 2 * (lane_run_offset(lane) + 64));
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    r.q[q] = p0[q];
    r.q[4 + q] = p1[q];
  }
}

// Common streaming loop: for every chunk of this block, `body(v, unit_index)` gets the
// lane's 64 unnormalised rotated values (unit_index < 0 for lanes past the end).
template <class Body>
__device__ __forceinline__ void stream_units(const uint16_t* __restrict__ X, int rows, int K, int64_t ldx,
                                             uint8_t* smem, int* status, Body body) {
  Stream st;
  st.ring = smem;
  st.bars = reinterpret_cast<uint64_t*>(smem + kDepth * kChunkBytes);
  st.X = X;
  st.ldx = ldx;
  st.gpr = K >> 8;
  st.units = static_cast<int64_t>(rows) * st.gpr;
  const int64_t nchunks = (st.units + kUnitsPerIter - 1) / kUnitsPerIter;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kDepth; ++i) mbar_init(smem_u32(st.bars + i), 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 0; i < kDepth; ++i) {
      const int64_t c = blockIdx.x + static_cast<int64_t>(i) * gridDim.x;
      if (c < nchunks) st.issue(c, i);
    }
  }
  volatile int never = 0;
  int it = 0;
  for (int64_t c = blockIdx.x; c < nchunks; c += gridDim.x, ++it) {
    const int slot = it % kDepth;
    if (!mbar_wait(smem_u32(st.bars + slot), static_cast<uint32_t>((it / kDepth) & 1), &never)) {
      record_status(status, CR_ERR_TIMEOUT);  // a copy never landed: give up on this block's chunks
      break;
    }
    const int64_t u = c * kUnitsPerIter + (threadIdx.x >> 2);
    const bool valid = u < st.units;
    Raw raw;
    if (valid) read_slot(st.ring + slot * kChunkBytes, lane, raw); else zero_raw(raw);
    __syncthreads();  // every thread has read the slot: refill it
    if (threadIdx.x == 0) {
      const int64_t cn = c + static_cast<int64_t>(kDepth) * gridDim.x;
      if (cn < nchunks) {
        fence_proxy_async_smem();
        st.issue(cn, slot);
      }
    }
    float v[64];
    widen(raw, v);
    fwht256_quad(v);
    body(v, valid ? u : -1);
  }
}

__global__ void __launch_bounds__(kThreads, 2) act_amax_kernel(const uint16_t* __restrict__ X, int rows, int K,
                                                               int64_t ldx, float* __restrict__ partial,
                                                               int* __restrict__ status) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float red[kThreads / 32];
  float amax = 0.f;
  stream_units(X, rows, K, ldx, smem, status, [&](const float (&v)[64], int64_t) {
#pragma unroll
    for (int i = 0; i < 64; ++i) amax = fmaxf(amax, fabsf(v[i]));
  });
  amax = block_max(amax, red);
  if (threadIdx.x == 0) partial[blockIdx.x] = amax;
}

__global__ void __launch_bounds__(kThreads, 2) act_quant_kernel(const uint16_t* __restrict__ X, int rows, int K,
                                                                int64_t ldx, const float* __restrict__ partial,
                                                                int npartial, uint8_t* __restrict__ Xq,
                                                                float* __restrict__ scale_out, int nscale,
                                                                int* __restrict__ status) {
  extern __shared__ __align__(128) uint8_t smem[];
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
  const int64_t ldq = K >> 1;
  const int lane = threadIdx.x & 31;
  stream_units(X, rows, K, ldx, smem, status, [&](const float (&v)[64], int64_t u) {
    if (u >= 0) {
      const int64_t r = u / gpr;
      quant_pack_store(v, s16, r16, Xq + r * ldq + ((u - r * gpr) << 7), lane);
    }
  });
}

// One block per row: pass 1 row max, pass 2 codes with the row's own scale.
__global__ void __launch_bounds__(kThreads, 2) pack_rows_kernel(const uint16_t* __restrict__ W, int K, int64_t ldw,
                                                                uint8_t* __restrict__ Wq,
                                                                float* __restrict__ w_scale) {
  __shared__ float red[kThreads / 32];
  const int row = blockIdx.x;
  const int gpr = K >> 8;
  const int lane = threadIdx.x & 31;
  const uint16_t* src = W + static_cast<int64_t>(row) * ldw;
  float amax = 0.f;
  for (int base = 0; base < gpr; base += kUnitsPerIter) {
    const int g = base + (threadIdx.x >> 2);
    Raw r;
    if (g < gpr) load_raw(src + (g << 8), lane, r); else zero_raw(r);
    float v[64];
    widen(r, v);
    fwht256_quad(v);
#pragma unroll
    for (int i = 0; i < 64; ++i) amax = fmaxf(amax, fabsf(v[i]));
  }
  const float amax16 = block_max(amax, red);
  float s16, r16;
  scale_from_amax16(amax16, s16, r16);
  if (threadIdx.x == 0) w_scale[row] = __fmul_rn(s16, 0.0625f);
  uint8_t* dst = Wq + static_cast<int64_t>(row) * (K >> 1);
  for (int base = 0; base < gpr; base += kUnitsPerIter) {
    const int g = base + (threadIdx.x >> 2);
    Raw r;
    if (g < gpr) load_raw(src + (g << 8), lane, r); else zero_raw(r);
    float v[64];
    widen(r, v);
    fwht256_quad(v);
    if (g < gpr) quant_pack_store(v, s16, r16, dst + (g << 7), lane);
  }
}

}  // namespace

int act_grid(int rows, int K, int num_sms) {
  const int64_t units = static_cast<int64_t>(rows) * (K >> 8);
  int64_t g = (units + kUnitsPerIter - 1) / kUnitsPerIter;
  int64_t cap = static_cast<int64_t>(num_sms) * 2;  // two resident blocks per SM
  if (cap > kMaxActBlocks) cap = kMaxActBlocks;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return static_cast<int>(g);
}

static bool stream_attrs_set(int dev) {
  static int done[64] = {};
  if (dev < 0 || dev >= 64) return false;
  if (!done[dev]) {
    if (cudaFuncSetAttribute(act_amax_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kStreamSmem) !=
            cudaSuccess ||
        cudaFuncSetAttribute(act_quant_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kStreamSmem) !=
            cudaSuccess)
      return false;
    done[dev] = 1;
  }
  return true;
}

cudaError_t launch_act_amax(const uint16_t* X, int rows, int K, int64_t ldx, float* partial, int grid, int* status,
                            cudaStream_t stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (!stream_attrs_set(dev)) return cudaErrorInvalidValue;
  act_amax_kernel<<<grid, kThreads, kStreamSmem, stream>>>(X, rows, K, ldx, partial, status);
  return cudaGetLastError();
}

cudaError_t launch_act_quant(const uint16_t* X, int rows, int K, int64_t ldx, const float* partial, int npartial,
                             uint8_t* Xq, float* scale_out, int nscale, int grid, int* status, cudaStream_t stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (!stream_attrs_set(dev)) return cudaErrorInvalidValue;
  act_quant_kernel<<<grid, kThreads, kStreamSmem, stream>>>(X, rows, K, ldx, partial, npartial, Xq, scale_out,
                                                            nscale, status);
  return cudaGetLastError();
}

cudaError_t launch_pack_rows(const uint16_t* W, int rows, int K, int64_t ldw, uint8_t* Wq, float* w_scale,
                             cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  pack_rows_kernel<<<rows, kThreads, 0, stream>>>(W, K, ldw, Wq, w_scale);
  return cudaGetLastError();
}

}  // namespace cr
