// act_device.cuh -- device helpers for one 256-element unit of the ConvRot
// rotation and its quantisation, shared by the activation kernels and the
// fused few-token layer.  Included inside an anonymous namespace of cr, after
// cr_device.cuh and cr_internal.h.
//
// The rotation multiplies every contiguous 256-wide slice of a row by the
// regular Hadamard matrix H256 = (J-2I)^(x4) / 16 ("Qwen-Image-Edit-2511 --
// INT4 tensorwise W4A4 (+ConvRot, mixed int8 fallback)", introduction),
// computed as a fast transform: one radix-4 pass per base-4 digit of the
// index, each pass replacing the four values that differ in that digit by
// (their sum) - 2 * (own value).  A unit belongs to 4 adjacent lanes; lane bit
// 0 selects element bit 5 and lane bit 1 element bit 7, so each lane holds two
// runs of 32 consecutive elements.
#pragma once

constexpr int kLanesPerUnit = 4;

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

// Unnormalised transform of the unit spread over 4 lanes: the first kDig base-4
// digit passes of H256, i.e. the block-diagonal rotation by H_g, g = 4^kDig, of
// every g consecutive elements, times 2^kDig (kDig = 4: 16 * x H256).
// Every lane of the warp must call this (it shuffles with the full mask).
template <int kDig>
__device__ __forceinline__ void fwht256_quad(float (&v)[64]) {
  static_assert(kDig >= 2 && kDig <= 5, "groups of 16, 64, 256 or 1024");
  // digit 0: elements 0-3 of each quad (local stride 1)
#pragma unroll
  for (int b = 0; b < 64; b += 4) radix4(v[b], v[b + 1], v[b + 2], v[b + 3]);
  // digit 1: local stride 4
#pragma unroll
  for (int b = 0; b < 64; b += 16) {
#pragma unroll
    for (int j = 0; j < 4; ++j) radix4(v[b + j], v[b + j + 4], v[b + j + 8], v[b + j + 12]);
  }
  if (kDig >= 3) radix4_split<16, 1>(v);  // digit 2: element bit 4 local (stride 16), bit 5 = lane bit 0
  if (kDig >= 4) radix4_split<32, 2>(v);  // digit 3: element bit 6 local (stride 32), bit 7 = lane bit 1
  if (kDig >= 5) {
    // digit 4 (groups of 1024): the unit's index bits 0-1 = lane bits 2-3; every lane holds the same
    // element positions of its unit, so the four values of a group sit in the same register of lanes
    // l, l^4, l^8, l^12 (the caller's units are 4-aligned within rows of a multiple of 4 units)
#pragma unroll
    for (int j = 0; j < 64; ++j) {
      const float t = __fadd_rn(v[j], __shfl_xor_sync(0xffffffffu, v[j], 4));
      const float S = __fadd_rn(t, __shfl_xor_sync(0xffffffffu, t, 8));
      v[j] = __fmaf_rn(-2.f, v[j], S);
    }
  }
}

__device__ __forceinline__ float warp_max(float a) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  return a;
}

// Block-wide max of `a` (kN threads); result valid in every thread.
template <int kN>
__device__ __forceinline__ float block_max_n(float a, float* red) {
  a = warp_max(a);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = a;
  __syncthreads();
  float b = (lane < kN / 32) ? red[lane] : 0.f;
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

// INT8 codes for the lane's 64 values: two runs of 32 bytes.  The magic add
// leaves round_half_even(t) in the low mantissa bits; its low byte is the
// two's-complement code.  With s = fl(amax / 127), |t| <= 127 (1 + 2^-23), so
// the code lies in [-127, 127] and needs no clamp.
__device__ __forceinline__ void quant_store8(const float (&v)[64], float s, float r, uint8_t* unit_q, int lane) {
  uint32_t w[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    uint32_t acc = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e)
      acc |= (__float_as_uint(__fadd_rn(div_rn_by(v[4 * k + e], s, r), 12582912.0f)) & 0xFFu) << (8 * e);
    w[k] = acc;
  }
  const int off = lane_run_offset(lane);  // bytes: one code per byte
  uint4* d0 = reinterpret_cast<uint4*>(unit_q + off);
  uint4* d1 = reinterpret_cast<uint4*>(unit_q + off + 64);
  d0[0] = make_uint4(w[0], w[1], w[2], w[3]);
  d0[1] = make_uint4(w[4], w[5], w[6], w[7]);
  d1[0] = make_uint4(w[8], w[9], w[10], w[11]);
  d1[1] = make_uint4(w[12], w[13], w[14], w[15]);
}

// Code formats (kFmt): symmetric INT4 (amax -> 7) packed two per byte, or
// symmetric INT8 (amax -> 127), one code per byte.  kDig = digit passes of the
// rotation (0: none, the stock INT8 path; 2, 3, 4: groups of 16, 64, 256), so
// the values are 2^kDig * (x H_g).  From the max of the values: the scale of
// the values s_v, its reciprocal and the scale written out (s_v / 2^kDig:
// exact).  All-zero input: scale 1.
template <int kFmt, int kDig>
__device__ __forceinline__ void value_scale(float amax_v, float& s_v, float& r_v, float& s_out) {
  constexpr float kQ = kFmt == kFmtByte8 ? 127.f : 7.f;
  constexpr float kF = static_cast<float>(1 << kDig);  // unnormalised factor of the rotation (1: none)
  s_v = (amax_v > 0.f) ? __fdiv_rn(amax_v, kQ) : kF;
  r_v = __frcp_rn(s_v);
  s_out = __fmul_rn(s_v, 1.f / kF);  // exact: power-of-two scaling
}

// ---------------------------------------------------------------------------
// The streaming kernels' lane mapping (4 lanes per unit, 8 units per warp): lane
// bits 0-1 are element bits 3-4; the thread's slot k (0..7) holds the 8
// consecutive elements of piece p = k ^ k0 (element bits 5-7 = p), k0 = the
// unit's index inside the warp's 8.  Transform on pairs of values.
// ---------------------------------------------------------------------------

// The lane's 64 values as 32 pairs W[i] = (v[i], v[i + 32]): the two halves of
// a pair sit in different groups of every digit pass except the last, so most
// of the transform runs on Blackwell's two-wide fp32 add / fma, with the same
// operations in the same order as the one-value-at-a-time form.
struct Pairs {
  float2 w[32];
};

__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// (J - 2I) on four pairs, elementwise.
__device__ __forceinline__ void radix4_2(float2& a, float2& b, float2& c, float2& d) {
  const float2 m2 = make_float2(-2.f, -2.f);
  const float2 s = add2(add2(a, b), add2(c, d));
  a = fma2(m2, a, s);
  b = fma2(m2, b, s);
  c = fma2(m2, c, s);
  d = fma2(m2, d, s);
}

// Split digit pass on pairs: one bit in-thread (pair stride `st`), one bit across lanes.
template <int st, int lane_mask>
__device__ __forceinline__ void radix4_split_2(float2 (&w)[32]) {
  const float2 m2 = make_float2(-2.f, -2.f);
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    if (i & st) continue;
    const float2 s = add2(w[i], w[i + st]);
    const float2 S = add2(s, make_float2(__shfl_xor_sync(0xffffffffu, s.x, lane_mask),
                                         __shfl_xor_sync(0xffffffffu, s.y, lane_mask)));
    w[i] = fma2(m2, w[i], S);
    w[i + st] = fma2(m2, w[i + st], S);
  }
}

// Digit 3 of the mapped transform: element bits 6-7 = j bits 4-5; the group of v[i] is v[i], v[i+16],
// v[i+32], v[i+48].
__device__ __forceinline__ void fwht_digit3_mapped(float2 (&w)[32]) {
  const float2 m2 = make_float2(-2.f, -2.f);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float2 h = add2(w[i], w[i + 16]);  // (v[i] + v[i+16], v[i+32] + v[i+48])
    const float s = __fadd_rn(h.x, h.y);
    const float2 S = make_float2(s, s);
    w[i] = fma2(m2, w[i], S);
    w[i + 16] = fma2(m2, w[i + 16], S);
  }
}

// Digit 4 of the mapped transform (groups of 1024): unit index bits 0-1 = lane bits 2-3 (the slot XOR
// k0 of a unit equals its index uw among the warp's 8 units).  Unit uw holds piece p in slot p ^ uw, so
// the partner unit uw ^ m (lane ^ 4m) holds the same element in pair index i ^ 8m.  With
// T(i) = w(i) + w_{lane^4}(i ^ 8), the group's sum is T(i) + T_{lane^8}(i ^ 16).
__device__ __forceinline__ void fwht_digit4_mapped(float2 (&w)[32]) {
  const float2 m2 = make_float2(-2.f, -2.f);
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    float2 t[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const float2 o = w[e + 8 * (m ^ 1)];
      t[m] = add2(w[e + 8 * m], make_float2(__shfl_xor_sync(0xffffffffu, o.x, 4), __shfl_xor_sync(0xffffffffu, o.y, 4)));
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const float2 o = t[m ^ 2];
      const float2 S = add2(t[m], make_float2(__shfl_xor_sync(0xffffffffu, o.x, 8), __shfl_xor_sync(0xffffffffu, o.y, 8)));
      w[e + 8 * m] = fma2(m2, w[e + 8 * m], S);
    }
  }
}

// Digit passes of the transform for this mapping: the first kDig of H256's
// (unnormalised; kDig = 4 gives 16 * x H256, 3 and 2 the groups of 64 and 16).
// Local index j of v: bits 0-2 = element bits 0-2, bits 3-5 = slot bits 0-2.
// The slot XOR of the mapping permutes element bits 5-7 alike on input and
// output, which each digit pass treats symmetrically (or, above the group,
// only relabels groups).
template <int kDig>
__device__ __forceinline__ void fwht256_mapped(Pairs& P) {
  static_assert(kDig >= 2 && kDig <= 5, "groups of 16, 64, 256 or 1024");
  float2(&w)[32] = P.w;
  // digit 0: element bits 0-1 = j bits 0-1
#pragma unroll
  for (int b = 0; b < 32; b += 4) radix4_2(w[b], w[b + 1], w[b + 2], w[b + 3]);
  radix4_split_2<4, 1>(w);  // digit 1: element bit 2 = j bit 2, bit 3 = lane bit 0
  if constexpr (kDig >= 3) radix4_split_2<8, 2>(w);  // digit 2: element bit 4 = lane bit 1, bit 5 = j bit 3
  if constexpr (kDig >= 4) fwht_digit3_mapped(w);
  if constexpr (kDig >= 5) fwht_digit4_mapped(w);
}

// bf16 -> float32 pairs: W[i] = (v[i], v[i+32]) with v[8k + e] = element e of slot k.  The low half
// moves up by a byte permute rather than a shift (which may be issued as an integer multiply-add on
// the pipe the transform's float adds and fmas need).
__device__ __forceinline__ void widen_pairs(const Raw& r, Pairs& P) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t a[4] = {r.q[k].x, r.q[k].y, r.q[k].z, r.q[k].w};
    const uint32_t b[4] = {r.q[k + 4].x, r.q[k + 4].y, r.q[k + 4].z, r.q[k + 4].w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      P.w[8 * k + 2 * h] = make_float2(__uint_as_float(__byte_perm(a[h], 0u, 0x1044)),
                                       __uint_as_float(__byte_perm(b[h], 0u, 0x1044)));
      P.w[8 * k + 2 * h + 1] = make_float2(__uint_as_float(a[h] & 0xFFFF0000u), __uint_as_float(b[h] & 0xFFFF0000u));
    }
  }
}

// Eight codes (low nibble of each word) -> one packed word, element 2b in the low nibble of byte b.
__device__ __forceinline__ uint32_t pack8(const uint32_t (&c)[8]) {
  const uint32_t e = __byte_perm(__byte_perm(c[0], c[2], 0x0040), __byte_perm(c[4], c[6], 0x0040), 0x5410);
  const uint32_t o = __byte_perm(__byte_perm(c[1], c[3], 0x0040), __byte_perm(c[5], c[7], 0x0040), 0x5410);
  return (e & 0x0F0F0F0Fu) | (__funnelshift_l(o, o, 4) & 0xF0F0F0F0u);  // rotate: the wrapped bits are masked off
}

// Lane's raw 64 values of unit `unit` straight from global memory, in the streaming mapping's slot
// order: slot k holds piece p = k ^ k0 (8 consecutive bf16, one 16-byte load).
__device__ __forceinline__ void load_unit_mapped(const uint16_t* __restrict__ unit, int k0, Raw& raw) {
  const int l = threadIdx.x & 3;
#pragma unroll
  for (int k = 0; k < 8; ++k) raw.q[k] = __ldg(reinterpret_cast<const uint4*>(unit + 32 * (k ^ k0) + 8 * l));
}

// Codes of the lane's 64 rotated values (pairs P, slot XOR k0 of the streaming mapping) straight to the
// unit's code bytes in global memory: correctly rounded y / s (one Markstein step, as div_rn_by), round
// half to even by the magic add, piece p = k ^ k0 at bytes 16p + 4l (INT4, packed) or 32p + 8l (INT8).
template <int kFmt>
__device__ __forceinline__ void codes_to_unit_global(const Pairs& P, int k0, float2 r2, float2 ns2,
                                                     uint8_t* __restrict__ unit_q) {
  const int l = threadIdx.x & 3;
  const float2 magic2 = make_float2(12582912.0f, 12582912.0f);
  uint32_t cx[32], cy[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const float2 y = P.w[i];
    const float2 q0 = __fmul2_rn(y, r2);
    const float2 e = fma2(q0, ns2, y);
    const float2 t = add2(fma2(e, r2, q0), magic2);
    cx[i] = __float_as_uint(t.x);
    cy[i] = __float_as_uint(t.y);
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    uint32_t c[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) c[e] = (k < 4) ? cx[8 * k + e] : cy[8 * (k - 4) + e];
    if constexpr (kFmt == kFmtPacked4) {
      *reinterpret_cast<uint32_t*>(unit_q + 16 * (k ^ k0) + 4 * l) = pack8(c);
    } else {
      const uint32_t lo = __byte_perm(__byte_perm(c[0], c[1], 0x0040), __byte_perm(c[2], c[3], 0x0040), 0x5410);
      const uint32_t hi = __byte_perm(__byte_perm(c[4], c[5], 0x0040), __byte_perm(c[6], c[7], 0x0040), 0x5410);
      *reinterpret_cast<uint2*>(unit_q + 32 * (k ^ k0) + 8 * l) = make_uint2(lo, hi);
    }
  }
}
