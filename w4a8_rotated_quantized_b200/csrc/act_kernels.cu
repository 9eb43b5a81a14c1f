// act_kernels.cu -- ConvRot rotation + dynamic quantisation of activations and weights on sm_100a.
//
// The rotation multiplies every contiguous 256-wide slice of a row by the
// regular Hadamard matrix H256 = (J-2I)^(x4) / 16 ("Qwen-Image-Edit-2511 --
// INT4 tensorwise W4A4 (+ConvRot, mixed int8 fallback)", introduction:
// group-256 regular-Hadamard rotation, activations rotated online and
// quantised dynamically to INT4).  It is computed as a fast transform: one
// radix-4 pass per base-4 digit of the index, each pass replacing the four
// values that differ in that digit by (their sum) - 2 * (own value).  A
// 256-slice ("unit") belongs to 4 adjacent lanes; the lane mappings and the
// per-unit transform and quantisation are in act_device.cuh.
//
// The 1/16 normalisation is never applied to the values: codes only depend on
// the ratio y / s, and scaling both by 16 is exact in float32.  The scale
// written out is divided by 16.
//
// Kernels:
// * act_pass_kernel -- the tensorwise path (activations, and weights with one
//   tensorwise scale): one persistent cooperative launch, one CTA per SM, the
//   rotated values of the last rounds kept on chip across a grid barrier
//   (described where it is defined).
// * act_amax_kernel + act_quant_kernel -- the same result in two streaming
//   passes through a bulk-copy ring (per-block partial maxima, then codes),
//   run only when the device refuses the cooperative launch.
// * pack_rows_kernel -- weights with one scale per row: a block per row.
// * pack_w4a8_kernel -- the W4A8 weight format (group-16 asymmetric codes).

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "cr_device.cuh"
#include "grid_sync.cuh"
#include "cr_internal.h"

namespace cr {
namespace {

#include "act_device.cuh"

constexpr int kThreads = 256;
constexpr int kUnitsPerIter = kThreads / kLanesPerUnit;  // 64

__device__ __forceinline__ float block_max(float a, float* red) { return block_max_n<kThreads>(a, red); }

// ---------------------------------------------------------------------------
// Streaming passes over the whole tensor: the fallback of the one-launch pass
// ---------------------------------------------------------------------------
// Block b owns the contiguous unit range [units*b/grid, units*(b+1)/grid) and
// walks it in chunks of 64 units (32 KB of bf16) through a 3-stage ring filled
// by bulk asynchronous copies (thread 0 issues them, one per row segment; an
// mbarrier counts the bytes).  Each warp releases a ring slot on a second
// mbarrier once its reads of the slot have completed, so no step waits for the
// whole block.
//
// Lane mapping inside a unit (4 lanes per unit, 8 units per warp): lane bits
// 0-1 are element bits 3-4; the thread's slot k (0..7) holds the 8 consecutive
// elements of piece p = k ^ (unit & 7), i.e. element bits 5-7 = p.  The XOR
// only permutes values inside groups the transform treats symmetrically, so
// the rotated values do not depend on it; it makes the 8 lanes of every
// quarter-warp read 8 different 16-byte bank groups, and the 32 lanes of a
// warp store their packed code words to 32 different banks.
constexpr int kDepth = 3;                          // chunks in flight per block
constexpr int kChunkUnits = kUnitsPerIter;         // 64
constexpr int kChunkBytes = kChunkUnits * 512;     // 32 KB of bf16 per chunk
constexpr int kWarps = kThreads / 32;
constexpr int kStageWarpBytes = 8 * 128;           // INT4 codes of a warp's 8 units (two buffers)
constexpr int kStageWarpBytes8 = 8 * 256;          // INT8 codes of a warp's 8 units (one buffer)
constexpr int kOffStage = kDepth * kChunkBytes;
constexpr int kOffBars = kOffStage + 2 * kWarps * kStageWarpBytes;
static_assert(2 * kStageWarpBytes == kStageWarpBytes8, "both code formats use the same staging area");
constexpr int kStreamSmem = kOffBars + 2 * kDepth * 8;

struct UnitRange {
  const uint16_t* X;
  int64_t ldx;
  int gpr;          // units per row
  int64_t u_begin;  // this block's units
  int64_t u_end;
};

// Thread 0: bulk-copy units [u0, u1) into `dst`, one copy per row segment.
__device__ __forceinline__ void issue_chunk(const UnitRange& ur, int64_t u0, int64_t u1, uint8_t* dst, uint32_t bar) {
  mbar_arrive_expect_tx(bar, static_cast<uint32_t>((u1 - u0) * 512));
  for (int64_t u = u0; u < u1;) {
    const int64_t r = u / ur.gpr;
    int64_t seg_end = (r + 1) * ur.gpr;
    if (seg_end > u1) seg_end = u1;
    const uint16_t* src = ur.X + r * ur.ldx + ((u - r * ur.gpr) << 8);
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst + (u - u0) * 512)),
                 "l"(src), "r"(static_cast<uint32_t>((seg_end - u) * 512)), "r"(bar)
                 : "memory");
    u = seg_end;
  }
}

// Common streaming loop.  For every chunk, `body(P, u, k0)` gets the lane's 64
// unnormalised rotated values of unit u as pairs (u < 0 for lanes past the
// block's range) and the XOR k0 = unit & 7 of its slot order.  `zero` must be 0 at run
// time; it ties each warp's slot release to the values it loaded.
template <int kDig, class Body>
__device__ __forceinline__ void stream_units(const UnitRange& ur, uint8_t* smem, int* status, int zero, Body body) {
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kOffBars);
  uint64_t* empty = full + kDepth;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int l = lane & 3;
  const int uc = threadIdx.x >> 2;  // unit inside the chunk
  const int k0 = uc & 7;
  const int64_t n = ur.u_end - ur.u_begin;
  const int64_t nchunks = (n + kChunkUnits - 1) / kChunkUnits;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kDepth; ++i) {
      mbar_init(smem_u32(full + i), 1);
      mbar_init(smem_u32(empty + i), kWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();
  auto chunk_units = [&](int64_t c, int64_t& u0, int64_t& u1) {
    u0 = ur.u_begin + c * kChunkUnits;
    u1 = u0 + kChunkUnits < ur.u_end ? u0 + kChunkUnits : ur.u_end;
  };
  if (threadIdx.x == 0) {
    for (int i = 0; i < kDepth && i < nchunks; ++i) {
      int64_t u0, u1;
      chunk_units(i, u0, u1);
      issue_chunk(ur, u0, u1, smem + i * kChunkBytes, smem_u32(full + i));
    }
  }
  volatile int never = 0;
  for (int64_t c = 0; c < nchunks; ++c) {
    const int slot = static_cast<int>(c % kDepth);
    const uint32_t par = static_cast<uint32_t>((c / kDepth) & 1);
    if (!mbar_wait(smem_u32(full + slot), par, &never)) {
      record_status(status, CR_ERR_TIMEOUT);  // a copy never landed: give up on this block's chunks
      break;
    }
    int64_t u0, u1;
    chunk_units(c, u0, u1);
    const int64_t u = u0 + uc;
    const bool valid = u < u1;
    Raw raw;
    if (valid) {
      const uint8_t* unit = smem + slot * kChunkBytes + uc * 512 + 16 * l;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int p = k ^ k0;
        raw.q[k] = *reinterpret_cast<const uint4*>(unit + 128 * (p >> 1) + 64 * (p & 1));
      }
    } else {
      zero_raw(raw);
    }
    // release the slot once every lane's reads have returned (the mask depends on the data)
    const uint32_t dep = raw.q[0].x ^ raw.q[1].x ^ raw.q[2].x ^ raw.q[3].x ^ raw.q[4].x ^ raw.q[5].x ^ raw.q[6].x ^
                         raw.q[7].x;
    __syncwarp(~(dep & static_cast<uint32_t>(zero)));
    if (lane == 0) mbar_arrive(smem_u32(empty + slot));
    if (threadIdx.x == 0 && c + kDepth < nchunks) {
      if (!mbar_wait(smem_u32(empty + slot), par, &never)) {
        record_status(status, CR_ERR_TIMEOUT);
      } else {
        int64_t v0, v1;
        chunk_units(c + kDepth, v0, v1);
        issue_chunk(ur, v0, v1, smem + slot * kChunkBytes, smem_u32(full + slot));
      }
    }
    Pairs P;
    widen_pairs(raw, P);
    if constexpr (kDig > 0) fwht256_mapped<kDig>(P);
    body(P, valid ? u : int64_t(-1), k0);
    (void)warp;
  }
}

// Units per alignment step of a block's range: groups of 1024 combine four consecutive units inside a
// warp's 8, so their ranges start on a multiple of 8 units (rows then hold a multiple of 4 units).
template <int kDig>
__host__ __device__ constexpr int range_align() { return kDig == 5 ? 8 : 1; }

template <int kAlign>
__device__ __forceinline__ UnitRange unit_range(const uint16_t* X, int rows, int K, int64_t ldx) {
  UnitRange ur;
  ur.X = X;
  ur.ldx = ldx;
  ur.gpr = K >> 8;
  const int64_t units = static_cast<int64_t>(rows) * ur.gpr;
  if constexpr (kAlign == 1) {
    ur.u_begin = units * blockIdx.x / gridDim.x;
    ur.u_end = units * (blockIdx.x + 1) / gridDim.x;
  } else {
    const int64_t steps = (units + kAlign - 1) / kAlign;
    const int64_t b = kAlign * (steps * blockIdx.x / gridDim.x);
    const int64_t e = kAlign * (steps * (blockIdx.x + 1) / gridDim.x);
    ur.u_begin = b < units ? b : units;
    ur.u_end = e < units ? e : units;
  }
  return ur;
}


// Codes of the lane's 64 rotated values (pairs P, slot XOR k0) -> the warp's staging buffer `stg`
// (its 8 units, 128 or 256 code bytes each, unit uw = lane / 4 at uw * unit bytes).  Every lane then
// makes its stores visible to the async proxy; the caller syncs the warp before a bulk store reads them.
template <int kFmt>
__device__ __forceinline__ void codes_to_stage(const Pairs& P, int k0, float2 r2, float2 ns2, uint8_t* stg) {
  const int lane = threadIdx.x & 31, l = lane & 3, uw = lane >> 2;
  const float2 magic2 = make_float2(12582912.0f, 12582912.0f);
  // codes: correctly rounded y / s (Markstein step, as div_rn_by), then round half to even
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
    // slot k = elements 8k .. 8k+7 of v: pairs 8(k&3) .. +7, half k >> 2
    uint32_t c[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) c[e] = (k < 4) ? cx[8 * k + e] : cy[8 * (k - 4) + e];
    if constexpr (kFmt == kFmtPacked4) {
      // piece p = k ^ k0 holds elements 32p + 8l .. +7 of the unit: packed bytes 16p + 4l .. +3
      *reinterpret_cast<uint32_t*>(stg + uw * 128 + 16 * (k ^ k0) + 4 * l) = pack8(c);
    } else {
      // one code per byte (the low byte of each word): bytes 32p + 8l .. +7
      const uint32_t lo = __byte_perm(__byte_perm(c[0], c[1], 0x0040), __byte_perm(c[2], c[3], 0x0040), 0x5410);
      const uint32_t hi = __byte_perm(__byte_perm(c[4], c[5], 0x0040), __byte_perm(c[6], c[7], 0x0040), 0x5410);
      *reinterpret_cast<uint2*>(stg + uw * 256 + 32 * (k ^ k0) + 8 * l) = make_uint2(lo, hi);
    }
  }
  fence_proxy_async_smem();
}

// codes_to_stage, then bulk copies of the staged codes to Xq, one per row segment of the warp's units
// (unit u of this lane; u < 0 marks lanes past the end, and a warp's existing units are a prefix of its
// 8).  Lane 0 commits one bulk group; the caller makes sure `stg` is no longer read by an earlier group.
template <int kFmt>
__device__ __forceinline__ void codes_to_global(const Pairs& P, int64_t u, int k0, float2 r2, float2 ns2,
                                                uint8_t* stg, const UnitRange& ur, uint8_t* __restrict__ Xq,
                                                int64_t ldq) {
  constexpr int kUnitBytes = kFmt == kFmtPacked4 ? 128 : 256;  // codes of one 256-element unit
  const int lane = threadIdx.x & 31;
  codes_to_stage<kFmt>(P, k0, r2, ns2, stg);
  const int64_t u0w = __shfl_sync(0xffffffffu, u, 0);
  const int cnt = __popc(__ballot_sync(0xffffffffu, u >= 0)) >> 2;
  if (lane == 0 && cnt > 0) {
    for (int64_t x = u0w; x < u0w + cnt;) {
      const int64_t r = x / ur.gpr;
      int64_t seg_end = (r + 1) * ur.gpr;
      if (seg_end > u0w + cnt) seg_end = u0w + cnt;
      uint8_t* dst = Xq + r * ldq + (x - r * ur.gpr) * kUnitBytes;
      asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
                   "r"(smem_u32(stg + (x - u0w) * kUnitBytes)),
                   "r"(static_cast<uint32_t>((seg_end - x) * kUnitBytes))
                   : "memory");
      x = seg_end;
    }
    bulk_commit_group();
  }
}

template <int kDig>
__global__ void __launch_bounds__(kThreads, 2) act_amax_kernel(const uint16_t* __restrict__ X, int rows, int K,
                                                               int64_t ldx, float* __restrict__ partial,
                                                               int* __restrict__ status, int zero) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float red[kThreads / 32];
  float amax = 0.f;
  stream_units<kDig>(unit_range<range_align<kDig>()>(X, rows, K, ldx), smem, status, zero,
                     [&](const Pairs& P, int64_t, int) {
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fmaxf(fabsf(P.w[i].x), fabsf(P.w[i].y)));
  });
  amax = block_max(amax, red);
  if (threadIdx.x == 0) partial[blockIdx.x] = amax;
}

template <int kFmt, int kDig>
__global__ void __launch_bounds__(kThreads, 2) act_quant_kernel(const uint16_t* __restrict__ X, int rows, int K,
                                                                int64_t ldx, const float* __restrict__ partial,
                                                                int npartial, uint8_t* __restrict__ Xq,
                                                                float* __restrict__ scale_out, int nscale,
                                                                int* __restrict__ status, int zero) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float red[kThreads / 32];
  float a = 0.f;
  for (int i = threadIdx.x; i < npartial; i += kThreads) a = fmaxf(a, partial[i]);
  const float amax_v = block_max(a, red);
  float s_v, r_v, s_out;
  value_scale<kFmt, kDig>(amax_v, s_v, r_v, s_out);
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < nscale; i += kThreads) scale_out[i] = s_out;
  const UnitRange ur = unit_range<range_align<kDig>()>(X, rows, K, ldx);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ldq = kFmt == kFmtPacked4 ? (K >> 1) : K;
  uint8_t* stage0 = smem + kOffStage + warp * 2 * kStageWarpBytes;
  int chunk = 0;
  const float2 r2 = make_float2(r_v, r_v), ns2 = make_float2(-s_v, -s_v);
  stream_units<kDig>(ur, smem, status, zero, [&](const Pairs& P, int64_t u, int k0) {
    // INT4: two 1 KB buffers per warp, alternating; INT8: one 2 KB buffer
    uint8_t* stg = kFmt == kFmtPacked4 ? stage0 + (chunk & 1) * kStageWarpBytes : stage0;
    if (lane == 0) {
      if (kFmt == kFmtPacked4) bulk_wait_group_read<1>(); else bulk_wait_group_read<0>();  // buffer no longer read
    }
    __syncwarp();
    codes_to_global<kFmt>(P, u, k0, r2, ns2, stg, ur, Xq, ldq);
    ++chunk;
  });
  if (lane == 0) bulk_wait_group<0>();  // every packed code has been written
}


// ---------------------------------------------------------------------------
// TMEM and shared-memory helpers of the one-launch pass
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_st_x32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// Pairs <-> 64 TMEM columns of this thread's lane: column 2i = pair i .x, 2i + 1 = .y.
__device__ __forceinline__ void pairs_to_tmem(const Pairs& P, uint32_t taddr) {
  uint32_t r[32];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      r[2 * i] = __float_as_uint(P.w[16 * h + i].x);
      r[2 * i + 1] = __float_as_uint(P.w[16 * h + i].y);
    }
    tmem_st_x32(taddr + 32u * h, r);
  }
}
__device__ __forceinline__ void pairs_from_tmem(Pairs& P, uint32_t taddr) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t r[32];
    tmem_ld32(taddr + 32u * h, r);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 16; ++i) P.w[16 * h + i] = make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
  }
}

// ---------------------------------------------------------------------------
// One-launch pass: persistent, one CTA of 16 warps per SM (cooperative launch)
// ---------------------------------------------------------------------------
// Units are numbered row by row and cut into tiles of 8 (one warp's share, 4 KB of bf16; for groups of
// 1024 a tile holds two whole groups, since rows hold a multiple of 4 units).  The grid has one CTA per SM
// (one per tile for a tensor of fewer tiles than SMs); CTA b owns a contiguous range of tiles and walks it
// in rounds of 16 tiles, tile t of a round going to warp t, so a round reads 64 KB of consecutive units.
// A warp whose tile of a round lies past its CTA's range (in the last round only) skips that round.
// Each lane loads its unit's 64 values straight from global memory into registers, the next round's while
// it works on this one: plain vector loads keep the DRAM busier than bulk or tensor copies, whose
// per-instruction cost caps them well below the HBM bandwidth at these sizes, and no shared-memory stage
// is needed.
//
// Phase 1 rotates every unit and takes the max; the rotated float32 values of the CTA's last two rounds
// stay in TMEM (512 columns x 128 lanes) and those of the round before in shared memory (128 KB).  A grid
// barrier (a weighted arrival counter and a running max in the workspace) publishes the global max;
// between arriving and waiting, each warp rotates the first round that phase 2 reads again (the rotation
// does not need the scale).  Phase 2 quantises that round and the three kept rounds, then loads the other
// rounds again in reverse order, the most recently read first, so on a tensor larger than L2 the second
// read finds its tail there.  Codes go from registers straight to Xq.  A programmatic dependent launch
// (the few-token GEMM of the one-call layer) may start as soon as every CTA has begun.
constexpr int kQThreads = 512;
constexpr int kQWarps = kQThreads / 32;
constexpr int kQTmemRounds = 2;
constexpr int kQKeepBytes = kQThreads * 64 * 4;  // one more round of rotated values in shared memory

// Every launch adds exactly kQBarWeight to the arrival counter (the CTAs' weights sum to it), so its
// barrier completes at base + kQBarWeight, base = the counter at launch start rounded down to a multiple
// of kQBarWeight; the launch's max slot alternates with the parity of base / kQBarWeight.
constexpr unsigned long long kQBarWeight = 1ull << 16;

struct QArgs {
  const uint16_t* x;
  int64_t ldx;
  uint8_t* xq;                    // codes [rows, K / 2] (INT4) or [rows, K] (INT8), dense
  int gpr;                        // units per row
  int units;                      // rows * gpr, below 2^31 (the launcher checks)
  int ntiles;                     // ceil(units / 8)
  float* scale_out;
  int nscale;
  unsigned long long* bar_count;  // weighted arrivals, never reset
  unsigned int* bar_max;          // [2] running max (float bits), by launch parity
  int* status;
};

template <int kFmt, int kDig>
__global__ void __launch_bounds__(kQThreads, 1) act_pass_kernel(const QArgs a) {
  extern __shared__ __align__(16) float4 keep[];  // [32 pairs / 2][kQThreads]: conflict-free 16-byte rows
  __shared__ float red[kQWarps + 4];
  __shared__ uint32_t tmem_slot;
  __shared__ int bar_ok;
  __shared__ unsigned long long bar_base;
  constexpr int kUnitBytes = kFmt == kFmtPacked4 ? 128 : 256;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k0 = lane >> 2;  // the lane's unit inside its warp's tile; also its slot XOR
  const int tb = static_cast<int>(static_cast<int64_t>(a.ntiles) * blockIdx.x / gridDim.x);
  const int te = static_cast<int>(static_cast<int64_t>(a.ntiles) * (blockIdx.x + 1) / gridDim.x);
  const int n = (te - tb + kQWarps - 1) / kQWarps;     // rounds of this CTA
  const int nt = n < kQTmemRounds ? n : kQTmemRounds;  // rounds kept in TMEM
  const int ns = n > nt ? 1 : 0;                       // and the round before them, in shared memory
  // the lane's unit in round c (-1 past the range or past the last unit)
  auto unit_of = [&](int c) {
    const int tile = tb + kQWarps * c + warp;
    const int u = 8 * tile + k0;
    return (tile < te && u < a.units) ? u : -1;
  };
  // a warp whose tile of round c lies past the CTA's range (only in a CTA's last round) skips that round
  // (not for groups of 1024, where the branch costs the register allocation more than it saves)
  auto active = [&](int c) { return kDig > 4 || tb + kQWarps * c + warp < te; };
  auto load = [&](int c, Raw& raw) {
    const int u = unit_of(c);
    if (u >= 0) {
      const int r = u / a.gpr;
      load_unit_mapped(a.x + r * a.ldx + (static_cast<int64_t>(u - r * a.gpr) << 8), k0, raw);
    } else {
      zero_raw(raw);
    }
  };

  // a programmatic dependent (the few-token GEMM of the one-call layer) may start now: it reads the codes
  // and the scale only after waiting for this grid to complete, and uses SMs this grid leaves free
  if (threadIdx.x == 0) griddep_launch_dependents();
  // the barrier's base: the counter rounded down to a multiple of kQBarWeight, the same from launch start
  // until this CTA arrives (the counter cannot reach base + kQBarWeight before then); read now, so that the
  // load's round trip is not on the way to the barrier
  unsigned long long count0 = 0;
  if (threadIdx.x == 0) count0 = ld_relaxed_gpu(a.bar_count);
  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
  auto tmem_cols = [&](int c) { return static_cast<uint32_t>((c - (n - nt)) * 256 + (warp >> 2) * 64); };

  // ---- phase 1: rotate, max; the last nt rounds' rotated values into TMEM
  float amax = 0.f;
  Raw nxt;
  if (n > 0) load(0, nxt);
  if (threadIdx.x == 0) bar_base = count0 & ~(kQBarWeight - 1);  // waits for the counter while round 0 loads
  for (int c = 0; c < n; ++c) {
    Raw raw = nxt;
    if (c + 1 < n) load(c + 1, nxt);  // in flight while this round is rotated
    if (!active(c)) continue;         // warp-uniform; its TMEM columns are never read back
    Pairs P;
    widen_pairs(raw, P);
    if constexpr (kDig > 0) fwht256_mapped<kDig>(P);
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fmaxf(fabsf(P.w[i].x), fabsf(P.w[i].y)));
    if (c >= n - nt) pairs_to_tmem(P, tmem + tmem_cols(c));
    if (ns && c == n - nt - 1) {
#pragma unroll
      for (int j = 0; j < 16; ++j)
        keep[j * kQThreads + threadIdx.x] = make_float4(P.w[2 * j].x, P.w[2 * j].y, P.w[2 * j + 1].x, P.w[2 * j + 1].y);
    }
  }
  // rounds m - 1 .. 0 are loaded again in phase 2 (m = n - nt - ns); the first is in flight across the barrier
  const int m = n - nt - ns;
  if (m > 0) load(m - 1, nxt);
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
  amax = warp_max(amax);
  if (lane == 0) red[warp] = amax;
  __syncthreads();

  // ---- grid barrier: every CTA's max is in the running max before any CTA reads it.  Thread 0 arrives
  // (a release reduction, no round trip), every warp rotates round m - 1, then thread 0 waits.
  unsigned long long base = 0;
  int par = 0;
  if (threadIdx.x == 0) {
    base = bar_base;
    float mx = 0.f;
    for (int w = 0; w < kQWarps; ++w) mx = fmaxf(mx, red[w]);
    par = static_cast<int>((base / kQBarWeight) & 1);
    red_max_relaxed_gpu(a.bar_max + par, __float_as_uint(mx));  // non-negative floats order like their bits
    const unsigned long long w = kQBarWeight / gridDim.x;
    red_add_release_gpu(a.bar_count, blockIdx.x == 0 ? kQBarWeight - w * (gridDim.x - 1) : w);
  }
  Pairs P0;
  if (m > 0) {
    Raw raw = nxt;
    if (m > 1) load(m - 2, nxt);
    widen_pairs(raw, P0);
    if constexpr (kDig > 0) fwht256_mapped<kDig>(P0);
  }
  if (threadIdx.x == 0) {
    const bool good = grid_wait(a.bar_count, base + kQBarWeight);
    red[kQWarps] = __uint_as_float(ld_relaxed_gpu(a.bar_max + par));
    // the other slot is the next launch's; the previous launch, its last user, has finished
    if (blockIdx.x == 0) st_relaxed_gpu(a.bar_max + (par ^ 1), 0u);
    bar_ok = good ? 1 : 0;
    if (!good) record_status(a.status, CR_ERR_TIMEOUT);
  }
  __syncthreads();
  float s_v, r_v, s_out;
  value_scale<kFmt, kDig>(red[kQWarps], s_v, r_v, s_out);
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < a.nscale; i += kQThreads) a.scale_out[i] = s_out;

  // ---- phase 2: codes, the TMEM rounds first, then the others again (reverse order)
  if (bar_ok) {
    const float2 r2 = make_float2(r_v, r_v), ns2 = make_float2(-s_v, -s_v);
    auto store = [&](const Pairs& P, int c) {
      const int u = unit_of(c);
      if (u >= 0) codes_to_unit_global<kFmt>(P, k0, r2, ns2, a.xq + static_cast<int64_t>(u) * kUnitBytes);
    };
    if (m > 0) store(P0, m - 1);
    for (int c = n - 1; c >= n - nt; --c) {
      if (!active(c)) continue;
      Pairs P;
      pairs_from_tmem(P, tmem + tmem_cols(c));
      store(P, c);
    }
    if (ns) {
      Pairs P;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float4 v = keep[j * kQThreads + threadIdx.x];
        P.w[2 * j] = make_float2(v.x, v.y);
        P.w[2 * j + 1] = make_float2(v.z, v.w);
      }
      store(P, m);
    }
    for (int c = m - 2; c >= 0; --c) {
      Raw raw = nxt;
      if (c > 0) load(c - 1, nxt);
      Pairs P;
      widen_pairs(raw, P);
      if constexpr (kDig > 0) fwht256_mapped<kDig>(P);
      store(P, c);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_slot, 512);
  }
}

// One block per row: pass 1 row max, pass 2 codes with the row's own scale.
template <int kFmt, int kDig>
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
    if constexpr (kDig > 0) fwht256_quad<kDig>(v);
#pragma unroll
    for (int i = 0; i < 64; ++i) amax = fmaxf(amax, fabsf(v[i]));
  }
  const float amax_v = block_max(amax, red);
  float s_v, r_v, s_out;
  value_scale<kFmt, kDig>(amax_v, s_v, r_v, s_out);
  if (threadIdx.x == 0) w_scale[row] = s_out;
  uint8_t* dst = Wq + static_cast<int64_t>(row) * (kFmt == kFmtPacked4 ? (K >> 1) : K);
  for (int base = 0; base < gpr; base += kUnitsPerIter) {
    const int g = base + (threadIdx.x >> 2);
    Raw r;
    if (g < gpr) load_raw(src + (g << 8), lane, r); else zero_raw(r);
    float v[64];
    widen(r, v);
    if constexpr (kDig > 0) fwht256_quad<kDig>(v);
    if (g < gpr) {
      if (kFmt == kFmtPacked4) quant_pack_store(v, s_v, r_v, dst + (g << 7), lane);
      else quant_store8(v, s_v, r_v, dst + (g << 8), lane);
    }
  }
}

// W4A8 weights ("Qwen-Image-Edit-2511 -- W4A8 ConvRot", build table and file layout:
// asymmetric 4-bit weights, group_size 16, convrot_groupsize 256).  One pass, four lanes per
// 256-element unit of a row; every group of 16 lies inside one lane's run of 32, so the group's
// min / max need no exchange.  Per group, with y the (rotated) float32 values:
//   s = fp16(fl(hi - lo) / 15), 1 if that is 0;  z = clamp(rne(-lo / s), 0, 15);
//   q = clamp(rne(y / s) + z, 0, 15)
// Outputs: Wq [N, K/2] (element 2j in the low nibble of byte j), gscale fp16 [N, K/16],
// gzero [N, K/32] (group 2j in the low nibble of byte j).
template <bool kRot>
__global__ void __launch_bounds__(kThreads) pack_w4a8_kernel(const uint16_t* __restrict__ W, int N, int K,
                                                               int64_t ldw, uint8_t* __restrict__ Wq,
                                                               __half* __restrict__ gscale,
                                                               uint8_t* __restrict__ gzero) {
  const int gpr = K >> 8;
  const int64_t units = static_cast<int64_t>(N) * gpr;
  const int lane = threadIdx.x & 31;
  const int off = lane_run_offset(lane);  // element offset of the lane's first run of 32
  for (int64_t u = static_cast<int64_t>(blockIdx.x) * kUnitsPerIter + (threadIdx.x >> 2); u < units;
       u += static_cast<int64_t>(gridDim.x) * kUnitsPerIter) {
    const int64_t row = u / gpr;
    const int g = static_cast<int>(u - row * gpr);
    Raw r;
    load_raw(W + row * ldw + (g << 8), lane, r);
    float v[64];
    widen(r, v);
    if (kRot) {
      fwht256_quad<4>(v);  // 16 * (x H): scale back to x H (exact)
#pragma unroll
      for (int i = 0; i < 64; ++i) v[i] = __fmul_rn(v[i], 0.0625f);
    }
    uint32_t words[8];
    uint32_t sc[2];
    uint32_t zb[2];
#pragma unroll
    for (int grp = 0; grp < 4; ++grp) {  // groups: run 0 -> 0, 1; run 1 -> 2, 3
      float lo = v[16 * grp], hi = v[16 * grp];
#pragma unroll
      for (int i = 1; i < 16; ++i) {
        lo = fminf(lo, v[16 * grp + i]);
        hi = fmaxf(hi, v[16 * grp + i]);
      }
      __half sh = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), 15.f));
      if (__half2float(sh) == 0.f) sh = __float2half_rn(1.f);
      const float sf = __half2float(sh);
      const float zf = fminf(fmaxf(rintf(__fdiv_rn(-lo, sf)), 0.f), 15.f);
      const uint32_t z = static_cast<uint32_t>(zf);
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        uint32_t acc = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float t = rintf(__fdiv_rn(v[16 * grp + 8 * w + e], sf)) + zf;
          acc |= static_cast<uint32_t>(fminf(fmaxf(t, 0.f), 15.f)) << (4 * e);
        }
        words[2 * grp + w] = acc;
      }
      const uint32_t sbits = static_cast<uint32_t>(__half_as_ushort(sh));
      if (grp & 1) {
        sc[grp >> 1] |= sbits << 16;
        zb[grp >> 1] |= z << 4;
      } else {
        sc[grp >> 1] = sbits;
        zb[grp >> 1] = z;
      }
    }
    uint8_t* q_unit = Wq + row * (K >> 1) + (g << 7);
    *reinterpret_cast<uint4*>(q_unit + (off >> 1)) = make_uint4(words[0], words[1], words[2], words[3]);
    *reinterpret_cast<uint4*>(q_unit + (off >> 1) + 32) = make_uint4(words[4], words[5], words[6], words[7]);
    // groups of the unit: 16; the lane's first run holds groups off/16, off/16 + 1, its second run
    // groups off/16 + 4, off/16 + 5 (off/16 is even)
    uint32_t* s_unit = reinterpret_cast<uint32_t*>(gscale + row * (K >> 4) + (g << 4));
    s_unit[off >> 5] = sc[0];
    s_unit[(off >> 5) + 2] = sc[1];
    uint8_t* z_unit = gzero + row * (K >> 5) + (g << 3);
    z_unit[off >> 5] = static_cast<uint8_t>(zb[0]);
    z_unit[(off >> 5) + 2] = static_cast<uint8_t>(zb[1]);
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

// Formats: (bits, rotate) in {(4, true), (8, true), (8, false)}; the fourth
// combination (INT4 without rotation) is accepted too and costs nothing extra.
template <int kFmt, int kDig>
static bool stream_attrs_set(int dev) {
  static int done[64] = {};
  if (dev < 0 || dev >= 64) return false;
  if (!done[dev]) {
    if (cudaFuncSetAttribute(act_amax_kernel<kDig>, cudaFuncAttributeMaxDynamicSharedMemorySize, kStreamSmem) !=
            cudaSuccess ||
        cudaFuncSetAttribute(act_quant_kernel<kFmt, kDig>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kStreamSmem) != cudaSuccess)
      return false;
    done[dev] = 1;
  }
  return true;
}

template <int kFmt, int kDig>
static cudaError_t act_two_pass(const uint16_t* X, int rows, int K, int64_t ldx, float* partial, int grid, uint8_t* Xq,
                                float* scale_out, int nscale, int* status, cudaStream_t stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (!stream_attrs_set<kFmt, kDig>(dev)) return cudaErrorInvalidValue;
  act_amax_kernel<kDig><<<grid, kThreads, kStreamSmem, stream>>>(X, rows, K, ldx, partial, status, 0);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  act_quant_kernel<kFmt, kDig><<<grid, kThreads, kStreamSmem, stream>>>(X, rows, K, ldx, partial, grid, Xq,
                                                                         scale_out, nscale, status, 0);
  return cudaGetLastError();
}

// The one-launch pass: a cooperative launch of one CTA per SM (fewer for a small tensor).  cudaErrorCooperativeLaunchTooLarge
// when the SMs cannot all hold one CTA (or the tensor has 2^31 units or more).
template <int kFmt, int kDig>
static cudaError_t act_one_launch(const uint16_t* X, int rows, int K, int64_t ldx, uint8_t* Xq, float* scale_out,
                                  int nscale, uint8_t* workspace, int num_sms, cudaStream_t stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static int done[64] = {};
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!done[dev]) {
    if ((e = cudaFuncSetAttribute(act_pass_kernel<kFmt, kDig>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  kQKeepBytes)) != cudaSuccess)
      return e;
    done[dev] = 1;
  }
  const int gpr = K >> 8;
  const int64_t units = static_cast<int64_t>(rows) * gpr;
  if (units >= (int64_t(1) << 31) - 8) return cudaErrorCooperativeLaunchTooLarge;
  QArgs a;
  a.x = X;
  a.ldx = ldx;
  a.xq = Xq;
  a.gpr = gpr;
  a.units = static_cast<int>(units);
  a.ntiles = static_cast<int>((units + 7) / 8);
  a.scale_out = scale_out;
  a.nscale = nscale;
  a.bar_count = reinterpret_cast<unsigned long long*>(workspace + kWsActBarOff);
  a.bar_max = reinterpret_cast<unsigned int*>(workspace + kWsActBarOff + 16);
  a.status = reinterpret_cast<int*>(workspace + kWsStatusOff);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident: the grid barrier cannot wait for an unlaunched CTA
  attr[0].val.cooperative = 1;
  // one CTA per SM, but no more CTAs than tiles: a small tensor (few tokens) spreads one warp's tile per
  // SM, keeps its grid barrier short and leaves the other SMs to the GEMM that may start beside it
  const int grid = a.ntiles < num_sms ? (a.ntiles < 1 ? 1 : a.ntiles) : num_sms;
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kQThreads, 1, 1);
  cfg.dynamicSmemBytes = kQKeepBytes;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, act_pass_kernel<kFmt, kDig>, a);
}

template <int kFmt, int kDig>
static cudaError_t act_any(const uint16_t* X, int rows, int K, int64_t ldx, uint8_t* Xq, float* scale_out, int nscale,
                           uint8_t* workspace, int num_sms, int path, cudaStream_t stream) {
  if (path != kActTwoPass && rows > 0 && num_sms > 0) {
    const cudaError_t e = act_one_launch<kFmt, kDig>(X, rows, K, ldx, Xq, scale_out, nscale, workspace, num_sms,
                                                     stream);
    if (e != cudaErrorCooperativeLaunchTooLarge || path == kActOneLaunch) return e;
    cudaGetLastError();  // the SMs are not all available for one CTA each: use the two streaming passes
  }
  float* partial = reinterpret_cast<float*>(workspace + kWsPartialOff);
  int* status = reinterpret_cast<int*>(workspace + kWsStatusOff);
  return act_two_pass<kFmt, kDig>(X, rows, K, ldx, partial, act_grid(rows, K, num_sms), Xq, scale_out, nscale,
                                   status, stream);
}

// Digit passes of the rotation for a group size (0: no rotation); -1 for a size that is not built.
static int rotation_digits(bool rotate, int group) {
  if (!rotate) return 0;
  return group == 1024 ? 5 : group == 256 ? 4 : group == 64 ? 3 : group == 16 ? 2 : -1;
}

cudaError_t launch_act_fmt(const uint16_t* X, int rows, int K, int64_t ldx, uint8_t* Xq, float* scale_out, int nscale,
                           int fmt, bool rotate, int group, uint8_t* workspace, int num_sms, int path,
                           cudaStream_t stream) {
  const int dig = rotation_digits(rotate, group);
#define CR_ACT_CASE(F, D)                                                                                   \
  if (fmt == F && dig == D)                                                                                \
    return act_any<F, D>(X, rows, K, ldx, Xq, scale_out, nscale, workspace, num_sms, path, stream);
  CR_ACT_CASE(kFmtPacked4, 5)
  CR_ACT_CASE(kFmtPacked4, 4)
  CR_ACT_CASE(kFmtPacked4, 3)
  CR_ACT_CASE(kFmtPacked4, 2)
  CR_ACT_CASE(kFmtPacked4, 0)
  CR_ACT_CASE(kFmtByte8, 5)
  CR_ACT_CASE(kFmtByte8, 4)
  CR_ACT_CASE(kFmtByte8, 3)
  CR_ACT_CASE(kFmtByte8, 2)
  CR_ACT_CASE(kFmtByte8, 0)
#undef CR_ACT_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_act(const uint16_t* X, int rows, int K, int64_t ldx, uint8_t* Xq, float* scale_out, int nscale,
                       uint8_t* workspace, int num_sms, cudaStream_t stream) {
  return act_any<kFmtPacked4, 4>(X, rows, K, ldx, Xq, scale_out, nscale, workspace, num_sms, kActAuto, stream);
}

cudaError_t launch_pack_rows_fmt(const uint16_t* W, int rows, int K, int64_t ldw, uint8_t* Wq, float* w_scale,
                                 int fmt, bool rotate, int group, cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  const int dig = rotation_digits(rotate, group);
#define CR_ROWS_CASE(F, D)                                                                  \
  if (fmt == F && dig == D) {                                                              \
    pack_rows_kernel<F, D><<<rows, kThreads, 0, stream>>>(W, K, ldw, Wq, w_scale);         \
    return cudaGetLastError();                                                             \
  }
  CR_ROWS_CASE(kFmtPacked4, 5)
  CR_ROWS_CASE(kFmtPacked4, 4)
  CR_ROWS_CASE(kFmtPacked4, 3)
  CR_ROWS_CASE(kFmtPacked4, 2)
  CR_ROWS_CASE(kFmtPacked4, 0)
  CR_ROWS_CASE(kFmtByte8, 5)
  CR_ROWS_CASE(kFmtByte8, 4)
  CR_ROWS_CASE(kFmtByte8, 3)
  CR_ROWS_CASE(kFmtByte8, 2)
  CR_ROWS_CASE(kFmtByte8, 0)
#undef CR_ROWS_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_pack_w4a8(const uint16_t* W, int N, int K, int64_t ldw, bool rotate, uint8_t* Wq, void* gscale,
                             uint8_t* gzero, int num_sms, cudaStream_t stream) {
  if (N <= 0) return cudaSuccess;
  const int64_t units = static_cast<int64_t>(N) * (K >> 8);
  int64_t grid = (units + kUnitsPerIter - 1) / kUnitsPerIter;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  if (grid > cap) grid = cap;
  __half* gs = static_cast<__half*>(gscale);
  if (rotate)
    pack_w4a8_kernel<true><<<static_cast<unsigned>(grid), kThreads, 0, stream>>>(W, N, K, ldw, Wq, gs, gzero);
  else
    pack_w4a8_kernel<false><<<static_cast<unsigned>(grid), kThreads, 0, stream>>>(W, N, K, ldw, Wq, gs, gzero);
  return cudaGetLastError();
}

cudaError_t launch_pack_rows(const uint16_t* W, int rows, int K, int64_t ldw, uint8_t* Wq, float* w_scale,
                             cudaStream_t stream) {
  return launch_pack_rows_fmt(W, rows, K, ldw, Wq, w_scale, kFmtPacked4, true, 256, stream);
}

}  // namespace cr
