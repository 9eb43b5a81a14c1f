// gemm_w4a4_small.cu -- INT4 x INT4 GEMM for few tokens (M <= 256) on sm_100a.
//
// Same product and epilogue as the CTA-pair kernel ("Qwen-Image-Edit-2511 --
// INT4 tensorwise W4A4 (+ConvRot, mixed int8 fallback)", section
// "Measurements": rank-one scaled s4 MMA).  With few tokens the layer is bound
// by streaming the packed weights from HBM ("Qwen3-4B -- ConvRot W4A4",
// "What it costs in speed": the fixed per-layer cost dominates at small token
// counts), so this kernel is arranged for that stream:
//
// * Operands swap roles: the MMA computes D[n, m] (weight row n, token m), so
//   the weights fill the MMA's M = 128 side and the tokens its N side (M
//   padded to Mp, a multiple of 16).  The output is written transposed.
// * Each CTA owns 128 weight rows.  K is split across a cluster of S CTAs
//   (S <= 8; two CTAs fit on an SM up to 128 tokens, one above) so that every
//   SM streams weights.  Each
//   CTA leaves its partial int32 sums in its own shared memory; after a
//   cluster barrier every CTA adds up one slice of the tile from all CTAs of
//   the cluster with distributed-shared-memory vector loads (exact integer
//   sums) and writes that slice's outputs.
// * Packed codes of both operands arrive by TMA (two k-blocks, i.e. 128 bytes
//   of every row, per box, 128-byte swizzle) in a ring sized to the shared
//   memory left by the widened-token ring.  A fill's weight half and its code
//   half complete on barriers of their own, so the weights are widened as soon
//   as they land, also while the codes are still being made.
// * The weights are widened into TMEM with one 32x32b store per row and
//   k-block (the MMA reads its A operand from TMEM); the tokens are widened
//   into the 128-byte-swizzled K-major layout the MMA reads from shared memory.
//   Widening places each nibble in the high half of a byte (int8 16*q), so the
//   MMA accumulates 256 * acc (exact in int32 for K <= 65536); codes are
//   permuted inside every group of 8 the same way for both operands.
//
// Fused layer (cr_w4a4_linear_ex in its one-launch mode, at most 256 tokens): the
// same kernel also rotates and quantises X, so the whole layer is one launch.  The producer
// starts the weight stream at once (weights do not depend on X); meanwhile
// warps 6-9 rotate this CTA's share of X's 256-element units and take their
// max, a grid-wide barrier publishes every CTA's max, the warps quantise their
// share with the global scale into packed codes in the workspace, and a second
// grid-wide barrier makes every code visible before the producer loads them.
// All CTAs are resident (cooperative launch), and both grid barriers are
// bounded waits like every other wait here.  The codes are those of
// cr_rotate_quant_act bit for bit (same transform, same division, same max).
//
// After the activation pass of the one-call layer (two launches), the GEMM launches as a programmatic
// dependent of that pass: its CTAs start on the SMs the pass leaves free, set up, load the first weight
// fills and widen them into the TMEM ring while the pass runs, and wait for the pass (griddepcontrol)
// before loading codes or reading the activation scale.
//
// Roles (320 threads per CTA):
//   warp 0       TMEM allocation (256 columns); MMA issuer
//   warp 1       TMA producer
//   warps 2-5    weight widening (one TMEM lane quarter each)
//   warps 6-9    the tile's weight scales and bias (loaded before the main loop);
//                token widening during the main loop; then accumulator -> shared
//                memory
//   all warps    the split-K sum and the epilogue
// Every wait is bounded; on expiry the CTA records CR_ERR_TIMEOUT in the
// device status word, skips its output and still takes part in every cluster
// barrier, so no CTA waits for another that gave up.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "cr_device.cuh"
#include "grid_sync.cuh"
#include "cr_internal.h"

namespace cr {
namespace {

#include "act_device.cuh"

constexpr int TM = 128;               // weight rows per CTA (MMA M)
constexpr int BK = 128;               // codes per k-block
constexpr int BKP = 64;               // packed bytes per row per k-block
constexpr int KPS = 2;                // k-blocks per packed fill
constexpr int PROW = KPS * BKP;       // packed bytes per row per fill (one 128-byte swizzle row)
constexpr int MAX_PST = 4;            // packed ring stages (runtime count <= this)
constexpr int MAX_ST = 4;             // widened ring stages (runtime count <= this)
constexpr int W_FILL = TM * PROW;     // 16 KB of packed weights per fill
constexpr int NUM_BARS = 3 * MAX_PST + 2 * MAX_ST + 2;
constexpr int NUM_THREADS = 320;
constexpr int PEMPTY_ARRIVALS = KPS * 8;  // per fill: 4 weight warps + 4 token warps, for each k-block
constexpr int FULL_ARRIVALS = 8;          // per k-block: the 4 weight warps and the 4 token warps
constexpr int EPI_WARP0 = 6;

// Two configurations: up to 128 tokens with two CTAs per SM (256 TMEM columns each), and up to 256
// tokens (kBig) with one CTA per SM, whose 512 TMEM columns hold an accumulator of up to 256 token
// columns, and larger rings.
template <bool kBig> struct SCfg {
  static constexpr int MAX_MP = kBig ? 256 : 128;               // padded tokens
  static constexpr int RING_BYTES = (kBig ? 128 : 64) * 1024;   // packed ring; after the main loop: partial sums
  static constexpr int BST_BYTES = (kBig ? 72 : 32) * 1024;     // widened tokens
  static constexpr int OFF_RING = 0;
  static constexpr int OFF_BST = OFF_RING + RING_BYTES;
  static constexpr int OFF_BAR = OFF_BST + BST_BYTES;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int OFF_EPI = OFF_MISC + 64;  // the tile's weight scales and bias, the activation scale
  static constexpr int SMEM_BYTES = OFF_EPI + 2 * TM * 4 + 16;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;
  static constexpr int CTAS_PER_SM = kBig ? 1 : 2;
  static constexpr int TMEM_COLS = kBig ? 512 : 256;
  static constexpr int A_COL0 = MAX_MP;  // accumulator: columns [0, Mp); weight ring from here, 32 per stage
  static_assert(A_COL0 + MAX_ST * 32 <= TMEM_COLS, "TMEM budget");
  static_assert(MAX_MP * TM * 4 <= RING_BYTES, "partial sums must fit in the packed ring");
  static_assert(CTAS_PER_SM * (SMEM_ALLOC + 1024) <= 233472, "shared memory per SM");
  static_assert(BST_BYTES >= 32 * 1024, "the fused layer keeps 32 units of rotated values in the token ring");
};

struct Smem {
  uint8_t* base;
  int fill_bytes;  // W_FILL + Mp * PROW
  int bst_bytes;   // Mp * BK
  int off_bst, off_bar, off_misc, off_epi;  // of the configuration (SCfg)
  __device__ uint8_t* wp(int p) const { return base + p * fill_bytes; }
  __device__ uint8_t* xp(int p) const { return base + p * fill_bytes + W_FILL; }
  __device__ uint8_t* bs(int s) const { return base + off_bst + s * bst_bytes; }
  __device__ int32_t* sum() const { return reinterpret_cast<int32_t*>(base); }  // [Mp][TM], over the ring
  __device__ uint32_t bar(int i) const { return smem_u32(base + off_bar + 8 * i); }
  __device__ uint32_t pfull(int p) const { return bar(p); }
  __device__ uint32_t pempty(int p) const { return bar(MAX_PST + p); }
  __device__ uint32_t full(int s) const { return bar(2 * MAX_PST + s); }
  __device__ uint32_t empty(int s) const { return bar(2 * MAX_PST + MAX_ST + s); }
  __device__ uint32_t acc_full() const { return bar(2 * MAX_PST + 2 * MAX_ST); }
  __device__ uint32_t x_ready() const { return bar(2 * MAX_PST + 2 * MAX_ST + 1); }  // fused: codes written
  __device__ uint32_t xfull(int p) const { return bar(2 * MAX_PST + 2 * MAX_ST + 2 + p); }  // a fill's codes
  __device__ uint32_t* tmem_slot() const { return reinterpret_cast<uint32_t*>(base + off_misc); }
  __device__ volatile int* abort_flag() const { return reinterpret_cast<volatile int*>(base + off_misc + 4); }
  __device__ float* act_red() const { return reinterpret_cast<float*>(base + off_misc + 16); }  // [9] (fused)
  __device__ float* epi_sw() const { return reinterpret_cast<float*>(base + off_epi); }           // [TM]
  __device__ float* epi_b() const { return reinterpret_cast<float*>(base + off_epi + 4 * TM); }   // [TM]
  __device__ float* epi_sa() const { return reinterpret_cast<float*>(base + off_epi + 8 * TM); }
};


__device__ __forceinline__ void fail(const Smem& sm, int* status) {
  record_status(status, CR_ERR_TIMEOUT);
  *sm.abort_flag() = 1;
}

// Activation side of the fused layer: X, the workspace codes the tensor map over Xq reads, the
// per-CTA maxima and the grid barrier's words.
struct FusedAct {
  const uint16_t* X;
  int64_t ldx;
  uint8_t* xq;          // packed codes [M, K/2], dense
  float* a_scale;       // the activation scale, written by CTA 0
  unsigned long long* bar_count;  // weighted arrivals, never reset: every launch adds exactly 2 * kBarWeight
  unsigned int* bar_max;          // [2] running max of the rotated values (float bits), by launch parity
};

// Every grid barrier of a launch adds exactly kBarWeight to the arrival counter (the CTAs' weights sum
// to it), so a launch's barriers complete at base + kBarWeight and base + 2 kBarWeight, where base is
// the counter at launch start rounded down to a multiple of 2 kBarWeight.
constexpr unsigned long long kBarWeight = 1ull << 16;

constexpr int ACT_WARP0 = 6;  // warps 6-9 run the activation phases of the fused layer
constexpr int ACT_THREADS = 128;
constexpr int ACT_UNITS = ACT_THREADS / kLanesPerUnit;  // 32 units per pass

// This CTA's share of kBarWeight (CTA 0 takes the remainder).
__device__ __forceinline__ unsigned long long bar_weight() {
  const unsigned long long w = kBarWeight / gridDim.x;
  return blockIdx.x == 0 ? kBarWeight - w * (gridDim.x - 1) : w;
}

// Grid-wide barrier over all CTAs of the launch (all resident), called by one thread per CTA: arrive
// with a release reduction of this CTA's weight (no round trip to wait for), then poll the counter
// with acquire loads until it reaches `target`.  Bounded: false after CR_WAIT_TIMEOUT_NS.
__device__ __forceinline__ bool grid_barrier(const FusedAct& fa, unsigned long long target) {
  return grid_arrive_wait(fa.bar_count, bar_weight(), target);
}

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Fused layer, warps 6-9, from kernel entry (they need none of the GEMM's set-up): the rotation
// of this CTA's units and their max, folded into a global running max as the CTA arrives at grid
// barrier 1; the global scale; the codes of the same units written to fa.xq; grid barrier 2, after
// which every code is visible to the producer's tensor-map loads.  The rotated values of up to 32
// units stay in shared memory (the widened-token ring, unused until the main loop) between the two
// phases; more units per CTA are rotated again.  The lane mapping, transform, division and
// rounding are those of the activation kernels, so the codes and the scale equal
// cr_rotate_quant_act's bit for bit.  Returns the activation scale (s_out); `ok` is false after a
// timeout (recorded, and the CTA's abort flag set).
template <int kDig>
__device__ float fused_act_phases(const FusedAct& fa, int M, int K, const Smem& sm, int* status, bool& ok) {
  const int t = threadIdx.x - ACT_WARP0 * 32;  // 0..127
  const int w = t >> 5, lane = threadIdx.x & 31;
  const int uc = t >> 2;   // unit of this lane inside a pass of 32
  const int k0 = uc & 7;   // its index inside the warp's 8 units
  const int gpr = K >> 8;
  const int64_t units = static_cast<int64_t>(M) * gpr;
  const int64_t u0 = units * blockIdx.x / gridDim.x, u1 = units * (blockIdx.x + 1) / gridDim.x;
  const bool keep = u1 - u0 <= ACT_UNITS;  // one pass: its rotated values wait in shared memory
  auto unit_ptr = [&](int64_t u) {
    const int64_t r = u / gpr;
    return fa.X + r * fa.ldx + ((u - r * gpr) << 8);
  };
  float2* kept = reinterpret_cast<float2*>(sm.bs(0)) + t;  // pair i at kept[128 i]: 32 KB, conflict-free
  float* red = sm.act_red();  // [0..3] per-warp maxima, [4] the global max, [5] the barrier outcome
  volatile int* flag = reinterpret_cast<volatile int*>(red + 5);
  // the counter before this launch's first barrier completes (it cannot without this CTA)
  const unsigned long long base = t == 0 ? ld_relaxed_gpu(fa.bar_count) & ~(2 * kBarWeight - 1) : 0ull;
  const int par = static_cast<int>((base / (2 * kBarWeight)) & 1);  // this launch's max slot
  // ---- phase A: max of the rotated values of this CTA's units
  float amax = 0.f;
  for (int64_t base = u0; base < u1; base += ACT_UNITS) {
    const int64_t u = base + uc;
    Raw raw;
    if (u < u1) load_unit_mapped(unit_ptr(u), k0, raw); else zero_raw(raw);
    Pairs P;
    widen_pairs(raw, P);
    fwht256_mapped<kDig>(P);
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fmaxf(fabsf(P.w[i].x), fabsf(P.w[i].y)));
    if (keep) {
#pragma unroll
      for (int i = 0; i < 32; ++i) kept[128 * i] = P.w[i];
    }
  }
  amax = warp_max(amax);
  if (lane == 0) red[w] = amax;
  named_bar_sync(1, ACT_THREADS);
  if (t == 0) {
    // non-negative floats order like their bit patterns
    red_max_relaxed_gpu(fa.bar_max + par, __float_as_uint(fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]))));
    const bool good = grid_barrier(fa, base + kBarWeight);
    red[4] = __uint_as_float(ld_relaxed_gpu(fa.bar_max + par));  // after the barrier's acquire: every CTA's max
    // the other slot is the next launch's; the previous launch, its last user, has finished
    if (blockIdx.x == 0) st_relaxed_gpu(fa.bar_max + (par ^ 1), 0u);
    *flag = good ? 1 : 0;
    if (!good) fail(sm, status);
  }
  named_bar_sync(1, ACT_THREADS);
  ok = *flag != 0;
  float s_v, r_v, s_out;
  value_scale<kFmtPacked4, kDig>(red[4], s_v, r_v, s_out);
  if (blockIdx.x == 0 && t == 0) *fa.a_scale = s_out;
  // ---- phase B: codes of the same units with the global scale
  if (ok) {
    const float2 r2 = make_float2(r_v, r_v), ns2 = make_float2(-s_v, -s_v);
    for (int64_t base = u0; base < u1; base += ACT_UNITS) {
      const int64_t u = base + uc;
      Pairs P;
      if (keep) {
#pragma unroll
        for (int i = 0; i < 32; ++i) P.w[i] = kept[128 * i];
      } else {
        Raw raw;
        if (u < u1) load_unit_mapped(unit_ptr(u), k0, raw); else zero_raw(raw);
        widen_pairs(raw, P);
        fwht256_mapped<kDig>(P);
      }
      if (u < u1) {
        const int64_t row = u / gpr;
        codes_to_unit_global<kFmtPacked4>(P, k0, r2, ns2, fa.xq + row * (K >> 1) + ((u - row * gpr) << 7));
      }
    }
  }
  // every code of this CTA is written: make them visible to tensor-map loads, then release them with
  // the arrival at grid barrier 2 (the CTA barrier orders every thread's stores before it)
  fence_proxy_async_global();
  named_bar_sync(1, ACT_THREADS);
  if (t == 0 && ok) {
    const bool good = grid_barrier(fa, base + 2 * kBarWeight);
    fence_proxy_async_global();
    if (!good) {
      *flag = 0;
      fail(sm, status);
    }
  }
  named_bar_sync(1, ACT_THREADS);
  ok = *flag != 0;
  return s_out;
}


__device__ __forceinline__ uint32_t widen_lo(uint32_t w) { return (w << 4) & 0xF0F0F0F0u; }
__device__ __forceinline__ uint32_t widen_hi(uint32_t w) { return w & 0xF0F0F0F0u; }

// Byte offset of 16-byte chunk c (0..3) of k-block half h (0..1) of row r in a
// packed box: rows of 128 bytes, chunk j of row r stored at chunk j ^ (r & 7).
__device__ __forceinline__ int packed_off(int r, int h, int c) { return r * PROW + ((((h << 2) | c) ^ (r & 7)) << 4); }

// D[tmem] (+)= A[tmem] * B[smem]^T, one CTA, issued by lane 0 of a converged warp.
__device__ __forceinline__ void umma_i8_ts_lane0(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                                 uint32_t accumulate, int lane) {
  asm volatile(
      "{ .reg .pred p, e; setp.ne.b32 p, %4, 0; setp.eq.s32 e, %5, 0; "
      "@e tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p; }" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(lane)
      : "memory");
}
__device__ __forceinline__ void umma_commit_lane0(uint32_t bar, int lane) {
  asm volatile(
      "{ .reg .pred e; setp.eq.s32 e, %1, 0; "
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0]; }" ::"r"(bar),
      "r"(lane)
      : "memory");
}

// Registers -> TMEM: this thread's lane, 32 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_st_row32(uint32_t taddr, const uint32_t (&r)[32]) {
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

// 16-byte load from the shared memory of a CTA of the cluster (address from mapa_shared).
__device__ __forceinline__ int4 ld_cluster_v4(uint32_t cluster_addr) {
  int4 v;
  asm volatile("ld.shared::cluster.v4.s32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(cluster_addr)
               : "memory");
  return v;
}

// kFusedDig = 0: the GEMM on codes already in memory; 2, 3, 4: the fused layer, whose activation
// phases rotate with that many base-4 digit passes (groups of 16, 64, 256) before quantising.
template <bool kOutS32, int kFusedDig, bool kBig>
__global__ void __launch_bounds__(NUM_THREADS, SCfg<kBig>::CTAS_PER_SM)
    w4a4_gemm_small_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                           const float* __restrict__ a_scale, const float* __restrict__ w_scale,
                           const uint16_t* __restrict__ bias, void* __restrict__ Yv, int64_t ldy, int M, int N, int K,
                           int Mp, int PS, int ST, int* __restrict__ status, const FusedAct fa, int pdl) {
  constexpr bool kFused = kFusedDig > 0;
  static_assert(!(kFused && kOutS32), "the fused layer writes bf16 outputs");
  using C = SCfg<kBig>;
  extern __shared__ uint8_t smem_raw[];
  Smem sm;
  sm.base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  sm.fill_bytes = W_FILL + Mp * PROW;
  sm.bst_bytes = Mp * BK;
  sm.off_bst = C::OFF_BST;
  sm.off_bar = C::OFF_BAR;
  sm.off_misc = C::OFF_MISC;
  sm.off_epi = C::OFF_EPI;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint32_t nct;
  asm("mov.u32 %0, %%cluster_nctarank;" : "=r"(nct));
  const int S = static_cast<int>(nct);  // CTAs of this tile's cluster = K splits
  const int split = S > 1 ? static_cast<int>(cluster_ctarank()) : 0;  // this CTA's K range
  const int tile = static_cast<int>(blockIdx.x) / S;
  const int n0 = tile * TM;
  const int nf = K / (BK * KPS);
  const int f0 = static_cast<int>(static_cast<int64_t>(nf) * split / S);
  const int f1 = static_cast<int>(static_cast<int64_t>(nf) * (split + 1) / S);
  const int n_fill = f1 - f0;  // >= 1: the host keeps S <= nf
  const int n_items = n_fill * KPS;

  if (threadIdx.x == 0) {
    for (int p = 0; p < PS; ++p) {
      // the weight and the code halves of a fill complete separately, so that the weights are widened
      // as soon as they land, also while the codes are still being made (fused, or programmatic dependent)
      mbar_init(sm.pfull(p), 1);
      mbar_init(sm.xfull(p), 1);
      mbar_init(sm.pempty(p), PEMPTY_ARRIVALS);
    }
    for (int s = 0; s < ST; ++s) {
      mbar_init(sm.full(s), FULL_ARRIVALS);
      mbar_init(sm.empty(s), 1);
    }
    mbar_init(sm.acc_full(), 1);
    mbar_init(sm.x_ready(), 1);
    *sm.abort_flag() = 0;
    fence_mbar_init();
  }
  if (warp == 1 && lane == 0) {
    prefetch_tmap(&tmap_w);
    prefetch_tmap(&tmap_x);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(sm.tmem_slot()), C::TMEM_COLS);
    tmem_relinquish();
  }
  volatile int* abort = sm.abort_flag();
  bool epi_ok = true;    // epilogue warps: the accumulator is complete and saved
  float sa_fused = 0.f;  // fused layer: the activation scale found by warps 6-9
  bool act_ok = true;    // fused layer: the activation phases completed
  uint32_t tmem_base = 0;
  if constexpr (kFused) {
    // warps 6-9 rotate and quantise X while the GEMM roles set up (named barrier 2, 192 threads);
    // they meet warp 0 at named barrier 3 (160 threads) once the codes are out, and only then use
    // TMEM or the mbarriers
    if (warp >= ACT_WARP0) {
      sa_fused = fused_act_phases<kFusedDig>(fa, M, K, sm, status, act_ok);
      tc_fence_before();
      named_bar_sync(3, 160);
      tc_fence_after();
      tmem_base = *sm.tmem_slot();
      if (threadIdx.x == ACT_WARP0 * 32 && act_ok) mbar_arrive(sm.x_ready());
    } else {
      tc_fence_before();
      named_bar_sync(2, 192);
      tc_fence_after();
      tmem_base = *sm.tmem_slot();
    }
  } else {
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    tmem_base = *sm.tmem_slot();
  }

  if (warp == 0) {
    // ------------------------------------------------------------ MMA issuer
    if constexpr (kFused) named_bar_sync(3, 160);  // the activation warps are done with their phases
    const uint32_t idesc = idesc_i8(TM, Mp);
    bool ok = true;
    int s = 0;
    uint32_t ph = 0;
    int last_s = -1;
    uint32_t last_ph = 0;
    for (int it = 0; it < n_items; ++it) {
      if (!mbar_wait(sm.full(s), ph, abort)) { ok = false; break; }
      __syncwarp();
      tc_fence_after();
      const uint64_t db = sw128_kmajor_desc(smem_u32(sm.bs(s)));
      const uint32_t a_tmem = tmem_base + static_cast<uint32_t>(C::A_COL0 + 32 * s);
#pragma unroll
      for (int kk = 0; kk < BK / 32; ++kk)
        umma_i8_ts_lane0(tmem_base, a_tmem + 8u * kk, db + 2u * kk, idesc, it | kk ? 1u : 0u, lane);
      umma_commit_lane0(sm.empty(s), lane);
      last_s = s;
      last_ph = ph;
      if (++s == ST) { s = 0; ph ^= 1u; }
    }
    if (ok) {
      umma_commit_lane0(sm.acc_full(), lane);
    } else {
      if (lane == 0) fail(sm, status);
      // let the MMAs already issued finish before TMEM is freed at the end
      if (last_s >= 0) {
        volatile int never = 0;
        mbar_wait(sm.empty(last_s), last_ph, &never);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      bool ok = true;
      int p = 0, issued = 0, x_issued = 0;
      uint32_t ph = 0;
      const uint32_t x_bytes = static_cast<uint32_t>(sm.fill_bytes - W_FILL);
      if (kFused || pdl) {
        // the weights of the first fills go out at once: they do not depend on X; the codes follow once
        // every CTA has written its share of them (fused), or once the activation pass this launch
        // depends on has completed (programmatic dependent)
        const int first = n_fill < PS ? n_fill : PS;
        for (int f = 0; f < first; ++f) {
          mbar_arrive_expect_tx(sm.pfull(f), W_FILL);
          tma_load_2d(smem_u32(sm.wp(f)), &tmap_w, (f0 + f) * PROW, n0, sm.pfull(f));
          ++issued;
        }
        bool x_ok = true;
        if constexpr (kFused) x_ok = mbar_wait(sm.x_ready(), 0, abort);
        else griddep_wait();
        if (!x_ok) {
          ok = false;
        } else {
          for (int f = 0; f < first; ++f) {
            mbar_arrive_expect_tx(sm.xfull(f), x_bytes);
            tma_load_2d(smem_u32(sm.xp(f)), &tmap_x, (f0 + f) * PROW, 0, sm.xfull(f));
            ++x_issued;
          }
          p = first % PS;
          ph = first == PS ? 1u : 0u;
        }
      }
      // a slot is free without a wait only on its first use (fused: the first PS fills went out above)
      bool next_free = n_fill > issued && (issued < PS || mbar_test(sm.pempty(p), ph ^ 1u));
      for (int f = issued; ok && f < n_fill; ++f) {
        if (!mbar_wait_from(sm.pempty(p), ph ^ 1u, next_free, abort)) { ok = false; break; }
        mbar_arrive_expect_tx(sm.pfull(p), W_FILL);
        tma_load_2d(smem_u32(sm.wp(p)), &tmap_w, (f0 + f) * PROW, n0, sm.pfull(p));
        mbar_arrive_expect_tx(sm.xfull(p), x_bytes);
        tma_load_2d(smem_u32(sm.xp(p)), &tmap_x, (f0 + f) * PROW, 0, sm.xfull(p));
        ++x_issued;
        ++issued;
        if (++p == PS) { p = 0; ph ^= 1u; }
        next_free = f + 1 < n_fill && (f + 1 < PS || mbar_test(sm.pempty(p), ph ^ 1u));
      }
      if (!ok) {
        fail(sm, status);
        // let the loads already issued land: the last weight and the last code half issued to each slot
        // (the code halves of the first fills may not have gone out)
        for (int q = 0; q < PS && q < issued; ++q) {
          const int last = q + PS * ((issued - 1 - q) / PS);
          volatile int never = 0;
          mbar_wait(sm.pfull(q), static_cast<uint32_t>((last / PS) & 1), &never);
          if (q < x_issued) {
            const int xlast = q + PS * ((x_issued - 1 - q) / PS);
            mbar_wait(sm.xfull(q), static_cast<uint32_t>((xlast / PS) & 1), &never);
          }
        }
      }
    }
  } else if (warp < EPI_WARP0) {
    // ------------------------------------------------------------ weights: packed ring -> widened TMEM (warps 2-5)
    const int q = warp & 3;       // TMEM lane quarter
    const int r = 32 * q + lane;  // weight row inside the tile (= TMEM lane)
    bool ok = true;
    int p = 0, s = 0;
    uint32_t pph = 0, eph = 1;
    for (int it = 0; it < n_items; ++it) {
      const int h = it & 1;
      if (!mbar_wait(sm.pfull(p), pph, abort)) { ok = false; break; }
      __syncwarp();
      const uint8_t* src = sm.wp(p);
      uint4 w4[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) w4[c] = *reinterpret_cast<const uint4*>(src + packed_off(r, h, c));
      if (!mbar_wait(sm.empty(s), eph, abort)) { ok = false; break; }
      uint32_t v[32];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint32_t w[4] = {w4[c].x, w4[c].y, w4[c].z, w4[c].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          v[8 * c + 2 * j] = widen_lo(w[j]);
          v[8 * c + 2 * j + 1] = widen_hi(w[j]);
        }
      }
      tmem_st_row32(tmem_base + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(C::A_COL0 + 32 * s), v);
      // the TMEM store consumed the widened words, hence the packed reads have completed
      __syncwarp();
      if (lane == 0) mbar_arrive(sm.pempty(p));
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sm.full(s));
      if (h == 1 && ++p == PS) { p = 0; pph ^= 1u; }
      if (++s == ST) { s = 0; eph ^= 1u; }
    }
    if (!ok) fail(sm, status);
  } else {
    // ------------------------------------------------------------ tokens: packed ring -> widened shared memory
    const int t = threadIdx.x - EPI_WARP0 * 32;  // 0..127
    // the tile's weight scale and bias of row n0 + t, for the epilogue: loaded now, in flight during the
    // main loop, and put in shared memory after it
    float ep_sw = 0.f, ep_b = 0.f;
    if (!kOutS32 && n0 + t < N) {
      ep_sw = __ldg(w_scale + n0 + t);
      if (bias) ep_b = __uint_as_float(static_cast<uint32_t>(__ldg(bias + n0 + t)) << 16);
    }
    bool ok = act_ok;
    int p = 0, s = 0;
    uint32_t pph = 0, eph = 1;
    for (int it = 0; ok && it < n_items; ++it) {
      const int h = it & 1;  // k-block inside the fill
      if (!mbar_wait(sm.xfull(p), pph, abort) || !mbar_wait(sm.empty(s), eph, abort)) { ok = false; break; }
      __syncwarp();
      const uint8_t* src = sm.xp(p);
      uint8_t* dst = sm.bs(s);
      for (int idx = t; idx < Mp * 4; idx += 128) {
        const int r = idx >> 2, c = idx & 3;
        const uint4 w = *reinterpret_cast<const uint4*>(src + packed_off(r, h, c));
        uint8_t* row = dst + (r >> 3) * 1024 + (r & 7) * 128;
        *reinterpret_cast<uint4*>(row + (((2 * c) ^ (r & 7)) << 4)) =
            make_uint4(widen_lo(w.x), widen_hi(w.x), widen_lo(w.y), widen_hi(w.y));
        *reinterpret_cast<uint4*>(row + (((2 * c + 1) ^ (r & 7)) << 4)) =
            make_uint4(widen_lo(w.z), widen_hi(w.z), widen_lo(w.w), widen_hi(w.w));
      }
      // the widened stores consumed the packed words: the packed reads have completed
      __syncwarp();
      if (lane == 0) mbar_arrive(sm.pempty(p));
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(sm.full(s));
      if (h == 1 && ++p == PS) { p = 0; pph ^= 1u; }
      if (++s == ST) { s = 0; eph ^= 1u; }
    }
    if (!ok) fail(sm, status);
    float ep_sa = 0.f;
    if (!kOutS32 && t == 0) {
      if constexpr (kFused) {
        ep_sa = sa_fused;
      } else {
        if (pdl) griddep_wait();  // a_scale comes from the activation pass this launch depends on
        ep_sa = __ldg(a_scale);   // in flight while the last MMAs complete
      }
    }
    // ------------------------------------------------------------ accumulator -> own shared memory
    epi_ok = ok && mbar_wait_warp(sm.acc_full(), 0, abort);
    if (!epi_ok && lane == 0) fail(sm, status);
    tc_fence_after();
    if (epi_ok) {
      const int q = warp & 3;
      const int rl = 32 * q + lane;  // weight row inside the tile
      const uint32_t trow = tmem_base + (static_cast<uint32_t>(32 * q) << 16);
      int32_t* sum = sm.sum();
      for (int ch = 0; ch < Mp; ch += 32) {
        uint32_t r[32];
        tmem_ld32(trow + static_cast<uint32_t>(ch), r);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (ch + j < Mp) sum[(ch + j) * TM + rl] = static_cast<int32_t>(r[j]);  // [token][row]
      }
    }
    if constexpr (!kOutS32) {
      sm.epi_sw()[t] = ep_sw;
      sm.epi_b()[t] = ep_b;
      if (t == 0) *sm.epi_sa() = ep_sa;
    }
  }

  // ---------------------------------------------------------------- split-K sum and epilogue
  // Every thread of every CTA of the cluster takes part in both cluster barriers, including
  // after a timeout, so no CTA waits for one that gave up.  Outputs (m, n0 + 4v .. 4v+3), m < M,
  // are vectors vi of M * TM/4; this CTA finishes vi in [V*split/S, V*(split+1)/S), every warp taking
  // part: thread t takes vi = v0 + t + NUM_THREADS j.
  static_assert(NUM_THREADS % (TM / 4) == 0, "a thread's vectors share its 4 output columns");
  const int t = threadIdx.x;
  const int V = M * (TM / 4);
  const int v0 = static_cast<int>(static_cast<int64_t>(V) * split / S);
  const int v1 = static_cast<int>(static_cast<int64_t>(V) * (split + 1) / S);
  __syncwarp();
  __syncthreads();  // this CTA's partial sums, scales and bias are in its shared memory (or it gave up)
  if (S > 1) cluster_sync();
  if (*abort == 0) {
    const uint32_t local = smem_u32(sm.sum());
    const int nl = 4 * ((v0 + t) % (TM / 4));
    const int n = n0 + nl;
    float pre_h[4] = {0.f, 0.f, 0.f, 0.f}, pre_l[4] = {0.f, 0.f, 0.f, 0.f}, pre_b[4] = {0.f, 0.f, 0.f, 0.f};
    if (!kOutS32 && v0 + t < v1 && n < N) {
      const float sa = *sm.epi_sa();
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float sw = sm.epi_sw()[nl + e];
        pre_h[e] = __fmul_rn(sa, sw);
        pre_l[e] = __fmaf_rn(sa, sw, -pre_h[e]);  // sa*sw = hi + lo exactly
        pre_b[e] = sm.epi_b()[nl + e];
      }
    }
    // Two vectors per step: both vectors' partial sums are loaded before either is added up.
    for (int vi = v0 + t; vi < v1 && n < N; vi += 2 * NUM_THREADS) {  // N is a multiple of 8: a vector is inside or outside
      const int nv = vi + NUM_THREADS < v1 ? 2 : 1;
      int4 sums[2] = {make_int4(0, 0, 0, 0), make_int4(0, 0, 0, 0)};  // exact integer sums over the K splits
#pragma unroll
      for (int c = 0; c < 8; ++c) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (h < nv && c < S) {
            const uint32_t off = 4u * static_cast<uint32_t>(((vi + NUM_THREADS * h) / (TM / 4)) * TM + nl);
            const int4 p = S > 1 ? ld_cluster_v4(mapa_shared(local + off, static_cast<uint32_t>(c)))
                                 : *reinterpret_cast<const int4*>(sm.sum() + off / 4);
            sums[h].x += p.x;
            sums[h].y += p.y;
            sums[h].z += p.z;
            sums[h].w += p.w;
          }
        }
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (h >= nv) break;
        const int m = (vi + NUM_THREADS * h) / (TM / 4);
        const int4 acc = sums[h];
        const int32_t a4[4] = {acc.x >> 8, acc.y >> 8, acc.z >> 8, acc.w >> 8};  // the MMA accumulated 256 * acc
        if constexpr (kOutS32) {
          *reinterpret_cast<int4*>(static_cast<int32_t*>(Yv) + static_cast<int64_t>(m) * ldy + n) =
              make_int4(a4[0], a4[1], a4[2], a4[3]);
        } else {
          uint32_t pk[2];
#pragma unroll
          for (int e2 = 0; e2 < 4; e2 += 2) {
            float y2[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              // |acc| < 2^22: adding 1.5 * 2^23 through the bit pattern converts to float exactly
              const float af = __fsub_rn(__int_as_float(a4[e2 + e] + 0x4B400000), 12582912.0f);
              y2[e] = __fmaf_rn(af, pre_l[e2 + e], __fmaf_rn(af, pre_h[e2 + e], pre_b[e2 + e]));
            }
            __nv_bfloat162 b2 = __floats2bfloat162_rn(y2[0], y2[1]);
            pk[e2 >> 1] = *reinterpret_cast<uint32_t*>(&b2);
          }
          *reinterpret_cast<uint2*>(static_cast<uint16_t*>(Yv) + static_cast<int64_t>(m) * ldy + n) =
              make_uint2(pk[0], pk[1]);
        }
      }
    }
  }
  if (S > 1) cluster_sync();  // no CTA leaves while another still reads its partial sums

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    // the MMAs have completed (acc_full, or the drain wait of the issuer on a timeout path)
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// 2-D uint8 tensor map over a dense [rows, cols] byte matrix: boxes of box_rows rows x 128 bytes,
// 128-byte swizzle; rows past the end read as zero codes.
bool packed_map(CUtensorMap* map, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  return make_tmap_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, ptr, rows, cols, cols, PROW, box_rows,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
}

// Largest number of resident clusters of `S` CTAs of one kernel configuration (cached per device and S).
template <bool kOutS32, int kFusedDig, bool kBig>
int max_clusters(int dev, int S, int num_sms, cudaStream_t stream) {
  static int cache[64][9] = {};
  if (cache[dev][S]) return cache[dev][S];
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(S);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(static_cast<unsigned>(S * (2 * num_sms / S)), 1, 1);
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = SCfg<kBig>::SMEM_ALLOC;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, w4a4_gemm_small_kernel<kOutS32, kFusedDig, kBig>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = -1;
  }
  cache[dev][S] = n;
  return n;
}

// The K split of a fused launch that the driver accepted (every CTA resident), per device and shape.
struct SplitCache {
  std::mutex mu;
  struct Entry { int dev, tiles, nf, S; } e[64];
  int n = 0;
  int find(int dev, int tiles, int nf) {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < n; ++i)
      if (e[i].dev == dev && e[i].tiles == tiles && e[i].nf == nf) return e[i].S;
    return 0;
  }
  void put(int dev, int tiles, int nf, int S) {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < n; ++i)
      if (e[i].dev == dev && e[i].tiles == tiles && e[i].nf == nf) return;
    if (n < 64) e[n++] = {dev, tiles, nf, S};
  }
};

// kFusedDig = 0: the GEMM on codes Xq already in memory.  Otherwise the fused layer: `fa` carries X
// and the workspace, Xq is the workspace's code area (read by the tensor map after the activation
// phases wrote it); returns kNotFused when the launch cannot keep every CTA resident, so that the
// caller runs the two-kernel path instead.
template <bool kOutS32, int kFusedDig, bool kBig>
int launch_small_impl(const void* Xq, const float* a_scale, const void* Wq, const float* w_scale, const void* bias,
                      void* Y, int64_t ldy, int M, int N, int K, int* status, int num_sms, cudaStream_t stream,
                      const FusedAct& fa, bool pdl = false) {
  constexpr bool kFused = kFusedDig > 0;
  using C = SCfg<kBig>;
  if (M == 0 || N == 0) return CR_OK;
  if (M > C::MAX_MP) return CR_ERR_UNSUPPORTED_SHAPE;
  static bool attr_done[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return CR_ERR_CUDA;
  auto kern = w4a4_gemm_small_kernel<kOutS32, kFusedDig, kBig>;
  if (!attr_done[dev]) {
    // all of the unified L1 / shared memory as shared memory: two CTAs per SM (also what the cluster
    // occupancy query below assumes)
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_ALLOC) != cudaSuccess ||
        cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
      return CR_ERR_CUDA;
    attr_done[dev] = true;
  }
  const int Mp = ((M + 15) / 16) * 16;
  const int tiles = (N + TM - 1) / TM;
  const int nf = K / (BK * KPS);
  int S = C::CTAS_PER_SM * num_sms / tiles;  // every SM streams weights
  if (S > 8) S = 8;
  if (S > nf) S = nf;
  if (S < 1) S = 1;
  // Fused: the grid barriers need every CTA resident, which the cooperative launch guarantees or
  // refuses.  Splits to try, largest first: the one the driver accepted before for this shape; else,
  // outside stream capture, every split from two CTAs per SM down; during a capture (where a refused
  // launch would invalidate the capture) only the split the cluster occupancy query vouches for.
  static SplitCache accepted;
  int s_hi = S, s_lo = 1;
  if constexpr (kBig && !kFused) {
    // one CTA per SM (what the occupancy query assumes for tensor-memory kernels): every cluster of the
    // split in one wave
    while (S > 1 && max_clusters<kOutS32, kFusedDig, kBig>(dev, S, num_sms, stream) < tiles) --S;
    s_hi = S;
  }
  if constexpr (kFused) {
    const int known = accepted.find(dev, tiles, nf);
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) {
      cudaGetLastError();
      cap = cudaStreamCaptureStatusActive;
    }
    if (known) {
      s_hi = s_lo = known;
    } else if (cap != cudaStreamCaptureStatusNone) {
      while (S >= 1 && max_clusters<kOutS32, kFusedDig, kBig>(dev, S, num_sms, stream) < tiles) --S;
      s_hi = s_lo = S;
    }
    if (s_hi < 1 || tiles * s_hi > kMaxActBlocks) return kNotFused;
  }
  const int fill = W_FILL + Mp * PROW;
  int PS = C::RING_BYTES / fill;
  if (PS > MAX_PST) PS = MAX_PST;
  int ST = C::BST_BYTES / (Mp * BK);
  if (ST > MAX_ST) ST = MAX_ST;
  if (PS < 2 || ST < 2) return CR_ERR_UNSUPPORTED_SHAPE;
  CUtensorMap tw, tx;
  if (!packed_map(&tw, Wq, static_cast<uint64_t>(N), static_cast<uint64_t>(K / 2), TM)) return CR_ERR_CUDA;
  if (!packed_map(&tx, Xq, static_cast<uint64_t>(M), static_cast<uint64_t>(K / 2), static_cast<uint32_t>(Mp)))
    return CR_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  if (kFused) {
    attr[1].id = cudaLaunchAttributeCooperative;  // fused: every CTA resident, or the launch is refused
    attr[1].val.cooperative = 1;
  } else {
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // start while the activation pass runs
    attr[1].val.programmaticStreamSerializationAllowed = 1;
  }
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM_ALLOC;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = kFused || pdl ? 2 : 1;
  for (S = s_hi; S >= s_lo; --S) {
    attr[0].val.clusterDim.x = static_cast<unsigned>(S);
    cfg.gridDim = dim3(static_cast<unsigned>(tiles * S), 1, 1);
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tw, tx, a_scale, w_scale, static_cast<const uint16_t*>(bias),
                                             Y, ldy, M, N, K, Mp, PS, ST, status, fa, pdl ? 1 : 0);
    if (e == cudaSuccess) {
      if (kFused) accepted.put(dev, tiles, nf, S);
      return CR_OK;
    }
    cudaGetLastError();  // a refused launch leaves no error behind
    if (!kFused) return CR_ERR_CUDA;
  }
  return kNotFused;  // no split could keep every CTA resident: the two-kernel path runs
}

}  // namespace

int launch_w4a4_gemm_small(const void* Xq, const float* a_scale, const void* Wq, const float* w_scale,
                           const void* bias, void* Y, int64_t ldy, int M, int N, int K, int* status, int num_sms,
                           cudaStream_t stream, bool after_act) {
  if (M > kSmallMaxM)
    return launch_small_impl<false, 0, true>(Xq, a_scale, Wq, w_scale, bias, Y, ldy, M, N, K, status, num_sms, stream,
                                             FusedAct{}, after_act);
  return launch_small_impl<false, 0, false>(Xq, a_scale, Wq, w_scale, bias, Y, ldy, M, N, K, status, num_sms, stream,
                                            FusedAct{}, after_act);
}

int launch_w4a4_gemm_small_s32(const void* Xq, const void* Wq, int32_t* C, int64_t ldc, int M, int N, int K,
                               int* status, int num_sms, cudaStream_t stream) {
  if (M > kSmallMaxM)
    return launch_small_impl<true, 0, true>(Xq, nullptr, Wq, nullptr, nullptr, C, ldc, M, N, K, status, num_sms,
                                            stream, FusedAct{});
  return launch_small_impl<true, 0, false>(Xq, nullptr, Wq, nullptr, nullptr, C, ldc, M, N, K, status, num_sms,
                                           stream, FusedAct{});
}

namespace {
template <bool kBig>
int linear_small_groups(const FusedAct& fa, const uint8_t* xq, const float* a_scale, const void* Wq,
                        const float* w_scale, const void* bias, void* Y, int64_t ldy, int M, int N, int K, int group,
                        int* status, int num_sms, cudaStream_t stream) {
  switch (group) {
    case 256:
      return launch_small_impl<false, 4, kBig>(xq, a_scale, Wq, w_scale, bias, Y, ldy, M, N, K, status, num_sms,
                                               stream, fa);
    case 64:
      return launch_small_impl<false, 3, kBig>(xq, a_scale, Wq, w_scale, bias, Y, ldy, M, N, K, status, num_sms,
                                               stream, fa);
    case 16:
      return launch_small_impl<false, 2, kBig>(xq, a_scale, Wq, w_scale, bias, Y, ldy, M, N, K, status, num_sms,
                                               stream, fa);
    default:
      return kNotFused;  // groups of 1024 combine units across lanes of a warp: the two-kernel path
  }
}
}  // namespace

int launch_w4a4_linear_small(const uint16_t* X, int64_t ldx, const void* Wq, const float* w_scale, const void* bias,
                             void* Y, int64_t ldy, int M, int N, int K, int group, uint8_t* workspace, uint8_t* xq,
                             float* a_scale, int num_sms, cudaStream_t stream) {
  if (M > kSmallBigMaxM) return kNotFused;
  FusedAct fa;
  fa.X = X;
  fa.ldx = ldx;
  fa.xq = xq;
  fa.a_scale = a_scale;
  fa.bar_count = reinterpret_cast<unsigned long long*>(workspace + kWsLayerBarOff);
  fa.bar_max = reinterpret_cast<unsigned int*>(workspace + kWsLayerBarOff + 32);
  int* status = reinterpret_cast<int*>(workspace + kWsStatusOff);
  if (M > kSmallMaxM)
    return linear_small_groups<true>(fa, xq, a_scale, Wq, w_scale, bias, Y, ldy, M, N, K, group, status, num_sms,
                                     stream);
  return linear_small_groups<false>(fa, xq, a_scale, Wq, w_scale, bias, Y, ldy, M, N, K, group, status, num_sms,
                                    stream);
}

}  // namespace cr
