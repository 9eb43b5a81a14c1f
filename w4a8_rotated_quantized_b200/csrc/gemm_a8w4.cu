// gemm_a8w4.cu -- one-byte activation codes against packed signed INT4 weights
// on a CTA pair (tcgen05 cta_group::2 kind::i8), with the layer's scale/bias
// epilogue.
//
// The "INT8 branch" of the W4A4 format: INT8 activation codes (amax / 127)
// against the format's INT4 weights ("Qwen3-4B -- ConvRot W4A4 (ComfyUI text
// encoder)", section "Hardware": on newer GPUs the format runs an INT8
// activation branch).  (Fed INT4 codes one per byte, the same kernel computes
// the W4A4 product; measured, it is not faster than the kernel that widens
// packed INT4 activations, so the W4A4 calls keep that one.)
//
//   acc[m, n] = sum_k qa[m, k] * qw[n, k]   (exact in int32)
//   Y[m, n]   = bf16(acc * s_a * s_w[n] + bias[n])
//
// The activation operand needs no conversion, so it goes from a TMA ring
// straight into the MMA (shared-memory descriptor), as in the INT8 kernel; both
// CTAs' activation loads of a stage complete on the leader's barrier.  Only the
// weights are widened: a nibble placed in the high half of a byte reads as the
// int8 value 16 q, so the MMA accumulates 16 * acc (exact for K <= 65536) and
// the epilogue shifts by 4.  The activation bytes are in K order, so the
// widening interleaves each packed word's even and odd codes back into K order
// with byte permutes: widened byte e of a row holds code e.
//
// Tiles 256 x 256 (MMA M = 256, N = 256, K = 32: 128 cycles per instruction).
// Four stages, each holding one k-block: activations (128 rows x 128 bytes,
// 128-byte swizzle) and packed weights (128 rows x 64 bytes, unswizzled) by
// TMA, and the widened weights (128 rows x 128 bytes, 128-byte swizzle).  One
// "full" barrier per stage in the leader counts both CTAs' activation bytes
// and the widening warps of both CTAs; one "empty" barrier per stage in each
// CTA is the MMA's commit, after which the producer refills the stage and the
// widening warps may overwrite its widened weights.  So the MMA issuer waits
// once and commits once per k-block: with separate barriers for the TMA and the
// widened rings (two waits and two commits) the same kernel was 10-11% slower.
//
// Roles (448 threads per CTA):
//   warp 0      TMEM allocation; in the leader CTA, the MMA issuer
//   warp 1      TMA producer (both CTAs)
//   warps 2-5   epilogue (TMEM -> scale, bias -> bf16 -> TMA stores, or int32 rows)
//   warps 6-9   weight widening, even k-blocks | warps 10-13 odd k-blocks
// Every wait is bounded; on expiry the CTA records CR_ERR_TIMEOUT in the
// device status word and winds down.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "cr_device.cuh"
#include "cr_internal.h"

namespace cr {
namespace {

constexpr int CM = 128;            // activation rows per CTA (pair: 256)
constexpr int PN = 256;            // output columns per pair tile
constexpr int CN = PN / 2;         // weight rows per CTA
constexpr int BK = 128;            // K elements per k-block (4 MMAs of K = 32)
constexpr int STAGES = 4;
constexpr int A_S = CM * BK;       // 16 KB
constexpr int BP_S = CN * BK / 2;  // 8 KB of packed weights
constexpr int P_STAGE = A_S + BP_S;  // 24 KB
constexpr int W_STAGE = CN * BK;   // 16 KB
constexpr int OFF_W = 0;
constexpr int OFF_P = OFF_W + STAGES * W_STAGE;
constexpr int OFF_PARAM = OFF_P + STAGES * P_STAGE;
constexpr int PARAM_BYTES = 4 * 3 * PN * 4;  // per epilogue warp: scale hi, scale lo, bias
constexpr int OFF_STAGE = OFF_PARAM + PARAM_BYTES;
constexpr int STAGE_BYTES = 32 * 32 * 2;
constexpr int OFF_BAR = OFF_STAGE + 4 * 2 * STAGE_BYTES;
constexpr int NUM_BARS = 3 * STAGES + 4;
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16;
constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;
constexpr int NUM_THREADS = 448;
constexpr int TMEM_COLS = 512;
constexpr int ACC_COLS = PN;
constexpr int WIDEN_WARPS = 4;     // per set
constexpr int WARP_W0 = 6;         // first widening warp
constexpr int FULL_ARRIVALS = 1 + 2 * WIDEN_WARPS;  // leader producer + widening warps of both CTAs
constexpr int EMPTY_ACC_ARRIVALS = 2 * 4;
constexpr uint32_t IDESC = idesc_i8(2 * CM, PN);

static_assert(2 * ACC_COLS <= TMEM_COLS, "TMEM budget");
static_assert(W_STAGE % 1024 == 0 && OFF_P % 1024 == 0 && A_S % 1024 == 0 && P_STAGE % 1024 == 0,
              "swizzle atoms need 1024-byte alignment");
static_assert(OFF_STAGE % 512 == 0, "64-byte-swizzled staging needs 512-byte alignment");
static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
static_assert(STAGES == 4, "widened-stage arithmetic uses masks");

struct Smem {
  uint8_t* base;
  __device__ uint8_t* w(int s) const { return base + OFF_W + s * W_STAGE; }
  __device__ uint8_t* a(int p) const { return base + OFF_P + p * P_STAGE; }
  __device__ uint8_t* bp(int p) const { return base + OFF_P + p * P_STAGE + A_S; }
  __device__ float* ph(int q) const { return reinterpret_cast<float*>(base + OFF_PARAM) + q * 3 * PN; }
  __device__ float* pl(int q) const { return ph(q) + PN; }
  __device__ float* pb(int q) const { return ph(q) + 2 * PN; }
  __device__ uint8_t* stage(int q, int buf) const { return base + OFF_STAGE + (2 * q + buf) * STAGE_BYTES; }
  __device__ uint32_t bar(int i) const { return smem_u32(base + OFF_BAR + 8 * i); }
  __device__ uint32_t full(int p) const { return bar(p); }                  // leader: activations + widened weights
  __device__ uint32_t pfull(int p) const { return bar(STAGES + p); }       // local: packed weight bytes
  __device__ uint32_t empty(int p) const { return bar(2 * STAGES + p); }   // both: the stage's MMAs completed
  __device__ uint32_t tmem_full(int b) const { return bar(3 * STAGES + b); }
  __device__ uint32_t tmem_empty(int b) const { return bar(3 * STAGES + 2 + b); }
  __device__ uint32_t* tmem_slot() const { return reinterpret_cast<uint32_t*>(base + OFF_MISC); }
  __device__ volatile int* abort_flag() const { return reinterpret_cast<volatile int*>(base + OFF_MISC + 4); }
};

__device__ __forceinline__ void fail(const Smem& sm, int* status) {
  record_status(status, CR_ERR_TIMEOUT);
  *sm.abort_flag() = 1;
}

// Packed word w (codes 8j .. 8j+7, code 8j+e in bits 4e .. 4e+3) -> 8 widened bytes 16 q in code order.
__device__ __forceinline__ uint2 widen8(uint32_t w) {
  const uint32_t lo = (w << 4) & 0xF0F0F0F0u;  // byte i: code 2i   (i = 0..3)
  const uint32_t hi = w & 0xF0F0F0F0u;         // byte i: code 2i+1
  // interleave: bytes (lo0, hi0, lo1, hi1) and (lo2, hi2, lo3, hi3)
  return make_uint2(__byte_perm(lo, hi, 0x5140), __byte_perm(lo, hi, 0x7362));
}

template <bool kOutS32>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    a8w4_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                          const __grid_constant__ CUtensorMap tmap_y, const float* __restrict__ a_scale,
                          const float* __restrict__ w_scale, const uint16_t* __restrict__ bias,
                          void* __restrict__ Yv, int64_t ldy, int M, int N, int K, int* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  Smem sm;
  sm.base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = static_cast<int>(cluster_id_x());
  const int npairs = static_cast<int>(num_clusters_x());
  const int num_m = (M + 2 * CM - 1) / (2 * CM);
  const int num_n = (N + PN - 1) / PN;
  const int num_tiles = num_m * num_n;
  const int nk = K / BK;
  const int my_tiles = pair < num_tiles ? (num_tiles - pair + npairs - 1) / npairs : 0;
  const int n_items = my_tiles * nk;

  if (threadIdx.x == 0) {
    for (int p = 0; p < STAGES; ++p) {
      mbar_init(sm.full(p), FULL_ARRIVALS);
      mbar_init(sm.pfull(p), 1);
      mbar_init(sm.empty(p), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(sm.tmem_full(b), 1);
      mbar_init(sm.tmem_empty(b), EMPTY_ACC_ARRIVALS);
    }
    *sm.abort_flag() = 0;
    fence_mbar_init();
  }
  if (warp == 1 && lane == 0) {
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
    if (!kOutS32) prefetch_tmap(&tmap_y);
  }
  if (warp == 0) {
    tmem_alloc_pair(smem_u32(sm.tmem_slot()), TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *sm.tmem_slot();
  volatile int* abort = sm.abort_flag();

  auto tile_of = [&](int local) { return pair + local * npairs; };

  if (warp == 0) {
    // ------------------------------------------------------------ MMA issuer (leader CTA)
    if (rank == 0) {
      bool ok = true;
      bool committed = false;
      uint32_t last_bar = 0, last_par = 0;
      int j = 0;
      bool ready = n_items > 0 && mbar_test(sm.full(0), 0);
      for (int t = 0; ok && t < my_tiles; ++t) {
        const int b = t & 1;
        if (!mbar_wait(sm.tmem_empty(b), static_cast<uint32_t>(((t >> 1) & 1) ^ 1), abort)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * ACC_COLS);
        for (int kb = 0; kb < nk; ++kb, ++j) {
          const int s = j & 3;
          const uint32_t ph = static_cast<uint32_t>((j >> 2) & 1);
          if (!mbar_wait_from(sm.full(s), ph, ready, abort)) { ok = false; break; }
          __syncwarp();
          tc_fence_after();
          const uint64_t da = sw128_kmajor_desc(smem_u32(sm.a(s)));
          const uint64_t db = sw128_kmajor_desc(smem_u32(sm.w(s)));
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk)
            umma_i8_pair_ss_lane0(d_tmem, da + 2u * kk, db + 2u * kk, IDESC, (kb | kk) ? 1u : 0u, lane);
          umma_commit_pair_mc_lane0(sm.empty(s), 0x3, lane);
          last_bar = sm.empty(s);
          last_par = ph;
          committed = true;
          if (j + 1 < n_items) ready = mbar_test(sm.full((j + 1) & 3), static_cast<uint32_t>(((j + 1) >> 2) & 1));
        }
        if (!ok) break;
        umma_commit_pair_mc_lane0(sm.tmem_full(b), 0x3, lane);
      }
      if (!ok) {
        if (lane == 0) fail(sm, status);
        if (committed) {
          volatile int never = 0;
          mbar_wait(last_bar, last_par, &never);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      bool ok = true;
      const uint32_t full_leader0 = mapa_shared(sm.full(0), 0);
      int f = 0, p = 0;
      uint32_t ph = 0;
      for (int t = 0; ok && t < my_tiles; ++t) {
        const int tile = tile_of(t);
        const int m0 = (tile / num_n) * 2 * CM + CM * static_cast<int>(rank);
        const int n0 = (tile % num_n) * PN + CN * static_cast<int>(rank);
        for (int x = 0; x < K; x += BK) {
          if (f >= STAGES && !mbar_wait(sm.empty(p), ph ^ 1u, abort)) { ok = false; break; }
          if (rank == 0) mbar_arrive_expect_tx(sm.full(p), 2 * A_S);  // both CTAs' activation bytes
          mbar_arrive_expect_tx(sm.pfull(p), BP_S);
          tma_load_2d_pair(smem_u32(sm.a(p)), &tmap_a, x, m0, full_leader0 + 8u * static_cast<uint32_t>(p));
          tma_load_2d(smem_u32(sm.bp(p)), &tmap_b, x / 2, n0, sm.pfull(p));
          ++f;
          if (++p == STAGES) { p = 0; ph ^= 1u; }
        }
      }
      if (!ok) {
        fail(sm, status);
        // loads already issued must land before the CTA exits; the activation loads complete on the
        // leader's barriers, so give them a bounded grace period (a tile load takes microseconds)
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 1000000ull) __nanosleep(1000);
      }
    }
  } else if (warp >= WARP_W0) {
    // ------------------------------------------------------------ weight widening (both CTAs)
    const int set = (warp - WARP_W0) / WIDEN_WARPS;  // k-blocks of this parity
    const int wb = (warp - WARP_W0) % WIDEN_WARPS;   // rows 32 wb .. 32 wb + 31 of the CTA's 128
    const int c = lane & 3;                          // 16-byte chunk of the 64 packed bytes of a row
    const uint32_t full_leader0 = mapa_shared(sm.full(0), 0);
    bool ok = true;
    bool ready = set < n_items && mbar_test(sm.pfull(set), 0);
    for (int j = set; j < n_items; j += 2) {
      const int s = j & 3;
      if (!mbar_wait_from(sm.pfull(s), static_cast<uint32_t>((j >> 2) & 1), ready, abort)) { ok = false; break; }
      __syncwarp();
      const uint8_t* src = sm.bp(s);
      uint4 w4[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        // a quarter-warp reads two consecutive rows: 8 distinct 16-byte bank groups
        const int r = 32 * wb + 8 * i + (lane >> 2);
        w4[i] = *reinterpret_cast<const uint4*>(src + r * (BK / 2) + 16 * c);
      }
      // the widened slot is free: the producer refilled this stage only after its MMAs completed
      uint8_t* ws = sm.w(s);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = 32 * wb + 8 * i + (lane >> 2);
        uint8_t* row = ws + (r >> 3) * 1024 + (r & 7) * 128;
        const uint4 w = w4[i];
        const uint2 e0 = widen8(w.x), e1 = widen8(w.y), e2 = widen8(w.z), e3 = widen8(w.w);
        // packed chunk c = codes 32c .. 32c+31 = widened bytes 32c .. 32c+31 = 16-byte chunks 2c, 2c+1
        *reinterpret_cast<uint4*>(row + (((2 * c) ^ (r & 7)) << 4)) = make_uint4(e0.x, e0.y, e1.x, e1.y);
        *reinterpret_cast<uint4*>(row + (((2 * c + 1) ^ (r & 7)) << 4)) = make_uint4(e2.x, e2.y, e3.x, e3.y);
      }
      if (j + 2 < n_items) ready = mbar_test(sm.pfull((j + 2) & 3), static_cast<uint32_t>(((j + 2) >> 2) & 1));
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(full_leader0 + 8u * static_cast<uint32_t>(s));
    }
    if (!ok) fail(sm, status);
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-5)
    const int q = warp & 3;
    const int lrow = lane;
    float* wph = sm.ph(q);
    float* wpl = sm.pl(q);
    float* wpb = sm.pb(q);
    const uint32_t empty_leader = mapa_shared(sm.tmem_empty(0), 0);
    const float sa = kOutS32 ? 0.f : __ldg(a_scale);
    bool ok = true;
    int nstore = 0;
    for (int t = 0; ok && t < my_tiles; ++t) {
      const int b = t & 1;
      const int tile = tile_of(t);
      const int m0 = (tile / num_n) * 2 * CM + CM * static_cast<int>(rank);
      const int n0 = (tile % num_n) * PN;
      __syncwarp();
      for (int col = lane; !kOutS32 && col < PN; col += 32) {
        const int n = n0 + col;
        float ph = 0.f, pl = 0.f, pb = 0.f;
        if (n < N) {
          const float sw = __ldg(w_scale + n);
          ph = __fmul_rn(sa, sw);
          pl = __fmaf_rn(sa, sw, -ph);
          if (bias) pb = __uint_as_float(static_cast<uint32_t>(__ldg(bias + n)) << 16);
        }
        wph[col] = ph;
        wpl[col] = pl;
        wpb[col] = pb;
      }
      __syncwarp();
      if (!mbar_wait_warp(sm.tmem_full(b), static_cast<uint32_t>((t >> 1) & 1), abort)) { ok = false; break; }
      tc_fence_after();
      const int row = m0 + 32 * q + lrow;
#pragma unroll 1
      for (int ch = 0; ch < PN / 32; ++ch) {
        if (n0 + ch * 32 >= N) break;
        uint32_t r[32];
        tmem_ld32(tmem_base + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(b * ACC_COLS + ch * 32), r);
        tmem_ld_wait();
        if constexpr (kOutS32) {
          int32_t* crow = static_cast<int32_t*>(Yv) + static_cast<int64_t>(row) * ldy;
          if (row < M) {
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
              const int n = n0 + ch * 32 + jj * 4;
              if (n < N)
                *reinterpret_cast<int4*>(crow + n) =
                    make_int4(static_cast<int32_t>(r[4 * jj]) >> 4, static_cast<int32_t>(r[4 * jj + 1]) >> 4,
                              static_cast<int32_t>(r[4 * jj + 2]) >> 4, static_cast<int32_t>(r[4 * jj + 3]) >> 4);
            }
          }
        } else {
          uint8_t* stg = sm.stage(q, nstore++ & 1);
          if (lane == 0) bulk_wait_group_read<1>();
          __syncwarp();
#pragma unroll
          for (int jj = 0; jj < 32; jj += 8) {
            uint32_t pk[4];
#pragma unroll
            for (int e2 = 0; e2 < 8; e2 += 2) {
              float y2[2];
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int col = ch * 32 + jj + e2 + e;
                // acc is 16 * (integer product); the product may exceed 2^24 (INT8 codes): one rounding
                const float af = __int2float_rn(static_cast<int32_t>(r[jj + e2 + e]) >> 4);
                y2[e] = __fmaf_rn(af, wpl[col], __fmaf_rn(af, wph[col], wpb[col]));
              }
              __nv_bfloat162 v = __floats2bfloat162_rn(y2[0], y2[1]);
              pk[e2 >> 1] = *reinterpret_cast<uint32_t*>(&v);
            }
            const int piece = (jj >> 3) ^ ((lrow >> 1) & 3);
            *reinterpret_cast<uint4*>(stg + lrow * 64 + piece * 16) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmap_y, n0 + ch * 32, m0 + 32 * q, smem_u32(stg));
            bulk_commit_group();
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(empty_leader + 8u * b);
    }
    if (!kOutS32 && lane == 0) bulk_wait_group<0>();
    if (!ok) fail(sm, status);
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

struct PairLaunch {
  int max_pairs = 0;
  bool attr_done = false;
};

template <bool kOutS32>
int launch_impl(const void* Xq, const float* a_scale, const void* Wq, const float* w_scale, const void* bias, void* Y,
                int64_t ldy, int M, int N, int K, int* status, int num_sms, cudaStream_t stream) {
  if (M == 0 || N == 0) return CR_OK;
  static PairLaunch info[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return CR_ERR_CUDA;
  CUtensorMap ta, tb, ty;
  if (!make_tmap_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, Xq, static_cast<uint64_t>(M), static_cast<uint64_t>(K),
                    static_cast<uint64_t>(K), BK, CM, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B))
    return CR_ERR_CUDA;
  if (!make_tmap_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq, static_cast<uint64_t>(N), static_cast<uint64_t>(K / 2),
                    static_cast<uint64_t>(K / 2), BK / 2, CN, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B))
    return CR_ERR_CUDA;
  memset(&ty, 0, sizeof(ty));
  if (!kOutS32 && !make_tmap_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Y, static_cast<uint64_t>(M),
                                static_cast<uint64_t>(N), static_cast<uint64_t>(ldy) * 2, 32, 32,
                                CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE))
    return CR_ERR_CUDA;
  auto kern = a8w4_gemm_pair_kernel<kOutS32>;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = SMEM_ALLOC;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (!info[dev].attr_done) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_ALLOC) != cudaSuccess)
      return CR_ERR_CUDA;
    cfg.gridDim = dim3(2 * (num_sms / 2), 1, 1);
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess || clusters < 1) {
      cudaGetLastError();
      clusters = num_sms / 2;
    }
    info[dev].max_pairs = clusters;
    info[dev].attr_done = true;
  }
  const int tiles = ((M + 2 * CM - 1) / (2 * CM)) * ((N + PN - 1) / PN);
  const int pairs = tiles < info[dev].max_pairs ? tiles : info[dev].max_pairs;
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, ta, tb, ty, a_scale, w_scale, static_cast<const uint16_t*>(bias), Y,
                                     ldy, M, N, K, status);
  return e == cudaSuccess ? CR_OK : CR_ERR_CUDA;
}

}  // namespace

int launch_a8w4_gemm(const void* Xq, const float* a_scale, const void* Wq, const float* w_scale, const void* bias,
                     void* Y, int64_t ldy, int M, int N, int K, int* status, int num_sms, cudaStream_t stream) {
  return launch_impl<false>(Xq, a_scale, Wq, w_scale, bias, Y, ldy, M, N, K, status, num_sms, stream);
}

int launch_a8w4_gemm_s32(const void* Xq, const void* Wq, int32_t* C, int64_t ldc, int M, int N, int K, int* status,
                         int num_sms, cudaStream_t stream) {
  return launch_impl<true>(Xq, nullptr, Wq, nullptr, nullptr, C, ldc, M, N, K, status, num_sms, stream);
}

}  // namespace cr
