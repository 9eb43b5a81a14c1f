// gemm_i8.cu -- INT8 x INT8 GEMM with the layer's scale/bias epilogue, on a
// CTA pair (tcgen05 cta_group::2).
//
// The INT8 tensorwise format, with or without the ConvRot rotation, is the
// fallback format of the same model cards ("Qwen-Image-Edit-2511 -- INT4
// tensorwise W4A4 (+ConvRot, mixed int8 fallback)", introduction: sensitive
// layers kept as int8_tensorwise; "Qwen Image 2.1 -- Hybrid W4A8 / INT8
// ConvRot", layer list: INT8 tensorwise + ConvRot).  The product is
//   acc[m, n] = sum_k qa[m, k] * qw[n, k]          (exact in int32)
//   Y[m, n]   = bf16(acc * s_a * s_w[n] + bias[n])
// with one code per byte, K-major rows for both operands.
//
// Unlike the INT4 path the codes need no widening: the tensor cores read both
// operands straight from the TMA ring.
//
// * A pair of CTAs (a cluster of 2) computes a 256 x 256 output tile with
//   tcgen05.mma.cta_group::2.kind::i8 (M = 256, N = 256, K = 32): 128 cycles
//   per instruction.  Each CTA loads 128 rows of A and 128 rows of B.
// * Each stage holds one k-block of 128 codes for every row (one 128-byte
//   swizzle row), loaded by TMA with the 128-byte swizzle.  Both CTAs' loads
//   of a stage complete on the leader's full barrier (the pair form of the
//   TMA load), which alone the MMA issuer waits on.  No multicast.
// * The MMA's completion frees the stage in both CTAs (multicast commit) and
//   hands finished accumulators to the epilogue (double-buffered, 2 x 256
//   TMEM columns).
//
// Roles (192 threads per CTA):
//   warp 0      TMEM allocation; in the leader CTA, the MMA issuer
//   warp 1      TMA producer (both CTAs)
//   warps 2-5   epilogue: TMEM -> int32 -> float -> scale, bias -> bf16 ->
//               swizzled staging -> TMA tensor stores (or raw int32 rows)
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

constexpr int CM = 128;            // A rows per CTA (pair: 256)
constexpr int PN = 256;            // output columns per pair tile
constexpr int CN = PN / 2;         // B rows per CTA
constexpr int BK = 128;            // codes (bytes) per row per stage
constexpr int STAGES = 6;
constexpr int A_S = CM * BK;       // 16 KB
constexpr int B_S = CN * BK;       // 16 KB
constexpr int STAGE = A_S + B_S;   // 32 KB
constexpr int OFF_RING = 0;
constexpr int OFF_PARAM = OFF_RING + STAGES * STAGE;
constexpr int PARAM_BYTES = 4 * 3 * PN * 4;          // per epilogue warp: scale hi, scale lo, bias
constexpr int OFF_STAGE = OFF_PARAM + PARAM_BYTES;   // epilogue output staging
constexpr int STAGE_BYTES = 32 * 32 * 2;             // 32 rows x 32 bf16 columns
constexpr int OFF_BAR = OFF_STAGE + 4 * 2 * STAGE_BYTES;
constexpr int NUM_BARS = 2 * STAGES + 4;
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16;
constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;
constexpr int NUM_THREADS = 192;
constexpr int TMEM_COLS = 512;
constexpr int ACC_COLS = PN;
constexpr int EMPTY_ACC_ARRIVALS = 2 * 4;  // 4 epilogue warps x 2 CTAs
constexpr uint32_t IDESC = idesc_i8(2 * CM, PN);

static_assert(2 * ACC_COLS <= TMEM_COLS, "TMEM budget");
static_assert(A_S % 1024 == 0 && STAGE % 1024 == 0, "swizzle atoms need 1024-byte alignment");
static_assert(OFF_STAGE % 512 == 0, "64-byte-swizzled staging needs 512-byte alignment");
static_assert(SMEM_ALLOC <= 232448, "shared memory budget");

struct Smem {
  uint8_t* base;
  __device__ uint8_t* a(int s) const { return base + OFF_RING + s * STAGE; }
  __device__ uint8_t* b(int s) const { return base + OFF_RING + s * STAGE + A_S; }
  __device__ float* ph(int q) const { return reinterpret_cast<float*>(base + OFF_PARAM) + q * 3 * PN; }
  __device__ float* pl(int q) const { return ph(q) + PN; }
  __device__ float* pb(int q) const { return ph(q) + 2 * PN; }
  __device__ uint8_t* stage(int q, int buf) const { return base + OFF_STAGE + (2 * q + buf) * STAGE_BYTES; }
  __device__ uint32_t bar(int i) const { return smem_u32(base + OFF_BAR + 8 * i); }
  __device__ uint32_t full(int s) const { return bar(s); }
  __device__ uint32_t empty(int s) const { return bar(STAGES + s); }
  __device__ uint32_t tmem_full(int b) const { return bar(2 * STAGES + b); }
  __device__ uint32_t tmem_empty(int b) const { return bar(2 * STAGES + 2 + b); }
  __device__ uint32_t* tmem_slot() const { return reinterpret_cast<uint32_t*>(base + OFF_MISC); }
  __device__ volatile int* abort_flag() const { return reinterpret_cast<volatile int*>(base + OFF_MISC + 4); }
};

__device__ __forceinline__ void fail(const Smem& sm, int* status) {
  record_status(status, CR_ERR_TIMEOUT);
  *sm.abort_flag() = 1;
}

template <bool kOutS32>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    i8_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                        const __grid_constant__ CUtensorMap tmap_y, const float* __restrict__ a_scale,
                        const float* __restrict__ w_scale, const uint16_t* __restrict__ bias, void* __restrict__ Yv,
                        int64_t ldy, int M, int N, int K, int* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  Smem sm;
  sm.base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0 = leader (issues the MMAs), 1 = peer
  const int pair = static_cast<int>(cluster_id_x());
  const int npairs = static_cast<int>(num_clusters_x());
  const int num_m = (M + 2 * CM - 1) / (2 * CM);
  const int num_n = (N + PN - 1) / PN;
  const int num_tiles = num_m * num_n;
  const int nk = K / BK;
  const int my_tiles = pair < num_tiles ? (num_tiles - pair + npairs - 1) / npairs : 0;
  const int n_items = my_tiles * nk;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(sm.full(s), 1);   // the leader producer's arrive (+ both CTAs' bytes)
      mbar_init(sm.empty(s), 1);  // the MMA commit
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
  cluster_sync();  // both CTAs' barriers exist before any cross-CTA arrive or load completion
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
      int it = 0;
      bool next_full = n_items > 0 && mbar_test(sm.full(0), 0);
      for (int t = 0; ok && t < my_tiles; ++t) {
        const int b = t & 1;
        if (!mbar_wait(sm.tmem_empty(b), static_cast<uint32_t>(((t >> 1) & 1) ^ 1), abort)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * ACC_COLS);
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = static_cast<uint32_t>((it / STAGES) & 1);
          if (!mbar_wait_from(sm.full(s), ph, next_full, abort)) { ok = false; break; }
          __syncwarp();
          tc_fence_after();
          const uint64_t da = sw128_kmajor_desc(smem_u32(sm.a(s)));
          const uint64_t db = sw128_kmajor_desc(smem_u32(sm.b(s)));
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk)
            umma_i8_pair_ss_lane0(d_tmem, da + 2u * kk, db + 2u * kk, IDESC, (kb | kk) ? 1u : 0u, lane);
          umma_commit_pair_mc_lane0(sm.empty(s), 0x3, lane);
          // test the next stage while these MMAs run
          const int s2 = (it + 1) % STAGES;
          next_full = it + 1 < n_items && mbar_test(sm.full(s2), static_cast<uint32_t>(((it + 1) / STAGES) & 1));
          last_bar = sm.empty(s);
          last_par = ph;
          committed = true;
        }
        if (!ok) break;
        umma_commit_pair_mc_lane0(sm.tmem_full(b), 0x3, lane);
      }
      if (!ok) {
        if (lane == 0) fail(sm, status);
        if (committed) {
          volatile int never = 0;
          mbar_wait(last_bar, last_par, &never);  // the MMAs issued so far have finished reading
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      bool ok = true;
      const uint32_t full_leader0 = mapa_shared(sm.full(0), 0);
      int f = 0, s = 0;
      uint32_t ph = 0;  // phase parity of stage s's current use
      for (int t = 0; ok && t < my_tiles; ++t) {
        const int tile = tile_of(t);
        const int m0 = (tile / num_n) * 2 * CM + CM * static_cast<int>(rank);
        const int n0 = (tile % num_n) * PN + CN * static_cast<int>(rank);
        for (int x = 0; x < K; x += BK) {
          if (f >= STAGES && !mbar_wait(sm.empty(s), ph ^ 1u, abort)) { ok = false; break; }
          // the leader's full barrier counts both CTAs' bytes of this stage
          if (rank == 0) mbar_arrive_expect_tx(sm.full(s), 2 * STAGE);
          const uint32_t fb = full_leader0 + 8u * static_cast<uint32_t>(s);
          tma_load_2d_pair(smem_u32(sm.a(s)), &tmap_a, x, m0, fb);
          tma_load_2d_pair(smem_u32(sm.b(s)), &tmap_b, x, n0, fb);
          ++f;
          if (++s == STAGES) { s = 0; ph ^= 1u; }
        }
      }
      if (!ok) {
        fail(sm, status);
        // Loads already issued must land before the CTA exits.  Their completion is counted on the
        // leader's barriers, which the peer cannot wait on, so each CTA gives them a bounded grace
        // period instead (a tile load takes microseconds).
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 1000000ull) __nanosleep(1000);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-5)
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int lrow = lane;   // TMEM lane 32q + lane holds tile row 32q + lane
    float* wph = sm.ph(q);
    float* wpl = sm.pl(q);
    float* wpb = sm.pb(q);
    const uint32_t empty_leader = mapa_shared(sm.tmem_empty(0), 0);
    const float sa = kOutS32 ? 0.f : __ldg(a_scale);
    bool ok = true;
    int nstore = 0;  // bf16 chunks stored by this warp: their staging buffers alternate
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
          pl = __fmaf_rn(sa, sw, -ph);  // sa*sw = ph + pl exactly
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
        if (n0 + ch * 32 >= N) break;  // columns past N: nothing to write
        uint32_t r[32];
        tmem_ld32(tmem_base + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(b * ACC_COLS + ch * 32), r);
        tmem_ld_wait();
        if constexpr (kOutS32) {
          int32_t* crow = static_cast<int32_t*>(Yv) + static_cast<int64_t>(row) * ldy;
          if (row < M) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int n = n0 + ch * 32 + j * 4;
              if (n < N)
                *reinterpret_cast<int4*>(crow + n) =
                    make_int4(static_cast<int32_t>(r[4 * j]), static_cast<int32_t>(r[4 * j + 1]),
                              static_cast<int32_t>(r[4 * j + 2]), static_cast<int32_t>(r[4 * j + 3]));
            }
          }
        } else {
          // bf16 row chunk -> staging buffer, 16-byte pieces XOR-swizzled like the 64-byte TMA swizzle
          uint8_t* stg = sm.stage(q, nstore++ & 1);
          if (lane == 0) bulk_wait_group_read<1>();  // the store that used this buffer has read it
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 32; j += 8) {
            uint32_t pk[4];
#pragma unroll
            for (int e2 = 0; e2 < 8; e2 += 2) {
              float y2[2];
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int col = ch * 32 + j + e2 + e;
                // |acc| <= 127^2 K may exceed 2^24: the conversion rounds once (correctly)
                const float af = __int2float_rn(static_cast<int32_t>(r[j + e2 + e]));
                y2[e] = __fmaf_rn(af, wpl[col], __fmaf_rn(af, wph[col], wpb[col]));
              }
              __nv_bfloat162 v = __floats2bfloat162_rn(y2[0], y2[1]);
              pk[e2 >> 1] = *reinterpret_cast<uint32_t*>(&v);
            }
            const int piece = (j >> 3) ^ ((lrow >> 1) & 3);
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
    if (!kOutS32 && lane == 0) bulk_wait_group<0>();  // every output tile has been written
    if (!ok) fail(sm, status);
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer no longer arrives on our barriers and the pair's MMAs are done
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
  // codes: [rows, K] bytes, boxes of 128 rows x 128 bytes, 128-byte swizzle
  if (!make_tmap_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, Xq, static_cast<uint64_t>(M), static_cast<uint64_t>(K),
                    static_cast<uint64_t>(K), BK, CM, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B))
    return CR_ERR_CUDA;
  if (!make_tmap_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq, static_cast<uint64_t>(N), static_cast<uint64_t>(K),
                    static_cast<uint64_t>(K), BK, CN, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B))
    return CR_ERR_CUDA;
  memset(&ty, 0, sizeof(ty));
  // bf16 output: 32 x 32 boxes, 64-byte swizzle
  if (!kOutS32 && !make_tmap_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Y, static_cast<uint64_t>(M),
                                static_cast<uint64_t>(N), static_cast<uint64_t>(ldy) * 2, 32, 32,
                                CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE))
    return CR_ERR_CUDA;
  auto kern = i8_gemm_pair_kernel<kOutS32>;
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

int launch_i8_gemm(const void* Xq, const float* a_scale, const void* Wq, const float* w_scale, const void* bias,
                   void* Y, int64_t ldy, int M, int N, int K, int* status, int num_sms, cudaStream_t stream) {
  return launch_impl<false>(Xq, a_scale, Wq, w_scale, bias, Y, ldy, M, N, K, status, num_sms, stream);
}

int launch_i8_gemm_s32(const void* Xq, const void* Wq, int32_t* C, int64_t ldc, int M, int N, int K, int* status,
                       int num_sms, cudaStream_t stream) {
  return launch_impl<true>(Xq, nullptr, Wq, nullptr, nullptr, C, ldc, M, N, K, status, num_sms, stream);
}

}  // namespace cr
