// gemm_w4a4.cu -- INT4 x INT4 GEMM with the rank-one scale + bias epilogue on
// sm_100a tensor cores (tcgen05.mma kind::i8, int32 accumulators in TMEM).
//
// "Qwen-Image-Edit-2511 -- INT4 tensorwise W4A4 (+ConvRot, mixed int8
// fallback)", section "Measurements": the layer's product is an s4 MMA scaled
// by a rank-one (activation scale x weight scale) factor.  B200 tensor cores
// have no 4-bit integer MMA, so the packed codes are widened to 8 bits in
// shared memory and multiplied with the 8-bit integer MMA, which is exact.
//
// Widening trick: a nibble placed in the high half of a byte, low half zero,
// reads as the int8 value 16*q.  So a packed word w gives the odd elements as
// (w & 0xF0F0F0F0) and the even elements as ((w << 4) & 0xF0F0F0F0): three
// ALU operations per 8 codes, no sign extension.  Both operands carry the
// factor 16, the MMA accumulates 256 * acc (exact in int32 for K <= 65536),
// and the epilogue shifts right by 8.  The byte order inside each group of 8
// codes becomes (0,2,4,6,1,3,5,7) on both operands; a dot product does not
// change under the same permutation of both factors.
//
// Structure (one CTA per SM, persistent over 128 x 256 output tiles):
//   warp 0      TMA producer: packed A [128 x 64 B] and B [256 x 64 B] tiles
//               into a 4-stage ring
//   warp 1      UMMA issuer: 4 x (128x256x32) MMAs per 128-deep k-block,
//               accumulating into one of two TMEM buffers (2 x 256 columns)
//   warps 2-5   unpackers: packed ring -> int8 operands in the 128-byte
//               swizzled K-major layout (2-stage ring)
//   warps 6-9   epilogue: TMEM -> registers -> scale, bias, bf16 -> global,
//               overlapping the next tile's main loop
// Every wait is bounded (CR_WAIT_TIMEOUT_NS); on expiry the CTA records
// CR_ERR_TIMEOUT in the device status word, drains its own copies and MMAs,
// frees TMEM and exits.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "cr_device.cuh"
#include "cr_internal.h"

namespace cr {
namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BKP = 64;    // packed bytes per row per k-block
constexpr int BK = 128;    // codes per row per k-block
constexpr int PSTAGES = 4;
constexpr int USTAGES = 2;
constexpr int A_P = BM * BKP;          // 8 KB
constexpr int B_P = BN * BKP;          // 16 KB
constexpr int P_STAGE = A_P + B_P;     // 24 KB
constexpr int A_U = BM * BK;           // 16 KB
constexpr int B_U = BN * BK;           // 32 KB
constexpr int U_STAGE = A_U + B_U;     // 48 KB
constexpr int OFF_U = 0;
constexpr int OFF_P = OFF_U + USTAGES * U_STAGE;
constexpr int OFF_PARAM = OFF_P + PSTAGES * P_STAGE;
constexpr int PARAM_BYTES = 4 * 3 * BN * 4;  // per epilogue warp: scale hi, scale lo, bias
constexpr int OFF_BAR = OFF_PARAM + PARAM_BYTES;
constexpr int NUM_BARS = 2 * PSTAGES + 2 * USTAGES + 4;
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16;
constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;  // slack for 1024-byte alignment
constexpr int NUM_THREADS = 320;
constexpr int TMEM_COLS = 512;
constexpr uint32_t IDESC = idesc_i8(BM, BN);

static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
static_assert(OFF_P % 1024 == 0 && U_STAGE % 1024 == 0 && A_U % 1024 == 0, "swizzle atoms need 1024-byte alignment");

struct Smem {
  uint8_t* base;
  __device__ uint8_t* a_u(int s) const { return base + OFF_U + s * U_STAGE; }
  __device__ uint8_t* b_u(int s) const { return base + OFF_U + s * U_STAGE + A_U; }
  __device__ uint8_t* a_p(int s) const { return base + OFF_P + s * P_STAGE; }
  __device__ uint8_t* b_p(int s) const { return base + OFF_P + s * P_STAGE + A_P; }
  // per-epilogue-warp column parameters (q = TMEM lane quarter of the warp)
  __device__ float* ph(int q) const { return reinterpret_cast<float*>(base + OFF_PARAM) + q * 3 * BN; }
  __device__ float* pl(int q) const { return ph(q) + BN; }
  __device__ float* pb(int q) const { return ph(q) + 2 * BN; }
  __device__ uint32_t bar(int i) const { return smem_u32(base + OFF_BAR + 8 * i); }
  __device__ uint32_t full_p(int s) const { return bar(s); }
  __device__ uint32_t empty_p(int s) const { return bar(PSTAGES + s); }
  __device__ uint32_t full_u(int s) const { return bar(2 * PSTAGES + s); }
  __device__ uint32_t empty_u(int s) const { return bar(2 * PSTAGES + USTAGES + s); }
  __device__ uint32_t tmem_full(int b) const { return bar(2 * PSTAGES + 2 * USTAGES + b); }
  __device__ uint32_t tmem_empty(int b) const { return bar(2 * PSTAGES + 2 * USTAGES + 2 + b); }
  __device__ uint32_t* tmem_slot() const { return reinterpret_cast<uint32_t*>(base + OFF_MISC); }
  __device__ volatile int* abort_flag() const { return reinterpret_cast<volatile int*>(base + OFF_MISC + 4); }
};

__device__ __forceinline__ void fail(const Smem& sm, int* status) {
  record_status(status, CR_ERR_TIMEOUT);
  *sm.abort_flag() = 1;
}

// Widen 16 packed bytes (32 codes) of one operand row into 32 int8 bytes of
// value 16*q, written as two 16-byte chunks of the 128-byte swizzled row.
__device__ __forceinline__ void unpack_chunk(const uint8_t* src_row, uint8_t* dst_atom_row, int c, int rsw) {
  const uint4 w = *reinterpret_cast<const uint4*>(src_row + 16 * c);
  const uint32_t m = 0xF0F0F0F0u;
  uint4 o0, o1;
  o0.x = (w.x << 4) & m; o0.y = w.x & m; o0.z = (w.y << 4) & m; o0.w = w.y & m;
  o1.x = (w.z << 4) & m; o1.y = w.z & m; o1.z = (w.w << 4) & m; o1.w = w.w & m;
  *reinterpret_cast<uint4*>(dst_atom_row + (((2 * c) ^ rsw) << 4)) = o0;
  *reinterpret_cast<uint4*>(dst_atom_row + (((2 * c + 1) ^ rsw) << 4)) = o1;
}

// kOutS32 = false: Y is bf16 [M, N] = acc * a_scale * w_scale[n] + bias[n].
// kOutS32 = true : Y is int32 [M, N] = acc (raw integer product, no scales).
template <bool kOutS32>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    w4a4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                     const float* __restrict__ a_scale, const float* __restrict__ w_scale,
                     const uint16_t* __restrict__ bias, void* __restrict__ Yv, int64_t ldy, int M, int N, int K,
                     int* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  Smem sm;
  sm.base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_m = (M + BM - 1) / BM;
  const int num_n = (N + BN - 1) / BN;
  const int num_tiles = num_m * num_n;
  const int nk = K / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < PSTAGES; ++s) {
      mbar_init(sm.full_p(s), 1);
      mbar_init(sm.empty_p(s), 4);  // one arrival per unpack warp
    }
    for (int s = 0; s < USTAGES; ++s) {
      mbar_init(sm.full_u(s), 4);
      mbar_init(sm.empty_u(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(sm.tmem_full(b), 1);
      mbar_init(sm.tmem_empty(b), 4);  // one arrival per epilogue warp
    }
    *sm.abort_flag() = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(sm.tmem_slot()), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *sm.tmem_slot();
  volatile int* abort = sm.abort_flag();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int ps = 0;
      uint32_t pph = 0;
      int fills[PSTAGES] = {0, 0, 0, 0};
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        const int m0 = (tile / num_n) * BM;
        const int n0 = (tile % num_n) * BN;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(sm.empty_p(ps), pph ^ 1u, abort)) { ok = false; break; }
          mbar_arrive_expect_tx(sm.full_p(ps), P_STAGE);
          tma_load_2d(smem_u32(sm.a_p(ps)), &tmap_a, kb * BKP, m0, sm.full_p(ps));
          tma_load_2d(smem_u32(sm.b_p(ps)), &tmap_b, kb * BKP, n0, sm.full_p(ps));
          ++fills[ps];
          if (++ps == PSTAGES) { ps = 0; pph ^= 1u; }
        }
      }
      if (!ok) {
        fail(sm, status);
        // let every copy this thread issued land before the CTA can exit
        for (int s = 0; s < PSTAGES; ++s)
          if (fills[s] > 0) {
            volatile int never = 0;
            mbar_wait(sm.full_p(s), static_cast<uint32_t>((fills[s] - 1) & 1), &never);
          }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int us = 0;
      uint32_t uph = 0;
      bool ok = true;
      uint32_t last_bar = 0, last_par = 0;
      bool committed = false;
      int t = 0;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x, ++t) {
        const int b = t & 1;
        const uint32_t bph = static_cast<uint32_t>((t >> 1) & 1);
        if (!mbar_wait(sm.tmem_empty(b), bph ^ 1u, abort)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * BN);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(sm.full_u(us), uph, abort)) { ok = false; break; }
          tc_fence_after();
          const uint64_t da = sw128_kmajor_desc(smem_u32(sm.a_u(us)));
          const uint64_t db = sw128_kmajor_desc(smem_u32(sm.b_u(us)));
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk) {
            // advance 32 bytes along K inside the swizzle atom (start address is in 16-byte units)
            umma_i8_ss(d_tmem, da + 2u * kk, db + 2u * kk, IDESC, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(sm.empty_u(us));
          last_bar = sm.empty_u(us);
          last_par = uph;
          committed = true;
          if (++us == USTAGES) { us = 0; uph ^= 1u; }
        }
        if (!ok) break;
        umma_commit(sm.tmem_full(b));
      }
      if (!ok) {
        fail(sm, status);
        if (committed) {
          volatile int never = 0;
          mbar_wait(last_bar, last_par, &never);  // all MMAs issued so far have completed
        }
      }
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ unpackers
    const int ut = threadIdx.x - 64;  // 0..127
    int ps = 0, us = 0;
    uint32_t pph = 0, uph = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
      for (int kb = 0; kb < nk; ++kb) {
        if (!mbar_wait_warp(sm.full_p(ps), pph, abort)) { ok = false; break; }
        if (!mbar_wait_warp(sm.empty_u(us), uph ^ 1u, abort)) { ok = false; break; }
        const uint8_t* ap = sm.a_p(ps);
        const uint8_t* bp = sm.b_p(ps);
        uint8_t* au = sm.a_u(us);
        uint8_t* bu = sm.b_u(us);
#pragma unroll
        for (int i = 0; i < (BM + BN) * 4 / 128; ++i) {
          const int item = ut + 128 * i;
          const int row = item >> 2;
          const int c = item & 3;
          if (row < BM) {
            unpack_chunk(ap + row * BKP, au + (row >> 3) * 1024 + (row & 7) * 128, c, row & 7);
          } else {
            const int r = row - BM;
            unpack_chunk(bp + r * BKP, bu + (r >> 3) * 1024 + (r & 7) * 128, c, r & 7);
          }
        }
        fence_proxy_async_smem();  // this thread's operand writes -> visible to the MMA (async proxy)
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(sm.empty_p(ps));
          mbar_arrive(sm.full_u(us));
        }
        if (++ps == PSTAGES) { ps = 0; pph ^= 1u; }
        if (++us == USTAGES) { us = 0; uph ^= 1u; }
      }
    }
    if (!ok) fail(sm, status);
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    float* wph = sm.ph(q);
    float* wpl = sm.pl(q);
    float* wpb = sm.pb(q);
    const float sa = kOutS32 ? 0.f : __ldg(a_scale);
    bool ok = true;
    int t = 0;
    for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x, ++t) {
      const int b = t & 1;
      const uint32_t bph = static_cast<uint32_t>((t >> 1) & 1);
      const int m0 = (tile / num_n) * BM;
      const int n0 = (tile % num_n) * BN;
      // column parameters of this tile, private to the warp (warp-level sync only)
      __syncwarp();
      for (int c = lane; !kOutS32 && c < BN; c += 32) {
        const int n = n0 + c;
        float ph = 0.f, pl = 0.f, pb = 0.f;
        if (n < N) {
          const float sw = __ldg(w_scale + n);
          ph = __fmul_rn(sa, sw);
          pl = __fmaf_rn(sa, sw, -ph);  // sa*sw = ph + pl exactly
          if (bias) pb = __uint_as_float(static_cast<uint32_t>(__ldg(bias + n)) << 16);
        }
        wph[c] = ph;
        wpl[c] = pl;
        wpb[c] = pb;
      }
      __syncwarp();
      if (!mbar_wait_warp(sm.tmem_full(b), bph, abort)) { ok = false; break; }
      tc_fence_after();
      const int row = m0 + q * 32 + lane;
      uint16_t* yrow = static_cast<uint16_t*>(Yv) + static_cast<int64_t>(row) * ldy;
#pragma unroll 1
      for (int ch = 0; ch < BN / 32; ++ch) {
        uint32_t r[32];
        tmem_ld32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(b * BN + ch * 32), r);
        tmem_ld_wait();
        if constexpr (kOutS32) {
          int32_t* crow = static_cast<int32_t*>(Yv) + static_cast<int64_t>(row) * ldy;
          if (row < M) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int n = n0 + ch * 32 + j * 4;
              if (n < N)
                *reinterpret_cast<int4*>(crow + n) =
                    make_int4(static_cast<int32_t>(r[4 * j]) >> 8, static_cast<int32_t>(r[4 * j + 1]) >> 8,
                              static_cast<int32_t>(r[4 * j + 2]) >> 8, static_cast<int32_t>(r[4 * j + 3]) >> 8);
            }
          }
        } else {
        uint32_t packed[16];
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          const int c0 = ch * 32 + j;
          const float4 h4 = *reinterpret_cast<const float4*>(wph + c0);
          const float4 l4 = *reinterpret_cast<const float4*>(wpl + c0);
          const float4 b4 = *reinterpret_cast<const float4*>(wpb + c0);
          const float hh[4] = {h4.x, h4.y, h4.z, h4.w};
          const float ll[4] = {l4.x, l4.y, l4.z, l4.w};
          const float bb[4] = {b4.x, b4.y, b4.z, b4.w};
          float y4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float af = static_cast<float>(static_cast<int32_t>(r[j + e]) >> 8);  // exact
            // y = acc*hi + acc*lo + bias with two fmas: within 2 float32 ulps of y
            y4[e] = __fmaf_rn(af, ll[e], __fmaf_rn(af, hh[e], bb[e]));
          }
          __nv_bfloat162 v0 = __floats2bfloat162_rn(y4[0], y4[1]);
          __nv_bfloat162 v1 = __floats2bfloat162_rn(y4[2], y4[3]);
          packed[j >> 1] = *reinterpret_cast<uint32_t*>(&v0);
          packed[(j >> 1) + 1] = *reinterpret_cast<uint32_t*>(&v1);
        }
        if (row < M) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int n = n0 + ch * 32 + j * 8;
            if (n < N)
              *reinterpret_cast<uint4*>(yrow + n) =
                  make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
          }
        }
        }  // bf16 epilogue
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sm.tmem_empty(b));
    }
    if (!ok) fail(sm, status);
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D uint8 tensor map over a dense [rows, cols] byte matrix, box [box_rows, box_cols].
bool make_u8_map(CUtensorMap* map, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows,
                 uint32_t box_cols) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <bool kOutS32>
int launch_gemm_impl(const void* Xq, const float* a_scale, const void* Wq, const float* w_scale, const void* bias,
                     void* Y, int64_t ldy, int M, int N, int K, int* status, int num_sms, cudaStream_t stream) {
  if (M == 0 || N == 0) return CR_OK;
  CUtensorMap ta, tb;
  if (!make_u8_map(&ta, Xq, static_cast<uint64_t>(M), static_cast<uint64_t>(K / 2), BM, BKP)) return CR_ERR_CUDA;
  if (!make_u8_map(&tb, Wq, static_cast<uint64_t>(N), static_cast<uint64_t>(K / 2), BN, BKP)) return CR_ERR_CUDA;
  static int attr_done_dev = -1;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return CR_ERR_CUDA;
  if (attr_done_dev != dev) {
    if (cudaFuncSetAttribute(w4a4_gemm_kernel<kOutS32>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_ALLOC) !=
        cudaSuccess)
      return CR_ERR_CUDA;
    attr_done_dev = dev;
  }
  const int tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  const int grid = tiles < num_sms ? tiles : num_sms;
  w4a4_gemm_kernel<kOutS32><<<grid, NUM_THREADS, SMEM_ALLOC, stream>>>(
      ta, tb, a_scale, w_scale, static_cast<const uint16_t*>(bias), Y, ldy, M, N, K, status);
  return cudaGetLastError() == cudaSuccess ? CR_OK : CR_ERR_CUDA;
}

}  // namespace

int launch_w4a4_gemm_1cta(const void* Xq, const float* a_scale, const void* Wq, const float* w_scale,
                          const void* bias, void* Y, int64_t ldy, int M, int N, int K, int* status, int num_sms,
                          cudaStream_t stream) {
  return launch_gemm_impl<false>(Xq, a_scale, Wq, w_scale, bias, Y, ldy, M, N, K, status, num_sms, stream);
}

// Few tokens (M <= kSmallMaxM): the weight stream bounds the layer, the swapped-operand kernel keeps
// every SM streaming; more tokens: the CTA-pair kernel.
int launch_w4a4_gemm(const void* Xq, const float* a_scale, const void* Wq, const float* w_scale, const void* bias,
                     void* Y, int64_t ldy, int M, int N, int K, int* status, int num_sms, cudaStream_t stream) {
  if (M <= kSmallMaxM)
    return launch_w4a4_gemm_small(Xq, a_scale, Wq, w_scale, bias, Y, ldy, M, N, K, status, num_sms, stream);
  return launch_w4a4_gemm_pair(Xq, a_scale, Wq, w_scale, bias, Y, ldy, M, N, K, status, num_sms, stream);
}

int launch_w4a4_gemm_s32(const void* Xq, const void* Wq, int32_t* C, int64_t ldc, int M, int N, int K, int* status,
                         int num_sms, cudaStream_t stream) {
  if (M <= kSmallMaxM) return launch_w4a4_gemm_small_s32(Xq, Wq, C, ldc, M, N, K, status, num_sms, stream);
  return launch_w4a4_gemm_pair_s32(Xq, Wq, C, ldc, M, N, K, status, num_sms, stream);
}

}  // namespace cr
