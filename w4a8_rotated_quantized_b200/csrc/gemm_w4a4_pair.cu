// gemm_w4a4_pair.cu -- INT4 x INT4 GEMM on a CTA pair (tcgen05 cta_group::2).
//
// The integer product of packed INT4 activation and weight codes with the
// rank-one scale + bias epilogue ("Qwen-Image-Edit-2511 -- INT4 tensorwise
// W4A4 (+ConvRot, mixed int8 fallback)", section "Measurements": rank-one
// scaled s4 MMA), for more than 128 tokens, arranged so that the tensor cores
// are never waiting for widened operands:
//
// * A pair of CTAs (a cluster of 2) computes a 256 x 192 output tile with
//   tcgen05.mma.cta_group::2.kind::i8 (M = 256, N = 192, K = 32).  Each CTA
//   owns 128 rows of A and 96 rows of B; the MMA reads both CTAs' B halves.
// * Wave quantisation: when the tiles' last round would leave more than half
//   of the pairs idle, that round's tiles are split along N into two 256 x 96
//   half tiles (the MMA's N is a field of the runtime instruction descriptor),
//   so the last round costs half a tile.  Small problems with at most half as
//   many tiles as pairs run as half tiles throughout.
// * Packed codes arrive by TMA in a 5-stage ring, two k-blocks (128 bytes of
//   every row) per stage and box, with the 128-byte swizzle.  A TMA box costs
//   issue time per row, so wide rows keep the single producer thread ahead of
//   the tensor cores; five stages cover the load latency.  No multicast.
// * A (activations) is widened from that ring into TMEM with tcgen05.st: the
//   MMA's A operand comes from TMEM, so widened A never touches shared memory.
// * B (weights) is widened into the 128-byte-swizzled K-major shared memory
//   layout the MMA reads.
// * Two sets of widening warps take alternate k-blocks, so each set has two
//   MMA k-block times to hide its load -> widen -> store -> signal latency.
//
// Widening: a nibble placed in the high half of a byte reads as the int8
// value 16*q, so a packed word w yields its odd codes as (w & 0xF0F0F0F0)
// and its even codes as ((w << 4) & 0xF0F0F0F0).  The MMA accumulates
// 256 * acc, exact in int32 for K <= 65536.  Codes are permuted inside every
// group of 8 the same way for A and B, which leaves the dot product
// unchanged: widened byte 8j + e holds code 8j + p(e) with
// p = (0,2,4,6,1,3,5,7) (the even codes of packed word j, then its odd codes).
// A thread widening A owns one row: its 32 widened words go to its TMEM lane
// with one 32x32b store.
//
// Roles (640 threads per CTA):
//   warp 0        TMEM allocation; in the leader CTA, the MMA issuer
//   warps 1-3     B widening, even k-blocks  | warps 17-19  B widening, odd k-blocks
//   warps 4-7     A widening, even k-blocks  | warps 8-11   A widening, odd k-blocks
//   warps 12-15   epilogue: TMEM -> scale, bias, bf16 -> swizzled shared-memory
//                 staging (2 x 2 KB per warp) -> TMA tensor stores
//   warp 16       TMA producer of the packed ring
// TMEM: accumulators 2 x 192 columns (double-buffered), A ring 4 x 32 columns.
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

constexpr int CM = 128;          // A rows per CTA (pair: 256)
constexpr int PN = 192;          // output columns per pair tile
constexpr int CN = PN / 2;       // B rows per CTA
constexpr int BK = 128;          // codes per k-block
constexpr int BKP = 64;          // packed bytes per row per k-block
constexpr int KPS = 2;           // k-blocks per packed stage
constexpr int PROW = KPS * BKP;  // packed bytes per row per stage (one 128-byte swizzle row)
constexpr int PSTAGES = 5;                 // packed (TMA) ring: 10 k-blocks
constexpr int STAGES = 4;                  // widened ring (A in TMEM, B in shared memory)
constexpr int A_P = CM * PROW;             // 16 KB
constexpr int B_P = CN * PROW;             // 12 KB
constexpr int P_STAGE = A_P + B_P;         // 28 KB
constexpr int B_STAGE = CN * BK;           // 12 KB
constexpr int OFF_B = 0;
constexpr int OFF_P = OFF_B + STAGES * B_STAGE;
constexpr int OFF_PARAM = OFF_P + PSTAGES * P_STAGE;
constexpr int PARAM_BYTES = 4 * 3 * PN * 4;  // per epilogue warp: scale hi, scale lo, bias
constexpr int OFF_STAGE = OFF_PARAM + PARAM_BYTES;  // epilogue output staging
constexpr int STAGE_BYTES = 32 * 32 * 2;            // 32 rows x 32 bf16 columns
constexpr int OFF_BAR = OFF_STAGE + 4 * 2 * STAGE_BYTES;
constexpr int NUM_BARS = 2 * PSTAGES + 2 * STAGES + 4;
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16;
constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;
constexpr int NUM_THREADS = 640;
constexpr int TMEM_COLS = 512;
constexpr int ACC_COLS = PN;                 // one accumulator buffer
constexpr int A_COL0 = 2 * ACC_COLS;         // first column of the A ring
constexpr int WIDEN_WARPS = 7;               // per set: 3 B + 4 A
constexpr int PEMPTY_ARRIVALS = KPS * WIDEN_WARPS;
constexpr int FULL_ARRIVALS = 2 * WIDEN_WARPS;
constexpr int EMPTY_ACC_ARRIVALS = 2 * 4;    // 4 epilogue warps x 2 CTAs
constexpr int PRODUCER_WARP = 16;
constexpr uint32_t IDESC = idesc_i8(2 * CM, PN);
constexpr uint32_t IDESC_HALF = idesc_i8(2 * CM, PN / 2);  // last-round half tiles: 48 B rows per CTA

// The output side of one launch: one to kMaxProj weight matrices that share the activation codes
// (projections of one input, e.g. the query, key and value weights).  Projection j has n[j] output
// columns, its own packed weights, scales, bias and output; its tiles follow those of projection j-1.
struct PairOut {
  CUtensorMap tmap_b[kMaxProj];  // packed weights [n[j], K/2]
  CUtensorMap tmap_y[kMaxProj];  // bf16 outputs [M, n[j]] (unused for int32 outputs)
  const float* w_scale[kMaxProj];
  const uint16_t* bias[kMaxProj];
  void* y[kMaxProj];
  int64_t ldy[kMaxProj];
  int n[kMaxProj];
  int num_n[kMaxProj];     // column tiles of projection j
  int tile_end[kMaxProj];  // tiles of projections 0..j
  int num_proj;
};

// Work items: the tiles of every projection in order, except that when the last round would leave
// more than half of the pairs idle, its tiles are split along N into two half tiles each, so that
// the last round takes half a tile's time.
struct Items {
  int full, total;
  __device__ void get(const PairOut& po, int g, int& proj, int& m_tile, int& n0, int& width) const {
    int tile = g, half = 0;
    width = PN;
    if (g >= full) {
      const int h = g - full;
      tile = full + (h >> 1);
      half = h & 1;
      width = PN / 2;
    }
    int j = 0;
    while (j + 1 < po.num_proj && tile >= po.tile_end[j]) ++j;
    const int local = tile - (j ? po.tile_end[j - 1] : 0);
    proj = j;
    m_tile = local / po.num_n[j];
    n0 = (local % po.num_n[j]) * PN + half * (PN / 2);
  }
};

static_assert(A_COL0 + STAGES * 32 <= TMEM_COLS, "TMEM budget");
static_assert(STAGES == 4 && KPS == 2, "widened-stage arithmetic below uses shifts for these sizes");
static_assert(B_STAGE % 1024 == 0 && OFF_P % 1024 == 0 && A_P % 1024 == 0 && P_STAGE % 1024 == 0,
              "swizzle atoms need 1024-byte alignment");
static_assert(OFF_STAGE % 512 == 0, "64-byte-swizzled staging needs 512-byte alignment");
static_assert(SMEM_ALLOC <= 232448, "shared memory budget");

struct Smem {
  uint8_t* base;
  __device__ uint8_t* b(int s) const { return base + OFF_B + s * B_STAGE; }
  __device__ uint8_t* ap(int p) const { return base + OFF_P + p * P_STAGE; }
  __device__ uint8_t* bp(int p) const { return base + OFF_P + p * P_STAGE + A_P; }
  __device__ float* ph(int q) const { return reinterpret_cast<float*>(base + OFF_PARAM) + q * 3 * PN; }
  __device__ float* pl(int q) const { return ph(q) + PN; }
  __device__ float* pb(int q) const { return ph(q) + 2 * PN; }
  __device__ uint8_t* stage(int q, int buf) const { return base + OFF_STAGE + (2 * q + buf) * STAGE_BYTES; }
  __device__ uint32_t bar(int i) const { return smem_u32(base + OFF_BAR + 8 * i); }
  __device__ uint32_t pfull(int p) const { return bar(p); }
  __device__ uint32_t pempty(int p) const { return bar(PSTAGES + p); }
  __device__ uint32_t full(int s) const { return bar(2 * PSTAGES + s); }
  __device__ uint32_t empty(int s) const { return bar(2 * PSTAGES + STAGES + s); }
  __device__ uint32_t tmem_full(int b) const { return bar(2 * PSTAGES + 2 * STAGES + b); }
  __device__ uint32_t tmem_empty(int b) const { return bar(2 * PSTAGES + 2 * STAGES + 2 + b); }
  __device__ uint32_t* tmem_slot() const { return reinterpret_cast<uint32_t*>(base + OFF_MISC); }
  __device__ volatile int* abort_flag() const { return reinterpret_cast<volatile int*>(base + OFF_MISC + 4); }
};

__device__ __forceinline__ void fail(const Smem& sm, int* status) {
  record_status(status, CR_ERR_TIMEOUT);
  *sm.abort_flag() = 1;
}

__device__ __forceinline__ uint32_t widen_lo(uint32_t w) { return (w << 4) & 0xF0F0F0F0u; }
__device__ __forceinline__ uint32_t widen_hi(uint32_t w) { return w & 0xF0F0F0F0u; }

// Byte offset of 16-byte chunk c (0..3) of k-block half h (0..1) of row r in a
// packed stage: rows of 128 bytes, chunk j of row r stored at chunk j ^ (r & 7).
__device__ __forceinline__ int packed_off(int r, int h, int c) { return r * PROW + ((((h << 2) | c) ^ (r & 7)) << 4); }

// Row of B (0..95 inside the CTA's half) widened by lane group a (0..7) in pass i (0..3) of warp wb.
// Each quarter-warp (lane groups 2k, 2k+1) takes two rows of an 8-row atom whose indices differ
// by 5: bit 2 differs, so their 16-byte packed reads fall in opposite halves of the swizzled
// row, and bit 0 differs, so their 16-byte widened stores (chunks 2c or 2c+1, swizzled) land on
// distinct banks.  No access of the B path has a bank conflict.
__device__ __forceinline__ int b_row(int wb, int i, int a) {
  constexpr uint32_t kPerm = 0x63724150u;  // nibbles: 0,5,1,4,2,7,3,6
  return 32 * wb + 8 * i + static_cast<int>((kPerm >> (4 * a)) & 7u);
}

// Registers -> TMEM: this thread's lane, 32 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
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



template <bool kOutS32>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    w4a4_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ PairOut po,
                          const float* __restrict__ a_scale, int M, int K, int* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  Smem sm;
  sm.base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0 = leader (issues the MMAs), 1 = peer
  const int pair = static_cast<int>(cluster_id_x());
  const int npairs = static_cast<int>(num_clusters_x());
  const int num_tiles = po.tile_end[po.num_proj - 1];
  const int nk = K / BK;  // even: K is a multiple of 256
  Items items;
  {
    const int rem = num_tiles % npairs;
    const bool split = rem > 0 && 2 * rem <= npairs;
    items.full = split ? num_tiles - rem : num_tiles;
    items.total = split ? num_tiles + rem : num_tiles;
  }
  const int my_tiles = pair < items.total ? (items.total - pair + npairs - 1) / npairs : 0;
  const int n_items = my_tiles * nk;

  if (threadIdx.x == 0) {
    for (int p = 0; p < PSTAGES; ++p) {
      mbar_init(sm.pfull(p), 1);
      mbar_init(sm.pempty(p), PEMPTY_ARRIVALS);
    }
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(sm.full(s), FULL_ARRIVALS);
      mbar_init(sm.empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(sm.tmem_full(b), 1);
      mbar_init(sm.tmem_empty(b), EMPTY_ACC_ARRIVALS);
    }
    *sm.abort_flag() = 0;
    fence_mbar_init();
  }
  if (warp == PRODUCER_WARP && lane == 0) {
    prefetch_tmap(&tmap_a);
    for (int j = 0; j < po.num_proj; ++j) {
      prefetch_tmap(&po.tmap_b[j]);
      if (!kOutS32) prefetch_tmap(&po.tmap_y[j]);
    }
  }
  if (warp == 0) {
    tmem_alloc_pair(smem_u32(sm.tmem_slot()), TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any cross-CTA arrive
  tc_fence_after();
  const uint32_t tmem_base = *sm.tmem_slot();
  volatile int* abort = sm.abort_flag();

  auto item_of = [&](int local, int& proj, int& m_tile, int& n0, int& width) {
    items.get(po, pair + local * npairs, proj, m_tile, n0, width);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ MMA issuer (leader CTA)
    if (rank == 0) {
      // The whole warp runs this loop so that the descriptor arithmetic stays warp-uniform;
      // lane 0 alone issues the MMAs and their commits.
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
        int pj_, mt_, n0_, width;
        item_of(t, pj_, mt_, n0_, width);
        const uint32_t idesc = width == PN ? IDESC : IDESC_HALF;
        // two k-blocks (two stages) per iteration
        for (int kb = 0; kb < nk; kb += 2, it += 2) {
          const int s0 = it & 3, s1 = (it + 1) & 3;
          const uint32_t ph0 = static_cast<uint32_t>((it >> 2) & 1);
          const uint32_t ph1 = static_cast<uint32_t>(((it + 1) >> 2) & 1);
          if (!mbar_wait_from(sm.full(s0), ph0, next_full, abort) || !mbar_wait(sm.full(s1), ph1, abort)) {
            ok = false;
            break;
          }
          __syncwarp();
          tc_fence_after();
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int sh = h ? s1 : s0;
            const uint64_t db = sw128_kmajor_desc(smem_u32(sm.b(sh)));
            const uint32_t a_tmem = tmem_base + static_cast<uint32_t>(A_COL0 + 32 * sh);
#pragma unroll
            for (int kk = 0; kk < BK / 32; ++kk)
              umma_i8_pair_ts_lane0(d_tmem, a_tmem + 8u * kk, db + 2u * kk, idesc, (kb + h) | kk ? 1u : 0u, lane);
            umma_commit_pair_mc_lane0(sm.empty(sh), 0x3, lane);
          }
          // test the next pair's first stage while these MMAs run
          next_full = it + 2 < n_items && mbar_test(sm.full((it + 2) & 3), static_cast<uint32_t>(((it + 2) >> 2) & 1));
          last_bar = sm.empty(s1);
          last_par = ph1;
          committed = true;
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
  } else if (warp == PRODUCER_WARP) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      bool ok = true;
      const int n_fill = n_items / KPS;
      int f = 0, p = 0;
      uint32_t ph = 0;  // phase parity of stage p's current use
      bool next_free = n_fill > 0;  // the first PSTAGES fills find their stages free
      for (int t = 0; ok && t < my_tiles; ++t) {
        int proj, m_tile, n0t, width;
        item_of(t, proj, m_tile, n0t, width);
        const int m0 = m_tile * 2 * CM + CM * static_cast<int>(rank);
        const int n0 = n0t + (width / 2) * static_cast<int>(rank);  // this CTA's half of the tile's B rows
        for (int x = 0; x < nk * BKP; x += PROW) {
          if (!mbar_wait_from(sm.pempty(p), ph ^ 1u, next_free, abort)) { ok = false; break; }
          mbar_arrive_expect_tx(sm.pfull(p), P_STAGE);
          tma_load_2d(smem_u32(sm.ap(p)), &tmap_a, x, m0, sm.pfull(p));
          tma_load_2d(smem_u32(sm.bp(p)), &po.tmap_b[proj], x, n0, sm.pfull(p));
          ++f;
          if (++p == PSTAGES) { p = 0; ph ^= 1u; }
          next_free = f < n_fill && (f < PSTAGES || mbar_test(sm.pempty(p), ph ^ 1u));
        }
      }
      if (!ok) {
        fail(sm, status);
        // wait for the loads already issued to land (the last use of each stage)
        for (int q = 0; q < PSTAGES && q < f; ++q) {
          const int last = q + PSTAGES * ((f - 1 - q) / PSTAGES);
          volatile int never = 0;
          mbar_wait(sm.pfull(q), static_cast<uint32_t>((last / PSTAGES) & 1), &never);
        }
      }
    }
  } else if (warp < 4 || warp > PRODUCER_WARP) {
    // ------------------------------------------------------------ B: packed ring -> widened shared memory
    const int set = warp > PRODUCER_WARP ? 1 : 0;  // k-blocks of this parity
    const int wb = set ? warp - (PRODUCER_WARP + 1) : warp - 1;  // rows 32wb .. 32wb+31 of the CTA's 96
    const int a = lane >> 2, c = lane & 3;
    const uint32_t full_leader = mapa_shared(sm.full(0), 0);
    bool ok = true;
    int p = 0;
    uint32_t pph = 0;
    bool p_ready = set < n_items && mbar_test(sm.pfull(0), 0);
    bool s_ready = set < n_items;  // the first STAGES k-blocks find their widened stages free
    for (int it = set; it < n_items; it += 2) {
      const int s = it & 3;
      if (!mbar_wait_from(sm.pfull(p), pph, p_ready, abort)) { ok = false; break; }
      __syncwarp();
      const uint8_t* src = sm.bp(p);
      uint8_t* bs = sm.b(s);
      uint4 w4[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) w4[i] = *reinterpret_cast<const uint4*>(src + packed_off(b_row(wb, i, a), set, c));
      // the widened stage must be free before it is written
      if (!mbar_wait_from(sm.empty(s), static_cast<uint32_t>(((it >> 2) & 1) ^ 1), s_ready, abort)) {
        ok = false;
        break;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = b_row(wb, i, a);
        uint8_t* row = bs + (r >> 3) * 1024 + (r & 7) * 128;
        const uint4 w = w4[i];
        *reinterpret_cast<uint4*>(row + (((2 * c) ^ (r & 7)) << 4)) =
            make_uint4(widen_lo(w.x), widen_hi(w.x), widen_lo(w.y), widen_hi(w.y));
        *reinterpret_cast<uint4*>(row + (((2 * c + 1) ^ (r & 7)) << 4)) =
            make_uint4(widen_lo(w.z), widen_hi(w.z), widen_lo(w.w), widen_hi(w.w));
      }
      // Every lane has issued its widened stores, which consume the packed words: its packed reads
      // have completed, so this k-block's half of the packed stage may be refilled.
      __syncwarp();
      if (lane == 0) mbar_arrive(sm.pempty(p));
      if (++p == PSTAGES) { p = 0; pph ^= 1u; }
      if (it + 2 < n_items) {
        p_ready = mbar_test(sm.pfull(p), pph);
        s_ready = mbar_test(sm.empty((it + 2) & 3), static_cast<uint32_t>((((it + 2) >> 2) & 1) ^ 1));
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(full_leader + 8u * s);
    }
    if (!ok) fail(sm, status);
  } else if (warp < 12) {
    // ------------------------------------------------------------ A: packed ring -> widened TMEM
    const int set = warp >= 8 ? 1 : 0;
    const int q = warp & 3;        // TMEM lane quarter: lanes 32q .. 32q+31
    const int r = 32 * q + lane;   // this thread's row of the CTA's 128 (= its TMEM lane)
    const uint32_t full_leader = mapa_shared(sm.full(0), 0);
    bool ok = true;
    int p = 0;
    uint32_t pph = 0;
    bool p_ready = set < n_items && mbar_test(sm.pfull(0), 0);
    bool s_ready = set < n_items;
    for (int it = set; it < n_items; it += 2) {
      const int s = it & 3;
      if (!mbar_wait_from(sm.pfull(p), pph, p_ready, abort)) { ok = false; break; }
      __syncwarp();
      const uint8_t* src = sm.ap(p);
      uint4 w4[4];  // the row's 64 packed bytes of this k-block
#pragma unroll
      for (int c = 0; c < 4; ++c) w4[c] = *reinterpret_cast<const uint4*>(src + packed_off(r, set, c));
      // the widened stage must be free before it is written
      if (!mbar_wait_from(sm.empty(s), static_cast<uint32_t>(((it >> 2) & 1) ^ 1), s_ready, abort)) {
        ok = false;
        break;
      }
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
      tmem_st_32x32b_x32(tmem_base + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(A_COL0 + 32 * s), v);
      // the TMEM store has consumed the widened words, hence the packed reads have completed
      __syncwarp();
      if (lane == 0) mbar_arrive(sm.pempty(p));
      if (++p == PSTAGES) { p = 0; pph ^= 1u; }
      if (it + 2 < n_items) {
        p_ready = mbar_test(sm.pfull(p), pph);
        s_ready = mbar_test(sm.empty((it + 2) & 3), static_cast<uint32_t>((((it + 2) >> 2) & 1) ^ 1));
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(full_leader + 8u * s);
    }
    if (!ok) fail(sm, status);
  } else {
    // ------------------------------------------------------------ epilogue (warps 12-15)
    const int q = warp & 3;
    const int lrow = lane;  // TMEM lane 32q + lane holds tile row 32q + lane
    float* wph = sm.ph(q);
    float* wpl = sm.pl(q);
    float* wpb = sm.pb(q);
    const uint32_t empty_leader = mapa_shared(sm.tmem_empty(0), 0);
    const float sa = kOutS32 ? 0.f : __ldg(a_scale);
    bool ok = true;
    int nstore = 0;  // bf16 chunks stored by this warp: their staging buffers alternate
    for (int t = 0; ok && t < my_tiles; ++t) {
      const int b = t & 1;
      int proj, m_tile, n0, width;
      item_of(t, proj, m_tile, n0, width);
      const int m0 = m_tile * 2 * CM + CM * static_cast<int>(rank);
      const int N = po.n[proj];
      const float* __restrict__ w_scale = po.w_scale[proj];
      const uint16_t* __restrict__ bias = po.bias[proj];
      __syncwarp();
      for (int col = lane; !kOutS32 && col < width; col += 32) {
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
      for (int ch = 0; ch < width / 32; ++ch) {
        if (n0 + ch * 32 >= N) break;  // columns past N (a half tile may lie wholly past them): nothing to write
        uint32_t r[32];
        tmem_ld32(tmem_base + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(b * ACC_COLS + ch * 32), r);
        tmem_ld_wait();
        if constexpr (kOutS32) {
          int32_t* crow = static_cast<int32_t*>(po.y[proj]) + static_cast<int64_t>(row) * po.ldy[proj];
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
                // acc is 256 * (integer product); |acc/256| < 2^22, so adding 1.5 * 2^23 through the
                // bit pattern and subtracting it again converts to float exactly
                const int32_t ai = (static_cast<int32_t>(r[j + e2 + e]) >> 8) + 0x4B400000;
                const float af = __fsub_rn(__int_as_float(ai), 12582912.0f);
                // y = acc*hi + acc*lo + bias with two fmas: within 2 float32 ulps of y
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
            tma_store_2d(&po.tmap_y[proj], n0 + ch * 32, m0 + 32 * q, smem_u32(stg));
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

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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

// 2-D uint8 tensor map over a dense [rows, cols] byte matrix: boxes of box_rows rows x 128 bytes
// (two k-blocks of codes), stored with the 128-byte swizzle.
bool packed_map(CUtensorMap* map, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(PROW), box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 output [rows, cols] with row stride ld (elements), 32 x 32 boxes, 64-byte swizzle.
bool output_map(CUtensorMap* map, void* ptr, uint64_t rows, uint64_t cols, uint64_t ld) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ptr, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

struct PairLaunch {
  int max_pairs = 0;
  bool attr_done = false;
};

// One launch over `num_proj` projections sharing the activation codes Xq [M, K/2].
template <bool kOutS32>
int launch_pair_impl(const void* Xq, const float* a_scale, int num_proj, const void* const* Wq,
                     const float* const* w_scale, const void* const* bias, void* const* Y, const int64_t* ldy,
                     const int* N, int M, int K, int* status, int num_sms, cudaStream_t stream) {
  if (num_proj < 1 || num_proj > kMaxProj) return CR_ERR_INVALID_ARG;
  static PairLaunch info[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return CR_ERR_CUDA;
  CUtensorMap ta;
  PairOut po;
  memset(&po, 0, sizeof(po));
  const int num_m = (M + 2 * CM - 1) / (2 * CM);
  int tiles = 0;
  for (int j = 0; j < num_proj; ++j) {
    if (N[j] == 0) continue;  // an empty projection has no tiles and is left out
    const int i = po.num_proj;
    if (!packed_map(&po.tmap_b[i], Wq[j], static_cast<uint64_t>(N[j]), static_cast<uint64_t>(K / 2), CN))
      return CR_ERR_CUDA;
    if (!kOutS32 && !output_map(&po.tmap_y[i], Y[j], static_cast<uint64_t>(M), static_cast<uint64_t>(N[j]),
                                static_cast<uint64_t>(ldy[j])))
      return CR_ERR_CUDA;
    po.w_scale[i] = w_scale ? w_scale[j] : nullptr;
    po.bias[i] = bias ? static_cast<const uint16_t*>(bias[j]) : nullptr;
    po.y[i] = Y[j];
    po.ldy[i] = ldy[j];
    po.n[i] = N[j];
    po.num_n[i] = (N[j] + PN - 1) / PN;
    tiles += num_m * po.num_n[i];
    po.tile_end[i] = tiles;
    po.num_proj = i + 1;
  }
  if (M == 0 || tiles == 0) return CR_OK;
  if (!packed_map(&ta, Xq, static_cast<uint64_t>(M), static_cast<uint64_t>(K / 2), CM)) return CR_ERR_CUDA;
  auto kern = w4a4_gemm_pair_kernel<kOutS32>;
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
  // pairs: all of them when the tiles outnumber them; twice the tiles (every tile split into two half
  // tiles by the kernel's item rule) when that still fits; else one pair per tile
  const int maxp = info[dev].max_pairs;
  const int pairs = tiles >= maxp ? maxp : (2 * tiles <= maxp ? 2 * tiles : tiles);
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, ta, po, a_scale, M, K, status);
  return e == cudaSuccess ? CR_OK : CR_ERR_CUDA;
}

}  // namespace

int launch_w4a4_gemm_pair(const void* Xq, const float* a_scale, const void* Wq, const float* w_scale,
                          const void* bias, void* Y, int64_t ldy, int M, int N, int K, int* status, int num_sms,
                          cudaStream_t stream) {
  return launch_pair_impl<false>(Xq, a_scale, 1, &Wq, &w_scale, &bias, &Y, &ldy, &N, M, K, status, num_sms, stream);
}

int launch_w4a4_gemm_pair_multi(const void* Xq, const float* a_scale, int num_proj, const void* const* Wq,
                                const float* const* w_scale, const void* const* bias, void* const* Y,
                                const int64_t* ldy, const int* N, int M, int K, int* status, int num_sms,
                                cudaStream_t stream) {
  return launch_pair_impl<false>(Xq, a_scale, num_proj, Wq, w_scale, bias, Y, ldy, N, M, K, status, num_sms, stream);
}

int launch_w4a4_gemm_pair_multi_s32(const void* Xq, int num_proj, const void* const* Wq, void* const* C,
                                    const int64_t* ldc, const int* N, int M, int K, int* status, int num_sms,
                                    cudaStream_t stream) {
  return launch_pair_impl<true>(Xq, nullptr, num_proj, Wq, nullptr, nullptr, C, ldc, N, M, K, status, num_sms,
                                stream);
}

int launch_w4a4_gemm_pair_s32(const void* Xq, const void* Wq, int32_t* C, int64_t ldc, int M, int N, int K,
                              int* status, int num_sms, cudaStream_t stream) {
  void* y = C;
  return launch_pair_impl<true>(Xq, nullptr, 1, &Wq, nullptr, nullptr, &y, &ldc, &N, M, K, status, num_sms, stream);
}

}  // namespace cr

