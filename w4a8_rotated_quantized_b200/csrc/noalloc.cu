// noalloc.cu -- the whole online layer without any caller-provided scratch.
//
// cr_w4a4_linear needs a workspace for the per-block partial maxima, the
// activation scale and the packed activation codes.  Some callers cannot
// provide one: code that runs where device allocation is forbidden or
// unavailable (inside another framework's CUDA-graph capture region, under a
// fixed memory pool that has no room for ad-hoc buffers, or in a host thread
// that must not call cudaMalloc because it synchronises the device).  For them
// this file keeps the scratch in one file-scope device array, allocated once
// when the library's module is loaded on a GPU and held until the process
// exits.  Nothing here calls cudaMalloc, cudaFree or any allocating routine.
//
// Limits and rules (also stated in include/convrot.h):
// - the packed activation codes must fit: M * K / 2 <= kNoAllocXqBytes (8 MiB);
//   larger calls are rejected with CR_ERR_WORKSPACE before anything is launched;
// - every call on a device shares the one array, so calls whose GPU work
//   overlaps (different streams, or different host threads) race on it;
// - the array keeps the last call's contents; nothing needs clearing between
//   calls, because every scratch byte a kernel reads is written earlier in the
//   same call, and the status word starts at zero when the module loads;
// - the first call on each device looks up the array's device address
//   (cudaGetSymbolAddress) with that device current; make that first call
//   before any stream capture.

#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/convrot.h"
#include "cr_internal.h"

namespace {

constexpr size_t kNoAllocXqBytes = size_t(8) << 20;
constexpr size_t kScaleOff = cr::kActWsBytes;            // one float, own 256-byte slot
constexpr size_t kXqOff = cr::kActWsBytes + 256;
constexpr size_t kScratchBytes = kXqOff + kNoAllocXqBytes;

// Host code must not use this name as a pointer: on the host it is only a
// stand-in symbol.  The device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
uint8_t* g_scratch_addr[kMaxDevices] = {};
int g_num_sms[kMaxDevices] = {};
std::mutex g_setup_mu;

// Once per device, with that device current: device check and the scratch's device address.
cr_status setup_current_device(uint8_t** scratch, int* num_sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return CR_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return CR_ERR_UNSUPPORTED_ARCH;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (!g_scratch_addr[dev]) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return CR_ERR_CUDA;
    }
    if (major != 10 || minor != 0) return CR_ERR_UNSUPPORTED_ARCH;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return CR_ERR_CUDA;
    }
    g_num_sms[dev] = sms;
    g_scratch_addr[dev] = static_cast<uint8_t*>(p);
  }
  *scratch = g_scratch_addr[dev];
  *num_sms = g_num_sms[dev];
  return CR_OK;
}

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" cr_status cr_w4a4_linear_noalloc(const void* X, int64_t ldx, const void* Wq, const float* w_scale,
                                            const void* bias, void* Y, int64_t ldy, int M, int N, int K, int group,
                                            void* stream) {
  if (M < 0 || N < 0 || K < 0 || ldx < 0 || ldy < 0) return CR_ERR_INVALID_ARG;
  if (M > 0 && N > 0 && (!X || !Wq || !w_scale || !Y)) return CR_ERR_INVALID_ARG;
  if ((group != CR_GROUP_256 && group != CR_GROUP_64 && group != CR_GROUP_16 && group != CR_GROUP_1024) || K < 256 ||
      K % 256 != 0 || K % group != 0 || K > CR_MAX_K || N % 8 != 0)
    return CR_ERR_UNSUPPORTED_SHAPE;
  if (ldx < K || ldy < N) return CR_ERR_INVALID_ARG;
  if (!aligned(X, 16) || !aligned(Wq, 16) || !aligned(Y, 16) || ldx % 8 != 0 || ldy % 8 != 0 ||
      !aligned(w_scale, 4) || (bias && !aligned(bias, 2)))
    return CR_ERR_MISALIGNED;
  if (static_cast<size_t>(M) * static_cast<size_t>(K) / 2 > kNoAllocXqBytes) return CR_ERR_WORKSPACE;
  if (M == 0 || N == 0) return CR_OK;
  uint8_t* scratch = nullptr;
  int nsm = 0;
  cr_status st = setup_current_device(&scratch, &nsm);
  if (st != CR_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* a_scale = reinterpret_cast<float*>(scratch + kScaleOff);
  uint8_t* xq = scratch + kXqOff;
  int* status = reinterpret_cast<int*>(scratch + cr::kWsStatusOff);
  const uint16_t* x = static_cast<const uint16_t*>(X);
  if (cr::launch_act_fmt(x, M, K, ldx, xq, a_scale, 1, cr::kFmtPacked4, true, group, scratch, nsm, cr::kActAuto, s) !=
      cudaSuccess)
    return CR_ERR_CUDA;
  return static_cast<cr_status>(cr::launch_w4a4_gemm(xq, a_scale, Wq, w_scale, bias, Y, ldy, M, N, K, status, nsm, s));
}
