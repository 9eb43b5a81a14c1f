// grid_sync.cuh -- grid-wide barriers of the persistent kernels (every CTA resident): GPU-scope
// loads, stores and reductions on words in the caller's workspace.  Inline PTX against the public
// PTX ISA; included after cr_device.cuh.
#pragma once

namespace cr {

__device__ __forceinline__ unsigned long long ld_acquire_gpu(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ unsigned long long ld_relaxed_gpu(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ unsigned int ld_relaxed_gpu(const unsigned int* p) {
  unsigned int v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed_gpu(unsigned int* p, unsigned int v) {
  asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void red_add_release_gpu(unsigned long long* p, unsigned long long v) {
  asm volatile("red.release.gpu.global.add.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ void red_max_relaxed_gpu(unsigned int* p, unsigned int v) {
  asm volatile("red.relaxed.gpu.global.max.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Wait at a grid-wide barrier whose arrivals are weights added to `count`: poll with acquire loads until
// the counter reaches `target`.  One thread per CTA.  Bounded: false after CR_WAIT_TIMEOUT_NS.
__device__ __forceinline__ bool grid_wait(const unsigned long long* count, unsigned long long target) {
  uint64_t t0 = 0;
#pragma unroll 1
  for (uint32_t i = 0; ld_acquire_gpu(count) < target; ++i) {
    if ((i & 63u) == 0) {
      const uint64_t t = globaltimer_ns();
      if (i == 0) t0 = t; else if (t - t0 > CR_WAIT_TIMEOUT_NS) return false;
    }
  }
  return true;
}

// Arrive (a release reduction adding `weight`: no round trip), then wait.
__device__ __forceinline__ bool grid_arrive_wait(unsigned long long* count, unsigned long long weight,
                                                 unsigned long long target) {
  red_add_release_gpu(count, weight);
  return grid_wait(count, target);
}

// Programmatic dependent launch: the next kernel on the stream, if launched as a programmatic dependent,
// may start once every CTA of this grid has executed launch_dependents (or exited); the dependent waits
// with griddep_wait until this grid has completed and its memory is visible before it reads this grid's
// results.
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

}  // namespace cr
