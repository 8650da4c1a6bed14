// kvq_selftest.cuh - the failure path of the library's bounded waits, run on
// purpose: a wait on a condition that nothing completes runs out, records
// KVQ_ERR_TIMEOUT in the device error word and returns, leaving the context
// usable. Used by tests only; no kernel of the hot path calls it.
#pragma once

#include "kvq_device.cuh"

namespace kvq {

// A 16-byte word that nothing ever writes (zero from program load): the
// poll below waits for it to become non-zero.
__device__ __align__(16) uint32_t g_never_written[4] = {0u, 0u, 0u, 0u};

// which = 0: mbar_wait_bounded on an mbarrier that nobody arrives on (the
//            wait of the write and prefill pipelines);
// which = 1: the split merge's poll (relaxed GPU-scope 16-byte loads, 64 ns
//            back-off, kMaxSpinRounds rounds) on a word that stays zero.
// One warp; the kernel returns once the wait has run out.
__global__ void __launch_bounds__(32, 1) kvq_selftest_wait_kernel(int which) {
  __shared__ __align__(8) uint64_t bar;
  if (which == 0) {
    const uint32_t b = smem_addr(&bar);
    if (threadIdx.x == 0) {
      mbar_init(b, 1);
      mbar_init_fence();
    }
    __syncwarp();
    if (threadIdx.x == 0) (void)mbar_wait_bounded(b, 0);
  } else {
    for (uint32_t rounds = 0;; ++rounds) {
      const uint4 v = ld_relaxed_gpu_v4(g_never_written);
      if (__all_sync(0xffffffffu, v.x && v.y && v.z && v.w)) break;
      if (rounds >= kMaxSpinRounds) {
        if (threadIdx.x == 0) record_error(KVQ_ERR_TIMEOUT);
        break;
      }
      __nanosleep(64);
    }
  }
}

// A kernel that holds SMs for a while and then ends on its own: each CTA
// (given most of an SM's shared memory, so that little else fits beside it)
// waits until `ns` nanoseconds of the global timer have passed, with a cap
// on its polls. Tests use it to fill SMs while a decode is launched on
// another stream.
__global__ void __launch_bounds__(32, 1) kvq_selftest_occupy_kernel(unsigned long long ns) {
  extern __shared__ uint8_t hold[];
  unsigned long long t0, t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  for (uint32_t i = 0; i < (1u << 22); ++i) {
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    if (t - t0 >= ns) break;
    __nanosleep(256);
  }
  if (threadIdx.x == 0 && ns == ~0ull) hold[0] = 0;  // never: keeps the allocation
}

}  // namespace kvq
