// work_queue.cuh -- the fused kernel's queue of published races and its
// bounded waits.
//
// Control words (VerifyArgs::ctl, zero at launch, each on its own 128-byte line):
//   kCtlPublished  races published so far; race j is request pubq[j] - 1
//   kCtlClaimed    race parts claimed so far (part i belongs to race i / parts)
//   kCtlScanned    requests whose accept scan is done (with or without a race)
// A producer writes the race description, then takes the next race slot j and
// writes pubq[j] = b + 1 with release semantics; it never waits in between.  A
// consumer claims part i with one atomic add, and may claim ahead of what is
// published (it then keeps the claim until the part is published, or until
// every request is scanned and the part turns out not to exist).
#pragma once
#include "sv_common.cuh"

namespace sv {

constexpr int kCtlPublished = 0 * 32;
constexpr int kCtlClaimed = 1 * 32;
constexpr int kCtlScanned = 2 * 32;
constexpr unsigned kNoPart = 0xFFFFFFFFu;

constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // every wait gives up after ~2 s

__device__ __forceinline__ unsigned load_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ unsigned load_volatile(const unsigned* p) {
  return *(const volatile unsigned*)p;
}

__device__ __forceinline__ void store_release_gpu(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Publish request b's race (one thread): the race description is written
// before the call.
__device__ __forceinline__ void publish_race(unsigned* ctl, unsigned* pubq, unsigned b) {
  __threadfence();
  const unsigned j = atomicAdd(&ctl[kCtlPublished], 1u);
  store_release_gpu(&pubq[j], b + 1);
}

// The request of published race j (one thread): pubq[j] is written right after
// the slot is taken, by a thread that does not wait in between, so this wait
// is short; bounded all the same (0 and SV_STATUS_TIMEOUT in *status if it runs
// out).
__device__ __forceinline__ unsigned wait_published(const unsigned* pubq, unsigned j,
                                                   unsigned* status) {
  unsigned v = load_acquire_gpu(&pubq[j]);
  if (v) return v;
  const unsigned long long t0 = globaltimer_ns();
  while (!(v = load_acquire_gpu(&pubq[j]))) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      atomicOr(status, kStatusTimeout);
      return 0u;
    }
    __nanosleep(32);
  }
  return v;
}

// A warp's idle wait (one call per idle turn of the work loop, by every lane):
// sleeps a growing interval (64 ns doubling to 2 us) and returns false, with
// SV_STATUS_TIMEOUT in *status, once the warp has been idle for longer than the
// limit since start().
struct WaitClock {
  unsigned long long t0;
  unsigned sleep_ns;
  __device__ __forceinline__ void start() {
    t0 = 0ull;
    sleep_ns = 64;
  }
  __device__ __forceinline__ bool wait(unsigned* status) {
    const unsigned long long now = globaltimer_ns();
    if (t0 == 0ull) t0 = now;
    if (now - t0 > kWaitLimitNs) {
      if ((threadIdx.x & 31) == 0) atomicOr(status, kStatusTimeout);
      return false;
    }
    __nanosleep(sleep_ns);
    if (sleep_ns < 2048) sleep_ns *= 2;
    return true;
  }
};

}  // namespace sv
