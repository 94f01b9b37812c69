// Bounded waits on mbarriers, shared by the kernels: every wait ends, either because the
// phase completed or because a time limit (%globaltimer) ran out; a wait that runs out
// records where in the device error word and raises the CTA's abort flag so that the other
// roles leave their loops.
#pragma once

#include <cstdint>

#include "kernels.h"
#include "sm100.cuh"

namespace hgx {
namespace waits {

using namespace sm100;

struct Ctx {
  uint32_t bars;           // shared address of barrier 0
  volatile uint32_t* abort_flag;
  uint32_t* err;
  uint64_t limit_ns;
};

__device__ __forceinline__ uint32_t bar_addr(const Ctx& c, uint32_t i) { return c.bars + 8 * i; }

// Bounded wait for the phase of the given parity. Returns false if the wait ran out (after
// recording it in the device error word and raising the CTA's abort flag) or if another
// role already raised the abort flag.
__device__ __forceinline__ bool wait_slow(uint32_t bar, uint32_t parity, volatile uint32_t* abort_flag,
                                       uint32_t* err, uint64_t limit_ns, uint32_t site) {
  uint64_t start = 0;
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if ((it & 63u) == 0) {
      const uint64_t now = globaltimer_ns();
      if (start == 0) {
        start = now;
      } else if (now - start > limit_ns) {
        *abort_flag = 1u;
        atomicOr(err, kErrTimeout | (site << 8));
        return false;
      }
    }
  }
}

__device__ __forceinline__ bool wait_bounded(const Ctx& c, uint32_t bar, uint32_t parity,
                                             uint32_t site) {
  if (mbar_try_wait(bar, parity)) return true;
  return wait_slow(bar, parity, c.abort_flag, c.err, c.limit_ns, site);
}

// Bounded wait that ignores the abort flag: used while draining copies and MMAs that are
// already in flight, which complete on their own.
__device__ __forceinline__ void wait_drain(const Ctx& c, uint32_t bar, uint32_t parity,
                                           uint32_t site) {
  const uint64_t start = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - start > c.limit_ns) {
      atomicOr(c.err, kErrTimeout | (site << 8));
      return;
    }
  }
}


}  // namespace waits
}  // namespace hgx
