// Device-side helpers shared by the library's kernels: shared-memory matrix
// descriptors for tcgen05 operands, and bounded mbarrier waits that record a
// status code instead of hanging.
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace wavei {

constexpr uint64_t kTimeoutNs = 2000000000ull;  // default: a wait gives up after 2 s
constexpr uint64_t kDrainNs = 200000000ull;     // waits while stopping: 0.2 s

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 version field.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// K-major operand (Q, K): rows of 128 bytes, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_k(uint32_t addr) { return smem_desc(addr, 16, 1024); }
// MN-major operand (V as [key][d]): 64-column groups one panel (16 KB) apart,
// 8-key groups 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_mn(uint32_t addr) { return smem_desc(addr, 16384, 1024); }

struct Ctl {
  volatile int* abort_flag;
  int32_t* status;
  uint64_t timeout_ns;  // how long one wait may take (the handle's wait limit)
};

// Bounded wait on an mbarrier phase. Returns false if this CTA is stopping:
// another thread gave up, or this one waited ctl.timeout_ns (it then sets the
// CTA's stop flag and records `code` in the status word, first code wins).
// A plain try_wait may suspend the thread for a system-dependent time, so
// after the first test every try_wait carries the remaining bound (at most
// kMaxSuspendNs) as its suspension limit and the clock is read after each:
// a bound far below the hardware's own suspension time still takes effect.
constexpr uint64_t kLongWaitNs = 1000000ull;   // bounds from 1 ms up: plain first test
constexpr uint32_t kMaxSuspendNs = 1000000u;   // one suspension lasts at most 1 ms
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, const Ctl& ctl, int code) {
  const uint32_t hint =
      ctl.timeout_ns < kMaxSuspendNs ? (uint32_t)ctl.timeout_ns : kMaxSuspendNs;
  if (ctl.timeout_ns >= kLongWaitNs && wptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = wptx::globaltimer_ns();
  while (!wptx::mbar_try_wait_hint(bar, parity, hint)) {
    if (*ctl.abort_flag) return false;
    if (wptx::globaltimer_ns() - t0 > ctl.timeout_ns) {
      *ctl.abort_flag = 1;
      atomicCAS(ctl.status, 0, code);
      return false;
    }
  }
  return true;
}

// Bounded wait that ignores the stop flag: used only while stopping, to let
// asynchronous copies or MMAs that were already issued complete.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = wptx::globaltimer_ns();
  while (!wptx::mbar_try_wait(bar, parity))
    if (wptx::globaltimer_ns() - t0 > kDrainNs) return;
}

}  // namespace wavei
