// status.cuh -- device status word and shared constants.
#pragma once

#include <cstdint>

namespace csa {

// Device-side status codes (match csa_status in csa.h).
constexpr uint32_t CSA_DEV_OK = 0;
constexpr uint32_t CSA_DEV_TIMEOUT = 4;
constexpr uint32_t CSA_DEV_BOUNDS = 6;

// A bounded wait gives up after this many SM clock cycles (about half a second at the
// B200's clocks), records CSA_DEV_TIMEOUT and lets the kernel unwind.
constexpr long long kWaitCycles = 1ll << 30;

// The status word lives in the first 256 bytes of every workspace.
constexpr size_t kStatusBytes = 256;

// Debugging builds (-DCSA_TRACE) may place the workspace in host-mapped memory, where device
// atomics are not available on every platform: they use plain stores instead.
__device__ __forceinline__ void record_status(uint32_t* status, uint32_t code) {
#ifdef CSA_TRACE
  if (status != nullptr) *reinterpret_cast<volatile uint32_t*>(status) = code;
#else
  if (status != nullptr) atomicCAS(status, CSA_DEV_OK, code);
#endif
}

// Where a bounded wait gave up (first one wins): status word 1.
__device__ __forceinline__ void record_site(uint32_t* status, uint32_t site) {
#ifdef CSA_TRACE
  if (status != nullptr) *reinterpret_cast<volatile uint32_t*>(status + 1) = site;
#else
  if (status != nullptr) atomicCAS(status + 1, 0u, site);
#endif
}

// Progress markers for debugging builds (-DCSA_TRACE): role `role` of the calling CTA stores `v`
// into status word 64 + 4*cta + role. Compiled out otherwise.
__device__ __forceinline__ void trace_mark(uint32_t* status, int role, uint32_t v) {
#ifdef CSA_TRACE
  if (status != nullptr) {
    const uint32_t cta = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
    volatile uint32_t* p = status + 64 + 4 * cta + role;
    *p = v;
  }
#else
  (void)status;
  (void)role;
  (void)v;
#endif
}

// Timeline for debugging builds (-DCSA_TRACE): CTA (0,0) stores the low word of %globaltimer (ns)
// into word kTraceWord + idx of the workspace (a debugging workspace of >= 8 MB). Compiled out
// otherwise.
constexpr size_t kTraceWord = size_t(1) << 20;
__device__ __forceinline__ void trace_time(uint32_t* status, int idx) {
#ifdef CSA_TRACE
  if (status != nullptr && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0) {
    uint32_t t;
    asm volatile("mov.u32 %0, %%globaltimer_lo;" : "=r"(t));
    *reinterpret_cast<volatile uint32_t*>(status + kTraceWord + idx) = t;
  }
#else
  (void)status;
  (void)idx;
#endif
}

// Step timeline for profiling builds (-DCSA_STEP_TIMELINE): thread 0 of every CTA folds the
// %globaltimer (ns) at kernel entry (min over CTAs), after its dependency wait (min) and at its end
// (max) into uint64 words 8 + 3*kernel + {0, 1, 2} of the status area (bytes 64..255 of the
// workspace, which the caller presets to ~0 / ~0 / 0). Kernel ids: see TimelineKernel. Compiled out
// otherwise.
enum TimelineKernel { kTlCompress = 0, kTlIndexer = 1, kTlTopk = 2, kTlTopkMerge = 3, kTlAttn = 4, kTlCombine = 5 };
enum TimelineWhat { kTlEntry = 0, kTlReady = 1, kTlExit = 2 };
__device__ __forceinline__ void timeline_mark(uint32_t* status, int kernel, int what) {
#ifdef CSA_STEP_TIMELINE
  if (status != nullptr && threadIdx.x == 0) {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    unsigned long long* w = reinterpret_cast<unsigned long long*>(status) + 8 + 3 * kernel + what;
    if (what == kTlExit) atomicMax(w, t);
    else atomicMin(w, t);
  }
#else
  (void)status;
  (void)kernel;
  (void)what;
#endif
}

}  // namespace csa
