// Shared device/host helpers of the MoGA sm_100a library.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/moga.h"

namespace moga {

// Host: record an error message for moga_last_error() and return `st`.
moga_status fail(moga_status st, const char* fmt, ...);
// Host: map the last launch error to MOGA_ERR_CUDA (with message) or MOGA_OK.
moga_status check_launch(const char* what);

// Device error word (one per device, lazily created by the CUDA runtime).
// The library is built as one translation unit (moga_lib.cu), so the word is
// defined here once.
__device__ int g_device_error = 0;

__device__ __forceinline__ void record_device_error(int code) {
  atomicCAS(&g_device_error, 0, code);
}

__host__ __device__ constexpr int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Index checks of the checking build (compiled with -DMOGA_DEBUG into
// libmoga_debug.so): kernels test every index they take from a caller's
// buffer (perm entries, cu_seqlens, token rows derived from them) before the
// access it guards.  A failed check records MOGA_ERR_BAD_INDEX in the device
// error word and skips that access (or, for a bad cu_seqlens, the whole
// launch); nothing traps.  In the default build the checks compile away.
#ifdef MOGA_DEBUG
constexpr bool kCheckIndices = true;
#else
constexpr bool kCheckIndices = false;
#endif

// Limit of every bounded wait on an mbarrier, in SM clock cycles: about two
// seconds at the maximum SM clock.  A wait that runs out records
// MOGA_ERR_TIMEOUT in the device error word and the kernel returns.
constexpr long long kWaitLimitCycles = 4000000000LL;

}  // namespace moga
