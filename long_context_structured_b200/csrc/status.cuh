// status.cuh -- device status word shared by every kernel of the library.
//
// The first 256 bytes of each workspace hold int32 status[64]:
//   status[0]  SATTN_OK or the first device-side error (SATTN_ERR_TIMEOUT)
//   status[1]  site id of the first failure (which wait gave up)
//   status[2]  scratch counter (uncertified top-k rows)
// Every entry point clears it before its first launch.
#pragma once

#include <stdint.h>

#include "../../include/sattn.h"

namespace sattn {

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per bounded wait
constexpr int kStatusWords = 64;
constexpr size_t kStatusBytes = 256;

__device__ __forceinline__ void report_timeout(int32_t* status, int where) {
  if (atomicCAS(status, 0, SATTN_ERR_TIMEOUT) == 0) {
    atomicExch(status + 1, where);
  }
}

__device__ __forceinline__ bool status_failed(const int32_t* status) {
  return *reinterpret_cast<const volatile int32_t*>(status) != 0;
}

}  // namespace sattn
