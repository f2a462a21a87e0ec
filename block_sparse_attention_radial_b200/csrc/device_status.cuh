// Per-device status word shared by every kernel of the library. A kernel that
// detects a problem it cannot return (a bounded wait that ran out, an
// out-of-range list entry, an output too small) records a bsa_status code
// here; the first code recorded wins until bsa_get_device_status() clears it.
#pragma once

#include <cstdint>

namespace bsa {

__device__ unsigned int g_status;
// Where the first bounded wait gave up: [0] = role (1 producer, 2 mma,
// 3 softmax), [1] = barrier id, [2] = block counter, [3] = CTA index.
__device__ unsigned int g_status_detail[4];

__device__ __forceinline__ void record_status(unsigned int code) {
  atomicCAS(&g_status, 0u, code);
}

}  // namespace bsa
