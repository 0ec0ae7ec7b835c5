// status.cuh -- device-side error recording shared by all DSA kernels.
// Kernels never trap: the first error of a call sequence is recorded in a
// 32-bit status word at the start of the caller's workspace and read back by
// dsa_get_device_status().  Codes equal the dsa_status_t values of dsa.h.
#pragma once
#include <cstdint>

namespace dsa {

enum : int {
    DSA_STATUS_OK = 0,
    DSA_STATUS_INVALID_ARG = 1,  // an argument only the device can check (dsa_prefill: rows of different sequences)
    DSA_STATUS_TIMEOUT = 5,
    DSA_STATUS_INDEX_OOB = 6,
    DSA_STATUS_LENGTH = 7,
};

// Wall-clock limit of every bounded wait inside a kernel (nanoseconds).
constexpr uint64_t kWaitBudgetNs = 2000000000ull;

__device__ __forceinline__ void record_status(int* status, int code) {
    if (status != nullptr) atomicCAS(status, 0, code);
}

}  // namespace dsa
