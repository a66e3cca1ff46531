// status.cuh -- the device status word kept at the start of every workspace.
//
// Layout (first 256 bytes of a workspace; the caller zeroes them once):
//   word 0: OR of SPTS_DEV_* flags raised by kernels since the last check
//   word 1: code of the first place that raised a flag (kernel-specific)
//   word 2: a value recorded with it (e.g. an out-of-range index)
#pragma once

#include <cstdint>

namespace spts {

constexpr uint32_t SPTS_DEV_TIMEOUT = 1u;   // a bounded wait gave up
constexpr uint32_t SPTS_DEV_BADINDEX = 2u;  // an index was out of range and skipped

constexpr size_t kStatusBytes = 256;              // reserved head of every workspace
constexpr uint64_t kDrainLimitNs = 1000000000ull;  // abort-path drains: 1 s
constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;

__device__ __forceinline__ void raise_status(uint32_t *status, uint32_t flag, uint32_t where,
                                             uint32_t value = 0) {
  if (status == nullptr) return;
  uint32_t old = atomicOr(status, flag);
  if (old == 0) {
    atomicExch(status + 1, where);
    atomicExch(status + 2, value);
  }
}

}  // namespace spts
