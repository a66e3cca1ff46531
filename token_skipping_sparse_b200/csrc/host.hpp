// host.hpp -- host-side plumbing shared by the C-ABI entry points:
// thread-local error messages, argument checks, workspace carving, device
// properties and TMA tensor-map encoding (through the driver entry point, so
// the library does not link libcuda and loads on machines without a GPU).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <string>

#include "spts.h"
#include "status.cuh"

namespace spts {

void set_error(const char *fmt, ...);
void clear_error();

#define SPTS_REQUIRE(cond, code, ...)   \
  do {                                  \
    if (!(cond)) {                      \
      ::spts::set_error(__VA_ARGS__);   \
      return (code);                    \
    }                                   \
  } while (0)

#define SPTS_CUDA_TRY(call)                                                                 \
  do {                                                                                      \
    cudaError_t e_ = (call);                                                                \
    if (e_ != cudaSuccess) {                                                                \
      ::spts::set_error("%s failed: %s (%s:%d)", #call, cudaGetErrorString(e_), __FILE__, __LINE__); \
      return SPTS_ERR_CUDA;                                                                 \
    }                                                                                       \
  } while (0)

#define SPTS_TRY(expr)                \
  do {                                \
    spts_status s_ = (expr);          \
    if (s_ != SPTS_OK) return s_;     \
  } while (0)

inline bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Carves 256-byte aligned sub-buffers out of a caller workspace; the first
// kStatusBytes are the status word.
struct Carver {
  char *base;
  size_t cap;
  size_t off;
  Carver(void *ws, size_t bytes) : base(static_cast<char *>(ws)), cap(bytes), off(kStatusBytes) {}
  static size_t round(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }
  void *take(size_t bytes) {
    void *p = base + off;
    off += round(bytes);
    return p;
  }
  bool ok() const { return off <= cap; }
  uint32_t *status() const { return reinterpret_cast<uint32_t *>(base); }
};

// Checks a workspace against the size its *_workspace() call returned.
spts_status check_ws(void *ws, size_t ws_bytes, size_t need, const char *who);

void note_launch();            // counts one kernel launch of this library
int num_sms();                 // SM count of the current device
uint64_t wait_limit_ns();      // bounded-wait limit handed to kernels
size_t max_smem_optin();       // per-block opt-in shared memory

// TMA tensor maps (row-major tensors; dims innermost first).
spts_status make_tmap(CUtensorMap *map, CUtensorMapDataType dtype, int rank, const void *ptr,
                      const uint64_t *dims, const uint64_t *strides_bytes /* rank-1 entries */,
                      const uint32_t *box, CUtensorMapSwizzle swizzle);

// 2-D bf16 tensor [rows, cols] (row stride ld elements), box {64, box_rows},
// 128-byte swizzle: the K-major UMMA operand layout.
spts_status tmap_bf16_2d(CUtensorMap *map, const void *ptr, uint64_t rows, uint64_t cols, uint64_t ld,
                         uint32_t box_rows);

}  // namespace spts
