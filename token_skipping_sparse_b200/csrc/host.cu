// host.cu -- implementation of the host-side plumbing (see host.hpp).
#include <atomic>
#include <cstring>
#include <mutex>
#include <vector>

#include "host.hpp"

namespace spts {

static thread_local std::string g_last_error;
static uint64_t g_wait_limit_ns = kDefaultWaitLimitNs;
static std::atomic<uint64_t> g_launches{0};

void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

void set_error(const char *fmt, ...) {
  char buf[1024];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
}

void clear_error() { g_last_error.clear(); }

spts_status check_ws(void *ws, size_t ws_bytes, size_t need, const char *who) {
  SPTS_REQUIRE(ws != nullptr, SPTS_ERR_WORKSPACE, "%s: workspace is NULL", who);
  SPTS_REQUIRE(aligned(ws, 256), SPTS_ERR_WORKSPACE, "%s: workspace must be 256-byte aligned", who);
  SPTS_REQUIRE(ws_bytes >= need, SPTS_ERR_WORKSPACE, "%s: workspace has %zu bytes, needs %zu", who, ws_bytes,
               need);
  return SPTS_OK;
}

int num_sms() {
  static std::mutex mu;
  static std::vector<int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  std::lock_guard<std::mutex> lk(mu);
  if (static_cast<int>(cache.size()) <= dev) cache.resize(dev + 1, 0);
  if (cache[dev] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = n > 0 ? n : 148;
  }
  return cache[dev];
}

size_t max_smem_optin() {
  int dev = 0, v = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  return static_cast<size_t>(v);
}

uint64_t wait_limit_ns() { return g_wait_limit_ns; }

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

spts_status make_tmap(CUtensorMap *map, CUtensorMapDataType dtype, int rank, const void *ptr,
                      const uint64_t *dims, const uint64_t *strides_bytes, const uint32_t *box,
                      CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  SPTS_REQUIRE(fn != nullptr, SPTS_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t d[5], s[4];
  cuuint32_t b[5], e[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    e[i] = 1;
  }
  for (int i = 0; i < rank - 1; ++i) s[i] = strides_bytes[i];
  CUresult r = fn(map, dtype, static_cast<cuuint32_t>(rank), const_cast<void *>(ptr), d, s, b, e,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  SPTS_REQUIRE(r == CUDA_SUCCESS, SPTS_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)",
               static_cast<int>(r));
  return SPTS_OK;
}

spts_status tmap_bf16_2d(CUtensorMap *map, const void *ptr, uint64_t rows, uint64_t cols, uint64_t ld,
                         uint32_t box_rows) {
  uint64_t dims[2] = {cols, rows};
  uint64_t strides[1] = {ld * 2};
  uint32_t box[2] = {64, box_rows};
  return make_tmap(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ptr, dims, strides, box,
                   CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace spts

extern "C" {

const char *spts_version(void) { return "0.1.0"; }

size_t spts_last_error(char *buf, size_t len) {
  const std::string &e = spts::g_last_error;
  if (buf != nullptr && len > 0) {
    size_t n = e.size() < len - 1 ? e.size() : len - 1;
    memcpy(buf, e.data(), n);
    buf[n] = '\0';
  }
  return e.size();
}

spts_status spts_check_device_status(void *ws, spts_stream stream) {
  SPTS_REQUIRE(ws != nullptr, SPTS_ERR_WORKSPACE, "spts_check_device_status: workspace is NULL");
  uint32_t word[4] = {0, 0, 0, 0};
  SPTS_CUDA_TRY(cudaStreamSynchronize(stream));
  SPTS_CUDA_TRY(cudaMemcpy(word, ws, sizeof(word), cudaMemcpyDeviceToHost));
  SPTS_CUDA_TRY(cudaMemset(ws, 0, sizeof(word)));
  if (word[0] & spts::SPTS_DEV_TIMEOUT) {
    spts::set_error("device: a bounded wait gave up (site 0x%x)", word[1]);
    return SPTS_ERR_TIMEOUT;
  }
  if (word[0] & spts::SPTS_DEV_BADINDEX) {
    spts::set_error("device: out-of-range index %u skipped (site 0x%x)", word[2], word[1]);
    return SPTS_ERR_INVALID;
  }
  return SPTS_OK;
}

// Test hook: the bounded-wait limit handed to pipelined kernels (0 makes
// every wait that is not already satisfied give up at once).
void spts_debug_set_wait_limit_ns(uint64_t ns) { spts::g_wait_limit_ns = ns; }
uint64_t spts_debug_get_wait_limit_ns(void) { return spts::g_wait_limit_ns; }

uint64_t spts_launch_count(void) { return spts::g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
