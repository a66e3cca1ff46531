// noalloc.cu -- spts_stage_prune_noalloc: the MSDP stage prune for callers
// that cannot allocate device memory when they call into the library.
//
// spts_stage_prune needs Nc int32 of scratch for the kept indices, which the
// caller normally provides as a workspace.  Some callers cannot obtain one:
// a plugin running inside a host framework that reserved the GPU's memory up
// front and forbids any further cudaMalloc, or a latency-critical loop where
// cudaMalloc's implicit device synchronisation is not acceptable.  This
// variant keeps that scratch in a fixed, file-scope device array instead,
// so it allocates nothing and takes no workspace.
//
// The array lives in every GPU that loads the library until the process
// exits (SPTS_NOALLOC_MAX_NC int32 = 1 MiB).  In host code the symbol
// `g_prune_scratch` is only a host-side stand-in, not a device address, so
// the device address is looked up once per device with cudaGetSymbolAddress
// (with that device current) and cached.
//
// CUDA loads device code lazily by default: the module holding the array is
// loaded on that first address lookup, and each kernel on its first launch
// or attribute query, and both take device memory.  A call with Nc == 0 is
// the set-up form: it does the lookup and loads the two kernels the prune
// launches, then returns, so a caller that reserves the GPU's memory makes it
// once per device before the reservation.
#include <mutex>

#include "host.hpp"
#include "rowops.cuh"

namespace spts {
namespace {

static __device__ __align__(256) int32_t g_prune_scratch[SPTS_NOALLOC_MAX_NC];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int32_t *g_addr[kMaxDevices] = {};

spts_status scratch_address(int32_t **out) {
  int dev = 0;
  SPTS_CUDA_TRY(cudaGetDevice(&dev));
  SPTS_REQUIRE(dev >= 0 && dev < kMaxDevices, SPTS_ERR_UNSUPPORTED,
               "spts_stage_prune_noalloc: device ordinal %d beyond %d", dev, kMaxDevices);
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_addr[dev] == nullptr) {
    void *p = nullptr;
    SPTS_CUDA_TRY(cudaGetSymbolAddress(&p, g_prune_scratch));
    g_addr[dev] = static_cast<int32_t *>(p);
  }
  *out = g_addr[dev];
  return SPTS_OK;
}

}  // namespace
}  // namespace spts

using namespace spts;

extern "C" spts_status spts_stage_prune_noalloc(const float *scores, int64_t Nc, int64_t k_keep, int64_t force_tail,
                                                const float *h_in, const int32_t *pos_in, int D, float *h_out,
                                                int32_t *pos_out, int32_t *kept_idx, spts_stream stream) {
  const char *who = "spts_stage_prune_noalloc";
  if (Nc == 0) {  // set-up only: resolve the array on this device, load the kernels
    int32_t *p = nullptr;
    SPTS_TRY(scratch_address(&p));
    SPTS_TRY(preload_select_topk());
    return preload_gather_rows();
  }
  SPTS_REQUIRE(scores && h_in && pos_in && h_out && pos_out, SPTS_ERR_INVALID, "%s: NULL argument", who);
  SPTS_REQUIRE(Nc <= SPTS_NOALLOC_MAX_NC, SPTS_ERR_SHAPE,
               "%s: Nc = %lld exceeds the fixed scratch of %d candidates; use spts_stage_prune with a workspace",
               who, static_cast<long long>(Nc), SPTS_NOALLOC_MAX_NC);
  SPTS_REQUIRE(0 <= force_tail && force_tail <= k_keep && k_keep <= Nc && D > 0 && D % 4 == 0, SPTS_ERR_SHAPE,
               "%s: need 0 <= force_tail <= k_keep <= Nc and D %% 4 == 0", who);
  SPTS_REQUIRE(aligned(h_in, 16) && aligned(h_out, 16) && aligned(scores, 4) && aligned(pos_in, 4) &&
                   aligned(pos_out, 4) && (!kept_idx || aligned(kept_idx, 4)),
               SPTS_ERR_INVALID, "%s: misaligned pointer", who);
  const char *hi = reinterpret_cast<const char *>(h_in), *ho = reinterpret_cast<const char *>(h_out);
  const size_t hb = static_cast<size_t>(Nc) * D * 4, ob = static_cast<size_t>(k_keep) * D * 4;
  SPTS_REQUIRE(ho + ob <= hi || hi + hb <= ho, SPTS_ERR_INVALID, "%s: h_out overlaps h_in", who);
  if (k_keep == 0) return SPTS_OK;
  int32_t *kept = kept_idx;
  if (kept == nullptr) SPTS_TRY(scratch_address(&kept));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // The selection writes all k_keep indices before the gather reads them, so
  // nothing in the scratch has to start at zero.  No status word is kept:
  // device-side index checks report nothing in this variant.
  SPTS_TRY(launch_select_topk(scores, nullptr, SPTS_FUSE_NONE, 0.f, 0.f, Nc, k_keep, force_tail, kept, nullptr,
                              nullptr, nullptr, nullptr, s));  // no scratch: the single-CTA selection
  return launch_gather_rows(h_in, Nc, kept, k_keep, static_cast<int64_t>(D) * 4, h_out, pos_in, pos_out, nullptr, s);
}
