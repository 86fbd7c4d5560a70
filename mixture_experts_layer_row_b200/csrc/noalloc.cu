// Routing metadata without any caller-provided workspace.
//
// Some callers cannot allocate device memory: for example an inference-engine plugin that is handed
// only its input and output tensors under a fixed memory plan, or a host runtime that has no device
// allocator of its own. They cannot supply the workspace moe_route_metadata takes for its per-chunk
// histograms, so this entry point keeps that scratch in a file-scope device array instead. The array
// is part of the library image: every GPU that loads the library holds it until the process exits.
//
// The kernels are the same three that moe_route_metadata launches; only the histogram scratch
// differs. The histogram kernel writes every scratch entry before the scan reads it, so nothing in the
// array has to start at zero and nothing is cleared between calls.
#include <atomic>
#include <mutex>

#include "internal.h"

namespace moe {
namespace {

// Capacity of the static scratch: ceil(T/256) * E int32 entries (256 KB per GPU).
constexpr int64_t kNoAllocScratchInts = 65536;

static __device__ __align__(256) int32_t g_route_scratch[kNoAllocScratchInts];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
int32_t* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device. In host code the array's name is only
// a host-side stand-in, so the address is looked up once per device, with that device current.
int scratch_for_current_device(int32_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
    g_scratch_ptr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_scratch_ptr[dev];
  return MOE_OK;
}

}  // namespace
}  // namespace moe

extern "C" MOE_API int moe_route_metadata_noalloc(const moe_config_t* cfg, const int32_t* idx,
                                                  int32_t* counts, int32_t* offsets, int32_t* poff,
                                                  int32_t* perm, int32_t* prow, int32_t* row_token,
                                                  void* stream) {
  if (!cfg || !idx || !counts || !offsets || !poff || !perm || !prow || !row_token)
    return MOE_ERR_INVALID_ARG;
  if (moe_max_rows(cfg) <= 0) return MOE_ERR_INVALID_ARG;  // same config rules as every entry point
  const int64_t nchunks = ((int64_t)cfg->T + 255) / 256;
  if (nchunks * cfg->E > moe::kNoAllocScratchInts) return MOE_ERR_WORKSPACE;
  int32_t* hist = nullptr;
  const int rc = moe::scratch_for_current_device(&hist);
  if (rc != MOE_OK) return rc;
  // Device-side routing errors are not reported by this variant (there is no workspace flag);
  // invalid expert ids are still skipped by the kernels.
  return moe::launch_metadata(idx, cfg->T, cfg->E, cfg->k, moe::group_align(cfg->dtype),
                              moe_max_rows(cfg), counts, offsets, poff, perm, prow, row_token, hist,
                              nullptr, reinterpret_cast<cudaStream_t>(stream));
}
