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
struct ScratchSlot {
  int32_t* ptr;
  unsigned long long ctx_id;  // the context the address belongs to
};
ScratchSlot g_scratch[kMaxDevices] = {};

// Unique id of the calling thread's current CUDA context (driver API through the runtime's entry
// point lookup, so the library links no extra library). False if there is none or the lookup fails.
bool current_context_id(unsigned long long* id) {
  typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
  typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  if (!get_current || !get_id) {
    void* a = nullptr;
    void* b = nullptr;
    cudaDriverEntryPointQueryResult qa, qb;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) != cudaSuccess ||
        qa != cudaDriverEntryPointSuccess ||
        cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) != cudaSuccess ||
        qb != cudaDriverEntryPointSuccess)
      return false;
    get_current = reinterpret_cast<CtxGetCurrentFn>(a);
    get_id = reinterpret_cast<CtxGetIdFn>(b);
  }
  CUcontext c = nullptr;
  if (get_current(&c) != CUDA_SUCCESS || !c) return false;
  return get_id(c, id) == CUDA_SUCCESS;
}

// Device address of the scratch array on the current device. In host code the array's name is only
// a host-side stand-in, so the address is looked up with the device current: once per device, and
// again whenever the device's context has been replaced (after cudaDeviceReset the module is loaded
// anew and the array may sit at another address).
int scratch_for_current_device(int32_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  unsigned long long ctx = 0;
  const bool have_ctx = current_context_id(&ctx);
  ScratchSlot& slot = g_scratch[dev];
  if (!slot.ptr || !have_ctx || slot.ctx_id != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
    // the lookup above makes the primary context current if none was
    if (!current_context_id(&ctx)) ctx = 0;
    slot.ptr = static_cast<int32_t*>(p);
    slot.ctx_id = ctx;
  }
  *out = slot.ptr;
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
  // entries with an expert id outside [0,E) still get perm = prow = -1 and no row.
  return moe::launch_metadata(idx, cfg->T, cfg->E, cfg->k, moe::group_align(cfg->dtype),
                              moe_max_rows(cfg), counts, offsets, poff, perm, prow, row_token, hist,
                              nullptr, reinterpret_cast<cudaStream_t>(stream));
}
