// gsg_noalloc.cu -- gsg_moe_route_permute_noalloc: the routing permutation for callers that
// cannot allocate device memory.
//
// Who needs it: code that may not call cudaMalloc (or any allocating library routine) at the
// point where it routes tokens -- a host loop whose device memory is owned and fully carved up
// by another component (a serving engine's pre-sized pool, a framework that forbids allocation
// after start-up), or code running in a process that must never grow its device footprint
// after initialisation.  gsg_moe_route_permute needs a caller-supplied workspace once
// R = T*k exceeds one routing chunk; this variant takes the same inputs and outputs but keeps
// that workspace in a fixed array that the library holds for the lifetime of the process.
//
// The scratch: g_route_scratch below, kNoAllocScratchBytes = 256 KiB, file-scope device memory.
// Every GPU that loads the library holds it until the process exits.  In host code the name
// g_route_scratch is a host-side stand-in for the device variable, not a device address: the
// device address comes from cudaGetSymbolAddress, taken once per device (with that device
// current) by the entry point's first call on that device.
//
// Limits: R <= 2048 uses no scratch.  Above that the routing needs the workspace that
// gsg_workspace_size(GSG_OP_ROUTE, ...) reports: at most 128 KiB while it cuts R into 1024-row
// chunks, else 2 * ceil(R / 8192) * E int32.  So a call is accepted when ceil(R / 8192) * E <=
// 32768 (E = 384: R up to 696,320 rows; E = 128: R up to 2,097,152); larger requests return
// GSG_ERR_UNSUPPORTED_SHAPE before anything is launched.
//
// Sharing: every call on a device uses the same array, which keeps the last call's contents.
// Nothing in it has to start at zero: the histogram launch writes every [chunk][expert] count
// and the scan launch every base before any launch reads them.  Calls whose launches overlap
// on the GPU (different streams without ordering between them) race on the array.
#include <mutex>

#include "gsg_internal.cuh"
#include "gsg_launch.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 256 * 1024;
constexpr int kNoAllocMaxDevices = 64;

static __device__ __align__(256) int32_t g_route_scratch[kNoAllocScratchBytes / sizeof(int32_t)];

std::mutex g_noalloc_mu;
void* g_scratch_ptr[kNoAllocMaxDevices] = {};

// Once per device, with that device current: the scratch's device address.
gsg_status_t scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices) return GSG_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress((void**)&ptr, g_route_scratch) != cudaSuccess || ptr == nullptr) return GSG_ERR_CUDA;
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return GSG_OK;
}

}  // namespace

extern "C" gsg_status_t gsg_moe_route_permute_noalloc(const int32_t* topk_ids, int T, int k, int E,
                                                      int32_t* expert_offsets, int32_t* perm_src,
                                                      int32_t* inv_perm, void* stream) {
  if (T < 0 || k < 1) return GSG_ERR_INVALID_ARG;
  if (!gsg::route_supported(E)) return GSG_ERR_UNSUPPORTED_SHAPE;
  if ((long long)T * k > (1ll << 30)) return GSG_ERR_UNSUPPORTED_SHAPE;
  if (!expert_offsets) return GSG_ERR_INVALID_ARG;
  const int R = T * k;
  if (T > 0 && (!topk_ids || !perm_src || !inv_perm)) return GSG_ERR_INVALID_ARG;
  if (gsg::route_workspace_bytes(R, E) > kNoAllocScratchBytes) return GSG_ERR_UNSUPPORTED_SHAPE;
  int* status = nullptr;
  int num_sms = 0;
  gsg_status_t st = gsg::device_setup(&status, &num_sms);
  if (st != GSG_OK) return st;
  void* scratch = nullptr;
  st = scratch_for_current_device(&scratch);
  if (st != GSG_OK) return st;
  const cudaError_t err = gsg::launch_route(topk_ids, R, E, expert_offsets, perm_src, inv_perm, scratch, status,
                                            reinterpret_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? GSG_OK : GSG_ERR_CUDA;
}
