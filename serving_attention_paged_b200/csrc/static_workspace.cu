// pa_run_static_workspace: the decode run stage for callers that cannot
// allocate device memory.
//
// Some callers have no way to obtain device memory for the workspace: a
// serving engine whose memory pool has already claimed every free byte of
// the GPU for its KV cache, a C host program embedded in a process whose
// allocator it does not own, or a latency-critical path that must not pay
// the implicit device synchronisation of cudaMalloc / cudaFree.  For them the
// workspace lives in a fixed array compiled into this library.
//
// The array is kStaticWorkspaceBytes on every GPU that loads the library and
// stays allocated until the process exits.  Its device address is looked up
// with cudaGetSymbolAddress on the first call made on each device (with that
// device current).  The address is cached per device for the life of the process: a
// cudaDeviceReset (or anything else that destroys the device's primary
// context) invalidates it, and the entry point must not be used on that
// device afterwards.  Every call shares the one array and leaves its contents
// behind; each call re-uploads the work list and re-zeroes the arrival
// counters and status words, so calls that run one after another are
// independent, but two calls whose work overlaps on the GPU (other streams,
// other threads) race.  pa_static_workspace_check reads the status words a
// call left there (a bad page index under PA_FLAG_CHECK_INDICES, an abandoned
// bounded wait) before the next call clears them.
#include <cuda_runtime.h>

#include <mutex>

#include "pa_internal.h"

namespace {

constexpr size_t kStaticWorkspaceBytes = size_t(8) << 20;  // 8 MiB per GPU

// In host code this name is only a stand-in for the symbol: the device
// address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_static_workspace[kStaticWorkspaceBytes];

constexpr int kMaxDevices = 64;
std::mutex g_lock;
void* g_address[kMaxDevices] = {};

pa_status static_workspace_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PA_ERR_CUDA;
  std::lock_guard<std::mutex> guard(g_lock);
  if (!g_address[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess || !p) return PA_ERR_CUDA;
    g_address[dev] = p;
  }
  *out = g_address[dev];
  return PA_OK;
}

}  // namespace

extern "C" pa_status pa_run_static_workspace(pa_plan_t plan, const void* q, const void* k_pool,
                                             const void* v_pool, const int32_t* d_kv_indices,
                                             void* o, float* lse, void* stream) {
  if (!plan || plan->cascade || plan->prefill) return PA_ERR_INVALID_ARG;
  if (plan->ws.total > kStaticWorkspaceBytes) return PA_ERR_WORKSPACE_TOO_SMALL;
  void* ws = nullptr;
  pa_status st = static_workspace_address(&ws);
  if (st != PA_OK) return st;
  st = pa_plan_upload(plan, ws, kStaticWorkspaceBytes, stream);
  if (st != PA_OK) return st;
  return pa_run(plan, q, k_pool, v_pool, d_kv_indices, o, lse, ws, kStaticWorkspaceBytes, stream);
}

extern "C" pa_status pa_static_workspace_check(pa_plan_t plan, int64_t* bad_position,
                                               void* stream) {
  if (!plan || plan->cascade || plan->prefill) return PA_ERR_INVALID_ARG;
  if (plan->ws.total > kStaticWorkspaceBytes) return PA_ERR_WORKSPACE_TOO_SMALL;
  void* ws = nullptr;
  const pa_status st = static_workspace_address(&ws);
  if (st != PA_OK) return st;
  return pa_plan_check(plan, ws, bad_position, stream);
}
