// sla_route_noalloc: the routing entry point for callers that cannot hand the
// library a device workspace. Its scratch (status word, pooled means, pooled
// scores) lives in one file-scope device array instead of caller memory.
#include <string.h>

#include <mutex>

#include <cuda.h>  // CUcontext (type only; the driver is reached through the runtime)

#include "sla_internal.h"

namespace sla {

// Held by every GPU that loads the library, until the process exits.
static __device__ __align__(256) unsigned char g_route_scratch[SLA_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};  // id of the context the address belongs to

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

}  // namespace

// Process-unique id of the current CUDA context (0 if it cannot be read). A device
// reset ends the primary context; the next one has another id, and the array then
// has another device address.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_cur = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static bool looked_up = false;
  if (!looked_up) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = (CtxGetCurrentFn)p;
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = (CtxGetIdFn)p;
    looked_up = true;
  }
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_cur && get_id && get_cur(&ctx) == CUDA_SUCCESS && ctx && get_id(ctx, &id) == CUDA_SUCCESS) return id;
  return 0;
}

namespace {

// Device address of g_route_scratch on the current device. The host-side name
// of the array is only a stand-in, so the address is looked up (with that device
// current) once per device and context, and cached.
cudaError_t scratch_for_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mutex);
  void* p = g_scratch_ptr[dev];
  const unsigned long long ctx = p != nullptr ? current_context_id() : 0;
  if (p == nullptr || ctx == 0 || ctx != g_scratch_ctx[dev]) {
    p = nullptr;
    e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = current_context_id();
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace sla

using namespace sla;

static bool aligned_to(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

extern "C" SLA_API sla_status sla_route_noalloc(const void* q, const void* k, const sla_config* cfg,
                                                int8_t* mask_out, int32_t* crit_idx,
                                                int32_t* neg_idx, void* stream) {
  const sla_status st = sla_validate_config(cfg);
  if (st != SLA_OK) return st;
  Plan p;
  make_plan(cfg, &p);
  if (!q || !k || !aligned_to(q, 16) || !aligned_to(k, 16)) return SLA_ERR_INVALID_ARG;
  const bool threeway = cfg->mode == SLA_MODE_THREEWAY;
  const int n_crit = threeway ? cfg->k_h : cfg->top_n;
  if (n_crit > 0 && (!crit_idx || !aligned_to(crit_idx, 4))) return SLA_ERR_INVALID_ARG;
  if (threeway && cfg->k_l > 0 && (!neg_idx || !aligned_to(neg_idx, 4))) return SLA_ERR_INVALID_ARG;
  // routing uses the status word, the pooled means and the pooled scores, which
  // the plan places before every other region
  if (p.off_crit > (size_t)SLA_NOALLOC_SCRATCH_BYTES) return SLA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (scratch_for_current_device(&scratch) != cudaSuccess) return SLA_ERR_CUDA;
  Args a;
  memset(&a, 0, sizeof(a));
  a.q = (const __nv_bfloat16*)q;
  a.k = (const __nv_bfloat16*)k;
  a.mask_out = mask_out;
  a.crit = n_crit > 0 ? crit_idx : nullptr;
  a.neg = threeway && cfg->k_l > 0 ? neg_idx : nullptr;
  a.ws = (char*)scratch;
  a.status = (int*)((char*)scratch + p.off_status);
  cudaStream_t s = (cudaStream_t)stream;
  // the array keeps the previous call's contents: the status word must start at zero
  if (cudaMemsetAsync(a.status, 0, 8, s) != cudaSuccess) return SLA_ERR_CUDA;
  return route_stages(p, a, s) == cudaSuccess ? SLA_OK : SLA_ERR_CUDA;
}

extern "C" SLA_API sla_status sla_route_noalloc_status(void* stream, int32_t* detail) {
  void* scratch = nullptr;
  if (scratch_for_current_device(&scratch) != cudaSuccess) return SLA_ERR_CUDA;
  // the status word is the first region of the routing plan (offset 0)
  return sla_check_device_status(scratch, stream, detail);
}
