// ffn_nvfp4_linear_noalloc: the bf16 (W4A16) tensor-core projection for
// callers that cannot allocate device memory on the call path -- for example
// a plugin whose host framework owns every device allocation and hands it no
// workspace, or latency-critical serving code that must not call cudaMalloc
// (which can synchronise the whole device) once it is running.  The split-K
// partial sums that ffn_nvfp4_linear keeps in the caller's workspace live
// here in one fixed device array instead.
#include <cuda.h>

#include <mutex>

#include "ffn_nvfp4.h"
#include "internal.h"

namespace {

// The fixed scratch: 16 MiB of device memory on every GPU whose context loads
// this module, held until the process exits.  Shared by all calls.
constexpr size_t kNoAllocScratchBytes = 16u << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device addresses of the scratch array, one per CUDA context.  The array
// lives in the module loaded into a context, so its address belongs to that
// context: after a device reset (or a primary context torn down and made
// again) the array is reloaded, possibly elsewhere.  The cache is keyed on the
// context's unique ID (never reused within a process, unlike the device
// ordinal or the context handle), so a stale address never reaches a kernel.
constexpr int kMaxContexts = 64;
struct ScratchEntry {
  unsigned long long ctx_id;
  void* addr;
};
std::mutex g_setup_mutex;
ScratchEntry g_scratch[kMaxContexts] = {};
int g_scratch_used = 0;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <class Fn>
Fn driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    return reinterpret_cast<Fn>(p);
  return nullptr;
}

// Unique ID of the calling thread's current context (false if none).
bool current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_cur = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    get_cur = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
    get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  });
  CUcontext ctx = nullptr;
  return get_cur && get_id && get_cur(&ctx) == CUDA_SUCCESS && ctx &&
         get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of the scratch array in the current context, looked up once
// per context with that context current.  (In host code the array's name is
// only a host-side stand-in, never a device address.)  With lazy module
// loading the first lookup in a context loads the module and so reserves the
// 16 MiB there: it can fail with cudaErrorMemoryAllocation.
cudaError_t scratch_for_current_context(void** out) {
  unsigned long long id = 0;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  const bool have_ctx = current_context_id(&id);
  if (have_ctx)
    for (int i = 0; i < g_scratch_used; ++i)
      if (g_scratch[i].ctx_id == id) {
        *out = g_scratch[i].addr;
        return cudaSuccess;
      }
  // First call in this context (the lookup also makes the device's primary
  // context current on this thread if no context was).
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess) return e;
  if ((have_ctx || current_context_id(&id)) && g_scratch_used < kMaxContexts)
    g_scratch[g_scratch_used++] = ScratchEntry{id, p};
  *out = p;
  return cudaSuccess;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return 148;
  }
  return n;
}

}  // namespace

extern "C" ffn_status ffn_nvfp4_linear_noalloc(const void* x, int64_t m,
                                               const ffn_nvfp4_weight* w, void* y,
                                               void* stream) {
  if (m < 0 || !w) return FFN_ERR_INVALID_ARG;
  ffn::TcWeight tw;
  bool gate_up = false;
  ffn::handle_tc_view(w, &tw, &gate_up);
  if (gate_up || !tw.tiled16) return FFN_ERR_UNSUPPORTED;
  if (m == 0) return FFN_OK;
  if (!x || !y) return FFN_ERR_INVALID_ARG;
  if (ffn_status st = ffn::handle_check_device(w)) return st;
  if ((reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(y) & 15u))
    return FFN_ERR_ALIGNMENT;
  const ffn::TcPlan plan = ffn::plan_tc(m, tw.n, tw.k, false, sm_count());
  if (plan.partial_bytes > kNoAllocScratchBytes) return FFN_ERR_WORKSPACE;
  if (cudaPeekAtLastError() != cudaSuccess) {
    cudaGetLastError();
    return FFN_ERR_CUDA;
  }
  void* scratch = nullptr;
  const cudaError_t se = scratch_for_current_context(&scratch);
  if (se != cudaSuccess) {
    cudaGetLastError();
    return se == cudaErrorMemoryAllocation ? FFN_ERR_OOM : FFN_ERR_CUDA;
  }
  const cudaError_t e = ffn::launch_tc_w4a16(x, m, tw, false, plan, y, scratch,
                                             reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FFN_OK : FFN_ERR_CUDA;
}
