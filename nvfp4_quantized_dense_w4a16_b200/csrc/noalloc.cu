// ffn_nvfp4_linear_noalloc: the bf16 (W4A16) tensor-core projection for
// callers that cannot allocate device memory on the call path -- for example
// a plugin whose host framework owns every device allocation and hands it no
// workspace, or latency-critical serving code that must not call cudaMalloc
// (which can synchronise the whole device) once it is running.  The split-K
// partial sums that ffn_nvfp4_linear keeps in the caller's workspace live
// here in one fixed device array instead.
#include <mutex>

#include "ffn_nvfp4.h"
#include "internal.h"

namespace {

// The fixed scratch: 16 MiB of device memory on every GPU that loads the
// library, held until the process exits.  Shared by all calls.
constexpr size_t kNoAllocScratchBytes = 16u << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array for the current device, looked up once
// per device with that device current.  (In host code the array's name is
// only a host-side stand-in, never a device address.)
cudaError_t scratch_for_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
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
  if (gate_up) return FFN_ERR_UNSUPPORTED;
  if (m == 0) return FFN_OK;
  if (!x || !y) return FFN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(y) & 15u))
    return FFN_ERR_ALIGNMENT;
  const ffn::TcPlan plan = ffn::plan_tc(m, tw.n, tw.k, false, sm_count());
  if (plan.partial_bytes > kNoAllocScratchBytes) return FFN_ERR_WORKSPACE;
  if (cudaPeekAtLastError() != cudaSuccess) {
    cudaGetLastError();
    return FFN_ERR_CUDA;
  }
  void* scratch = nullptr;
  if (scratch_for_current_device(&scratch) != cudaSuccess) {
    cudaGetLastError();
    return FFN_ERR_CUDA;
  }
  const cudaError_t e = ffn::launch_tc_w4a16(x, m, tw, false, plan, y, scratch,
                                             reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FFN_OK : FFN_ERR_CUDA;
}
