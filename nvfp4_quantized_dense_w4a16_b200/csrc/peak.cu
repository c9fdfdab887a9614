// Dense tensor-core throughput probe for the two MMA kinds the library
// issues: kind::f16 (bf16 x bf16, fp32 accumulate; the W4A16 kernels) and
// kind::mxf4nvf4 with UE4M3 scales per 16 elements (E2M1 x E2M1; the
// fixed-format kernels).  It gives the roofline denominator of the FP4
// kernels, which a library GEMM cannot: no library on this machine exposes
// the block-scaled FP4 MMA.
//
// One CTA per SM.  NT threads each issue `iters` MMAs back to back into their
// own fp32 accumulator in TMEM, with both operands in shared memory (filled
// with finite values; the probe measures issue and math rate, not data
// movement), then commit and wait (bounded) for completion.
#include <stdint.h>

#include "ffn_nvfp4.h"
#include "sm100.cuh"

namespace ffn {
namespace {

using namespace sm100;

constexpr int kProbeThreads = 128;

// Operand tile bytes: A = 128 rows x 32 B, B = N rows x 32 B (one MMA's K:
// 16 bf16 or 64 E2M1), no-swizzle K-major: the second 16-byte K half of all
// rows follows the first (LBO), 8-row groups are 128 B apart (SBO).
template <int KIND>
struct ProbeCfg {
  static constexpr int N = KIND == 0 ? 256 : 128;
  static constexpr int kABytes = 128 * 32;
  static constexpr int kBBytes = N * 32;
  static constexpr int kSfBytes = 512;   // one 32-row x 16-byte scale block
  static constexpr int kSmem = kABytes + kBBytes + 2 * kSfBytes + 64;
  // requested (mostly unused) so that only one CTA fits per SM
  static constexpr int kSmemLaunch = 160 * 1024;
  static constexpr uint64_t kFlops = 2ull * 128 * N * (KIND == 0 ? 16 : 64);
};

template <int KIND, int NT>
__global__ void __launch_bounds__(kProbeThreads, 1) mma_probe_kernel(int iters, int* err) {
  using C = ProbeCfg<KIND>;
  static_assert(NT * C::N + (KIND == 1 ? 8 : 0) <= 512, "TMEM budget");
  static_assert(C::kSmem + 1024 <= C::kSmemLaunch, "shared memory");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint8_t* A = sm;
  uint8_t* B = sm + C::kABytes;
  uint8_t* SF = B + C::kBBytes;
  uint64_t* done = reinterpret_cast<uint64_t*>(SF + 2 * C::kSfBytes);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + NT);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // finite operand values: bf16 0x3C00..0x3CFF (about 0.0078..0.0087), E2M1
  // codes of any pattern, scale bytes 0x38 (1.0)
  for (int i = threadIdx.x; i < (C::kABytes + C::kBBytes) / 4; i += blockDim.x) {
    const uint32_t h = (uint32_t)i * 2654435761u;
    reinterpret_cast<uint32_t*>(A)[i] =
        KIND == 0 ? (0x3C003C00u | (h & 0x00FF00FFu)) : (h & 0x77777777u);
  }
  for (int i = threadIdx.x; i < 2 * C::kSfBytes / 4; i += blockDim.x)
    reinterpret_cast<uint32_t*>(SF)[i] = 0x38383838u;
  if (threadIdx.x == 0) {
    for (int j = 0; j < NT; ++j) mbar_init(&done[j], 1);
    fence_mbar_init();
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // generic writes -> MMA reads
  if (warp == 0) {
    tmem_alloc(tslot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t sf_col = NT * C::N;  // SFA at sf_col, SFB at sf_col + 4

  if (KIND == 1 && warp == 1 && lane == 0) {
    tmem_cp_32x128b_x4(tmem + sf_col, smem_desc_interleave(smem_u32(SF), 16, 128));
    tmem_cp_32x128b_x4(tmem + sf_col + 4, smem_desc_interleave(smem_u32(SF + C::kSfBytes), 16, 128));
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp < NT && lane == 0) {
    const uint32_t d = tmem + warp * C::N;
    const uint64_t ad = smem_desc_interleave(smem_u32(A), C::kABytes / 2, 128);
    const uint64_t bd = smem_desc_interleave(smem_u32(B), C::kBBytes / 2, 128);
    if (KIND == 0) {
      const uint32_t id = idesc_bf16_f32(128, C::N);
      for (int i = 0; i < iters; ++i) {
        // A from shared memory: the ss form of kind::f16
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
            "l"(ad), "l"(bd), "r"(id), "r"(i > 0 ? 1u : 0u)
            : "memory");
      }
    } else {
      const uint32_t id = idesc_mxf4nvf4(128, C::N);
      for (int i = 0; i < iters; ++i)
        mma_mxf4nvf4(d, ad, bd, id, tmem + sf_col, tmem + sf_col + 4, i > 0 ? 1u : 0u);
    }
    mma_commit(&done[warp]);
    const long long t0 = clock64();
    while (!mbar_try_wait(&done[warp], 0)) {
      if (clock64() - t0 > kWaitLimitCycles) {
        atomicOr(err, 1);
        break;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int KIND, int NT>
cudaError_t run_probe(int sms, int iters, int* err, cudaStream_t s, float* ms) {
  cudaEvent_t e0, e1;
  cudaError_t e = cudaEventCreate(&e0);
  if (e != cudaSuccess) return e;
  e = cudaEventCreate(&e1);
  if (e != cudaSuccess) {
    cudaEventDestroy(e0);
    return e;
  }
  const int smem = ProbeCfg<KIND>::kSmemLaunch;
  e = cudaFuncSetAttribute(mma_probe_kernel<KIND, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) {
    cudaEventDestroy(e0);
    cudaEventDestroy(e1);
    return e;
  }
  mma_probe_kernel<KIND, NT><<<sms, kProbeThreads, smem, s>>>(iters / 8 > 0 ? iters / 8 : 1, err);  // warm-up
  cudaEventRecord(e0, s);
  mma_probe_kernel<KIND, NT><<<sms, kProbeThreads, smem, s>>>(iters, err);
  cudaEventRecord(e1, s);
  e = cudaGetLastError();
  if (e == cudaSuccess) e = cudaEventSynchronize(e1);
  if (e == cudaSuccess) e = cudaEventElapsedTime(ms, e0, e1);
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  return e;
}

}  // namespace
}  // namespace ffn

extern "C" ffn_status ffn_nvfp4_tensor_peak(int kind, int issuers, int iters, double* tflops) {
  if (!tflops || (kind != 0 && kind != 1) || (issuers != 1 && issuers != 2) || iters < 1 ||
      iters > (1 << 24))
    return FFN_ERR_INVALID_ARG;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return FFN_ERR_CUDA;
  }
  int* err = nullptr;
  if (cudaMalloc(&err, sizeof(int)) != cudaSuccess) {
    cudaGetLastError();
    return FFN_ERR_OOM;
  }
  cudaStream_t s = nullptr;
  cudaError_t e = cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaMemsetAsync(err, 0, sizeof(int), s);
  float ms = 0.0f;
  uint64_t flops = 0;
  if (e == cudaSuccess) {
    if (kind == 0) {
      flops = ffn::ProbeCfg<0>::kFlops;
      e = issuers == 1 ? ffn::run_probe<0, 1>(sms, iters, err, s, &ms)
                       : ffn::run_probe<0, 2>(sms, iters, err, s, &ms);
    } else {
      flops = ffn::ProbeCfg<1>::kFlops;
      e = issuers == 1 ? ffn::run_probe<1, 1>(sms, iters, err, s, &ms)
                       : ffn::run_probe<1, 2>(sms, iters, err, s, &ms);
    }
  }
  int flag = 0;
  if (e == cudaSuccess) e = cudaMemcpy(&flag, err, sizeof(int), cudaMemcpyDeviceToHost);
  if (s) cudaStreamDestroy(s);
  cudaFree(err);
  if (e != cudaSuccess || flag != 0 || ms <= 0.0f) {
    cudaGetLastError();
    return FFN_ERR_CUDA;
  }
  *tflops = (double)flops * sms * issuers * iters / (ms * 1e-3) / 1e12;
  return FFN_OK;
}
