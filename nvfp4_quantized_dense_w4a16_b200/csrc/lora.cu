// LoRA adapters on the NVFP4 FFN ("metrale_model_layers/layers/
// dense_ffn_overlays.rs", set_lora_weights / apply_lora_gate_up /
// apply_lora_down): a projection's delta is (x A^T) B^T with A [r, in] and
// B [out, r] in bf16.  This file holds the adapter handle and the kernel of
// the first, rank-r product xa = bf16(x A^T); the second product and the add
// into the projection's output happen in the projection kernels' epilogues
// (lora_delta in common.cuh).
#include <new>

#include "common.cuh"
#include "ffn_nvfp4.h"
#include "internal.h"
#include "launch.cuh"
#include "profile.h"

struct ffn_lora {
  int64_t rank = 0, hidden = 0, inter = 0;
  int device = 0;
  // gate and up A stacked: rows [0, r) gate, [r, 2r) up (zero rows for an
  // absent adapter); down A [r, inter]; B matrices [out, r]
  uint16_t* a_gu = nullptr;
  uint16_t* a_d = nullptr;
  uint16_t* b_g = nullptr;
  uint16_t* b_u = nullptr;
  uint16_t* b_d = nullptr;
};

namespace ffn {
namespace {

constexpr int kXaRows = 8;     // activation rows per CTA (one warp each)
constexpr int kXaOuts = 32;    // rank-r outputs per pass (one accumulator each per lane)
constexpr int kXaKTile = 256;  // K elements staged per pass

// xa[j, i] = bf16(sum_k x[j, k] * A[i, k]) for i < R: each warp owns one row
// j; lane l accumulates K elements 8l..8l+7 of every 256-element tile for all
// outputs of the pass (A's tile staged in shared memory), then the warp sums
// the lanes in a fixed butterfly order.  K % 8 == 0.
__global__ void __launch_bounds__(kXaRows * 32) lora_xa_kernel(const uint16_t* __restrict__ x, int m,
                                                               int64_t K, const uint16_t* __restrict__ A,
                                                               int R, uint16_t* __restrict__ xa) {
  // the next kernel may launch now: it waits for this one before reading
  // its results; x may come from the previous kernel
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ __align__(16) uint16_t As[kXaOuts][kXaKTile];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x * kXaRows + warp;
  for (int i0 = 0; i0 < R; i0 += kXaOuts) {
    const int nout = min(kXaOuts, R - i0);
    float acc[kXaOuts];
#pragma unroll
    for (int i = 0; i < kXaOuts; ++i) acc[i] = 0.0f;
    for (int64_t k0 = 0; k0 < K; k0 += kXaKTile) {
      const int kt = (int)min((int64_t)kXaKTile, K - k0);
      __syncthreads();
      for (int idx = threadIdx.x; idx < nout * (kXaKTile / 8); idx += blockDim.x) {
        const int i = idx / (kXaKTile / 8), c = idx % (kXaKTile / 8);
        uint4 v = make_uint4(0, 0, 0, 0);
        if (8 * c < kt) v = *reinterpret_cast<const uint4*>(A + (size_t)(i0 + i) * K + k0 + 8 * c);
        *reinterpret_cast<uint4*>(&As[i][8 * c]) = v;
      }
      __syncthreads();
      if (j < m && 8 * lane < kt) {
        const uint4 xv = *reinterpret_cast<const uint4*>(x + (size_t)j * K + k0 + 8 * lane);
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
        float xf[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          xf[2 * e] = bf16_bits_to_float(xw[e] & 0xffffu);
          xf[2 * e + 1] = bf16_bits_to_float(xw[e] >> 16);
        }
#pragma unroll
        for (int i = 0; i < kXaOuts; ++i) {
          if (i < nout) {
            const uint4 av = *reinterpret_cast<const uint4*>(&As[i][8 * lane]);
            const uint32_t aw[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              acc[i] = fmaf(xf[2 * e], bf16_bits_to_float(aw[e] & 0xffffu), acc[i]);
              acc[i] = fmaf(xf[2 * e + 1], bf16_bits_to_float(aw[e] >> 16), acc[i]);
            }
          }
        }
      }
    }
#pragma unroll
    for (int i = 0; i < kXaOuts; ++i) acc[i] = warp_sum(acc[i]);
    if (j < m && lane == 0)
#pragma unroll
      for (int i = 0; i < kXaOuts; ++i)
        if (i < nout) xa[(size_t)j * R + i0 + i] = f32_to_bf16_bits(acc[i]);
  }
}

}  // namespace

cudaError_t launch_lora_xa(const void* x, int64_t m, int64_t k, const uint16_t* a, int rows, void* xa,
                           cudaStream_t s) {
  ProfScope prof(s, "lora_xa");
  return launch_pdl(lora_xa_kernel, dim3((unsigned)((m + kXaRows - 1) / kXaRows)), dim3(kXaRows * 32), 0, s,
                    static_cast<const uint16_t*>(x), (int)m, k, a, rows, static_cast<uint16_t*>(xa));
}

bool lora_dims_mismatch(const ffn_lora* l, int64_t hidden, int64_t inter) {
  return l->hidden != hidden || l->inter != inter;
}

LoraView lora_view(const ffn_lora* l) {
  LoraView v;
  if (!l) return v;
  v.rank = (int)l->rank;
  v.a_gu = l->a_gu;
  v.a_d = l->a_d;
  v.b_g = l->b_g;
  v.b_u = l->b_u;
  v.b_d = l->b_d;
  v.device = l->device;
  return v;
}

}  // namespace ffn

namespace {

void free_lora(ffn_lora* l) {
  if (!l) return;
  cudaFree(l->a_gu);
  cudaFree(l->a_d);
  cudaFree(l->b_g);
  cudaFree(l->b_u);
  cudaFree(l->b_d);
  delete l;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" {

ffn_status ffn_nvfp4_lora_create(int64_t rank, int64_t hidden, int64_t inter, const void* gate_a,
                                 const void* gate_b, const void* up_a, const void* up_b,
                                 const void* down_a, const void* down_b, void* stream,
                                 ffn_lora** out) {
  if (!out) return FFN_ERR_INVALID_ARG;
  *out = nullptr;
  if (rank < 1 || rank > FFN_LORA_MAX_RANK) return FFN_ERR_UNSUPPORTED;
  if (hidden <= 0 || inter <= 0 || hidden % 32 || inter % 32) return FFN_ERR_SHAPE;
  if (!gate_a != !gate_b || !up_a != !up_b || !down_a != !down_b) return FFN_ERR_INVALID_ARG;
  if (!gate_a && !up_a && !down_a) return FFN_ERR_INVALID_ARG;
  for (const void* p : {gate_a, gate_b, up_a, up_b, down_a, down_b})
    if (p && !aligned16(p)) return FFN_ERR_ALIGNMENT;
  if (cudaPeekAtLastError() != cudaSuccess) {
    cudaGetLastError();
    return FFN_ERR_CUDA;
  }
  auto* l = new (std::nothrow) ffn_lora;
  if (!l) return FFN_ERR_OOM;
  l->rank = rank;
  l->hidden = hidden;
  l->inter = inter;
  cudaGetDevice(&l->device);
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t r = (size_t)rank;
  auto get = [&](uint16_t** p, size_t elems) {
    if (cudaMalloc(reinterpret_cast<void**>(p), elems * 2) != cudaSuccess) {
      cudaGetLastError();
      *p = nullptr;
      return false;
    }
    return true;
  };
  cudaError_t e = cudaSuccess;
  bool ok = true;
  if (gate_a || up_a) {
    ok = get(&l->a_gu, 2 * r * hidden);
    if (ok) e = cudaMemsetAsync(l->a_gu, 0, 2 * r * hidden * 2, s);
    if (ok && e == cudaSuccess && gate_a)
      e = cudaMemcpyAsync(l->a_gu, gate_a, r * hidden * 2, cudaMemcpyDeviceToDevice, s);
    if (ok && e == cudaSuccess && up_a)
      e = cudaMemcpyAsync(l->a_gu + r * hidden, up_a, r * hidden * 2, cudaMemcpyDeviceToDevice, s);
  }
  if (ok && e == cudaSuccess && gate_b) {
    ok = get(&l->b_g, (size_t)inter * r);
    if (ok) e = cudaMemcpyAsync(l->b_g, gate_b, (size_t)inter * r * 2, cudaMemcpyDeviceToDevice, s);
  }
  if (ok && e == cudaSuccess && up_b) {
    ok = get(&l->b_u, (size_t)inter * r);
    if (ok) e = cudaMemcpyAsync(l->b_u, up_b, (size_t)inter * r * 2, cudaMemcpyDeviceToDevice, s);
  }
  if (ok && e == cudaSuccess && down_a) {
    ok = get(&l->a_d, r * inter) && get(&l->b_d, (size_t)hidden * r);
    if (ok) e = cudaMemcpyAsync(l->a_d, down_a, r * inter * 2, cudaMemcpyDeviceToDevice, s);
    if (ok && e == cudaSuccess)
      e = cudaMemcpyAsync(l->b_d, down_b, (size_t)hidden * r * 2, cudaMemcpyDeviceToDevice, s);
  }
  if (!ok) {
    free_lora(l);
    return FFN_ERR_OOM;
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    free_lora(l);
    return FFN_ERR_CUDA;
  }
  *out = l;
  return FFN_OK;
}

ffn_status ffn_nvfp4_lora_destroy(ffn_lora* l) {
  if (!l) return FFN_OK;
  const cudaError_t e = cudaDeviceSynchronize();
  free_lora(l);
  return e == cudaSuccess ? FFN_OK : FFN_ERR_CUDA;
}

}  // extern "C"
