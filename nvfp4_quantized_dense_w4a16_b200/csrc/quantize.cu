// NVFP4 quantisers: weights (with a per-tensor fp32 scale) and per-row
// activations for the fixed W4A4 format.  Every integer decision (block scale
// byte, element code) is taken in fp32 with IEEE round-to-nearest-even
// division and multiplication, so the result is bit-reproducible.
//
// The weight conventions are this library's (the source pages only name the
// quantiser): gs = amax / 2688, t = (block amax / gs) / 6, s = E4M3(t),
// sdec = E4M3value(s) * gs, code = E2M1(w / sdec).  Activations (fixed format,
// "metrale_model_layers/layers/dense_ffn_fixed.rs", nvfp4_proj_mx inputs):
// s = E4M3(block amax / 6), code = E2M1(x / E4M3value(s)).
#include "common.cuh"
#include "internal.h"
#include "launch.cuh"
#include "profile.h"

namespace ffn {

// Each thread owns one 16-element block: 32 bytes of bf16 in, 8 bytes of
// codes and one scale byte out; a warp touches 1 KB of contiguous input.
struct Block16 {
  float v[16];
  float amax;
};

__device__ __forceinline__ void load_block16(const uint16_t* src, Block16& b) {
  const uint4* p = reinterpret_cast<const uint4*>(src);
  const uint4 a = __ldg(p), c = __ldg(p + 1);
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
  b.amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    b.v[2 * i] = bf16_bits_to_float(w[i] & 0xffffu);
    b.v[2 * i + 1] = bf16_bits_to_float(w[i] >> 16);
    b.amax = fmaxf(b.amax, fmaxf(fabsf(b.v[2 * i]), fabsf(b.v[2 * i + 1])));
  }
}

// Encode a block whose decoded scale is sdec (0 => all codes 0).
__device__ __forceinline__ uint2 encode_block16(const Block16& b, float sdec, bool zero) {
  return e2m1_encode_block16(b.v, sdec, zero);
}

__global__ void amax_bf16_kernel(const uint16_t* __restrict__ w, int64_t count8,
                                 unsigned int* __restrict__ amax_bits) {
  // count8 = number of 8-element (16-byte) groups
  unsigned int best = 0;
  const uint4* p = reinterpret_cast<const uint4*>(w);
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < count8;
       i += (int64_t)gridDim.x * blockDim.x) {
    const uint4 a = __ldg(p + i);
    const uint32_t v[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      // |bf16| as fp32 bits: non-negative floats order like unsigned ints
      best = max(best, (v[j] & 0x7fffu) << 16);
      best = max(best, (v[j] >> 16 & 0x7fffu) << 16);
    }
  }
  best = __reduce_max_sync(0xffffffffu, best);
  if ((threadIdx.x & 31) == 0 && best) atomicMax(amax_bits, best);
}

__device__ __forceinline__ float tensor_scale_from_amax(float amax) {
  return amax == 0.0f ? 1.0f : __fdiv_rn(amax, 2688.0f);
}

__global__ void quantize_weight_blocks_kernel(const uint16_t* __restrict__ w, int64_t nblocks,
                                              const unsigned int* __restrict__ amax_bits,
                                              uint8_t* __restrict__ codes,
                                              uint8_t* __restrict__ scales) {
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= nblocks) return;
  const float gs = tensor_scale_from_amax(__uint_as_float(*amax_bits));
  Block16 b;
  load_block16(w + 16 * i, b);
  const float t = __fdiv_rn(__fdiv_rn(b.amax, gs), 6.0f);
  const uint32_t s8 = e4m3_encode_satfinite(t);
  const float sdec = __fmul_rn(e4m3_decode(s8), gs);
  const uint2 c = encode_block16(b, sdec, s8 == 0 || sdec == 0.0f);
  reinterpret_cast<uint2*>(codes)[i] = c;
  scales[i] = (uint8_t)s8;
}

__global__ void finalize_tensor_scale_kernel(float* gs_inout) {
  // the buffer held amax's bits during the two passes above
  const float amax = __uint_as_float(*reinterpret_cast<unsigned int*>(gs_inout));
  *gs_inout = tensor_scale_from_amax(amax);
}

__global__ void quantize_act_blocks_kernel(const uint16_t* __restrict__ x, int64_t nblocks,
                                           uint8_t* __restrict__ codes,
                                           uint8_t* __restrict__ scales) {
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= nblocks) return;
  Block16 b;
  load_block16(x + 16 * i, b);
  const uint32_t s8 = e4m3_encode_satfinite(__fdiv_rn(b.amax, 6.0f));
  const uint2 c = encode_block16(b, e4m3_decode(s8), s8 == 0);
  reinterpret_cast<uint2*>(codes)[i] = c;
  scales[i] = (uint8_t)s8;
}

// As above, with the scale byte of (row r, 16-block kb) stored at
// ((r / 128) * kc + kb / 4) * 512 + 16 * (r % 32) + 4 * ((r % 128) / 32) + kb % 4.
__global__ void quantize_act_blocked_kernel(const uint16_t* __restrict__ x, int64_t nblocks,
                                            int64_t kb_per_row, int kc,
                                            uint8_t* __restrict__ codes,
                                            uint8_t* __restrict__ sf_blocks) {
  // x comes from the previous kernel (with programmatic dependent launch)
  // the next kernel may launch now: it waits for this one before reading
  // its results
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= nblocks) return;
  Block16 b;
  load_block16(x + 16 * i, b);
  const uint32_t s8 = e4m3_encode_satfinite(__fdiv_rn(b.amax, 6.0f));
  const uint2 c = encode_block16(b, e4m3_decode(s8), s8 == 0);
  reinterpret_cast<uint2*>(codes)[i] = c;
  sf_blocks[sf_blocked_offset(i / kb_per_row, i % kb_per_row, kc)] = (uint8_t)s8;
}

cudaError_t launch_quantize_activations_blocked(const void* x, int64_t m, int64_t k, void* codes,
                                                void* sf_blocks, cudaStream_t s) {
  const int64_t nblocks = m * k / 16;
  if (nblocks == 0) return cudaSuccess;
  const int threads = 256;
  const int kc = (int)((k + 63) / 64);
  ProfScope prof(s, "quantize_activations");
  return launch_pdl(quantize_act_blocked_kernel, dim3((unsigned)((nblocks + threads - 1) / threads)),
                    dim3(threads), 0, s, (const uint16_t*)x, nblocks, (int64_t)(k / 16), kc,
                    (uint8_t*)codes, (uint8_t*)sf_blocks);
}

cudaError_t launch_quantize_weights(const void* w, int64_t n, int64_t k, void* codes,
                                    void* scales, float* gs, cudaStream_t s) {
  const int64_t count = n * k;
  cudaError_t e = cudaMemsetAsync(gs, 0, sizeof(float), s);
  if (e != cudaSuccess) return e;
  ProfScope prof(s, "quantize_weights");
  const int64_t count8 = count / 8;
  const int threads = 256;
  int grid = (int)((count8 + threads - 1) / threads);
  if (grid > 148 * 16) grid = 148 * 16;
  amax_bf16_kernel<<<grid, threads, 0, s>>>((const uint16_t*)w, count8, (unsigned int*)gs);
  const int64_t nblocks = count / 16;
  quantize_weight_blocks_kernel<<<(unsigned)((nblocks + threads - 1) / threads), threads, 0, s>>>(
      (const uint16_t*)w, nblocks, (const unsigned int*)gs, (uint8_t*)codes, (uint8_t*)scales);
  finalize_tensor_scale_kernel<<<1, 1, 0, s>>>(gs);
  return cudaGetLastError();
}

cudaError_t launch_quantize_activations(const void* x, int64_t m, int64_t k, void* codes,
                                        void* scales, cudaStream_t s) {
  const int64_t nblocks = m * k / 16;
  if (nblocks == 0) return cudaSuccess;
  const int threads = 256;
  ProfScope prof(s, "quantize_activations");
  quantize_act_blocks_kernel<<<(unsigned)((nblocks + threads - 1) / threads), threads, 0, s>>>(
      (const uint16_t*)x, nblocks, (uint8_t*)codes, (uint8_t*)scales);
  return cudaGetLastError();
}

}  // namespace ffn
