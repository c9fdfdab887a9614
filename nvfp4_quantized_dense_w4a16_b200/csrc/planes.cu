// Activation planes for the few-row W4A16 path on the block-scaled FP4
// tensor core.
//
// The NVFP4 weights are multiplied by the tensor core's kind::mxf4nvf4 MMA
// as they are stored (E2M1 codes, one UE4M3 scale per 16 elements along K):
// no software dequantisation.  The bf16 activation row x is written as a sum
// of P NVFP4 "planes", x = sum_p g_p * (s_p,b * q_p,k) + r_P, each plane one
// extra MMA column: plane p quantises the residual left by planes 0..p-1 with
// a per-row power-of-two factor g_p (fp32, so that every plane's block scales
// sit in E4M3's range), a power-of-two block scale s = 2^ceil(log2(amax / 6 /
// g_p)) (exact in E4M3; the residual then divides exactly) and codes
// q = E2M1(r / (g_p * s)), then subtracts what it represents (exactly: the
// represented value has at most two significant bits and lies within a
// factor two of the residual).  Each plane takes the next one to three
// significant bits of the elements near its block's maximum, so P planes
// leave a residual below about 3^-P of each block's maximum (P = 8 or 16
// here); seeded N(0, 1) bf16 rows are represented exactly by 8 planes, and
// values on a coarse binary grid, such as small integers, by the first.  The epilogue adds the plane
// columns back with their factors (y = sum_p g_p * D_p).
#include "common.cuh"
#include "internal.h"
#include "launch.cuh"
#include "profile.h"

namespace ffn {
namespace {

constexpr int kPlaneThreads = 256;
constexpr int kMaxPerThread = 96;  // K <= 256 * 96 = 24576 elements per row

__device__ __forceinline__ float block_reduce_max(float v, float* red) {
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float m = 0.0f;
  for (int w = 0; w < kPlaneThreads / 32; ++w) m = fmaxf(m, red[w]);
  return m;
}

// One CTA per activation row j.  Thread t owns the 16-element blocks
// t, t + 256, ... of the row and keeps their residuals in registers.
// Outputs: codes [m * P][K/2] (row j * P + p), scale bytes in the blocked
// layout of the MMA's scale-factor copy (rows j * P + p), g [m][P] (fp32).
// After its griddep_wait the kernel also zeroes the counters of the
// projection that follows it (split-K tile counters), if given.
template <int P>
__global__ void __launch_bounds__(kPlaneThreads) quantize_planes_kernel(
    const uint16_t* __restrict__ x, int m, int K, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ sf_blocks, float* __restrict__ g, int* zero_ptr, int zero_count) {
  asm volatile("griddepcontrol.wait;" ::: "memory");  // x may come from the previous kernel
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ float red[kPlaneThreads / 32];
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < zero_count; i += gridDim.x * blockDim.x)
    zero_ptr[i] = 0;
  const int j = blockIdx.x;
  const int nb = K / 16;
  const int kc = (K + 63) / 64;
  constexpr int kBlocks = kMaxPerThread / 16;  // blocks per thread
  float r[kBlocks][16];
#pragma unroll
  for (int bi = 0; bi < kBlocks; ++bi) {
    const int b = threadIdx.x + bi * kPlaneThreads;
#pragma unroll
    for (int e = 0; e < 16; ++e) r[bi][e] = 0.0f;
    if (b < nb) {
      const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)j * K + 16 * b);
      const uint4 a = src[0], c = src[1];
      const uint32_t w[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        r[bi][2 * e] = bf16_bits_to_float(w[e] & 0xffffu);
        r[bi][2 * e + 1] = bf16_bits_to_float(w[e] >> 16);
      }
    }
  }
  for (int p = 0; p < P; ++p) {
    float local = 0.0f;
#pragma unroll
    for (int bi = 0; bi < kBlocks; ++bi)
#pragma unroll
      for (int e = 0; e < 16; ++e) local = fmaxf(local, fabsf(r[bi][e]));
    const float rowmax = block_reduce_max(local, red);
    // g_p = 2^(floor(log2 rowmax) - 8): the largest block scale is then
    // amax / 6 / g_p < 2^9 / 6 < 448, and blocks down to ~2^-14 of the row's
    // maximum still get a normal or subnormal E4M3 scale; smaller ones wait
    // for a later plane.  An all-zero residual gives g = 0 and zero planes.
    const float gp = rowmax > 0.0f ? exp2f((float)(ilogbf(rowmax) - 8)) : 0.0f;
    const int row = j * P + p;
    if (threadIdx.x == 0) g[j * P + p] = gp;
#pragma unroll
    for (int bi = 0; bi < kBlocks; ++bi) {
      const int b = threadIdx.x + bi * kPlaneThreads;
      if (b >= nb) continue;
      float amax = 0.0f;
#pragma unroll
      for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(r[bi][e]));
      uint32_t s8 = 0;
      float sdec = 0.0f;
      if (gp > 0.0f && amax > 0.0f) {
        // smallest power of two 2^e >= amax / 6 / g_p, e in [-9, 8] (E4M3's
        // powers of two: subnormal 2^-9..2^-7, normal 2^-6..2^8)
        const float t = __fdiv_rn(__fdiv_rn(amax, 6.0f), gp);
        int ex;
        const float fr = frexpf(t, &ex);  // t = fr * 2^ex, fr in [0.5, 1)
        int e = fr == 0.5f ? ex - 1 : ex;
        e = e < -9 ? -9 : (e > 8 ? 8 : e);
        s8 = e >= -6 ? (uint32_t)(e + 7) << 3 : (1u << (e + 9));
        sdec = ldexpf(gp, e);
      }
      const bool zero = s8 == 0;
      const uint2 c = e2m1_encode_block16(r[bi], zero ? 1.0f : sdec, zero);
      if (!zero) {
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const uint32_t nib = ((e < 8 ? c.x : c.y) >> (4 * (e & 7))) & 15u;
          const float v = (nib & 8u ? -1.0f : 1.0f) * e2m1_mag(nib & 7u);
          r[bi][e] -= v * sdec;  // v * sdec has at most 6 significant bits: exact
        }
      }
      *reinterpret_cast<uint2*>(codes + (size_t)row * (K / 2) + 8 * b) = c;
      sf_blocks[sf_blocked_offset(row, b, kc)] = (uint8_t)s8;
    }
  }
}

}  // namespace

// Planes per row: 8 represent bf16 rows of normal spread exactly (each plane
// takes the next two to three bits near its block maximum); one row gets 16,
// which fill the narrowest MMA (N = 16) at no extra cost.
int planes_for_rows(int64_t m) { return m == 1 ? 16 : m <= 8 ? 8 : 0; }

cudaError_t launch_quantize_planes(const void* x, int64_t m, int64_t k, int planes, void* codes, void* sf_blocks,
                                   float* g, int* zero_ptr, int zero_count, cudaStream_t s) {
  if (k > (int64_t)kPlaneThreads * kMaxPerThread || k % 16) return cudaErrorInvalidValue;
  ProfScope prof(s, "quantize_planes");
  const dim3 grid((unsigned)m), block(kPlaneThreads);
  const auto* xp = static_cast<const uint16_t*>(x);
  auto* cp = static_cast<uint8_t*>(codes);
  auto* sp = static_cast<uint8_t*>(sf_blocks);
  if (planes == 16)
    return launch_pdl(quantize_planes_kernel<16>, grid, block, 0, s, xp, (int)m, (int)k, cp, sp, g, zero_ptr,
                      zero_count);
  if (planes == 8)
    return launch_pdl(quantize_planes_kernel<8>, grid, block, 0, s, xp, (int)m, (int)k, cp, sp, g, zero_ptr,
                      zero_count);
  return cudaErrorInvalidValue;
}

}  // namespace ffn
