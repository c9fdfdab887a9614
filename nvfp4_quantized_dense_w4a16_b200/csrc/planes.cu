// Activation planes for the few-row W4A16 path on the block-scaled FP4
// tensor core.
//
// The NVFP4 weights are multiplied by the tensor core's kind::mxf4nvf4 MMA
// as they are stored (E2M1 codes, one UE4M3 scale per 16 elements along K):
// no software dequantisation.  The bf16 activation row x is written as a sum
// of P = 8 NVFP4 "planes", x = sum_p g_p * (s_p,b * q_p,k) + r_P, each plane
// one extra MMA column:
//  * g_p = 2^(E - 8 - floor(3p / 2)) with E = floor(log2 max|x|): a per-row
//    power-of-two factor (fp32, applied in the epilogue) that keeps every
//    block scale of the plane within E4M3's powers of two 2^-9..2^8;
//  * per 16-block a power-of-two scale s = 2^ceil(log2(amax / 6 / g_p)) of
//    the residual r left by planes 0..p-1 (exact in E4M3, and the residual
//    then scales exactly), codes q = E2M1(r / (g_p * s)), and
//    r -= g_p * s * q (exact: the represented value has at most two
//    significant bits and lies within a factor two of r).
// Each plane removes at least a factor 3 from every block's residual while
// the schedule of g_p lowers the planes' range by 2^1.5 per plane, so no
// block outgrows its plane; in practice a plane takes the next two to three
// bits near each block's maximum, and 8 planes represent seeded bf16 rows
// (normal, outlier-channel and cubed-normal values) exactly or to ~1e-9 of
// the row maximum; small integers need the first plane only.  The epilogue
// folds the plane columns back with their factors (y = sum_p g_p * D_p).
#include "common.cuh"
#include "internal.h"
#include "launch.cuh"
#include "profile.h"

namespace ffn {
namespace {

constexpr int kPlaneThreads = 128;  // eight threads per 16-element block
constexpr int kBlocksPerCta = kPlaneThreads / 8;
constexpr int kPlanes = 8;

__device__ __forceinline__ float block_reduce_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float m = 0.0f;
#pragma unroll
  for (int w = 0; w < kPlaneThreads / 32; ++w) m = fmaxf(m, red[w]);
  return m;
}

// 2^k as fp32 (exact; built from the exponent bits in the normal range).
__device__ __forceinline__ float exp2i(int k) {
  return k >= -126 && k <= 127 ? __int_as_float((k + 127) << 23) : ldexpf(1.0f, k);
}

// Smallest e with 6 * 2^e >= a, for a > 0 normal: with a in [2^k, 2^(k+1)),
// e = k - 2 when a <= 1.5 * 2^k (6 * 2^(k-2) = 1.5 * 2^k), else k - 1
// (3 * 2^k > a); e = k - 3 never suffices (0.75 * 2^k < a).  Integer work on
// the bits of a, no division.
__device__ __forceinline__ int ceil_log2_over_6(float a) {
  const uint32_t bits = __float_as_uint(a);
  const int k = (int)((bits >> 23) & 0xffu) - 127;
  return (bits & 0x7fffffu) <= 0x400000u ? k - 2 : k - 1;
}

// grid (m, ceil(K / 16 / 16)): CTA (j, c) handles the 16-element blocks
// 16c .. 16c + 15 of row j, eight threads per block (two elements each),
// after reading the whole row for its maximum (every CTA of the row finds the
// same E).  Outputs: codes [m * P][K/2] (row j * P + p), scale bytes in the
// blocked layout of the MMA's scale-factor copy (rows j * P + p), g [m][P]
// (fp32).  The next kernel may launch at once (it waits for this one before
// reading the planes); after its own wait for the previous kernel this one
// also zeroes the counters of the projection that follows it, if given.
__global__ void __launch_bounds__(kPlaneThreads) quantize_planes_kernel(
    const uint16_t* __restrict__ x, int m, int K, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ sf_blocks, float* __restrict__ g, int* zero_ptr, int zero_count) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");  // x may come from the previous kernel
  __shared__ float red[kPlaneThreads / 32];
  const int cta = blockIdx.x * gridDim.y + blockIdx.y;
  for (int i = cta * kPlaneThreads + threadIdx.x; i < zero_count; i += gridDim.x * gridDim.y * kPlaneThreads)
    zero_ptr[i] = 0;
  const int j = blockIdx.x;
  const int nb = K / 16, kc = (K + 63) / 64;
  const uint16_t* row = x + (size_t)j * K;
  // the row's maximum |x|: eight bf16 per 16-byte load, eight independent
  // loads in flight per thread (|bf16| bits order like the values)
  uint32_t mx[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  const uint4* r16 = reinterpret_cast<const uint4*>(row);
  const int n16 = K / 8;
  for (int i0 = threadIdx.x; i0 < n16; i0 += 8 * kPlaneThreads) {
    uint4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * kPlaneThreads;
      v[u] = i < n16 ? r16[i] : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) mx[u] = max(mx[u], max(w[e] & 0x7fffu, (w[e] >> 16) & 0x7fffu));
    }
  }
  uint32_t mbits = 0;
#pragma unroll
  for (int u = 0; u < 8; ++u) mbits = max(mbits, mx[u]);
  const float rowmax = block_reduce_max(bf16_bits_to_float(mbits), red);
  const int E = rowmax > 0.0f ? ilogbf(rowmax) : 0;
  if (blockIdx.y == 0 && threadIdx.x < kPlanes)
    g[j * kPlanes + threadIdx.x] = rowmax > 0.0f ? exp2i(E - 8 - (3 * (int)threadIdx.x) / 2) : 0.0f;
  const int b = blockIdx.y * kBlocksPerCta + (threadIdx.x >> 3);
  const int part = threadIdx.x & 7;  // elements 2 part, 2 part + 1 of the block
  const bool valid = b < nb;         // whole groups of eight lanes share validity
  float r0 = 0.0f, r1 = 0.0f;
  if (valid) {
    const uint32_t v = *reinterpret_cast<const uint32_t*>(row + 16 * b + 2 * part);
    r0 = bf16_bits_to_float(v & 0xffffu);
    r1 = bf16_bits_to_float(v >> 16);
  }
#pragma unroll 1
  for (int p = 0; p < kPlanes; ++p) {
    float amax = fmaxf(fabsf(r0), fabsf(r1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
    uint32_t s8 = 0, byte = 0;
    if (amax > 0.0f) {
      const int ge = E - 8 - (3 * p) / 2;  // log2 g_p
      // smallest power of two 2^e >= amax / 6 / g_p, clamped to E4M3's 2^-9..2^8
      int e = ceil_log2_over_6(amax * exp2i(-ge));
      e = e < -9 ? -9 : (e > 8 ? 8 : e);
      s8 = e >= -6 ? (uint32_t)(e + 7) << 3 : (1u << (e + 9));
      // r / (g_p * 2^e) and the represented values are exact power-of-two scalings
      const float down = exp2i(-(ge + e)), up = exp2i(ge + e);
      const uint32_t q0 = e2m1_encode(r0 * down), q1 = e2m1_encode(r1 * down);
      r0 -= ((q0 & 8u) ? -e2m1_mag(q0 & 7u) : e2m1_mag(q0 & 7u)) * up;
      r1 -= ((q1 & 8u) ? -e2m1_mag(q1 & 7u) : e2m1_mag(q1 & 7u)) * up;
      byte = q0 | (q1 << 4);
    }
    if (valid) {
      const int rowp = j * kPlanes + p;
      codes[(size_t)rowp * (K / 2) + 8 * b + part] = (uint8_t)byte;
      if (part == 0) sf_blocks[sf_blocked_offset(rowp, b, kc)] = (uint8_t)s8;
    }
  }
}

}  // namespace

// Planes per activation row (0: the few-row block-scaled path does not apply).
int planes_for_rows(int64_t m) { return m <= 8 ? kPlanes : 0; }

cudaError_t launch_quantize_planes(const void* x, int64_t m, int64_t k, int planes, void* codes, void* sf_blocks,
                                   float* g, int* zero_ptr, int zero_count, cudaStream_t s) {
  if (planes != kPlanes || k % 16) return cudaErrorInvalidValue;
  ProfScope prof(s, "quantize_planes");
  const dim3 grid((unsigned)m, (unsigned)((k / 16 + kBlocksPerCta - 1) / kBlocksPerCta));
  return launch_pdl(quantize_planes_kernel, grid, dim3(kPlaneThreads), 0, s, static_cast<const uint16_t*>(x),
                    (int)m, (int)k, static_cast<uint8_t*>(codes), static_cast<uint8_t*>(sf_blocks), g, zero_ptr,
                    zero_count);
}

}  // namespace ffn
