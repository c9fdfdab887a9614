// Device helpers shared by the NVFP4 FFN kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lora_args.h"

namespace ffn {

// ---------------------------------------------------------------------------
// Formats.  FP4 E2M1 (OCP MX v1.0): nibble bit 3 = sign, bits 0-2 index the
// magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}.  E4M3 (OCP OFP8 v1.0): bias 7, no
// infinities, max 448.
// ---------------------------------------------------------------------------

// E2M1 code of q: nearest magnitude, ties to the even magnitude index,
// saturating at 6, sign bit copied from q.  Each comparison counts the
// midpoints below |q|; '>' at a midpoint whose lower neighbour has an even
// index and '>=' where the upper one is even gives ties-to-even.
__device__ __forceinline__ uint32_t e2m1_encode(float q) {
  const float a = fabsf(q);
  uint32_t idx = (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) +
                 (a > 2.5f) + (a >= 3.5f) + (a > 5.0f);
  return idx | (signbit(q) ? 8u : 0u);
}

// fp32 -> E4M3 byte, round to nearest even, saturating to 448 (CUDA's own
// conversion; inputs here are non-negative).
__device__ __forceinline__ uint32_t e4m3_encode_satfinite(float t) {
  return (uint32_t)__nv_cvt_float_to_fp8(t, __NV_SATFINITE, __NV_E4M3);
}

// Value of a non-negative E4M3 byte (exact in fp32).
__device__ __forceinline__ float e4m3_decode(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  if (e == 0) return (float)m * 0.001953125f;  // m * 2^-9
  return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// Codes of one 16-element block under the decoded scale sdec (fp32 IEEE
// division per element); all zero when `zero`.  Element i in nibble i.
__device__ __forceinline__ uint2 e2m1_encode_block16(const float (&v)[16], float sdec, bool zero) {
  uint32_t lo = 0, hi = 0;
  if (!zero) {
#pragma unroll
    for (int i = 0; i < 8; ++i) lo |= e2m1_encode(__fdiv_rn(v[i], sdec)) << (4 * i);
#pragma unroll
    for (int i = 0; i < 8; ++i) hi |= e2m1_encode(__fdiv_rn(v[8 + i], sdec)) << (4 * i);
  }
  return make_uint2(lo, hi);
}

// Scale-factor byte position of (row r, 16-element block kb) in the blocked
// layout the block-scaled FP4 kernel copies to TMEM: one 512-byte block per
// 128 rows and 64 elements (kc such blocks per 128 rows), row r's four scales
// at 16 * (r % 32) + 4 * ((r % 128) / 32).
__host__ __device__ __forceinline__ int64_t sf_blocked_offset(int64_t r, int64_t kb, int64_t kc) {
  const int rr = (int)(r & 127);
  return ((r >> 7) * kc + kb / 4) * 512 + 16 * (rr & 31) + 4 * (rr >> 5) + (kb & 3);
}

// E2M1 magnitude of a 3-bit index as fp32 (exact).
__device__ __forceinline__ float e2m1_mag(uint32_t i) {
  // 0, .5, 1, 1.5, 2, 3, 4, 6 = (i < 2 ? 0.5*i : 2^(e-1)*(1+m/2)) with e = i>>1
  return i < 2 ? 0.5f * (float)i : __uint_as_float(((i >> 1) + 126u) << 23 | ((i & 1u) << 22));
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t bits16) {
  return __uint_as_float(bits16 << 16);
}

__device__ __forceinline__ float bf16_round(float v) {
  return __bfloat162float(__float2bfloat16_rn(v));
}

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float v) {
  __nv_bfloat16 b = __float2bfloat16_rn(v);
  return *reinterpret_cast<uint16_t*>(&b);
}

__device__ __forceinline__ float lora_dot(const uint16_t* xa_row, const uint16_t* b_row, int r) {
  float d = 0.0f;
  for (int i = 0; i < r; ++i)
    d = fmaf(__uint_as_float((uint32_t)xa_row[i] << 16), __uint_as_float((uint32_t)b_row[i] << 16), d);
  return d;
}

// y (a bf16 value as fp32) + delta of output n for activation row j, rounded
// to bf16; unchanged without an adapter.
__device__ __forceinline__ float lora_add(float y, const uint16_t* b, int off, const LoraArgs& l, int64_t j,
                                          int64_t n) {
  if (!b) return y;
  const float d = lora_dot(l.xa + j * l.xa_ld + off, b + n * l.r, l.r);
  return __bfloat162float(__float2bfloat16_rn(y + d));
}

// SiLU in fp32: z / (1 + exp(-z)).
__device__ __forceinline__ float silu_f32(float z) { return z / (1.0f + expf(-z)); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace ffn
