// CUDA-core NVFP4 projections for few rows (decode) and the general
// fallback-free path for any row count.
//
// One warp owns one output column j (one weight row; for the fused gate+up
// weight the pair gate j / up j, so the SiLU*mul epilogue is warp-local).
// Lane l streams 32 consecutive K elements per step (16 bytes of codes, two
// E4M3 scale bytes) with 128-bit loads, decodes them in registers and
// multiplies by MR rows of activations; the warp reduces with shuffles.
// The reduction order for an output element depends only on K, never on m or
// on the other rows, so results are reproducible.
//
// W4A16 numerics: per 16-element block p = sum_i e2m1(c_i) * x_i (fp32),
// acc += s_b * p; y = bf16(gs * acc).  W4A4: the block sum of products of
// codes is an exact integer S, acc += (S/4) * (sa * sw) (sa * sw exact).
#include "common.cuh"
#include "internal.h"
#include "profile.h"

namespace ffn {

namespace {

constexpr int kWarps = 8;

// E2M1 values of the 16 codes (fp32) and twice them as integers.
__device__ __forceinline__ void fill_luts(float* lut, int* lut2) {
  if (threadIdx.x < 16) {
    const uint32_t c = threadIdx.x;
    const float v = e2m1_mag(c & 7u);
    lut[c] = (c & 8u) ? -v : v;
    lut2[c] = (int)((c & 8u) ? -2.0f * v : 2.0f * v);
  }
  __syncthreads();
}

template <int MR>
__device__ __forceinline__ void load_x32(const uint16_t* __restrict__ x, int64_t ldx, int r0,
                                         int rows, int64_t k, uint4 (&xv)[MR][4]) {
#pragma unroll
  for (int r = 0; r < MR; ++r) {
    if (r < rows) {
      const uint4* p = reinterpret_cast<const uint4*>(x + (int64_t)(r0 + r) * ldx + k);
#pragma unroll
      for (int q = 0; q < 4; ++q) xv[r][q] = __ldg(p + q);
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) xv[r][q] = make_uint4(0, 0, 0, 0);
    }
  }
}

// acc[r] += sum over the two blocks of this 32-element chunk.
template <int MR>
__device__ __forceinline__ void dot32_w4a16(const float* lut, uint4 cw, uint32_t sc2,
                                            const uint4 (&xv)[MR][4], float (&acc)[MR]) {
  const uint32_t cwords[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    const float s = e4m3_decode((sc2 >> (8 * b)) & 0xffu);
    float wv[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) wv[i] = lut[(cwords[2 * b + i / 8] >> (4 * (i % 8))) & 15u];
#pragma unroll
    for (int r = 0; r < MR; ++r) {
      const uint32_t xw[8] = {xv[r][2 * b].x, xv[r][2 * b].y, xv[r][2 * b].z, xv[r][2 * b].w,
                              xv[r][2 * b + 1].x, xv[r][2 * b + 1].y, xv[r][2 * b + 1].z,
                              xv[r][2 * b + 1].w};
      float p = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        p = fmaf(wv[2 * i], bf16_bits_to_float(xw[i] & 0xffffu), p);
        p = fmaf(wv[2 * i + 1], bf16_bits_to_float(xw[i] >> 16), p);
      }
      acc[r] = fmaf(s, p, acc[r]);
    }
  }
}

template <int MR, bool kGateUp>
__global__ void __launch_bounds__(kWarps * 32)
gemv_w4a16_kernel(const uint16_t* __restrict__ x, int m, const uint8_t* __restrict__ codes,
                  const uint8_t* __restrict__ scales, const float* __restrict__ gs,
                  int64_t ncols, int64_t k, uint16_t* __restrict__ y) {
  __shared__ float lut[16];
  __shared__ int lut2[16];
  fill_luts(lut, lut2);
  const int lane = threadIdx.x & 31;
  const int64_t j = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (j >= ncols) return;
  const int64_t ldc = k / 2, lds = k / 16;
  const uint8_t* c0 = codes + j * ldc;
  const uint8_t* s0 = scales + j * lds;
  const uint8_t* c1 = codes + (j + ncols) * ldc;  // up row (gate+up only)
  const uint8_t* s1 = scales + (j + ncols) * lds;
  const float gs0 = gs[0];
  const float gs1 = kGateUp ? gs[1] : 0.0f;
  for (int r0 = 0; r0 < m; r0 += MR) {
    const int rows = min(MR, m - r0);
    float a0[MR], a1[MR];
#pragma unroll
    for (int r = 0; r < MR; ++r) a0[r] = a1[r] = 0.0f;
    for (int64_t kk = (int64_t)lane * 32; kk < k; kk += 1024) {
      uint4 xv[MR][4];
      load_x32<MR>(x, k, r0, rows, kk, xv);
      const uint4 cw0 = __ldg(reinterpret_cast<const uint4*>(c0 + kk / 2));
      const uint32_t sc0 = __ldg(reinterpret_cast<const uint16_t*>(s0 + kk / 16));
      dot32_w4a16<MR>(lut, cw0, sc0, xv, a0);
      if (kGateUp) {
        const uint4 cw1 = __ldg(reinterpret_cast<const uint4*>(c1 + kk / 2));
        const uint32_t sc1 = __ldg(reinterpret_cast<const uint16_t*>(s1 + kk / 16));
        dot32_w4a16<MR>(lut, cw1, sc1, xv, a1);
      }
    }
#pragma unroll
    for (int r = 0; r < MR; ++r) {
      a0[r] = warp_sum(a0[r]);
      if (kGateUp) a1[r] = warp_sum(a1[r]);
    }
    if (lane == 0) {
#pragma unroll
      for (int r = 0; r < MR; ++r) {
        if (r < rows) {
          float v;
          if (kGateUp) {
            const float g = bf16_round(gs0 * a0[r]);
            const float u = bf16_round(gs1 * a1[r]);
            v = silu_f32(g) * u;
          } else {
            v = gs0 * a0[r];
          }
          y[(int64_t)(r0 + r) * ncols + j] = f32_to_bf16_bits(v);
        }
      }
    }
  }
}

// ---- fixed format (W4A4) ----------------------------------------------------

template <int MR>
__device__ __forceinline__ void dot32_w4a4(const int* lut2, uint4 cw, uint32_t sc2,
                                           const uint4 (&xc)[MR], const uint32_t (&xs)[MR],
                                           float (&acc)[MR]) {
  const uint32_t cwords[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    const float sw = e4m3_decode((sc2 >> (8 * b)) & 0xffu);
    int wv[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) wv[i] = lut2[(cwords[2 * b + i / 8] >> (4 * (i % 8))) & 15u];
#pragma unroll
    for (int r = 0; r < MR; ++r) {
      const uint32_t aw[2] = {b == 0 ? xc[r].x : xc[r].z, b == 0 ? xc[r].y : xc[r].w};
      int S = 0;
#pragma unroll
      for (int i = 0; i < 16; ++i) S += wv[i] * lut2[(aw[i / 8] >> (4 * (i % 8))) & 15u];
      const float sa = e4m3_decode((xs[r] >> (8 * b)) & 0xffu);
      acc[r] += __fmul_rn((float)S * 0.25f, __fmul_rn(sa, sw));
    }
  }
}

template <int MR, bool kGateUp>
__global__ void __launch_bounds__(kWarps * 32)
gemv_w4a4_kernel(const uint8_t* __restrict__ xcodes, const uint8_t* __restrict__ xscales, int m,
                 const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                 const float* __restrict__ gs, int64_t ncols, int64_t k,
                 uint16_t* __restrict__ y) {
  __shared__ float lut[16];
  __shared__ int lut2[16];
  fill_luts(lut, lut2);
  const int lane = threadIdx.x & 31;
  const int64_t j = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (j >= ncols) return;
  const int64_t ldc = k / 2, lds = k / 16;
  const uint8_t* c0 = codes + j * ldc;
  const uint8_t* s0 = scales + j * lds;
  const uint8_t* c1 = codes + (j + ncols) * ldc;
  const uint8_t* s1 = scales + (j + ncols) * lds;
  const float gs0 = gs[0];
  const float gs1 = kGateUp ? gs[1] : 0.0f;
  for (int r0 = 0; r0 < m; r0 += MR) {
    const int rows = min(MR, m - r0);
    float a0[MR], a1[MR];
#pragma unroll
    for (int r = 0; r < MR; ++r) a0[r] = a1[r] = 0.0f;
    for (int64_t kk = (int64_t)lane * 32; kk < k; kk += 1024) {
      uint4 xc[MR];
      uint32_t xs[MR];
#pragma unroll
      for (int r = 0; r < MR; ++r) {
        if (r < rows) {
          xc[r] = __ldg(reinterpret_cast<const uint4*>(xcodes + (int64_t)(r0 + r) * ldc + kk / 2));
          xs[r] = __ldg(reinterpret_cast<const uint16_t*>(xscales + (int64_t)(r0 + r) * lds + kk / 16));
        } else {
          xc[r] = make_uint4(0, 0, 0, 0);
          xs[r] = 0;
        }
      }
      const uint4 cw0 = __ldg(reinterpret_cast<const uint4*>(c0 + kk / 2));
      const uint32_t sc0 = __ldg(reinterpret_cast<const uint16_t*>(s0 + kk / 16));
      dot32_w4a4<MR>(lut2, cw0, sc0, xc, xs, a0);
      if (kGateUp) {
        const uint4 cw1 = __ldg(reinterpret_cast<const uint4*>(c1 + kk / 2));
        const uint32_t sc1 = __ldg(reinterpret_cast<const uint16_t*>(s1 + kk / 16));
        dot32_w4a4<MR>(lut2, cw1, sc1, xc, xs, a1);
      }
    }
#pragma unroll
    for (int r = 0; r < MR; ++r) {
      a0[r] = warp_sum(a0[r]);
      if (kGateUp) a1[r] = warp_sum(a1[r]);
    }
    if (lane == 0) {
#pragma unroll
      for (int r = 0; r < MR; ++r) {
        if (r < rows) {
          float v;
          if (kGateUp) {
            const float g = bf16_round(gs0 * a0[r]);
            const float u = bf16_round(gs1 * a1[r]);
            v = silu_f32(g) * u;
          } else {
            v = gs0 * a0[r];
          }
          y[(int64_t)(r0 + r) * ncols + j] = f32_to_bf16_bits(v);
        }
      }
    }
  }
}

template <int MR>
cudaError_t gemv16(const void* x, int64_t m, const WeightView& w, Epilogue ep, void* y,
                   cudaStream_t s) {
  const bool gu = ep == Epilogue::kSiluMul;
  const int64_t ncols = gu ? w.n / 2 : w.n;
  const unsigned grid = (unsigned)((ncols + kWarps - 1) / kWarps);
  ProfScope prof(s, gu ? "gemv_w4a16_gate_up_silu" : "gemv_w4a16");
  if (gu)
    gemv_w4a16_kernel<MR, true><<<grid, kWarps * 32, 0, s>>>(
        (const uint16_t*)x, (int)m, w.codes, w.scales, w.gs, ncols, w.k, (uint16_t*)y);
  else
    gemv_w4a16_kernel<MR, false><<<grid, kWarps * 32, 0, s>>>(
        (const uint16_t*)x, (int)m, w.codes, w.scales, w.gs, ncols, w.k, (uint16_t*)y);
  return cudaGetLastError();
}

}  // namespace

int gemv_grid(int64_t ncols) { return (int)((ncols + kWarps - 1) / kWarps); }

cudaError_t launch_gemv_w4a16(const void* x, int64_t m, const WeightView& w, Epilogue ep,
                              void* y, cudaStream_t s) {
  if (m <= 1) return gemv16<1>(x, m, w, ep, y, s);
  if (m <= 2) return gemv16<2>(x, m, w, ep, y, s);
  return gemv16<4>(x, m, w, ep, y, s);
}

cudaError_t launch_gemv_w4a4(const uint8_t* xcodes, const uint8_t* xscales, int64_t m,
                             const WeightView& w, Epilogue ep, void* y, cudaStream_t s) {
  // One row chunk size for every m: the per-row arithmetic must not depend
  // on how many rows share the launch.
  constexpr int MR = 4;
  const bool gu = ep == Epilogue::kSiluMul;
  const int64_t ncols = gu ? w.n / 2 : w.n;
  const unsigned grid = (unsigned)((ncols + kWarps - 1) / kWarps);
  ProfScope prof(s, gu ? "gemv_w4a4_gate_up_silu" : "gemv_w4a4");
  if (gu)
    gemv_w4a4_kernel<MR, true><<<grid, kWarps * 32, 0, s>>>(
        xcodes, xscales, (int)m, w.codes, w.scales, w.gs, ncols, w.k, (uint16_t*)y);
  else
    gemv_w4a4_kernel<MR, false><<<grid, kWarps * 32, 0, s>>>(
        xcodes, xscales, (int)m, w.codes, w.scales, w.gs, ncols, w.k, (uint16_t*)y);
  return cudaGetLastError();
}

}  // namespace ffn
