// tcgen05 (5th-generation tensor core) NVFP4-weight x bf16-activation GEMM
// for sm_100a: one projection D[n, r] = sum_k W[n, k] * X[r, k] of the FFN
// ("metrale_model_layers/layers/dense_ffn_prefill.rs", w4a16_prefill_gemm:
// the NVFP4 projection GEMM the layer runs for m rows).
//
// Design (one CTA per 128-weight-row tile x BN activation rows x K range):
//  * weights are streamed in a pre-tiled layout (per 128-row tile and
//    64-element K chunk: 128 x 16 B low codes, 128 x 16 B high codes,
//    128 x 4 B E4M3 scales = 4608 B) by bulk async copies.  The natural-code
//    copy is the canonical no-swizzle K-major operand of the block-scaled FP4
//    MMA with its 512-byte scale-factor block (row r at byte
//    16*(r%32) + 4*(r/32)), streamed by the W4A4 kernel; the bf16-activation
//    kernel streams a second copy whose code bits are rearranged for a cheap
//    decode (see "W4A16 operand decoding");
//  * activations X [m, K] bf16 arrive by 2-D TMA with the 128-byte swizzle
//    (box 64 x BN), the layout the MMA reads directly;
//  * dequant warpgroups (four warps, one per TMEM lane quarter) turn each
//    thread's row of codes into exact bf16 values (E2M1 * E4M3 scale * 2^-8:
//    at most 6 significant bits) with rotations, masks and one bf16x2
//    multiply, and write them straight into tensor memory, where they are the
//    MMA's A operand (M = 128 weight rows) -- so the dequantised weights never
//    occupy shared-memory bandwidth;
//  * one to three threads issue tcgen05.mma kind::f16 (A from TMEM, B = X
//    tile from shared memory, an fp32 accumulator each in TMEM, N = BN);
//  * the dequant warps then read the accumulators back (tcgen05.ld), add them
//    in a fixed order and run the epilogue: y = bf16(gs * acc); or for the
//    fused gate+up weight (64 gate rows then the matching 64 up rows per tile)
//    h = bf16(silu(bf16(gs_g*g)) * bf16(gs_u*u)); or fp32 split-K partials;
//  * the kernels are launched with programmatic dependent launch and wait for
//    the previous kernel only before reading activations and writing results.
// Pipelines are mbarrier-driven; every wait is bounded and, on timeout, sets
// a device error bit and lets the CTA free its TMEM and exit.
#include <cudaTypedefs.h>
#include <stdlib.h>

#include <mutex>
#include <utility>

#include "common.cuh"
#include "internal.h"
#include "launch.cuh"
#include "profile.h"
#include "sm100.cuh"

namespace ffn {

__device__ int g_ffn_device_error = 0;

using namespace sm100;

namespace {

constexpr int kChunkK = 64;        // K elements per stage
constexpr int kTileRows = 128;     // weight rows per tile = TMEM lanes
constexpr int kChunkBytes = 4608;  // 128 x (16 + 16 + 4) bytes

enum : int { kEpiStore = 0, kEpiSiluMul = 1, kEpiPartial = 2, kEpiSiluMulQuant = 3 };

// Pipeline shape.  The K range of a CTA is a sequence of 64-element chunks,
// grouped into units of UA consecutive chunks; unit u is dequantised by
// warpgroup u % DQG (its four warps cover the 128 TMEM lanes) into TMEM slot
// u % SA and multiplied by MMA-issuing thread u % NI into that thread's own
// accumulator (the epilogue adds them).  Three rings, each with its own
// granularity:
//  * weights: SWS stages of one round (DQG consecutive units, one per
//    warpgroup), released once every warpgroup has read its unit;
//  * activations: SXS stages of XC chunks, released when the MMAs that read
//    them complete and waited for either by the MMA threads (once per stage)
//    or, with DQX (one stage per unit), by the unit's dequant warps before
//    they hand the slot over -- which keeps that wait off the MMA thread, the
//    critical role of wide tiles;
//  * TMEM: SA A slots of one unit, released when their MMAs complete, so a
//    warpgroup can dequantise its next units while earlier ones are still in
//    the tensor pipe.
// Every mbarrier wait and tcgen05 fence costs ~0.1 us even when nothing is
// pending, so the dequant warps wait on two barriers per unit (slot free,
// weights landed) and the MMA threads on one (plus one per activation stage).
template <int BN, int SXS, int XC, int SWS, int SA, int DQG, int UA, int NI, bool DQX>
struct TcCfg {
  static constexpr int kThreads = 128 + 128 * DQG;
  static constexpr int kXStageBytes = XC * BN * 128;   // XC chunk tiles of BN rows x 128 B
  static constexpr int kUnitBytes = UA * kChunkBytes;
  static constexpr int kWStageBytes = DQG * kUnitBytes;
  static constexpr int kAColBase = NI * BN < 32 ? 32 : NI * BN;  // TMEM column of A slot 0
  static constexpr int kSlotCols = 32 * UA;
  static constexpr int kTmemNeed = kAColBase + kSlotCols * SA;
  static constexpr int kTmemCols = kTmemNeed <= 64 ? 64 : kTmemNeed <= 128 ? 128 : kTmemNeed <= 256 ? 256 : 512;
  // The epilogue staging buffers (16 KB per dequant warpgroup) reuse the start
  // of the rings: the epilogue runs after every MMA has completed, and those
  // MMAs consumed every copy the producers issued.
  static constexpr int kEpiBytes = 16384;
  static constexpr int kSmemW = SXS * kXStageBytes;
  static constexpr int kSmemRings = kSmemW + SWS * kWStageBytes;
  static constexpr int kSmemBar = kSmemRings;
  static constexpr int kNumBars = 2 * SXS + 2 * SWS + 2 * SA + NI;
  static constexpr int kSmemBytes = kSmemBar + kNumBars * 8 + 16;
  static constexpr int kSmemAlloc = kSmemBytes + 1024;  // slack for 1024-byte alignment
  // two CTAs per SM when both fit (228 KB of shared memory, 512 TMEM columns)
  static constexpr int kMinBlocks = (2 * (kSmemAlloc + 1024) <= 233472 && kTmemCols <= 256) ? 2 : 1;
  static_assert(kTmemNeed <= 512, "TMEM budget");
  static_assert(kSmemAlloc <= 232448, "shared memory budget");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N");
  static_assert(DQG >= 1 && DQG <= 3 && (NI == 1 || NI == 2) && UA >= 1, "roles");
  static_assert(kSmemRings >= DQG * kEpiBytes, "epilogue buffers alias the rings");
  // A parity wait can only tell the awaited phase from the one before it, so
  // the previous phase must be known complete when a thread starts waiting.
  // Slot u % SA is reused by unit u + SA: with SA a multiple of DQG and of NI
  // that unit has the same warpgroup and the same MMA thread, each of which
  // waited for the slot's previous phase itself.  Every warpgroup waits for
  // every weight round and (XC a multiple of UA * NI) every MMA thread for
  // every activation stage, in order, which covers those rings.
  // With DQX, stage u % SXS is reused by unit u + SXS of the same warpgroup.
  static_assert(SA % DQG == 0 && SA % NI == 0 &&
                    (DQX ? (XC == UA && SXS % DQG == 0) : XC % (UA * NI) == 0),
                "ring depths");
};

struct TcArgs {
  const uint8_t* wt;   // tiled weight [tiles][kc_total][4608]
  const float* gs;     // tensor scale(s)
  void* out;           // bf16 [m, ldo] or fp32 partials [splits][m][n_pad]
  int m, n_out, ldo, kc_total, kc_per_split, n_pad;
  // Activation rows one TMA box carries: min(m, tile rows).  Boxes never
  // extend past row m (no zero fill); shared-memory rows beyond them keep
  // stale data, which only reaches accumulator columns of rows >= m -- MMA
  // columns are independent and those columns are never stored.
  int x_box_rows;
  // kEpiSiluMulQuant: h is quantised per row to NVFP4 as it is produced
  // (the fixed format's input of the down projection): codes [m, n_out/2]
  // and scale bytes in the blocked layout with q_kc 64-element chunks per row.
  uint8_t* q_codes = nullptr;
  uint8_t* q_sf = nullptr;
  int q_kc = 0;
  LoraArgs lora;  // adapter deltas added to the bf16 outputs (store / SiLU*mul)
};

__device__ __forceinline__ uint32_t bmul2(uint32_t a, uint32_t b) {
  __nv_bfloat162 r = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&a),
                             *reinterpret_cast<__nv_bfloat162*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

// ------------------------------------------------ W4A16 operand decoding
//
// The bf16-activation path streams a second copy of the weight tiles whose
// code bits are rearranged inside every 32-bit word (eight E2M1 codes) so
// that each bf16x2 pair of the A operand comes out of one or two rotations
// and a mask.  The decoded half-word of a code (s, e1, e0, m) is
//   bit 15 = s, bits 8..6 = e1 e0 m, all other bits 0,
// which as a bf16 number is exactly the E2M1 value times 2^-126: the two
// exponent bits land in the exponent field and m in the top mantissa bit, and
// the e = 0 codes (0 and 0.5) become the bf16 subnormals 0 and 2^-127.  The
// block scale is applied as the bf16 number s * 2^118 (at most 448 * 2^118 <
// bf16 max), so every A element equals (E2M1 * s) * 2^-8 exactly, and the
// epilogue multiplies the fp32 accumulator by gs * 2^8.
//
// Within a word, output pair k (elements 2k, 2k+1) is read from
//   k = 0: c & M,  k = 1: (c << 4) & M,  k = 2: rotr(c, 6) & M,
//   k = 3: ((c << 6) & MA) | (rotr(c, 2) & MB)
// with M the eight destination bits {6,7,8,15,22,23,24,31}; these source
// positions are disjoint and cover the word (permute_codes_w4a16 writes it).
// The left shifts are written as multiplies, which the compiler can issue on
// the FMA pipe: the integer pipe, the bottleneck at small m, does 7 operations
// per eight codes.
constexpr uint32_t kPairMask = 0x81C081C0u;
constexpr uint32_t kPairMaskA = 0x80C080C0u;  // bits 6, 7, 15 of each half
constexpr uint32_t kPairMaskB = 0x01000100u;  // bit 8 of each half
constexpr float kW4A16Unscale = 256.0f;        // 2^8

__device__ __forceinline__ uint32_t rotr32(uint32_t x, int r) { return __funnelshift_r(x, x, r); }

// Source bit of destination bit p of output pair k.
__host__ __device__ constexpr int w4a16_src_bit(int k, int p) {
  return k == 0 ? p
       : k == 1 ? p - 4
       : k == 2 ? (p + 6) & 31
       : ((p & 15) == 8 ? (p + 2) & 31 : p - 6);
}

// Natural word (element e in bits 4e..4e+3) -> the rearranged word.
__device__ __forceinline__ uint32_t permute_codes_w4a16(uint32_t nat) {
  uint32_t out = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int p = (b == 3 ? 15 : 6 + b) + 16 * (e & 1);
      out |= ((nat >> (4 * e + b)) & 1u) << w4a16_src_bit(e >> 1, p);
    }
  }
  return out;
}

__device__ __forceinline__ uint32_t cvt_e4m3x2_f16x2(uint32_t two) {
  uint32_t r;
  asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(r) : "r"(two));
  return r;
}

// Two E4M3 scales (low byte -> low half) -> bf16 bits of s * 2^118 in each
// half: the f16 value is exact, and shifting its bits right by 3 leaves the
// bf16 layout with the exponent re-biased by -112; adding 230 << 7 sets the
// bias to +118.  (A zero scale yields 2^103; its codes are zero.)
__device__ __forceinline__ uint32_t scale2_w4a16(uint32_t two_e4m3) {
  const uint32_t h = cvt_e4m3x2_f16x2(two_e4m3);
  return ((h >> 3) & 0x1FFF1FFFu) + 0x73007300u;
}

__device__ __forceinline__ void dequant8_w4a16(uint32_t c, uint32_t s2, uint32_t* o) {
  o[0] = bmul2(c & kPairMask, s2);
  o[1] = bmul2((c * 16u) & kPairMask, s2);
  o[2] = bmul2(rotr32(c, 6) & kPairMask, s2);
  o[3] = bmul2(((c * 64u) & kPairMaskA) | (rotr32(c, 2) & kPairMaskB), s2);
}

// One thread's 64-element chunk (rearranged codes, four scales) -> 32 columns.
__device__ __forceinline__ void dequant64_w4a16(const uint4 lo, const uint4 hi, uint32_t sc,
                                                uint32_t (&v)[32]) {
  const uint32_t t01 = scale2_w4a16(sc & 0xffffu), t23 = scale2_w4a16(sc >> 16);
  const uint32_t s0 = __byte_perm(t01, 0, 0x1010), s1 = __byte_perm(t01, 0, 0x3232);
  const uint32_t s2 = __byte_perm(t23, 0, 0x1010), s3 = __byte_perm(t23, 0, 0x3232);
  dequant8_w4a16(lo.x, s0, v + 0);
  dequant8_w4a16(lo.y, s0, v + 4);
  dequant8_w4a16(lo.z, s1, v + 8);
  dequant8_w4a16(lo.w, s1, v + 12);
  dequant8_w4a16(hi.x, s2, v + 16);
  dequant8_w4a16(hi.y, s2, v + 20);
  dequant8_w4a16(hi.z, s3, v + 24);
  dequant8_w4a16(hi.w, s3, v + 28);
}

// SiLU with the fast exponential and division (a few ulp in fp32; the result
// is rounded to bf16 right after).
__device__ __forceinline__ float silu_fast(float z) {
  return z < -88.0f ? 0.0f * z : __fdividef(z, 1.0f + __expf(-z));
}

// Bounded wait that ignores the abort flag (used to drain in-flight work).
__device__ __forceinline__ bool wait_drain(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitLimitCycles) {
      atomicOr(&g_ffn_device_error, 16);
      return false;
    }
  }
  return true;
}

// Epilogue of one (128 weight rows) x (BN activation rows) accumulator tile
// held in TMEM columns [0, BN): warpgroup g of NG takes every NG-th 32-column
// chunk; thread (q, lane) owns tile row 32q + lane.  kEpiStore writes
// y = bf16(gs * acc); kEpiSiluMul (rows 0-63 gate, 64-127 the matching up rows)
// writes h = bf16(silu(bf16(gs_g * g)) * bf16(gs_u * u)); kEpiPartial writes
// fp32 split-K partials (gs_mul: a power of two folded into the operands,
// applied with gs); kEpiSiluMulQuant computes h like kEpiSiluMul and writes
// its per-row NVFP4 quantisation instead (per 16-block: s = E4M3(amax/6),
// codes = E2M1(h / s), the same arithmetic as the activation quantiser).
// Stores are staged through shared memory (ebuf, 16 KB per warpgroup) so that
// global writes are 16-byte and row-contiguous.
template <int BN, int EPI, int NG, int NACC = 1, bool LORA = false>
__device__ __forceinline__ void epilogue_tile(const TcArgs& a, uint32_t tmem, int q, int lane,
                                              int g, uint8_t* ebuf, int xtile, int wtile,
                                              int nacc_used = 1, float gs_mul = 1.0f) {
  const int row = 32 * q + lane;
  const uint32_t lane_addr = (uint32_t)(32 * q) << 16;
  const int rbase = xtile * BN;
  const int nchunks = (BN + 31) / 32;
  const int et = 32 * q + lane;  // 0..127 within this warpgroup
  for (int c = g; c < nchunks; c += NG) {
    const int r0 = rbase + 32 * c;
    if (r0 >= a.m) break;
    const int jmax = min(32, BN - 32 * c);
    uint32_t v[32];
    tmem_ld32(tmem + lane_addr + 32 * c, v);
    tmem_ld_wait();
    // accumulators 1..NACC-1 hold the other K steps: add them in a fixed order
#pragma unroll
    for (int acc = 1; acc < NACC; ++acc) {
      if (acc >= nacc_used) break;  // an issuer that had no unit left its accumulator unwritten
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t u[16];
        tmem_ld16(tmem + lane_addr + acc * BN + 32 * c + 16 * h, u);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j)
          v[16 * h + j] = __float_as_uint(__uint_as_float(v[16 * h + j]) + __uint_as_float(u[j]));
      }
    }
    if (EPI == kEpiPartial) {
      float* P = static_cast<float*>(a.out) + (size_t)blockIdx.z * a.m * a.n_pad;
      const int col = kTileRows * wtile + row;
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (j < jmax && r0 + j < a.m) P[(size_t)(r0 + j) * a.n_pad + col] = __uint_as_float(v[j]);
    } else if (EPI == kEpiStore) {
      uint16_t* T = reinterpret_cast<uint16_t*>(ebuf);  // [32][128] bf16
      const float gs = a.gs[0] * gs_mul;
      const int64_t nrow = (int64_t)kTileRows * wtile + row;
      const bool lv = LORA && a.lora.b0 != nullptr && nrow < a.n_out;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        float y = gs * __uint_as_float(v[j]);
        if (lv && r0 + j < a.m) y = lora_add(bf16_round(y), a.lora.b0, a.lora.off0, a.lora, r0 + j, nrow);
        T[j * 128 + row] = f32_to_bf16_bits(y);
      }
      named_bar_sync(1 + g, 128);
      const int n0 = kTileRows * wtile;
      for (int idx = et; idx < 32 * 16; idx += 128) {
        const int j = idx >> 4, ch = idx & 15;
        const int r = r0 + j, n = n0 + 8 * ch;
        if (j < jmax && r < a.m && n < a.n_out)
          *reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.out) + (size_t)r * a.ldo + n) =
              *reinterpret_cast<const uint4*>(T + j * 128 + 8 * ch);
      }
      named_bar_sync(1 + g, 128);
    } else {  // kEpiSiluMul
      float* U = reinterpret_cast<float*>(ebuf);                  // [32][64] fp32
      uint16_t* Hs = reinterpret_cast<uint16_t*>(ebuf + 8192);    // [32][64] bf16
      if (q >= 2) {
        const float gsu = a.gs[1] * gs_mul;
        const int64_t nu = 64 * (int64_t)wtile + row - 64;
        const bool lv = LORA && a.lora.b1 != nullptr && nu < a.n_out;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          float uv = bf16_round(gsu * __uint_as_float(v[j]));
          if (lv && r0 + j < a.m) uv = lora_add(uv, a.lora.b1, a.lora.off1, a.lora, r0 + j, nu);
          U[j * 64 + (row - 64)] = uv;
        }
      }
      named_bar_sync(1 + g, 128);
      if (q < 2) {
        const float gsg = a.gs[0] * gs_mul;
        const int64_t ng = 64 * (int64_t)wtile + row;
        const bool lv = LORA && a.lora.b0 != nullptr && ng < a.n_out;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          float gv = bf16_round(gsg * __uint_as_float(v[j]));
          if (lv && r0 + j < a.m) gv = lora_add(gv, a.lora.b0, a.lora.off0, a.lora, r0 + j, ng);
          Hs[j * 64 + row] = f32_to_bf16_bits(silu_fast(gv) * U[j * 64 + row]);
        }
      }
      named_bar_sync(1 + g, 128);
      const int n0 = 64 * wtile;
      if (EPI == kEpiSiluMulQuant) {
        // thread et: activation row j = et / 4 of this chunk, 16-block b = et % 4
        const int j = et >> 2, b = et & 3;
        const int r = r0 + j, n = n0 + 16 * b;
        if (j < jmax && r < a.m && n < a.n_out) {
          float hv[16];
          float amax = 0.0f;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            hv[i] = bf16_bits_to_float(Hs[j * 64 + 16 * b + i]);
            amax = fmaxf(amax, fabsf(hv[i]));
          }
          const uint32_t s8 = e4m3_encode_satfinite(__fdiv_rn(amax, 6.0f));
          const uint2 c = e2m1_encode_block16(hv, e4m3_decode(s8), s8 == 0);
          *reinterpret_cast<uint2*>(a.q_codes + (size_t)r * (a.n_out / 2) + n / 2) = c;
          a.q_sf[sf_blocked_offset(r, n / 16, a.q_kc)] = (uint8_t)s8;
        }
      } else {
        for (int idx = et; idx < 32 * 8; idx += 128) {
          const int j = idx >> 3, ch = idx & 7;
          const int r = r0 + j, n = n0 + 8 * ch;
          if (j < jmax && r < a.m && n < a.n_out)
            *reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.out) + (size_t)r * a.ldo + n) =
                *reinterpret_cast<const uint4*>(Hs + j * 64 + 8 * ch);
        }
      }
      named_bar_sync(1 + g, 128);
    }
  }
}

template <int BN, int SXS, int XC, int SWS, int SA, int DQG, int UA, int NI, bool DQX, int EPI,
          bool LORA = false>
__global__ void __launch_bounds__(TcCfg<BN, SXS, XC, SWS, SA, DQG, UA, NI, DQX>::kThreads,
                                  TcCfg<BN, SXS, XC, SWS, SA, DQG, UA, NI, DQX>::kMinBlocks)
tc_w4a16_kernel(const __grid_constant__ CUtensorMap xmap, const TcArgs a) {
  using C = TcCfg<BN, SXS, XC, SWS, SA, DQG, UA, NI, DQX>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* xs = smem;
  uint8_t* wsm = smem + C::kSmemW;
  uint8_t* epi = smem;  // aliases the rings; used only after the last MMA
  uint64_t* xfull = reinterpret_cast<uint64_t*>(smem + C::kSmemBar);
  uint64_t* xempty = xfull + SXS;
  uint64_t* wfull = xempty + SXS;
  uint64_t* wempty = wfull + SWS;
  uint64_t* afull = wempty + SWS;
  uint64_t* aempty = afull + SA;
  uint64_t* accum = aempty + SA;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + NI);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* err = &g_ffn_device_error;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int xtile = blockIdx.x, wtile = blockIdx.y;
  const int kc0 = blockIdx.z * a.kc_per_split;
  const int nk = min(a.kc_total, kc0 + a.kc_per_split) - kc0;  // >= 1 by the plan
  const int nunits = (nk + UA - 1) / UA;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SXS; ++s) {
      mbar_init(&xfull[s], 1);
      mbar_init(&xempty[s], DQX ? 1 : NI);  // one commit per MMA thread using the stage
    }
    for (int s = 0; s < SWS; ++s) {
      mbar_init(&wfull[s], 1);
      mbar_init(&wempty[s], 4 * DQG);  // every dequant warp
    }
    for (int s = 0; s < SA; ++s) {
      mbar_init(&afull[s], 4);
      mbar_init(&aempty[s], 1);
    }
    for (int j = 0; j < NI; ++j) mbar_init(&accum[j], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 3 && lane == 0) tma_prefetch_desc(&xmap);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // The next kernel may be scheduled now; the weights streamed here do not
  // depend on the previous kernel, the activations and the output do.
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------- weight producer
    if (lane == 0) {
      const uint8_t* wsrc = a.wt + ((size_t)wtile * a.kc_total + kc0) * kChunkBytes;
      const int rounds = (nunits + DQG - 1) / DQG;
      int issued = 0;
      for (int r = 0; r < rounds; ++r) {
        const int s = r % SWS;
        const int nc = min(DQG * UA, nk - r * DQG * UA);
        if (r >= SWS && !mbar_wait(&wempty[s], ((r / SWS) - 1) & 1, abort_flag, err, 1)) break;
        mbar_arrive_expect_tx(&wfull[s], nc * kChunkBytes);
        bulk_load(wsm + s * C::kWStageBytes, wsrc + (size_t)r * C::kWStageBytes, nc * kChunkBytes,
                  &wfull[s]);
        ++issued;
      }
      // no copy into this CTA's shared memory may outlive it
      for (int r = max(0, issued - SWS); r < issued; ++r) wait_drain(&wfull[r % SWS], (r / SWS) & 1);
    }
  } else if (warp == 3) {
    // --------------------------------------------- activation producer
    if (lane == 0) {
      griddep_wait();  // the activations may come from the previous kernel
      const int stages = (nk + XC - 1) / XC;
      int issued = 0;
      for (int t = 0; t < stages; ++t) {
        const int s = t % SXS;
        const int nc = min(XC, nk - t * XC);
        if (t >= SXS && !mbar_wait(&xempty[s], ((t / SXS) - 1) & 1, abort_flag, err, 1)) break;
        mbar_arrive_expect_tx(&xfull[s], nc * a.x_box_rows * 128);
        for (int c = 0; c < nc; ++c)
          tma_load_2d(xs + s * C::kXStageBytes + c * BN * 128, &xmap, (kc0 + t * XC + c) * kChunkK,
                      xtile * BN, &xfull[s]);
        ++issued;
      }
      for (int t = max(0, issued - SXS); t < issued; ++t) wait_drain(&xfull[t % SXS], (t / SXS) & 1);
    }
  } else if (warp == 1 || (NI == 2 && warp == 2)) {
    // -------------------------------------------------- MMA issuer(s)
    if (lane == 0) {
      const int j = warp - 1;  // units u = j, j + NI, ...
      const uint32_t idesc = idesc_bf16_f32(kTileRows, BN);
      const uint32_t d = tmem + j * BN;  // this thread's accumulator
      constexpr int kUnitsPerX = XC / UA;
      for (int u = j; u < nunits; u += NI) {
        const int t = u / kUnitsPerX, sx = t % SXS, sa = u % SA;
        if (!DQX && u % kUnitsPerX == j && !mbar_wait(&xfull[sx], (t / SXS) & 1, abort_flag, err, 2))
          break;
        if (!mbar_wait(&afull[sa], (u / SA) & 1, abort_flag, err, 2)) break;
        tc_fence_after();
        const int nc = min(UA, nk - u * UA);
        for (int c = 0; c < nc; ++c) {
          const uint32_t a_base = tmem + C::kAColBase + C::kSlotCols * sa + 32 * c;
          const uint64_t b_base = smem_desc_sw128(
              smem_u32(xs + sx * C::kXStageBytes + ((u % kUnitsPerX) * UA + c) * BN * 128));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ts(d, a_base + 8 * kk, b_base + 2 * kk, idesc,
                        (u == j && c == 0 && kk == 0) ? 0u : 1u);
        }
        mma_commit(&aempty[sa]);
        if (DQX || u + NI >= (t + 1) * kUnitsPerX || u + NI >= nunits)
          mma_commit(&xempty[sx]);  // this thread's last unit of the stage
      }
      mma_commit(&accum[j]);  // fires once every MMA this thread issued has completed
    }
  } else if (warp >= 4) {
    // ------------------------------------------- dequant, then epilogue
    const int g = (warp - 4) >> 2;                // dequant warpgroup
    const int q = warp & 3;                       // TMEM lane quarter
    const int row = 32 * q + lane;                // tile row == TMEM lane
    const uint32_t lane_addr = (uint32_t)(32 * q) << 16;
    const int sf_off = 16 * lane + 4 * q;         // this row's 4 scale bytes (block layout)
    for (int u = g; u < nunits; u += DQG) {
      const int r = u / DQG, sw = r % SWS, sa = u % SA;
      if (u >= SA) {  // the MMAs that read this TMEM slot SA units ago are done
        const bool ok = mbar_wait(&aempty[sa], ((u / SA) - 1) & 1, abort_flag, err, 4);
        if (!__all_sync(0xffffffffu, ok)) break;
        tc_fence_after();
      }
      const bool ok = mbar_wait(&wfull[sw], (r / SWS) & 1, abort_flag, err, 4);
      if (!__all_sync(0xffffffffu, ok)) break;  // stay converged for tcgen05.st
      const uint8_t* wu = wsm + sw * C::kWStageBytes + g * C::kUnitBytes;
      const int nc = min(UA, nk - u * UA);
      for (int c = 0; c < nc; ++c) {
        const uint8_t* w = wu + c * kChunkBytes;
        const uint4 lo = *reinterpret_cast<const uint4*>(w + 16 * row);
        const uint4 hi = *reinterpret_cast<const uint4*>(w + 2048 + 16 * row);
        const uint32_t sc = *reinterpret_cast<const uint32_t*>(w + 4096 + sf_off);
        uint32_t v[32];
        dequant64_w4a16(lo, hi, sc, v);
        tmem_st32(tmem + lane_addr + C::kAColBase + C::kSlotCols * sa + 32 * c, v);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&wempty[sw]);   // the shared-memory stage may be refilled
      if (DQX) {  // the unit's activations, on the MMA thread's behalf
        const bool okx = mbar_wait(&xfull[u % SXS], (u / SXS) & 1, abort_flag, err, 4);
        if (!__all_sync(0xffffffffu, okx)) break;
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&afull[sa]);
    }
    bool done = true;
    for (int j = 0; j < NI; ++j) done = wait_drain(&accum[j], 0) && done;
    done = __all_sync(0xffffffffu, done);
    tc_fence_after();
    griddep_wait();  // the previous kernel may still read the output buffer
    if (done && !*abort_flag)
      epilogue_tile<BN, EPI, DQG, NI, LORA>(a, tmem, q, lane, g, epi + g * C::kEpiBytes, xtile, wtile,
                                      min(NI, nunits), kW4A16Unscale);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Persistent narrow-tile W4A16 projection (m <= 64, one activation tile): the
// two projections of an FFN layer for few rows, each one launch.  Every CTA
// walks a list of segments -- (weight tile, range of 64-element K chunks) --
// with its pipelines running straight through from one segment to the next
// (the rings are indexed by the CTA's global unit count), so the weight
// stream never stops at a tile boundary and each CTA pays its prologue once.
//  * kModeTiles (the fused gate+up weight): the tiles are dealt round-robin
//    to the CTAs, each whole (all K chunks); the epilogue of each tile writes
//    h = bf16(silu(bf16 g) * bf16 u).  After its griddep_wait the kernel also
//    zeroes the tile counters of the projection that follows it in the
//    stream (the down projection of the same layer).
//  * kModeRanges (the down projection, K = inter deep, few tiles): the
//    (tile, chunk) space is cut into one contiguous, equal range per CTA;
//    each segment's fp32 partial sums go to the workspace, slot (CTA + tile),
//    and the CTA whose segment completes a tile's count (an atomic counter,
//    zeroed by the preceding gate+up kernel) adds that tile's partials in K
//    order -- a fixed order, whichever CTA finishes last -- and writes
//    out = bf16(gs * sum).  No separate reduction launch.
// ---------------------------------------------------------------------------
enum : int { kModeTiles = 0, kModeRanges = 1 };

struct PArgs {
  const uint8_t* wt;   // tiled weight [ntiles][kc][4608] (W4A16 code arrangement)
  const float* gs;     // tensor scale(s)
  uint16_t* out;       // bf16 [m, ldo]
  int m, n_out, ldo, kc, ntiles, x_box_rows;
  float* partials;     // kModeRanges: [gridDim.x + ntiles][m][128]
  int* counters;       // kModeRanges: [ntiles], zero on entry
  int* zero_ptr;       // kModeTiles: counters of the next projection (or null)
  int zero_count;
  LoraArgs lora;       // adapter deltas added to the bf16 outputs
};

struct Seg {
  int tile, c0, nk;
};

// Segment j of this CTA; false once there are no more.  kModeRanges needs
// ntiles * kc >= gridDim.x (the host sizes the grid so).
template <int MODE>
__device__ __forceinline__ bool cta_segment(const PArgs& a, int j, Seg& s) {
  const int G = gridDim.x, g = blockIdx.x;
  if (MODE == kModeTiles) {
    const int t = g + j * G;
    if (t >= a.ntiles) return false;
    s.tile = t;
    s.c0 = 0;
    s.nk = a.kc;
    return true;
  }
  const int64_t W = (int64_t)a.ntiles * a.kc;
  const int64_t lo = W * g / G, hi = W * (g + 1) / G;
  const int t = (int)(lo / a.kc) + j;
  const int64_t b = lo > (int64_t)t * a.kc ? lo : (int64_t)t * a.kc;
  const int64_t e = hi < (int64_t)(t + 1) * a.kc ? hi : (int64_t)(t + 1) * a.kc;
  if (b >= e) return false;
  s.tile = t;
  s.c0 = (int)(b - (int64_t)t * a.kc);
  s.nk = (int)(e - b);
  return true;
}

// kModeRanges: the CTA that owns unit u of the flattened (tile, chunk) space.
__device__ __forceinline__ int range_owner(int64_t u, int64_t W, int G) {
  return (int)(((u + 1) * G - 1) / W);
}

// Shared-memory layout of the persistent kernel: the rings (as TcCfg), the
// barriers, then DQG epilogue buffers of 8 KB that do not alias the rings
// (the epilogue of a segment runs while the next segment streams in).
template <int BN, int SXS, int XC, int SWS, int SA, int DQG, int NI>
struct PCfg {
  using C = TcCfg<BN, SXS, XC, SWS, SA, DQG, 1, NI, false>;
  static constexpr int kBarBytes = (C::kNumBars + 1) * 8 + 32;  // + accfree; TMEM slot, flags
  static constexpr int kEpiOff = (C::kSmemRings + kBarBytes + 127) / 128 * 128;
  static constexpr int kSmemAlloc = kEpiOff + DQG * 8192 + 1024;
  static_assert(kSmemAlloc <= 232448, "shared memory budget");
  static_assert(BN <= 64, "one activation tile of at most 64 rows");
};

template <int BN, int SXS, int XC, int SWS, int SA, int DQG, int NI, int MODE>
__global__ void __launch_bounds__(TcCfg<BN, SXS, XC, SWS, SA, DQG, 1, NI, false>::kThreads, 1)
tc_w4a16_persistent_kernel(const __grid_constant__ CUtensorMap xmap, const PArgs a) {
  using C = TcCfg<BN, SXS, XC, SWS, SA, DQG, 1, NI, false>;
  using PC = PCfg<BN, SXS, XC, SWS, SA, DQG, NI>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* xs = smem;
  uint8_t* wsm = smem + C::kSmemW;
  uint64_t* xfull = reinterpret_cast<uint64_t*>(smem + C::kSmemBar);
  uint64_t* xempty = xfull + SXS;
  uint64_t* wfull = xempty + SXS;
  uint64_t* wempty = wfull + SWS;
  uint64_t* afull = wempty + SWS;
  uint64_t* aempty = afull + SA;
  uint64_t* accfull = aempty + SA;        // NI barriers: one per MMA thread
  uint64_t* accfree = accfull + NI;       // 1 barrier: the epilogue has read the accumulators
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accfree + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);
  int* err = &g_ffn_device_error;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // units (= chunks) of this CTA over all its segments
  int total = 0, nseg = 0;
  {
    Seg sg;
    while (cta_segment<MODE>(a, nseg, sg)) {
      total += sg.nk;
      ++nseg;
    }
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < SXS; ++s) {
      mbar_init(&xfull[s], 1);
      mbar_init(&xempty[s], NI);
    }
    for (int s = 0; s < SWS; ++s) {
      mbar_init(&wfull[s], 1);
      mbar_init(&wempty[s], 4 * DQG);
    }
    for (int s = 0; s < SA; ++s) {
      mbar_init(&afull[s], 4);
      mbar_init(&aempty[s], 1);
    }
    for (int j = 0; j < NI; ++j) mbar_init(&accfull[j], 1);
    mbar_init(accfree, 4 * DQG);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 3 && lane == 0) tma_prefetch_desc(&xmap);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------- weight producer
    if (lane == 0) {
      int u = 0, issued_rounds = 0;
      bool ok = true;
      Seg sg;
      for (int j = 0; ok && cta_segment<MODE>(a, j, sg); ++j) {
        const uint8_t* src = a.wt + ((size_t)sg.tile * a.kc + sg.c0) * kChunkBytes;
        for (int c = 0; c < sg.nk; ++c, ++u) {
          const int r = u / DQG, slot = u % DQG, st = r % SWS;
          if (slot == 0) {
            if (r >= SWS && !mbar_wait(&wempty[st], ((r / SWS) - 1) & 1, abort_flag, err, 1)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&wfull[st], min(DQG, total - u) * kChunkBytes);
            ++issued_rounds;
          }
          bulk_load(wsm + st * C::kWStageBytes + slot * kChunkBytes, src + (size_t)c * kChunkBytes,
                    kChunkBytes, &wfull[st]);
        }
      }
      for (int r = max(0, issued_rounds - SWS); r < issued_rounds; ++r)
        wait_drain(&wfull[r % SWS], (r / SWS) & 1);
    }
  } else if (warp == 3) {
    // --------------------------------------------- activation producer
    if (lane == 0) {
      griddep_wait();  // x (or h) comes from the previous kernel
      if (MODE == kModeTiles)
        for (int i = blockIdx.x; i < a.zero_count; i += gridDim.x) a.zero_ptr[i] = 0;
      int u = 0, issued = 0;
      bool ok = true;
      Seg sg;
      for (int j = 0; ok && cta_segment<MODE>(a, j, sg); ++j) {
        for (int c = 0; c < sg.nk; ++c, ++u) {
          const int t = u / XC, pos = u % XC, st = t % SXS;
          if (pos == 0) {
            if (t >= SXS && !mbar_wait(&xempty[st], ((t / SXS) - 1) & 1, abort_flag, err, 1)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&xfull[st], min(XC, total - u) * a.x_box_rows * 128);
            ++issued;
          }
          tma_load_2d(xs + st * C::kXStageBytes + pos * BN * 128, &xmap, (sg.c0 + c) * kChunkK, 0,
                      &xfull[st]);
        }
      }
      for (int t = max(0, issued - SXS); t < issued; ++t) wait_drain(&xfull[t % SXS], (t / SXS) & 1);
    }
  } else if (warp == 1 || (NI == 2 && warp == 2)) {
    // -------------------------------------------------- MMA issuer(s)
    if (lane == 0) {
      const int jt = warp - 1;  // units u with u % NI == jt
      const uint32_t idesc = idesc_bf16_f32(kTileRows, BN);
      const uint32_t d = tmem + jt * BN;
      int u = 0;
      bool ok = true;
      Seg sg;
      for (int j = 0; ok && cta_segment<MODE>(a, j, sg); ++j) {
        if (j > 0 && !mbar_wait(accfree, (j - 1) & 1, abort_flag, err, 2)) break;
        tc_fence_after();
        bool first = true;
        for (int c = 0; c < sg.nk; ++c, ++u) {
          if (u % NI != jt) continue;
          const int t = u / XC, sx = t % SXS, sa = u % SA;
          if (u % XC == jt && !mbar_wait(&xfull[sx], (t / SXS) & 1, abort_flag, err, 2)) {
            ok = false;
            break;
          }
          if (!mbar_wait(&afull[sa], (u / SA) & 1, abort_flag, err, 2)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = tmem + C::kAColBase + C::kSlotCols * sa;
          const uint64_t b_base = smem_desc_sw128(smem_u32(xs + sx * C::kXStageBytes + (u % XC) * BN * 128));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ts(d, a_base + 8 * kk, b_base + 2 * kk, idesc, (first && kk == 0) ? 0u : 1u);
          first = false;
          mma_commit(&aempty[sa]);
          if (u + NI >= (t + 1) * XC || u + NI >= total) mma_commit(&xempty[sx]);
        }
        mma_commit(&accfull[jt]);  // this segment's MMAs of this thread are complete
      }
    }
  } else if (warp >= 4) {
    // ------------------------------- dequant, then each segment's epilogue
    const int g = (warp - 4) >> 2;
    const int q = warp & 3;
    const int row = 32 * q + lane;
    const int tid = threadIdx.x - 128;  // 0 .. 128 * DQG - 1
    const uint32_t lane_addr = (uint32_t)(32 * q) << 16;
    const int sf_off = 16 * lane + 4 * q;
    int u = 0;
    bool ok = true;
    bool waited = false;
    Seg sg;
    for (int j = 0; ok && cta_segment<MODE>(a, j, sg); ++j) {
      const int u0 = u;
      for (int c = 0; c < sg.nk; ++c, ++u) {
        if (u % DQG != g) continue;
        const int r = u / DQG, sw = r % SWS, sa = u % SA;
        if (u >= SA) {
          const bool okw = mbar_wait(&aempty[sa], ((u / SA) - 1) & 1, abort_flag, err, 4);
          if (!__all_sync(0xffffffffu, okw)) { ok = false; break; }
          tc_fence_after();
        }
        const bool okw = mbar_wait(&wfull[sw], (r / SWS) & 1, abort_flag, err, 4);
        if (!__all_sync(0xffffffffu, okw)) { ok = false; break; }
        const uint8_t* w = wsm + sw * C::kWStageBytes + g * kChunkBytes;
        const uint4 lo = *reinterpret_cast<const uint4*>(w + 16 * row);
        const uint4 hi = *reinterpret_cast<const uint4*>(w + 2048 + 16 * row);
        const uint32_t sc = *reinterpret_cast<const uint32_t*>(w + 4096 + sf_off);
        uint32_t v[32];
        dequant64_w4a16(lo, hi, sc, v);
        tmem_st32(tmem + lane_addr + C::kAColBase + C::kSlotCols * sa, v);
        __syncwarp();
        if (lane == 0) mbar_arrive(&wempty[sw]);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&afull[sa]);
      }
      if (!ok) break;
      // ---- epilogue of segment j: accumulators -> h, or partials (+ finalise)
      bool done = true;
      for (int jt = 0; jt < NI; ++jt) done = mbar_wait(&accfull[jt], j & 1, abort_flag, err, 8) && done;
      done = __all_sync(0xffffffffu, done);
      tc_fence_after();
      if (!waited) {
        griddep_wait();  // the previous kernel may still read this kernel's outputs
        waited = true;
      }
      if (!done || *abort_flag) { ok = false; break; }
      // accumulator jt holds units u0 + i with (u0 + i) % NI == jt, i < nk
      unsigned used = 0;
      for (int jt = 0; jt < NI; ++jt)
        if (((jt - u0) % NI + NI) % NI < sg.nk) used |= 1u << jt;
      const int cols = min(a.m, BN);
      if (MODE == kModeTiles) {
        // gate rows 0..63 and up rows 64..127 of tile t: h[:, 64t + row]
        float* U = reinterpret_cast<float*>(smem + PC::kEpiOff) + g * 2048;  // [32][64]
        for (int c = g; c * 32 < cols; c += DQG) {
          const int jmax = min(32, cols - 32 * c);
          float acc[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) acc[i] = 0.0f;
          for (int jt = 0; jt < NI; ++jt) {
            if (!(used >> jt & 1)) continue;
            uint32_t v0[16], v1[16];
            tmem_ld16(tmem + lane_addr + jt * BN + 32 * c, v0);
            if (BN - 32 * c > 16) tmem_ld16(tmem + lane_addr + jt * BN + 32 * c + 16, v1);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              acc[i] += __uint_as_float(v0[i]);
              if (BN - 32 * c > 16) acc[16 + i] += __uint_as_float(v1[i]);
            }
          }
          // rows 64..127 (up) hand bf16(gs_u * u) to rows 0..63 (gate)
          if (q >= 2) {
            const float gsu = a.gs[1] * kW4A16Unscale;
            const int nu = 64 * sg.tile + row - 64;
            const bool lv = a.lora.b1 != nullptr && nu < a.n_out;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              float uv = bf16_round(gsu * acc[i]);
              if (lv && i < jmax) uv = lora_add(uv, a.lora.b1, a.lora.off1, a.lora, 32 * c + i, nu);
              U[i * 64 + (row - 64)] = uv;
            }
          }
          named_bar_sync(1 + g, 128);
          if (q < 2) {
            const float gsg = a.gs[0] * kW4A16Unscale;
            const int n = 64 * sg.tile + row;
            if (n < a.n_out) {
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                if (i < jmax) {
                  float gv = bf16_round(gsg * acc[i]);
                  if (a.lora.b0) gv = lora_add(gv, a.lora.b0, a.lora.off0, a.lora, 32 * c + i, n);
                  a.out[(size_t)(32 * c + i) * a.ldo + n] = f32_to_bf16_bits(silu_fast(gv) * U[i * 64 + row]);
                }
              }
            }
          }
          named_bar_sync(1 + g, 128);
        }
      } else {
        // this segment's partial sums -> slot (CTA + tile), rows [act row][tile row]
        float* P = a.partials + (size_t)(blockIdx.x + sg.tile) * a.m * kTileRows;
        for (int c = g; c * 32 < cols; c += DQG) {
          const int jmax = min(32, cols - 32 * c);
          float acc[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) acc[i] = 0.0f;
          for (int jt = 0; jt < NI; ++jt) {
            if (!(used >> jt & 1)) continue;
            uint32_t v0[16], v1[16];
            tmem_ld16(tmem + lane_addr + jt * BN + 32 * c, v0);
            if (BN - 32 * c > 16) tmem_ld16(tmem + lane_addr + jt * BN + 32 * c + 16, v1);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              acc[i] += __uint_as_float(v0[i]);
              if (BN - 32 * c > 16) acc[16 + i] += __uint_as_float(v1[i]);
            }
          }
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (i < jmax) P[(size_t)(32 * c + i) * kTileRows + row] = acc[i];
        }
        __threadfence();
        named_bar_sync(1 + DQG, 128 * DQG);
        if (tid == 0) {
          const int64_t W = (int64_t)a.ntiles * a.kc;
          const int G = gridDim.x;
          const int g0 = range_owner((int64_t)sg.tile * a.kc, W, G);
          const int g1 = range_owner((int64_t)sg.tile * a.kc + a.kc - 1, W, G);
          *last_flag = atomicAdd(&a.counters[sg.tile], 1) == g1 - g0 ? 1 : 0;
        }
        named_bar_sync(1 + DQG, 128 * DQG);
        if (*last_flag) {
          __threadfence();
          const int64_t W = (int64_t)a.ntiles * a.kc;
          const int G = gridDim.x;
          const int g0 = range_owner((int64_t)sg.tile * a.kc, W, G);
          const int g1 = range_owner((int64_t)sg.tile * a.kc + a.kc - 1, W, G);
          const float gsd = a.gs[0] * kW4A16Unscale;
          for (int idx = tid; idx < a.m * kTileRows; idx += 128 * DQG) {
            const int jr = idx / kTileRows, rr = idx % kTileRows;
            const int n = kTileRows * sg.tile + rr;
            float sum = 0.0f;
            for (int gg = g0; gg <= g1; ++gg)
              sum += __ldcg(a.partials + ((size_t)(gg + sg.tile) * a.m + jr) * kTileRows + rr);
            if (n < a.n_out) {
              float y = gsd * sum;
              if (a.lora.b0) y = lora_add(bf16_round(y), a.lora.b0, a.lora.off0, a.lora, jr, n);
              a.out[(size_t)jr * a.ldo + n] = f32_to_bf16_bits(y);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(accfree);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Fixed-format (W4A4) projection on the block-scaled FP4 tensor core
// ("metrale_model_layers/layers/dense_ffn_fixed.rs", forward_fixed: the
// nvfp4_proj_mx projections).  D[n, r] = sum_k (wq * sw)[n, k] (xq * sx)[r, k]
// with kind::mxf4nvf4 (E2M1 x E2M1, UE4M3 scale per 16 elements, fp32 in TMEM).
//  * A = weights: the same 4608-byte tiled chunks as above, read by one bulk
//    copy per stage of kW4Chunks chunks; the codes are the no-swizzle K-major
//    operand (16-byte rows, 8-row groups 128 B apart, second K half 2048 B
//    away) and the chunk's 512-byte scale block is copied to TMEM as SFA;
//  * B = quantised activations: codes [m, K/2] by 2-D TMA (128-byte rows of
//    256 elements, 128-byte swizzle), scale blocks (one 512-byte block per
//    128 rows and 64 elements, written by the activation quantiser) by bulk
//    copy, copied to TMEM as SFB;
//  * the K split and the K order depend only on (n, K), never on m, and every
//    output column of an MMA depends only on its own activation row, so a
//    row's result is the same whatever m is;
//  * one activation tile per CTA, 128 rows (MMA N = 128, a 3-stage ring of
//    36 KB stages) or 16 rows for m <= 16 (N = 16, 5 stages of 22.5 KB), and
//    two CTAs per SM: one CTA's epilogue overlaps the other's main loop, the
//    few-row grids stream every weight tile at once instead of in waves, and
//    the next kernel's CTAs find room beside this one's as soon as one of
//    them ends.
// ---------------------------------------------------------------------------
constexpr int kW4BN = 128;        // activation rows per tile
constexpr int kW4BNSmall = 16;    // activation rows per tile for m <= 16
constexpr int kW4Chunks = 4;      // 64-element chunks per stage

// XT activation tiles per CTA would share each weight stage (one MMA per tile
// and chunk, an accumulator each; every activation row stays the N column of
// an MMA with the same K order, so XT changes no result bit); the shapes in
// use take one tile (XT = 1), which lets two CTAs share an SM.
template <int XT, int BN, int S>
struct W4Cfg {
  static constexpr int kStages = S;
  static constexpr int kWBytes = kW4Chunks * kChunkBytes;  // 18432
  static constexpr int kXBytes = BN * 128;                 // BN rows x 256 elements
  static constexpr int kSfbBytes = kW4Chunks * 512;        // 2048
  static constexpr int kStageBytes = kWBytes + XT * (kXBytes + kSfbBytes);
  static constexpr int kSmemEpi = kStages * kStageBytes;
  static constexpr int kSmemBar = kSmemEpi + (kSmemEpi >= 16384 ? 0 : 16384);
  static constexpr int kSmemBytes = kSmemBar + (2 * kStages + 1) * 8 + 16;
  static constexpr int kSmemAlloc = kSmemBytes + 1024;
  // TMEM columns: XT accumulators, then per activation tile (one MMA-issuing
  // warp each) its own copy of the weight scales, then its activation scales
  static constexpr int kSlotCols = 4 * kW4Chunks * kStages;
  static constexpr int kSfaCol = XT * BN < 32 ? 32 : XT * BN;
  static constexpr int kSfbCol = kSfaCol + XT * kSlotCols;
  static constexpr int kTmemCols = kSfbCol + XT * kSlotCols <= 256 ? 256 : 512;
  // two CTAs per SM when both fit (228 KB of shared memory, 512 TMEM columns)
  static constexpr int kMinBlocks = (2 * (kSmemAlloc + 1024) <= 233472 && kTmemCols <= 256) ? 2 : 1;
  static_assert(kSfbCol + XT * kSlotCols <= kTmemCols, "TMEM budget");
  static_assert(BN == kW4BN || XT == 1, "narrow tiles: one per CTA");
  static_assert(kStageBytes % 1024 == 0, "stage alignment");
  static_assert(kSmemAlloc <= 232448, "shared memory budget");
  static_assert(kSmemEpi >= 2 * 16384, "the two epilogue buffers alias the rings");
};

struct W4Args {
  TcArgs t;
  const uint8_t* sfb;   // activation scale blocks [ceil(m/128)][kc][512]
  int xtiles;           // activation tiles (of BN rows)
};

template <int EPI, int XT, int BN, int S>
__global__ void __launch_bounds__(256, W4Cfg<XT, BN, S>::kMinBlocks)
tc_w4a4_kernel(const __grid_constant__ CUtensorMap xmap, const W4Args w4) {
  using C = W4Cfg<XT, BN, S>;
  const TcArgs& a = w4.t;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* epi = smem;  // aliases the rings; used only after the last MMA
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kSmemBar);
  uint64_t* empty = full + S;
  uint64_t* accum = empty + S;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* err = &g_ffn_device_error;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int xt0 = blockIdx.x * XT, wtile = blockIdx.y;
  const int nxt = min(XT, w4.xtiles - xt0);                        // activation tiles of this CTA
  const int kc0 = blockIdx.z * a.kc_per_split;
  const int nk = min(a.kc_total, kc0 + a.kc_per_split) - kc0;     // chunks of this CTA
  const int nstage = (nk + kW4Chunks - 1) / kW4Chunks;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], nxt);  // one commit per MMA-issuing warp
    }
    mbar_init(accum, nxt);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&xmap);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      const uint8_t* wsrc = a.wt + ((size_t)wtile * a.kc_total + kc0) * kChunkBytes;
      auto stage_bytes = [&](int i) {
        const int nch = min(kW4Chunks, nk - kW4Chunks * i);
        return (uint32_t)(nch * kChunkBytes + nxt * (nch * 512 + a.x_box_rows * 128));
      };
      // the first ring's weights do not depend on the previous kernel: stream
      // them before waiting for it (the activation codes and scales do)
      const int pre = min(nstage, S);
      for (int i = 0; i < pre; ++i) {
        const int nch = min(kW4Chunks, nk - kW4Chunks * i);
        mbar_arrive_expect_tx(&full[i], stage_bytes(i));
        bulk_load(smem + i * C::kStageBytes, wsrc + (size_t)kW4Chunks * i * kChunkBytes, nch * kChunkBytes,
                  &full[i]);
      }
      griddep_wait();
      int issued = 0;
      for (int i = 0; i < nstage; ++i) {
        const int s = i % S;
        const int nch = min(kW4Chunks, nk - kW4Chunks * i);
        uint8_t* st = smem + s * C::kStageBytes;
        if (i >= pre) {
          if (!mbar_wait(&empty[s], ((i / S) - 1) & 1, abort_flag, err, 1)) break;
          mbar_arrive_expect_tx(&full[s], stage_bytes(i));
          bulk_load(st, wsrc + (size_t)kW4Chunks * i * kChunkBytes, nch * kChunkBytes, &full[s]);
        }
        for (int t = 0; t < nxt; ++t) {
          uint8_t* xt = st + C::kWBytes + t * (C::kXBytes + C::kSfbBytes);
          tma_load_2d(xt, &xmap, 32 * (kc0 + kW4Chunks * i), (xt0 + t) * BN, &full[s]);
          // (scale blocks cover 128 rows; a narrow tile is the only one: m <= BN)
          bulk_load(xt + C::kXBytes,
                    w4.sfb + ((size_t)(xt0 + t) * a.kc_total + kc0 + kW4Chunks * i) * 512, nch * 512, &full[s]);
        }
        ++issued;
      }
      for (int i = max(0, issued - S); i < issued; ++i) wait_drain(&full[i % S], (i / S) & 1);
    }
  } else if ((warp == 1 || warp == 3) && lane == 0 && (warp == 1 ? 0 : 1) < nxt) {
    // MMA issuers: warp 1 for activation tile 0, warp 3 for tile 1 (two
    // tcgen05 instruction streams; one thread's issue rate is the limit),
    // each with its own copy of the weight scales
    const int t = warp == 1 ? 0 : 1;
    const uint32_t idesc = idesc_mxf4nvf4(kTileRows, BN);
    const uint32_t sfa0 = tmem + C::kSfaCol + t * C::kSlotCols, sfb0 = tmem + C::kSfbCol + t * C::kSlotCols;
    for (int i = 0; i < nstage; ++i) {
      const int s = i % S;
      const int nch = min(kW4Chunks, nk - kW4Chunks * i);
      if (!mbar_wait(&full[s], (i / S) & 1, abort_flag, err, 2)) break;
      tc_fence_after();
      const uint8_t* st = smem + s * C::kStageBytes;
      const uint8_t* xt = st + C::kWBytes + t * (C::kXBytes + C::kSfbBytes);
      // the stage's scale copies first, then its MMAs
      for (int c = 0; c < nch; ++c) {
        const uint32_t slot = 4 * (s * kW4Chunks + c);
        tmem_cp_32x128b_x4(sfa0 + slot, smem_desc_interleave(smem_u32(st + c * kChunkBytes + 4096), 16, 128));
        tmem_cp_32x128b_x4(sfb0 + slot, smem_desc_interleave(smem_u32(xt + C::kXBytes + 512 * c), 16, 128));
      }
      for (int c = 0; c < nch; ++c) {
        const uint32_t slot = 4 * (s * kW4Chunks + c);
        mma_mxf4nvf4(tmem + t * BN, smem_desc_interleave(smem_u32(st + c * kChunkBytes), 2048, 128),
                     smem_desc_sw128(smem_u32(xt)) + 2 * c, idesc, sfa0 + slot, sfb0 + slot, (i | c) != 0 ? 1u : 0u);
      }
      mma_commit(&empty[s]);
    }
    mma_commit(accum);
  }
  // epilogue on all eight warps once the last MMA is done: warpgroup g takes
  // every other 32-row chunk of each activation tile (warp w reads TMEM
  // lanes 32 (w % 4) ..), each with its own 16 KB buffer
  __syncwarp();
  {
    const int q = warp & 3, g = warp < 4 ? 1 : 0;
    const bool done = __all_sync(0xffffffffu, wait_drain(accum, 0));
    tc_fence_after();
    griddep_wait();  // the previous kernel may still read this kernel's outputs
    if (done && !*abort_flag)
      for (int t = 0; t < nxt; ++t)
        epilogue_tile<BN, EPI, 2>(a, tmem + t * BN, q, lane, g, epi + g * 16384, xt0 + t, wtile);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Few-row W4A16 layer on the block-scaled FP4 tensor core.
//
// The NVFP4 weights go to tcgen05 kind::mxf4nvf4 as stored (natural tiled
// chunks: the codes are the A operand, the chunk's 512-byte scale block is
// SFA) -- no software dequantisation.  Each bf16 activation row becomes the B
// operand as P = 8 NVFP4 "planes", each one MMA column (N = 8m, at least 16):
// a 16-bit window of every 16-block's values, starting at the block's top
// bit, cut into 2-bit digits.  With E = floor(log2 max|x|) of the row and T
// the largest exponent in the block, an element x = M * 2^(e - 7) (M its
// 8-bit significand) is the integer A = M * 2^(e - T + 8) < 2^16 in units of
// 2^(T - 15), and plane p holds its digit d_p = (A >> (14 - 2p)) & 3 with the
// element's sign: E2M1 values 0, 1, 2, 3 (exact), block scale s = 2^(T - E +
// 8) (a power of two within E4M3's 2^-9..2^8 for T >= E - 17; smaller blocks
// are flushed), plane factor g_p = 2^(E - 2p - 9) applied in the epilogue,
// so that d_p * s * g_p = d_p * 2^(T - 2p - 1) and sum_p = A * 2^(T - 15) = x.
// Exact when every element of a block lies within 2^8 of the block's largest
// (the window holds all 8 significant bits); a smaller element loses the
// bits below 2^(T - 15) (truncation).  The digits of the 8 planes are
// independent of each other: no chain of residuals.  The epilogue folds the
// planes back, y[j] = sum_p g_p * D_j,p.
//
// One layer is two launches.  A small prologue kernel builds x's planes
// with one exponent per row (codes [m P][H/2], scale bytes [H/64][m P][4],
// E[m]) and zeroes the layer's counters.  Then one persistent kernel, two
// CTAs per SM, all resident, runs both projections:
//  * gate+up: whole tiles (gate rows 64t.., then the matching up rows), one
//    per CTA, when there are no more tiles than CTAs, else equal ranges of
//    the (tile, 64-element chunk) space with split-K partial sums that the
//    CTA completing a tile's count adds in K order.  The CTA that finishes
//    tile t computes h = bf16(silu(bf16 g) * bf16 u) for its 64 columns and
//    at once the planes of that 64-column chunk of h, with the chunk's own
//    exponent per row, then counts the tile as done;
//  * down: equal ranges of its (tile, chunk) space, started once every
//    gate+up tile is counted (one word, polled by one thread per CTA with a
//    back-off; no grid-wide barrier otherwise).  The copy warps re-base each
//    chunk's power-of-two scale bytes onto the row's largest chunk exponent
//    (kept with an atomic maximum), so a segment keeps one accumulator;
//    split-K partial sums as above.
// Each CTA's weight stream runs through both projections without a break.
// Every wait is bounded and raises a device error bit when it expires.
// ---------------------------------------------------------------------------
constexpr int kQChunks = 4;   // 64-element chunks per stage
constexpr int kQPlanes = 8;   // activation planes per row
constexpr int kSegZero = -1000;      // the row is all zero
constexpr int kSegNonFinite = 1000;  // the row holds an Inf or NaN

// Fixed configuration: up to two activation rows (N = 16 plane columns).
struct QCfg {
  static constexpr int kNT = 16;                          // MMA N
  static constexpr int kMR = kNT / kQPlanes;              // activation rows
  static constexpr int kXBytes = kNT * 128;               // 16 plane rows x 256 elements (128-byte swizzle)
  static constexpr int kStageBytes = kQChunks * kChunkBytes + kXBytes + kQChunks * 512;
  static constexpr int kStages = 4;
  static constexpr int kSmemMisc = kStages * kStageBytes;
  // misc: 16 words, Y [kMR][128] fp32 (a tile's sums)
  static constexpr int kSmemY = kSmemMisc + 64;
  static constexpr int kSmemBar = kSmemY + kMR * 128 * 4;
  static constexpr int kNumBars = 2 * kStages + 4;       // full, empty, accfull[2], accfree[2]
  static constexpr int kSmemAlloc = kSmemBar + kNumBars * 8 + 32 + 1024;
  // TMEM: two accumulator buffers (one accumulator per MMA-issuing warp in
  // each), then the scale-factor columns
  static constexpr int kIssuers = 2;
  static constexpr int kAccBuf = kIssuers * kNT;
  static constexpr int kSfaCol = 2 * kAccBuf;
  static constexpr int kSfbCol = kSfaCol + 4 * kQChunks * kStages;
  static constexpr int kTmemCols = 256;
  static_assert(kSfbCol + 4 * kQChunks * kStages <= kTmemCols, "TMEM budget");
  static_assert(kStageBytes % 1024 == 0, "stage alignment (128-byte swizzle)");
  static_assert(2 * (kSmemAlloc + 1024) <= 233472, "two CTAs per SM");
};

// 2^k as fp32 (exact; built from the exponent bits in the normal range).
__device__ __forceinline__ float exp2i(int k) {
  return k >= -126 && k <= 127 ? __int_as_float((k + 127) << 23) : ldexpf(1.0f, k);
}

// Row exponent from the largest |bf16| bit pattern of the row.
__device__ __forceinline__ int row_exponent(uint32_t max_bits) {
  return max_bits == 0 ? kSegZero : max_bits >= 0x7f80u ? kSegNonFinite : ilogbf(bf16_bits_to_float(max_bits));
}

// log2 of plane p's factor g_p for a row (or chunk) exponent E.
__device__ __forceinline__ int plane_log2_factor(int E, int p) { return E - 2 * p - 9; }

// The P planes of one 16-element block (the bit window described above), by
// the four lanes part = 0..3 of an aligned group of four (four elements each,
// v[0..3] = elements 4 part ..; exact bf16 values; every lane of the warp
// calls).  Writes bytes 8 b + 2 part, +1 of plane row j P + p (rows of
// row_bytes) and, from part 0, the block's scale byte at [b / 4][rows][4] +
// b % 4 for every plane.
__device__ __forceinline__ void block_planes(const float (&v)[4], int E, bool valid, int part, int j, int b,
                                             uint8_t* codes, size_t row_bytes, uint8_t* sf, int rows) {
  // significand M and exponent e of each element (M = 0 for zero)
  uint32_t M[4], sgn[4];
  int ev[4], T = -1000;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t bits = __float_as_uint(v[i]);
    const uint32_t fe = (bits >> 23) & 0xffu, mant = (bits >> 16) & 0x7fu;
    sgn[i] = bits >> 31;
    M[i] = fe ? (0x80u | mant) : mant;  // bf16 subnormals: 0.mant * 2^-126
    ev[i] = fe ? (int)fe - 127 : -126;
    if (M[i]) T = max(T, ev[i]);
  }
  T = max(T, __shfl_xor_sync(0xffffffffu, T, 1));
  T = max(T, __shfl_xor_sync(0xffffffffu, T, 2));
  const int es = T - E + 8;  // block scale 2^es
  const bool keep = T > -1000 && es >= -9;
  const uint32_t s8 = !keep ? 0u : es >= -6 ? (uint32_t)(es + 7) << 3 : (1u << (es + 9));
  uint32_t A[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int sh = ev[i] - T + 8;  // <= 8
    A[i] = !keep || M[i] == 0 ? 0u : sh >= 0 ? M[i] << sh : (sh > -16 ? M[i] >> -sh : 0u);
  }
  if (valid) {
#pragma unroll
    for (int p = 0; p < kQPlanes; ++p) {
      uint32_t pair = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t d = (A[i] >> (14 - 2 * p)) & 3u;  // E2M1 code of d: 0, 2 (1.0), 4 (2.0), 5 (3.0)
        const uint32_t c = d ? ((0x5420u >> (4 * d)) & 0xfu) | (sgn[i] << 3) : 0u;
        pair |= c << (4 * i);
      }
      const int rowp = j * kQPlanes + p;
      *reinterpret_cast<uint16_t*>(codes + (size_t)rowp * row_bytes + 8 * b + 2 * part) = (uint16_t)pair;
      if (part == 0) sf[((size_t)(b >> 2) * rows + rowp) * 4 + (b & 3)] = (uint8_t)s8;
    }
  }
}

// Prologue: grid (m, ceil(K / 16 / 32)), 128 threads; CTA (j, c) builds the
// planes of blocks 32c .. 32c + 31 of row j (four threads per block) after
// finding the row's maximum (every CTA of the row finds the same E), CTA
// (j, 0) writes E[j], and the CTAs zero the next kernel's counters.  It lets
// the next kernel launch at once (that one waits for this one before reading
// anything it writes).
constexpr int kPlaneThreads = 128;
constexpr int kPlaneBlocksPerCta = kPlaneThreads / 4;
__global__ void __launch_bounds__(kPlaneThreads) planes_prologue_kernel(const uint16_t* __restrict__ x, int m, int K,
                                                                        uint8_t* __restrict__ codes,
                                                                        uint8_t* __restrict__ sf, int* __restrict__ E_out,
                                                                        int* zero_ptr, int zero_count) {
  griddep_launch_dependents();
  griddep_wait();  // x comes from the previous kernel, which may also still use the counters
  __shared__ uint32_t red[kPlaneThreads / 32];
  const int cta = blockIdx.x * gridDim.y + blockIdx.y;
  for (int i = cta * kPlaneThreads + threadIdx.x; i < zero_count; i += gridDim.x * gridDim.y * kPlaneThreads)
    zero_ptr[i] = 0;
  const int j = blockIdx.x;
  const uint16_t* row = x + (size_t)j * K;
  // the row's maximum |x|: eight bf16 per 16-byte load, eight independent
  // loads in flight per thread (|bf16| bit patterns order like the values)
  uint32_t mx = 0;
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
      for (int e = 0; e < 4; ++e) mx = max(mx, max(w[e] & 0x7fffu, (w[e] >> 16) & 0x7fffu));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  mx = max(max(red[0], red[1]), max(red[2], red[3]));
  const int E = row_exponent(mx);
  if (blockIdx.y == 0 && threadIdx.x == 0) E_out[j] = E;
  const int nb = K / 16;
  const int b = blockIdx.y * kPlaneBlocksPerCta + (threadIdx.x >> 2);
  const int part = threadIdx.x & 3;  // elements 4 part .. 4 part + 3 of the block
  const bool valid = b < nb;         // whole groups of four lanes share validity
  float v[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  if (valid && E != kSegNonFinite) {
    const uint2 w = *reinterpret_cast<const uint2*>(row + 16 * b + 4 * part);
    v[0] = bf16_bits_to_float(w.x & 0xffffu);
    v[1] = bf16_bits_to_float(w.x >> 16);
    v[2] = bf16_bits_to_float(w.y & 0xffffu);
    v[3] = bf16_bits_to_float(w.y >> 16);
  }
  block_planes(v, E, valid, part, j, b, codes, (size_t)K / 2, sf, m * kQPlanes);
}

struct LArgs {
  const uint8_t* wt_gu;  // natural tiled gate+up weight [gu_tiles][gu_kc][4608] (gate/up interleaved by 64)
  const uint8_t* wt_dn;  // natural tiled down weight [dn_tiles][dn_kc][4608]
  const float* gs_gu;    // gate and up tensor scales
  const float* gs_dn;
  const uint8_t* xq;     // x planes (prologue): codes [m P][H/2], scales [H/64][m P][4], E [m]
  const uint8_t* xs;
  const int* xe;
  uint8_t* hq;           // h planes: codes [m P][I/2], scales [I/64][m P][4], E [I/64][m]
  uint8_t* hs;
  int* he;
  uint16_t* out;         // bf16 [m, H]
  float* part_gu;        // split-K partial sums [gu_parts + gu_tiles][m][128]
  float* part_dn;        // [gridDim.x + dn_tiles][m][128]
  int* cnt_gu;           // [gu_tiles] chunks done, zero on entry
  int* cnt_dn;           // [dn_tiles]
  uint32_t* gu_done;     // gate+up tiles whose h planes are written, zero on entry
  int* he_max;           // [m] largest chunk exponent of h per row, + 1001 (0: none yet), zero on entry
  int m, hidden, inter, gu_tiles, gu_kc, gu_parts, dn_tiles, dn_kc;
};

// Segment j of part g's equal share of the (tile, chunk) space split into
// `parts` shares (parts * tiles * kc < 2^32, checked by the host).
__device__ __forceinline__ bool range_segment(int ntiles, int kc, int parts, int g, int j, Seg& s) {
  if (g >= parts) return false;
  const uint32_t W = (uint32_t)ntiles * kc;
  const uint32_t lo = W * (uint32_t)g / parts, hi = W * (uint32_t)(g + 1) / parts;
  const uint32_t t = lo / kc + j;
  const uint32_t b = max(lo, t * kc), e = min(hi, (t + 1) * kc);
  if (b >= e) return false;
  s.tile = (int)t;
  s.c0 = (int)(b - t * kc);
  s.nk = (int)(e - b);
  return true;
}

__device__ __forceinline__ bool q_segment(const LArgs& a, int ph, int j, Seg& s) {
  return ph ? range_segment(a.dn_tiles, a.dn_kc, gridDim.x, blockIdx.x, j, s)
            : range_segment(a.gu_tiles, a.gu_kc, a.gu_parts, blockIdx.x, j, s);
}

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Bounded wait until *ctr reaches `target`, polling with a back-off (one
// thread per CTA polls one word).
__device__ __forceinline__ bool wait_count(const uint32_t* ctr, uint32_t target, volatile int* abort, int* err) {
  const long long t0 = clock64();
  for (;;) {
    if ((uint32_t)ld_acquire(reinterpret_cast<const int*>(ctr)) >= target) return true;
    if (*abort) return false;
    if (clock64() - t0 > kWaitLimitCycles) {
      *abort = 1;
      atomicOr(err, 32);
      return false;
    }
    __nanosleep(256);
  }
}

// Row exponent of h: the largest chunk exponent (stored + 1001; 0 = none).
__device__ __forceinline__ int he_row(const int* he_max, int jr) {
  const int v = __ldcg(he_max + jr);
  return v == 0 ? kSegZero : v - 1001;
}

// Sum of the split-K partial slots of tile t (CTAs g0..g1 of `parts` that
// own a non-empty share of it), in K order; the loads of eight slots at a
// time are in flight together (one L2 round trip instead of eight).
__device__ __forceinline__ float sum_partials(const float* part, int m, int jr, int rr, int t, uint32_t W, int parts,
                                              int g0, int g1) {
  float sum = 0.0f;
  for (int g = g0; g <= g1; g += 8) {
    float v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int gg = g + k;
      v[k] = gg <= g1 && W * (uint32_t)gg / parts != W * (uint32_t)(gg + 1) / parts
                 ? __ldcg(part + ((size_t)(gg + t) * m + jr) * kTileRows + rr)
                 : 0.0f;
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) sum += v[k];  // (+0 for an empty share: the sum never is -0)
  }
  return sum;
}

constexpr int kLayerThreads = 288;  // 9 warps
__global__ void __launch_bounds__(kLayerThreads, 2) tc_planes_layer_kernel(const LArgs a) {
  using C = QCfg;
  constexpr int S = C::kStages, P = kQPlanes, MR = C::kMR, NT = C::kNT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  int* misc = reinterpret_cast<int*>(smem + C::kSmemMisc);
  volatile int* sh_fail = misc;            // [2] epilogue stop flags by segment parity
  volatile int* last_flag = misc + 2;
  volatile int* sh_ready = misc + 3;      // the down phase's inputs are final
  float* Y = reinterpret_cast<float*>(smem + C::kSmemY);  // [MR][128] a finished tile's sums
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kSmemBar);
  uint64_t* empty = full + S;
  uint64_t* accfull = empty + S;   // [2]
  uint64_t* accfree = accfull + 2; // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accfree + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* err = &g_ffn_device_error;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rows = a.m * P;  // plane rows in use

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 2);  // the weights' expect_tx arrival + the stage's operand warp
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accfull[b], C::kIssuers);
      mbar_init(&accfree[b], 4);
    }
    *abort_flag = 0;
    sh_fail[0] = sh_fail[1] = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------- weight producer
    // (weights never depend on the previous kernel: no wait; gate+up then
    // down without a break)
    if (lane == 0) {
      int st_i = 0;
      bool ok = true;
      for (int ph = 0; ph < 2 && ok; ++ph) {
        const uint8_t* wt = ph ? a.wt_dn : a.wt_gu;
        const int kc = ph ? a.dn_kc : a.gu_kc;
        Seg sg;
        for (int j = 0; ok && q_segment(a, ph, j, sg); ++j) {
          for (int c = 0; c < sg.nk; c += kQChunks, ++st_i) {
            const int s = st_i % S, nch = min(kQChunks, sg.nk - c);
            if (st_i >= S && !mbar_wait(&empty[s], ((st_i / S) - 1) & 1, abort_flag, err, 1)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&full[s], nch * kChunkBytes);
            bulk_load(smem + s * C::kStageBytes, wt + ((size_t)sg.tile * kc + sg.c0 + c) * kChunkBytes,
                      nch * kChunkBytes, &full[s]);
          }
        }
      }
      for (int i = max(0, st_i - S); i < st_i; ++i) wait_drain(&full[i % S], (i / S) & 1);
    }
  } else if (warp == 1 || warp == 8) {
    // ---------------------- MMA issuers: warp 1 the even stages, warp 8 the
    // odd ones, each into its own accumulator of the segment's buffer (two
    // instruction streams: one thread's tcgen05 issue rate is the limit)
    // accumulator use u: one per segment
    if (lane == 0) {
      const int mi = warp == 1 ? 0 : 1;
      const uint32_t idesc = idesc_mxf4nvf4(kTileRows, NT);
      int st_i = 0, u = 0;
      bool ok = true;
      for (int ph = 0; ph < 2 && ok; ++ph) {
        Seg sg;
        for (int j = 0; ok && q_segment(a, ph, j, sg); ++j, ++u) {
          const int buf = u & 1;
          // every issuer waits for every segment's buffer (parity waits must
          // not skip a phase)
          if (u >= 2 && !mbar_wait(&accfree[buf], ((u >> 1) - 1) & 1, abort_flag, err, 2)) {
            ok = false;
            break;
          }
          tc_fence_after();
          bool first = true;
          for (int c = 0; c < sg.nk; c += kQChunks, ++st_i) {
            if ((st_i & 1) != mi) continue;
            const int s = st_i % S, nch = min(kQChunks, sg.nk - c);
            if (!mbar_wait(&full[s], (st_i / S) & 1, abort_flag, err, 2)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint8_t* st = smem + s * C::kStageBytes;
            const uint8_t* xs = st + kQChunks * kChunkBytes;
            const uint64_t b_base = smem_desc_sw128(smem_u32(xs));
            for (int cc = 0; cc < nch; ++cc) {  // the stage's scale copies, then its MMAs
              const uint32_t slot = 4 * (s * kQChunks + cc);
              tmem_cp_32x128b_x4(tmem + C::kSfaCol + slot,
                                 smem_desc_interleave(smem_u32(st + cc * kChunkBytes + 4096), 16, 128));
              tmem_cp_32x128b_x4(tmem + C::kSfbCol + slot,
                                 smem_desc_interleave(smem_u32(xs + C::kXBytes + 512 * cc), 16, 128));
            }
            for (int cc = 0; cc < nch; ++cc) {
              const uint32_t slot = 4 * (s * kQChunks + cc);
              mma_mxf4nvf4(tmem + buf * C::kAccBuf + mi * NT,
                           smem_desc_interleave(smem_u32(st + cc * kChunkBytes), 2048, 128), b_base + 2 * cc, idesc,
                           tmem + C::kSfaCol + slot, tmem + C::kSfbCol + slot, (!first || cc != 0) ? 1u : 0u);
            }
            first = false;
            mma_commit(&empty[s]);
          }
          if (ok) mma_commit(&accfull[buf]);  // (also when this issuer had no stage in the segment)
        }
      }
    }
  } else if (warp < 4) {
    // ------- warps 2-3: each stage's B operand (plane codes, 128-byte
    // swizzle) and SFB, copied from the planes in global memory; warp 2
    // fills the even stages, warp 3 the odd ones, each with all of a
    // stage's loads in flight at once.  Down: once every h chunk of this
    // CTA's range is final, each chunk's scale bytes are re-based from its
    // own exponent E_c to the row's E = max E_c (2^-(E - E_c) times, exact
    // while the scale stays >= 2^-9; a smaller one is flushed to 0)
    constexpr int kMaxU = NT * 8 / 32;         // 16-byte code units per lane
    constexpr int kMaxW = NT * kQChunks / 32;  // scale words per lane
    const int pt = threadIdx.x - 64;
    const int mine = warp - 2;
    // plane rows >= m P stay zero (their MMA columns are never read)
    for (int s = 0; s < S; ++s)
      for (int i = pt; i < (C::kXBytes + kQChunks * 512) / 16; i += 64)
        reinterpret_cast<uint4*>(smem + s * C::kStageBytes + kQChunks * kChunkBytes)[i] = make_uint4(0, 0, 0, 0);
    named_bar_sync(2, 64);  // both warps zeroed before either fills
    griddep_wait();         // x's planes come from the prologue
    int st_i = 0;
    bool ok = true;
    for (int ph = 0; ph < 2; ++ph) {
      const uint8_t* q = ph ? a.hq : a.xq;
      const uint8_t* qs = ph ? a.hs : a.xs;
      const int K = ph ? a.inter : a.hidden;
      Seg sg;
      if (ph == 1) {
        // every h chunk is final once all gate+up tiles are counted: warp 2
        // polls, warp 3 waits at the barrier (both always reach it)
        if (mine == 0 && lane == 0) {
          const bool has_down = q_segment(a, 1, 0, sg);
          *sh_ready = ok && (!has_down || wait_count(a.gu_done, a.gu_tiles, abort_flag, err)) ? 1 : 0;
        }
        named_bar_sync(2, 64);
        if (!*sh_ready) ok = false;
      }
      for (int j = 0; ok && q_segment(a, ph, j, sg); ++j) {
        int eseg[MR];  // down: the row's exponent, E = max E_c over all chunks of h
#pragma unroll
        for (int jr = 0; jr < MR; ++jr) eseg[jr] = ph == 1 && jr < a.m ? he_row(a.he_max, jr) : kSegZero;
        for (int c = 0; c < sg.nk; c += kQChunks, ++st_i) {
          if ((st_i & 1) != mine) continue;
          const int s = st_i % S, nch = min(kQChunks, sg.nk - c);
          const int cg = sg.c0 + c;  // first chunk of the stage
          if (st_i >= S &&
              !__all_sync(0xffffffffu, mbar_wait(&empty[s], ((st_i / S) - 1) & 1, abort_flag, err, 4))) {
            ok = false;
            break;
          }
          uint8_t* xs = smem + s * C::kStageBytes + kQChunks * kChunkBytes;
          uint8_t* sfb = xs + C::kXBytes;
          // codes: 16-byte units (row, u) of the stage's 128-byte rows
          uint4 v[kMaxU];
#pragma unroll
          for (int k = 0; k < kMaxU; ++k) {
            const int i = lane + 32 * k, r = i >> 3, u = i & 7;
            const int byte = cg * 32 + 16 * u;
            v[k] = make_uint4(0, 0, 0, 0);
            if (r < rows && u < 2 * nch && byte < K / 2)
              v[k] = __ldcg(reinterpret_cast<const uint4*>(q + (size_t)r * (K / 2) + byte));
          }
          // scale bytes: four per (chunk, row), masked past K; down: with the
          // chunk's exponent
          uint32_t w[kMaxW];
          int ec[kMaxW];
#pragma unroll
          for (int k = 0; k < kMaxW; ++k) {
            const int i = lane + 32 * k, cc = i / rows, r = i - cc * rows;
            w[k] = 0;
            ec[k] = kSegZero;
            if (cc < nch) {
              const int kleft = K - 64 * (cg + cc);  // > 0
              w[k] = __ldcg(reinterpret_cast<const uint32_t*>(qs + ((size_t)(cg + cc) * rows + r) * 4));
              if (kleft < 64) w[k] &= (1u << (8 * (kleft / 16))) - 1u;
              if (ph == 1) ec[k] = __ldcg(a.he + (size_t)(cg + cc) * a.m + r / P);
            }
          }
#pragma unroll
          for (int k = 0; k < kMaxU; ++k) {
            const int i = lane + 32 * k, r = i >> 3, u = i & 7;
            if (r < rows && u < 2 * nch) *reinterpret_cast<uint4*>(xs + r * 128 + ((u ^ (r & 7)) << 4)) = v[k];
          }
#pragma unroll
          for (int k = 0; k < kMaxW; ++k) {
            const int i = lane + 32 * k, cc = i / rows, r = i - cc * rows;
            if (cc < nch) {
              uint32_t wv = w[k];
              if (ph == 1 && wv != 0) {
                const int jr = r / P;
                const int es = jr == 0 ? eseg[0] : eseg[MR - 1];
                const int delta = es - ec[k];  // >= 0 (E = max E_c)
                if (delta != 0 && es != kSegNonFinite) {
                  uint32_t o = 0;
#pragma unroll
                  for (int bi = 0; bi < 4; ++bi) {
                    const uint32_t b8 = (wv >> (8 * bi)) & 0xffu;
                    if (b8 == 0) continue;
                    // power-of-two E4M3: normal (e + 7) << 3, subnormal 1 << (e + 9)
                    const int e = b8 >= 8 ? (int)(b8 >> 3) - 7 : (b8 == 1 ? -9 : b8 == 2 ? -8 : -7);
                    const int e2 = e - delta;
                    const uint32_t n8 = e2 >= -6 ? (uint32_t)(e2 + 7) << 3 : e2 >= -9 ? 1u << (e2 + 9) : 0u;
                    o |= n8 << (8 * bi);
                  }
                  wv = o;
                }
              }
              *reinterpret_cast<uint32_t*>(sfb + 512 * cc + 16 * (r & 31) + 4 * (r >> 5)) = wv;
            }
          }
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // generic writes -> MMA reads
          __syncwarp();
          if (lane == 0) mbar_arrive(&full[s]);
        }
      }
    }
  } else {
    // ------------- epilogues: gate+up segments (h and its chunk planes),
    // down stages (fold per chunk), split-K finalisation
    const int q = warp & 3;
    const int row = 32 * q + lane;
    const int tid = threadIdx.x - 128;
    const uint32_t lane_addr = (uint32_t)(32 * q) << 16;
    griddep_wait();  // the prologue (and so every earlier kernel) is complete
    int xe[MR];
#pragma unroll
    for (int jr = 0; jr < MR; ++jr) xe[jr] = jr < a.m ? __ldcg(a.xe + jr) : kSegZero;
    int u = 0, segs = 0, st_i = 0;
    bool dead = false;  // a wait of this warp expired: skip the remaining waits
    bool fail = false;
    for (int ph = 0; ph < 2 && !fail; ++ph) {
      const int nt = ph ? a.dn_tiles : a.gu_tiles, kc = ph ? a.dn_kc : a.gu_kc;
      const int parts = ph ? (int)gridDim.x : a.gu_parts;
      const uint32_t W = (uint32_t)nt * kc;
      Seg sg;
      for (int j = 0; q_segment(a, ph, j, sg); ++j, ++segs) {
        float y[MR];
#pragma unroll
        for (int jr = 0; jr < MR; ++jr) y[jr] = 0.0f;
        // the segment's accumulators, after its last stage: issuer mi wrote
        // one iff the segment has a stage of its parity
        const int ns = (sg.nk + kQChunks - 1) / kQChunks;
        const bool had[2] = {ns >= 2 || (st_i & 1) == 0, ns >= 2 || (st_i & 1) == 1};
        st_i += ns;
        {
          const int buf = u & 1;
          if (!dead) dead = !__all_sync(0xffffffffu, mbar_wait(&accfull[buf], (u >> 1) & 1, abort_flag, err, 16));
          tc_fence_after();
          uint32_t d0[NT], d1[NT];
          tmem_ld16(tmem + lane_addr + buf * C::kAccBuf, d0);
          tmem_ld16(tmem + lane_addr + buf * C::kAccBuf + NT, d1);
          // down: the row's exponent, E = max E_c over all chunks of h (final:
          // their planes fed these MMAs)
          int E[MR];
#pragma unroll
          for (int jr = 0; jr < MR; ++jr) E[jr] = ph ? (jr < a.m ? he_row(a.he_max, jr) : kSegZero) : xe[jr];
          tmem_ld_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&accfree[buf]);  // the MMAs may reuse the accumulators
          ++u;
          // fold the planes (p ascending): y[jr] = sum_p g_p * D[row, jr P + p],
          // D the sum of the two issuers' accumulators
#pragma unroll
          for (int jr = 0; jr < MR; ++jr) {
            if (jr < a.m) {
              if (E[jr] == kSegNonFinite) {
                y[jr] = __int_as_float(0x7fc00000);  // a non-finite activation
              } else if (E[jr] != kSegZero) {
#pragma unroll
                for (int p = 0; p < P; ++p) {
                  const float dv = (had[0] ? __uint_as_float(d0[jr * P + p]) : 0.0f) +
                                   (had[1] ? __uint_as_float(d1[jr * P + p]) : 0.0f);
                  y[jr] = fmaf(exp2i(plane_log2_factor(E[jr], p)), dv, y[jr]);
                }
              }
            }
          }
        }
        // the segment's sums are in y: stop together if a wait expired
        if (lane == 0 && (dead || *abort_flag)) sh_fail[segs & 1] = 1;
        named_bar_sync(1, 128);
        if (sh_fail[segs & 1]) {
          fail = true;
          break;
        }
        const int g0 = (int)((((uint64_t)sg.tile * kc + 1) * parts - 1) / W);  // owner of the tile's first chunk
        const int g1 = (int)((((uint64_t)sg.tile * kc + kc) * parts - 1) / W);  // and of its last
        bool have = sg.nk == kc;  // a whole tile: its sums are final here
        float* part = ph ? a.part_dn : a.part_gu;
        if (!have) {
          float* Pp = part + (size_t)(blockIdx.x + sg.tile) * a.m * kTileRows;
#pragma unroll
          for (int jr = 0; jr < MR; ++jr)
            if (jr < a.m) Pp[(size_t)jr * kTileRows + row] = y[jr];
          // the barrier orders the four warps' stores before thread 0's fence
          // and count (cumulative at GPU scope)
          named_bar_sync(1, 128);
          // the tile is complete when its counter reaches kc chunks
          if (tid == 0) {
            __threadfence();
            *last_flag = atomicAdd((ph ? a.cnt_dn : a.cnt_gu) + sg.tile, sg.nk) + sg.nk == kc ? 1 : 0;
          }
          named_bar_sync(1, 128);
          have = *last_flag != 0;
          if (have) __threadfence();
        }
        if (!have) continue;
        if (ph == 1) {
          // out[jr, 128 t + r]
          if (sg.nk == kc) {
            const int n = kTileRows * sg.tile + row;
#pragma unroll
            for (int jr = 0; jr < MR; ++jr)
              if (jr < a.m && n < a.hidden) a.out[(size_t)jr * a.hidden + n] = f32_to_bf16_bits(a.gs_dn[0] * y[jr]);
          } else {
            for (int idx = tid; idx < a.m * kTileRows; idx += 128) {
              const int jr = idx / kTileRows, rr = idx % kTileRows;
              const int n = kTileRows * sg.tile + rr;
              if (n < a.hidden)
                a.out[(size_t)jr * a.hidden + n] =
                    f32_to_bf16_bits(a.gs_dn[0] * sum_partials(part, a.m, jr, rr, sg.tile, W, parts, g0, g1));
            }
          }
          continue;
        }
        // gate+up tile t final: Y[jr][r] = its sums (gate r, up r + 64)
        if (sg.nk == kc) {
#pragma unroll
          for (int jr = 0; jr < MR; ++jr)
            if (jr < a.m) Y[jr * kTileRows + row] = y[jr];
        } else {
          for (int idx = tid; idx < a.m * kTileRows; idx += 128) {
            const int jr = idx / kTileRows, rr = idx % kTileRows;
            Y[jr * kTileRows + rr] = sum_partials(part, a.m, jr, rr, sg.tile, W, parts, g0, g1);
          }
        }
        named_bar_sync(1, 128);
        // warp q = activation row jr: lanes 0..15 take h columns 64 t + 4 lane
        // .. + 3, find the chunk's exponent and write its planes (four lanes
        // per 16-block)
        if (q < a.m) {
          const int jr = q;
          float hv[4] = {0.0f, 0.0f, 0.0f, 0.0f};
          uint32_t mx = 0;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int r = 4 * lane + e, n = 64 * sg.tile + r;
            if (lane < 16 && n < a.inter) {
              const float gv = bf16_round(a.gs_gu[0] * Y[jr * kTileRows + r]);
              const float uv = bf16_round(a.gs_gu[1] * Y[jr * kTileRows + 64 + r]);
              hv[e] = bf16_round(silu_fast(gv) * uv);
              mx = max(mx, (uint32_t)(f32_to_bf16_bits(hv[e]) & 0x7fffu));
            }
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          const int E = row_exponent(mx);
          if (E == kSegNonFinite) hv[0] = hv[1] = hv[2] = hv[3] = 0.0f;
          const int b = 4 * sg.tile + (lane >> 2);
          block_planes(hv, E, lane < 16 && b < a.inter / 16, lane & 3, jr, b, a.hq, (size_t)a.inter / 2, a.hs, rows);
          if (lane == 0) {
            a.he[(size_t)sg.tile * a.m + jr] = E;
            atomicMax(a.he_max + jr, E + 1001);
          }
        }
        named_bar_sync(1, 128);  // the planes are written (ordered before the release below)
        if (tid == 0) {
          __threadfence();
          asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(a.gu_done) : "memory");
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// Split-K reduction in a fixed order (z = 0, 1, ...), then the epilogue.
template <bool kGateUp>
__global__ void splitk_reduce_kernel(const float* __restrict__ P, int splits, int m, int n_pad,
                                     int n_out, const float* __restrict__ gs, float gs_mul,
                                     uint16_t* __restrict__ out, int ldo, const LoraArgs lora) {
  griddep_wait();  // the partial sums come from the previous kernel
  griddep_launch_dependents();
  const int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (idx >= (int64_t)m * n_out) return;
  const int r = (int)(idx / n_out), n = (int)(idx % n_out);
  const size_t plane = (size_t)m * n_pad;
  if (kGateUp) {
    const int gcol = kTileRows * (n / 64) + (n % 64), ucol = gcol + 64;
    float g = 0.0f, u = 0.0f;
    for (int z = 0; z < splits; ++z) {
      g += P[z * plane + (size_t)r * n_pad + gcol];
      u += P[z * plane + (size_t)r * n_pad + ucol];
    }
    const float gb = lora_add(bf16_round(gs[0] * gs_mul * g), lora.b0, lora.off0, lora, r, n);
    const float ub = lora_add(bf16_round(gs[1] * gs_mul * u), lora.b1, lora.off1, lora, r, n);
    out[(size_t)r * ldo + n] = f32_to_bf16_bits(silu_fast(gb) * ub);
  } else {
    float acc = 0.0f;
    for (int z = 0; z < splits; ++z) acc += P[z * plane + (size_t)r * n_pad + n];
    float y = gs[0] * gs_mul * acc;
    if (lora.b0) y = lora_add(bf16_round(y), lora.b0, lora.off0, lora, r, n);
    out[(size_t)r * ldo + n] = f32_to_bf16_bits(y);
  }
}

// The same reduction, four adjacent outputs per thread (16-byte partial loads,
// one 8-byte store); each output's sum and epilogue are those above, in the
// same order, so the results are identical.  Needs n_out and ldo divisible by
// 4 (a group of four never crosses a 64-column gate/up block).
template <bool kGateUp>
__global__ void splitk_reduce4_kernel(const float* __restrict__ P, int splits, int m, int n_pad,
                                      int n_out, const float* __restrict__ gs, float gs_mul,
                                      uint16_t* __restrict__ out, int ldo, const LoraArgs lora) {
  griddep_wait();  // the partial sums come from the previous kernel
  griddep_launch_dependents();
  const int nq = n_out / 4;
  const int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (idx >= (int64_t)m * nq) return;
  const int r = (int)(idx / nq), n = 4 * (int)(idx % nq);
  const size_t plane = (size_t)m * n_pad;
  uint16_t o[4];
  if (kGateUp) {
    const int gcol = kTileRows * (n / 64) + (n % 64), ucol = gcol + 64;
    float g[4] = {0.0f, 0.0f, 0.0f, 0.0f}, u[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    for (int z = 0; z < splits; ++z) {
      const float4 gv = *reinterpret_cast<const float4*>(P + z * plane + (size_t)r * n_pad + gcol);
      const float4 uv = *reinterpret_cast<const float4*>(P + z * plane + (size_t)r * n_pad + ucol);
      g[0] += gv.x; g[1] += gv.y; g[2] += gv.z; g[3] += gv.w;
      u[0] += uv.x; u[1] += uv.y; u[2] += uv.z; u[3] += uv.w;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float gb = lora_add(bf16_round(gs[0] * gs_mul * g[i]), lora.b0, lora.off0, lora, r, n + i);
      const float ub = lora_add(bf16_round(gs[1] * gs_mul * u[i]), lora.b1, lora.off1, lora, r, n + i);
      o[i] = f32_to_bf16_bits(silu_fast(gb) * ub);
    }
  } else {
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    for (int z = 0; z < splits; ++z) {
      const float4 v = *reinterpret_cast<const float4*>(P + z * plane + (size_t)r * n_pad + n);
      acc[0] += v.x; acc[1] += v.y; acc[2] += v.z; acc[3] += v.w;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float y = gs[0] * gs_mul * acc[i];
      if (lora.b0) y = lora_add(bf16_round(y), lora.b0, lora.off0, lora, r, n + i);
      o[i] = f32_to_bf16_bits(y);
    }
  }
  *reinterpret_cast<uint2*>(out + (size_t)r * ldo + n) =
      make_uint2((uint32_t)o[0] | ((uint32_t)o[1] << 16), (uint32_t)o[2] | ((uint32_t)o[3] << 16));
}

// Launch the split-K reduction (four outputs per thread when the shapes allow).
cudaError_t launch_splitk_reduce(bool gate_up, const float* P, int splits, int64_t m, int n_pad, int n_out,
                                 const float* gs, float gs_mul, uint16_t* y, int ldo, const LoraArgs& lora,
                                 cudaStream_t s) {
  if (n_out % 4 == 0 && ldo % 4 == 0) {
    const dim3 rgrid((unsigned)((m * (n_out / 4) + 255) / 256));
    return gate_up ? launch_pdl(splitk_reduce4_kernel<true>, rgrid, dim3(256), 0, s, P, splits, (int)m, n_pad,
                                n_out, gs, gs_mul, y, ldo, lora)
                   : launch_pdl(splitk_reduce4_kernel<false>, rgrid, dim3(256), 0, s, P, splits, (int)m, n_pad,
                                n_out, gs, gs_mul, y, ldo, lora);
  }
  const dim3 rgrid((unsigned)((m * n_out + 255) / 256));
  return gate_up ? launch_pdl(splitk_reduce_kernel<true>, rgrid, dim3(256), 0, s, P, splits, (int)m, n_pad, n_out,
                              gs, gs_mul, y, ldo, lora)
                 : launch_pdl(splitk_reduce_kernel<false>, rgrid, dim3(256), 0, s, P, splits, (int)m, n_pad, n_out,
                              gs, gs_mul, y, ldo, lora);
}

// Re-tile a canonical NVFP4 weight (codes [n, k/2], scales [n, k/16]) into the
// per-(128-row tile, 64-element chunk) layout the kernel streams.  For a fused
// gate+up weight (half = inter), tile t holds gate rows [64t, 64t+64) followed
// by the up rows with the same indices.  Padding rows / K tails are zero.
__global__ void tile_weight_kernel(const uint8_t* __restrict__ codes,
                                   const uint8_t* __restrict__ scales, int64_t nrows, int64_t k,
                                   int64_t half, int ntiles, int kc, bool for_w4a16,
                                   uint8_t* __restrict__ out) {
  const int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (idx >= (int64_t)ntiles * kc * kTileRows) return;
  const int r = (int)(idx % kTileRows);
  const int64_t tj = idx / kTileRows;
  const int j = (int)(tj % kc);
  const int t = (int)(tj / kc);
  int64_t src;
  bool valid;
  if (half > 0) {
    const int64_t i = 64 * (int64_t)t + (r & 63);
    src = r < 64 ? i : half + i;
    valid = i < half;
  } else {
    src = (int64_t)kTileRows * t + r;
    valid = src < nrows;
  }
  uint4 lo = make_uint4(0, 0, 0, 0), hi = lo;
  uint32_t sc = 0;
  if (valid) {
    const int64_t cb = k / 2, sb = k / 16;
    const uint8_t* crow = codes + src * cb;
    const uint8_t* srow = scales + src * sb;
    const int64_t off = 32 * (int64_t)j;
    if (off + 16 <= cb) lo = *reinterpret_cast<const uint4*>(crow + off);
    if (off + 32 <= cb) hi = *reinterpret_cast<const uint4*>(crow + off + 16);
    for (int b = 0; b < 4; ++b)
      if (4 * (int64_t)j + b < sb) sc |= (uint32_t)srow[4 * j + b] << (8 * b);
  }
  if (for_w4a16) {
    // The bf16-activation copy: scales lose the sign bit (scales are
    // magnitudes), a block whose scale is zero gets zero codes (the decoded
    // scale of such a block is not zero), and the code bits are rearranged.
    uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
    sc &= 0x7F7F7F7Fu;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (((sc >> (8 * (i >> 1))) & 0xFFu) == 0) w[i] = 0;
      w[i] = permute_codes_w4a16(w[i]);
    }
    lo = make_uint4(w[0], w[1], w[2], w[3]);
    hi = make_uint4(w[4], w[5], w[6], w[7]);
  }
  uint8_t* base = out + ((int64_t)t * kc + j) * kChunkBytes;
  *reinterpret_cast<uint4*>(base + 16 * r) = lo;
  *reinterpret_cast<uint4*>(base + 2048 + 16 * r) = hi;
  // scale bytes in the 512-byte block arrangement of the block-scaled MMA's
  // scale-factor copy: row r's four scales at 16 * (r % 32) + 4 * (r / 32)
  *reinterpret_cast<uint32_t*>(base + 4096 + 16 * (r & 31) + 4 * (r >> 5)) = sc;
}

// Fused gate+up tiles from two plain tiled weights [inter, k] of the same
// kind: fused tile t, row r < 64 is gate row 64t + r, row r >= 64 is up row
// 64t + r - 64 (zero past inter); codes and scale bytes are moved unchanged.
__global__ void retile_gate_up_kernel(const uint8_t* __restrict__ gate, const uint8_t* __restrict__ up,
                                      int64_t inter, int kc, int ntiles, uint8_t* __restrict__ out) {
  const int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (idx >= (int64_t)ntiles * kc * kTileRows) return;
  const int r = (int)(idx % kTileRows);
  const int64_t tj = idx / kTileRows;
  const int j = (int)(tj % kc);
  const int t = (int)(tj / kc);
  const int64_t i = 64 * (int64_t)t + (r & 63);
  uint4 lo = make_uint4(0, 0, 0, 0), hi = lo;
  uint32_t sc = 0;
  if (i < inter) {
    const int sr = (int)(i % kTileRows);
    const uint8_t* src = (r < 64 ? gate : up) + ((i / kTileRows) * kc + j) * kChunkBytes;
    lo = *reinterpret_cast<const uint4*>(src + 16 * sr);
    hi = *reinterpret_cast<const uint4*>(src + 2048 + 16 * sr);
    sc = *reinterpret_cast<const uint32_t*>(src + 4096 + 16 * (sr & 31) + 4 * (sr >> 5));
  }
  uint8_t* dst = out + ((int64_t)t * kc + j) * kChunkBytes;
  *reinterpret_cast<uint4*>(dst + 16 * r) = lo;
  *reinterpret_cast<uint4*>(dst + 2048 + 16 * r) = hi;
  *reinterpret_cast<uint32_t*>(dst + 4096 + 16 * (r & 31) + 4 * (r >> 5)) = sc;
}

// ----------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D map over X [m, k] bf16 with a 64 x box_rows box and the 128-byte swizzle.
bool make_x_map(CUtensorMap* map, const void* x, int64_t m, int64_t k, int box_rows) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)k, (cuuint64_t)m};
  cuuint64_t strides[1] = {(cuuint64_t)k * 2};
  cuuint32_t box[2] = {(cuuint32_t)kChunkK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN, int SXS, int XC, int SWS, int SA, int DQG, int UA, int NI, bool DQX, int EPI>
cudaError_t launch_cfg(const CUtensorMap& map, const TcArgs& a, dim3 grid, cudaStream_t s) {
  using C = TcCfg<BN, SXS, XC, SWS, SA, DQG, UA, NI, DQX>;
  // the LoRA epilogue is a separate instantiation: its code must not weigh on
  // the plain epilogue (registers, instruction cache)
  const bool lora = EPI != kEpiPartial && (a.lora.b0 || a.lora.b1);
  auto kern = lora ? tc_w4a16_kernel<BN, SXS, XC, SWS, SA, DQG, UA, NI, DQX, EPI, EPI != kEpiPartial>
                   : tc_w4a16_kernel<BN, SXS, XC, SWS, SA, DQG, UA, NI, DQX, EPI, false>;
  // The attribute belongs to the current device's context, so it is set on
  // every launch (a host-side call): correct on any device and after a reset.
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemAlloc);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, grid, dim3(C::kThreads), C::kSmemAlloc, s, map, a);
}

// Pipeline variant of the 256-row tile (read once from FFN_NVFP4_WIDE_CFG;
// 0 = the default): alternatives kept selectable so that they can be timed
// against each other on the same build.
int wide_variant() {
  static const int v = [] {
    const char* e = getenv("FFN_NVFP4_WIDE_CFG");
    return e ? atoi(e) : 0;
  }();
  return v;
}

template <int EPI>
cudaError_t launch_bn(int bn, const CUtensorMap& map, const TcArgs& a, dim3 grid, cudaStream_t s) {
  if (bn == 256) switch (wide_variant()) {
    // two dequant warpgroups, 4 two-chunk TMEM slots, the dequant warps wait
    // for the activations on the MMA thread's behalf (gate+up 7% slower at
    // m = 4096 than the default below)
    case 1: return launch_cfg<256, 2, 2, 4, 4, 2, 2, 1, true, EPI>(map, a, grid, s);
    // three dequant warpgroups, 6 one-chunk TMEM slots
    case 2: return launch_cfg<256, 2, 2, 6, 6, 3, 1, 1, false, EPI>(map, a, grid, s);
    // variant 1 with a deeper weight ring
    case 3: return launch_cfg<256, 2, 2, 5, 4, 2, 2, 1, true, EPI>(map, a, grid, s);
    default: break;
  }
  switch (bn) {
    // BN, activation stages, chunks per activation stage, weight stages
    // (rounds), TMEM A slots (units), dequant warpgroups, chunks per unit, MMA
    // threads, activation wait by the dequant warps.  TMEM: max(32, NI*BN) +
    // 32*UA*SA columns (<= 256 for two CTAs per SM).
    case 16: return launch_cfg<16, 2, 8, 8, 6, 2, 1, 2, false, EPI>(map, a, grid, s);
    case 32: return launch_cfg<32, 2, 4, 8, 6, 2, 1, 2, false, EPI>(map, a, grid, s);
    case 64: return launch_cfg<64, 2, 2, 8, 4, 2, 1, 2, false, EPI>(map, a, grid, s);
    case 128: return launch_cfg<128, 4, 2, 3, 4, 2, 2, 1, true, EPI>(map, a, grid, s);
    // three dequant warpgroups, 3 two-chunk TMEM slots (256 + 192 columns),
    // the MMA thread waits for each two-chunk activation stage itself
    default: return launch_cfg<256, 2, 2, 3, 3, 3, 2, 1, false, EPI>(map, a, grid, s);
  }
}

template <int BN, int SXS, int XC, int SWS, int SA, int DQG, int NI, int MODE>
cudaError_t launch_persist_cfg(const CUtensorMap& map, const PArgs& a, int grid, cudaStream_t s) {
  using C = TcCfg<BN, SXS, XC, SWS, SA, DQG, 1, NI, false>;
  using PC = PCfg<BN, SXS, XC, SWS, SA, DQG, NI>;
  auto kern = tc_w4a16_persistent_kernel<BN, SXS, XC, SWS, SA, DQG, NI, MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, PC::kSmemAlloc);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(grid), dim3(C::kThreads), PC::kSmemAlloc, s, map, a);
}

template <int MODE>
cudaError_t launch_persist_bn(int bn, const CUtensorMap& map, const PArgs& a, int grid, cudaStream_t s) {
  switch (bn) {
    // BN, activation stages, chunks per activation stage, weight stages
    // (rounds of DQG chunks), TMEM A slots (chunks), dequant warpgroups, MMA
    // threads.  One CTA per SM: TMEM NI*BN + 32*SA columns of 512.
    case 16: return launch_persist_cfg<16, 4, 6, 10, 12, 3, 2, MODE>(map, a, grid, s);
    case 32: return launch_persist_cfg<32, 3, 6, 8, 12, 3, 2, MODE>(map, a, grid, s);
    default: return launch_persist_cfg<64, 3, 4, 8, 6, 2, 2, MODE>(map, a, grid, s);
  }
}

// The down phase waits for chunks that other CTAs finish, so every CTA must
// be resident at once: the grid is the occupancy (two CTAs per SM, with the
// shared-memory carveout at its maximum) times the SMs, at most `max_grid`
// (what the workspace was sized for).
cudaError_t launch_layer(LArgs a, int max_grid, int num_sms, cudaStream_t s) {
  using C = QCfg;
  auto kern = tc_planes_layer_kernel;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemAlloc);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  int dev = 0, smem_sm = 0;
  if (e == cudaSuccess) e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
  if (e != cudaSuccess) return e;
  // registers: __launch_bounds__(kLayerThreads, 2) keeps two CTAs within the
  // register file; threads: 576 of 2048; shared memory (1 KB per CTA
  // reserved; two CTAs of the 4-stage ring leave about 40 KB of an SM free):
  const int occupancy = 2 * (C::kSmemAlloc + 1024) <= smem_sm ? 2 : 1;
  const int grid = min(max_grid, occupancy * num_sms);
  if (grid < 1) return cudaErrorInvalidConfiguration;
  a.gu_parts = min(a.gu_parts, grid);
  return launch_pdl(kern, dim3(grid), dim3(kLayerThreads), C::kSmemAlloc, s, a);
}

}  // namespace

int tc_tile_bytes_per_row_chunk() { return kChunkBytes; }

int planes_for_rows(int64_t m) { return m <= QCfg::kMR ? kQPlanes : 0; }

PlanesPlan plan_planes(int64_t m, int64_t hidden, int64_t inter, int num_sms) {
  PlanesPlan p;
  p.planes = planes_for_rows(m);
  if (!p.planes) return p;
  p.nt = QCfg::kNT;
  p.rows = (int)(m * p.planes);
  p.gu_tiles = (int)((inter + 63) / 64);
  p.gu_kc = (int)((hidden + kChunkK - 1) / kChunkK);
  p.dn_tiles = (int)((hidden + kTileRows - 1) / kTileRows);
  p.dn_kc = (int)((inter + kChunkK - 1) / kChunkK);
  p.grid = 2 * num_sms;  // at most two CTAs per SM, all resident
  // gate+up: whole tiles when they do not outnumber the CTAs
  p.gu_parts = p.gu_tiles <= p.grid ? p.gu_tiles : p.grid;
  p.gu_partial_bytes = (size_t)(p.gu_parts + p.gu_tiles) * m * kTileRows * sizeof(float);
  p.dn_partial_bytes = (size_t)(p.grid + p.dn_tiles) * m * kTileRows * sizeof(float);
  p.x_code_bytes = (size_t)p.rows * (size_t)(hidden / 2);
  p.x_sf_bytes = (size_t)p.gu_kc * p.rows * 4;
  p.h_code_bytes = (size_t)p.rows * (size_t)(inter / 2);
  p.h_sf_bytes = (size_t)p.dn_kc * p.rows * 4;
  p.zero_ints = p.gu_tiles + p.dn_tiles + 1 + (int)m;  // tile counters, finished gate+up tiles, h row exponents
  p.other_ints = (int)m + p.gu_tiles * (int)m;          // x's row exponents, h's chunk exponents
  return p;
}

cudaError_t launch_planes_ffn(const void* x, int64_t m, const TcWeight& gate_up, const TcWeight& down,
                              const PlanesPlan& p, const PlanesBuffers& b, void* out, cudaStream_t s) {
  const int64_t hidden = down.n, inter = gate_up.n / 2;
  if (hidden % 32 || inter % 32) return cudaErrorInvalidValue;
  // 32-bit range arithmetic in the kernel
  if ((uint64_t)p.gu_tiles * p.gu_kc * p.grid >= (1ull << 32) || (uint64_t)p.dn_tiles * p.dn_kc * p.grid >= (1ull << 32))
    return cudaErrorInvalidValue;
  int* zero = b.ints;  // [cnt_gu][cnt_dn][gu_done][he_max m] zeroed, then x's E [m], h's E [gu_tiles][m]
  int* xe = zero + p.zero_ints;
  cudaError_t e;
  {
    ProfScope prof(s, "planes_prologue");
    // the same shared-memory carveout as the layer kernel, so that SMs need
    // no reconfiguration between the two
    e = cudaFuncSetAttribute(planes_prologue_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)m, (unsigned)((hidden / 16 + kPlaneBlocksPerCta - 1) / kPlaneBlocksPerCta));
    e = launch_pdl(planes_prologue_kernel, grid, dim3(kPlaneThreads), 0, s, static_cast<const uint16_t*>(x),
                   (int)m, (int)hidden, static_cast<uint8_t*>(b.xq), static_cast<uint8_t*>(b.xs), xe, zero,
                   p.zero_ints);
  }
  if (e != cudaSuccess) return e;
  LArgs a{};
  a.wt_gu = gate_up.tiled;
  a.wt_dn = down.tiled;
  a.gs_gu = gate_up.gs;
  a.gs_dn = down.gs;
  a.xq = static_cast<const uint8_t*>(b.xq);
  a.xs = static_cast<const uint8_t*>(b.xs);
  a.xe = xe;
  a.hq = static_cast<uint8_t*>(b.hq);
  a.hs = static_cast<uint8_t*>(b.hs);
  a.he = xe + m;
  a.out = static_cast<uint16_t*>(out);
  a.part_gu = static_cast<float*>(b.part_gu);
  a.part_dn = static_cast<float*>(b.part_dn);
  a.cnt_gu = zero;
  a.cnt_dn = zero + p.gu_tiles;
  a.gu_done = reinterpret_cast<uint32_t*>(a.cnt_dn + p.dn_tiles);
  a.he_max = a.cnt_dn + p.dn_tiles + 1;
  a.m = (int)m;
  a.hidden = (int)hidden;
  a.inter = (int)inter;
  a.gu_tiles = p.gu_tiles;
  a.gu_kc = p.gu_kc;
  a.gu_parts = p.gu_parts;
  a.dn_tiles = p.dn_tiles;
  a.dn_kc = p.dn_kc;
  ProfScope prof(s, "tc_planes_layer");
  return launch_layer(a, p.grid, p.grid / 2, s);
}

PersistPlan plan_persist(int64_t m, int64_t hidden, int64_t inter, int num_sms) {
  PersistPlan p;
  p.bn = m <= 16 ? 16 : m <= 32 ? 32 : 64;
  p.gu_tiles = (int)((inter + 63) / 64);
  p.gu_kc = (int)((hidden + kChunkK - 1) / kChunkK);
  p.gu_grid = p.gu_tiles < num_sms ? p.gu_tiles : num_sms;
  p.dn_tiles = (int)((hidden + kTileRows - 1) / kTileRows);
  p.dn_kc = (int)((inter + kChunkK - 1) / kChunkK);
  const int64_t W = (int64_t)p.dn_tiles * p.dn_kc;
  p.dn_grid = (int)(W < num_sms ? W : num_sms);
  p.partial_bytes = (size_t)(p.dn_grid + p.dn_tiles) * m * kTileRows * sizeof(float);
  p.counter_bytes = (size_t)p.dn_tiles * sizeof(int);
  return p;
}

cudaError_t launch_persist_ffn(const void* x, int64_t m, const TcWeight& gate_up, const TcWeight& down,
                               const PersistPlan& p, void* h, void* partials, int* counters, void* out,
                               cudaStream_t s, const LoraView& lv, void* xa_gu, void* xa_d) {
  const int box_rows = (int)m;
  const int64_t inter = gate_up.n / 2, hidden = down.n;
  CUtensorMap xm, hm;
  if (!make_x_map(&xm, x, m, gate_up.k, box_rows) || !make_x_map(&hm, h, m, down.k, box_rows))
    return cudaErrorInvalidValue;
  PArgs a{};
  a.wt = gate_up.tiled16;
  a.gs = gate_up.gs;
  a.out = static_cast<uint16_t*>(h);
  a.m = (int)m;
  a.n_out = (int)inter;
  a.ldo = (int)inter;
  a.kc = p.gu_kc;
  a.ntiles = p.gu_tiles;
  a.x_box_rows = box_rows;
  a.zero_ptr = counters;
  a.zero_count = p.dn_tiles;
  cudaError_t e = cudaSuccess;
  if (lv.rank > 0 && lv.a_gu) {
    e = launch_lora_xa(x, m, gate_up.k, lv.a_gu, 2 * lv.rank, xa_gu, s);
    a.lora.xa = static_cast<const uint16_t*>(xa_gu);
    a.lora.xa_ld = 2 * lv.rank;
    a.lora.b0 = lv.b_g;
    a.lora.b1 = lv.b_u;
    a.lora.off0 = 0;
    a.lora.off1 = lv.rank;
    a.lora.r = lv.rank;
  }
  if (e != cudaSuccess) return e;
  {
    ProfScope prof(s, "tc_w4a16_gate_up_silu_persistent");
    e = launch_persist_bn<kModeTiles>(p.bn, xm, a, p.gu_grid, s);
  }
  if (e != cudaSuccess) return e;
  if (lv.rank > 0 && lv.a_d) {
    e = launch_lora_xa(h, m, down.k, lv.a_d, lv.rank, xa_d, s);
    if (e != cudaSuccess) return e;
  }
  PArgs b{};
  b.wt = down.tiled16;
  b.gs = down.gs;
  b.out = static_cast<uint16_t*>(out);
  b.m = (int)m;
  b.n_out = (int)hidden;
  b.ldo = (int)hidden;
  b.kc = p.dn_kc;
  b.ntiles = p.dn_tiles;
  b.x_box_rows = box_rows;
  b.partials = static_cast<float*>(partials);
  b.counters = counters;
  if (lv.rank > 0 && lv.a_d) {
    b.lora.xa = static_cast<const uint16_t*>(xa_d);
    b.lora.xa_ld = lv.rank;
    b.lora.b0 = lv.b_d;
    b.lora.r = lv.rank;
  }
  ProfScope prof(s, "tc_w4a16_down_persistent");
  return launch_persist_bn<kModeRanges>(p.bn, hm, b, p.dn_grid, s);
}

int64_t tc_tiled_bytes(int64_t n, int64_t k, bool gate_up) {
  const int64_t tiles = gate_up ? (n / 2 + 63) / 64 : (n + kTileRows - 1) / kTileRows;
  const int64_t kc = (k + kChunkK - 1) / kChunkK;
  return tiles * kc * kChunkBytes;
}

cudaError_t launch_tile_weight(const uint8_t* codes, const uint8_t* scales, int64_t n, int64_t k,
                               bool gate_up, bool for_w4a16, uint8_t* out, cudaStream_t s) {
  const int64_t half = gate_up ? n / 2 : 0;
  const int ntiles = (int)(gate_up ? (half + 63) / 64 : (n + kTileRows - 1) / kTileRows);
  const int kc = (int)((k + kChunkK - 1) / kChunkK);
  const int64_t total = (int64_t)ntiles * kc * kTileRows;
  tile_weight_kernel<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(codes, scales, n, k, half, ntiles,
                                                                   kc, for_w4a16, out);
  return cudaGetLastError();
}

cudaError_t launch_retile_gate_up(const uint8_t* gate_tiled, const uint8_t* up_tiled, int64_t inter,
                                  int64_t k, uint8_t* out, cudaStream_t s) {
  const int ntiles = (int)((inter + 63) / 64);
  const int kc = (int)((k + kChunkK - 1) / kChunkK);
  const int64_t total = (int64_t)ntiles * kc * kTileRows;
  retile_gate_up_kernel<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(gate_tiled, up_tiled, inter, kc,
                                                                       ntiles, out);
  return cudaGetLastError();
}

TcPlan plan_tc(int64_t m, int64_t n, int64_t k, bool gate_up, int num_sms) {
  TcPlan p;
  p.bn = m <= 16 ? 16 : m <= 32 ? 32 : m <= 64 ? 64 : m <= 128 ? 128 : 256;
  p.xtiles = (int)((m + p.bn - 1) / p.bn);
  p.wtiles = (int)(gate_up ? (n / 2 + 63) / 64 : (n + kTileRows - 1) / kTileRows);
  p.kc = (int)((k + kChunkK - 1) / kChunkK);
  p.n_pad = p.wtiles * kTileRows;
  const int ctas_per_sm = p.bn <= 64 ? 2 : 1;
  const int64_t slots = (int64_t)num_sms * ctas_per_sm;
  const int64_t ctas = (int64_t)p.xtiles * p.wtiles;
  int splits = 1;
  if (ctas < slots) {
    splits = (int)(slots / ctas);
    const int max_splits = p.kc / 8 > 1 ? p.kc / 8 : 1;  // keep >= 8 chunks per split
    if (splits > max_splits) splits = max_splits;
  }
  p.kc_per_split = (p.kc + splits - 1) / splits;
  p.splits = (p.kc + p.kc_per_split - 1) / p.kc_per_split;
  p.partial_bytes = p.splits > 1 ? (size_t)p.splits * m * p.n_pad * sizeof(float) : 0;
  return p;
}

cudaError_t launch_tc_w4a16(const void* x, int64_t m, const TcWeight& w, bool silu_mul,
                            const TcPlan& p, void* y, void* partials, cudaStream_t s,
                            const LoraArgs& lora) {
  CUtensorMap map;
  const int box_rows = (int)(m < p.bn ? m : p.bn);
  if (!make_x_map(&map, x, m, w.k, box_rows)) return cudaErrorInvalidValue;
  TcArgs a;
  a.x_box_rows = box_rows;
  a.wt = w.tiled16;
  a.gs = w.gs;
  a.m = (int)m;
  a.n_out = (int)(silu_mul ? w.n / 2 : w.n);
  a.ldo = a.n_out;
  a.kc_total = p.kc;
  a.kc_per_split = p.kc_per_split;
  a.n_pad = p.n_pad;
  a.lora = lora;
  const dim3 grid(p.xtiles, p.wtiles, p.splits);
  cudaError_t e;
  if (p.splits > 1) {
    a.out = partials;
    {
      ProfScope prof(s, silu_mul ? "tc_w4a16_gate_up_partial" : "tc_w4a16_partial");
      e = launch_bn<kEpiPartial>(p.bn, map, a, grid, s);
    }
    if (e != cudaSuccess) return e;
    ProfScope prof(s, silu_mul ? "splitk_reduce_silu_mul" : "splitk_reduce");
    return launch_splitk_reduce(silu_mul, static_cast<const float*>(partials), p.splits, m, p.n_pad, a.n_out,
                                w.gs, kW4A16Unscale, static_cast<uint16_t*>(y), a.ldo, lora, s);
  }
  a.out = y;
  ProfScope prof(s, silu_mul ? "tc_w4a16_gate_up_silu" : "tc_w4a16");
  return silu_mul ? launch_bn<kEpiSiluMul>(p.bn, map, a, grid, s)
                  : launch_bn<kEpiStore>(p.bn, map, a, grid, s);
}


TcPlan plan_w4a4(int64_t m, int64_t n, int64_t k, bool gate_up, int num_sms) {
  // The K split depends on (n, k) only; the tile width and count on m.
  TcPlan p;
  p.bn = m <= kW4BNSmall ? kW4BNSmall : kW4BN;
  p.xtiles = (int)((m + p.bn - 1) / p.bn);
  p.wtiles = (int)(gate_up ? (n / 2 + 63) / 64 : (n + kTileRows - 1) / kTileRows);
  p.kc = (int)((k + kChunkK - 1) / kChunkK);
  p.n_pad = p.wtiles * kTileRows;
  int splits = num_sms / p.wtiles;
  const int max_splits = p.kc / (2 * kW4Chunks) > 1 ? p.kc / (2 * kW4Chunks) : 1;
  if (splits > max_splits) splits = max_splits;
  if (splits < 1) splits = 1;
  p.kc_per_split = (p.kc + splits - 1) / splits;
  p.kc_per_split = (p.kc_per_split + kW4Chunks - 1) / kW4Chunks * kW4Chunks;
  p.splits = (p.kc + p.kc_per_split - 1) / p.kc_per_split;
  p.partial_bytes = p.splits > 1 ? (size_t)p.splits * m * p.n_pad * sizeof(float) : 0;
  return p;
}

size_t w4a4_sf_block_bytes(int64_t m, int64_t k) {
  return (size_t)((m + kW4BN - 1) / kW4BN) * ((k + kChunkK - 1) / kChunkK) * 512;
}

cudaError_t launch_tc_w4a4(const uint8_t* xcodes, const uint8_t* xsf_blocks, int64_t m,
                           const TcWeight& w, bool silu_mul, const TcPlan& p, void* y,
                           void* partials, cudaStream_t s, uint8_t* hq_codes, uint8_t* hq_sf) {
  auto enc = get_encode();
  if (!enc) return cudaErrorInvalidValue;
  CUtensorMap map;
  {
    cuuint64_t dims[2] = {(cuuint64_t)(w.k / 2), (cuuint64_t)m};
    cuuint64_t strides[1] = {(cuuint64_t)(w.k / 2)};
    cuuint32_t box[2] = {128, (cuuint32_t)(m < p.bn ? m : p.bn)};
    cuuint32_t estr[2] = {1, 1};
    if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(xcodes), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  W4Args a;
  a.xtiles = p.xtiles;
  a.t.x_box_rows = (int)(m < p.bn ? m : p.bn);
  if (p.bn != kW4BN && (p.bn != kW4BNSmall || m > p.bn)) return cudaErrorInvalidValue;
  a.t.wt = w.tiled;
  a.t.gs = w.gs;
  a.t.m = (int)m;
  a.t.n_out = (int)(silu_mul ? w.n / 2 : w.n);
  a.t.ldo = a.t.n_out;
  a.t.kc_total = p.kc;
  a.t.kc_per_split = p.kc_per_split;
  a.t.n_pad = p.n_pad;
  a.sfb = xsf_blocks;
  const dim3 grid(p.xtiles, p.wtiles, p.splits);
  using CWide = W4Cfg<1, kW4BN, 3>;
  using CNarrow = W4Cfg<1, kW4BNSmall, 5>;
  auto launch = [&](auto kern_wide, auto kern_narrow) -> cudaError_t {
    // set on every launch: the attributes belong to the current device's context
    auto go = [&](auto kern, int smem) -> cudaError_t {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
      return e == cudaSuccess ? launch_pdl(kern, grid, dim3(256), smem, s, map, a) : e;
    };
    return p.bn == kW4BNSmall ? go(kern_narrow, CNarrow::kSmemAlloc) : go(kern_wide, CWide::kSmemAlloc);
  };
  cudaError_t e;
  if (p.splits > 1) {
    a.t.out = partials;
    {
      ProfScope prof(s, silu_mul ? "tc_w4a4_gate_up_partial" : "tc_w4a4_partial");
      e = launch(tc_w4a4_kernel<kEpiPartial, 1, kW4BN, 3>, tc_w4a4_kernel<kEpiPartial, 1, kW4BNSmall, 5>);
    }
    if (e != cudaSuccess) return e;
    ProfScope prof(s, silu_mul ? "splitk_reduce_silu_mul" : "splitk_reduce");
    return launch_splitk_reduce(silu_mul, static_cast<const float*>(partials), p.splits, m, p.n_pad, a.t.n_out,
                                w.gs, 1.0f, static_cast<uint16_t*>(y), a.t.ldo, LoraArgs(), s);
  }
  a.t.out = y;
  if (silu_mul && hq_codes && hq_sf) {
    a.t.q_codes = hq_codes;
    a.t.q_sf = hq_sf;
    a.t.q_kc = (int)((a.t.n_out + kChunkK - 1) / kChunkK);
    ProfScope prof(s, "tc_w4a4_gate_up_silu_quant");
    return launch(tc_w4a4_kernel<kEpiSiluMulQuant, 1, kW4BN, 3>, tc_w4a4_kernel<kEpiSiluMulQuant, 1, kW4BNSmall, 5>);
  }
  ProfScope prof(s, silu_mul ? "tc_w4a4_gate_up_silu" : "tc_w4a4");
  return silu_mul ? launch(tc_w4a4_kernel<kEpiSiluMul, 1, kW4BN, 3>, tc_w4a4_kernel<kEpiSiluMul, 1, kW4BNSmall, 5>)
                  : launch(tc_w4a4_kernel<kEpiStore, 1, kW4BN, 3>, tc_w4a4_kernel<kEpiStore, 1, kW4BNSmall, 5>);
}

cudaError_t read_device_error(int* flags, bool clear) {
  cudaError_t e = cudaMemcpyFromSymbol(flags, g_ffn_device_error, sizeof(int));
  if (e == cudaSuccess && clear) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_ffn_device_error, &zero, sizeof(int));
  }
  return e;
}

}  // namespace ffn
