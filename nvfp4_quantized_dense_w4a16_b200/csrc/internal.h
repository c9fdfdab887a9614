// Host-side declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "ffn_nvfp4.h"
#include "lora_args.h"

namespace ffn {

// Operand of one projection: canonical NVFP4 layout of a [n, k] weight.
// For a fused gate+up weight, rows [0, n/2) are gate and [n/2, n) are up and
// gs points at two floats (gate, up).
struct WeightView {
  const uint8_t* codes;   // [n, k/2]
  const uint8_t* scales;  // [n, k/16]
  const float* gs;        // 1 or 2 device floats
  int64_t n, k;
};

enum class Epilogue : int {
  kStore = 0,   // y[r, j] = bf16(gs * acc)
  kSiluMul = 1  // h[r, j] = bf16(silu(bf16(gs_g*acc_g)) * bf16(gs_u*acc_u)), j < n/2
};

// Tensor-core (tcgen05) projection over the pre-tiled weight layout.
struct TcWeight {
  const uint8_t* tiled;    // [tiles][ceil(k/64)][4608], natural codes (W4A4)
  const uint8_t* tiled16;  // same layout, code bits rearranged for the W4A16 decode
  const float* gs;       // 1 or 2 device floats
  int64_t n, k;          // logical dims (n = 2*inter for a fused gate+up weight)
};

struct TcPlan {
  int bn = 0;            // activation rows per tile (MMA N)
  int xtiles = 0, wtiles = 0, kc = 0, kc_per_split = 0, splits = 1, n_pad = 0;
  size_t partial_bytes = 0;  // fp32 split-K partials needed in the workspace
};

// LoRA adapters of one layer (device copies; see lora.cu).
struct LoraView {
  int rank = 0, device = 0;
  const uint16_t* a_gu = nullptr;  // [2r, hidden]: gate rows then up rows
  const uint16_t* a_d = nullptr;   // [r, inter]
  const uint16_t* b_g = nullptr;   // [inter, r]
  const uint16_t* b_u = nullptr;
  const uint16_t* b_d = nullptr;   // [hidden, r]
};
LoraView lora_view(const ffn_lora* l);
bool lora_dims_mismatch(const ffn_lora* l, int64_t hidden, int64_t inter);
// xa[j, i] = bf16(x[j, :] . a[i, :]) for i < rows (x [m, k], a [rows, k]).
cudaError_t launch_lora_xa(const void* x, int64_t m, int64_t k, const uint16_t* a, int rows, void* xa,
                           cudaStream_t s);

TcPlan plan_tc(int64_t m, int64_t n, int64_t k, bool gate_up, int num_sms);
int64_t tc_tiled_bytes(int64_t n, int64_t k, bool gate_up);
// Fused gate+up tiles from the gate and up handles' tiles of the same kind.
cudaError_t launch_retile_gate_up(const uint8_t* gate_tiled, const uint8_t* up_tiled, int64_t inter,
                                  int64_t k, uint8_t* out, cudaStream_t s);
cudaError_t launch_tile_weight(const uint8_t* codes, const uint8_t* scales, int64_t n, int64_t k,
                               bool gate_up, bool for_w4a16, uint8_t* out, cudaStream_t s);
cudaError_t launch_tc_w4a16(const void* x, int64_t m, const TcWeight& w, bool silu_mul,
                            const TcPlan& p, void* y, void* partials, cudaStream_t s,
                            const LoraArgs& lora = LoraArgs());
// Few-row FFN layer (m <= 64): two persistent launches, one CTA per SM --
// gate+up over whole tiles dealt round-robin (SiLU*mul epilogue into h), then
// down over equal contiguous (tile, K chunk) ranges with the split-K sums
// added in K order by the CTA that completes each tile.
constexpr int64_t kPersistMaxRows = 64;
struct PersistPlan {
  int bn = 0;
  int gu_tiles = 0, gu_kc = 0, gu_grid = 0;
  int dn_tiles = 0, dn_kc = 0, dn_grid = 0;
  size_t partial_bytes = 0, counter_bytes = 0;
};
PersistPlan plan_persist(int64_t m, int64_t hidden, int64_t inter, int num_sms);
// With LoRA adapters (lv.rank > 0): xa_gu [m, 2r] and xa_d [m, r] workspace
// buffers receive the rank-r products, computed by lora_xa launches before
// each projection, and the projections' epilogues add the deltas.
cudaError_t launch_persist_ffn(const void* x, int64_t m, const TcWeight& gate_up, const TcWeight& down,
                               const PersistPlan& p, void* h, void* partials, int* counters, void* out,
                               cudaStream_t s, const LoraView& lv = LoraView(), void* xa_gu = nullptr,
                               void* xa_d = nullptr);
// Few-row W4A16 layer on the block-scaled FP4 tensor core (natural tiled
// weights as the MMA's A operand, activations as NVFP4 planes built in the
// GEMM kernel's shared memory).
int planes_for_rows(int64_t m);  // planes per activation row, 0 when the path does not apply
struct PlanesPlan {
  int planes = 0, nt = 0, rows = 0, grid = 0;
  int gu_tiles = 0, gu_kc = 0, gu_parts = 0, dn_tiles = 0, dn_kc = 0;
  size_t gu_partial_bytes = 0, dn_partial_bytes = 0, x_code_bytes = 0, x_sf_bytes = 0, h_code_bytes = 0,
         h_sf_bytes = 0;
  int zero_ints = 0;   // ints the prologue zeroes
  int other_ints = 0;  // ints after them (row and chunk exponents)
};
struct PlanesBuffers {  // workspace regions of the few-row block-scaled layer
  void *xq, *xs, *hq, *hs, *part_gu, *part_dn;
  int* ints;
};
PlanesPlan plan_planes(int64_t m, int64_t hidden, int64_t inter, int num_sms);
// Requires hidden and inter multiples of 32, and no LoRA adapter.
cudaError_t launch_planes_ffn(const void* x, int64_t m, const TcWeight& gate_up, const TcWeight& down,
                              const PlanesPlan& p, const PlanesBuffers& b, void* out, cudaStream_t s);
// Fixed-format (W4A4) projection on the block-scaled FP4 tensor core.  The
// K split depends on (n, k) only; the activation tile (16 rows for m <= 16,
// else 128) and the number of tiles on m, neither of which changes a result
// bit.
TcPlan plan_w4a4(int64_t m, int64_t n, int64_t k, bool gate_up, int num_sms);
size_t w4a4_sf_block_bytes(int64_t m, int64_t k);
// With silu_mul, no K split and hq_codes/hq_sf given, the epilogue writes the
// per-row NVFP4 quantisation of h (codes [m, n/4], blocked scales) instead
// of h itself.
cudaError_t launch_tc_w4a4(const uint8_t* xcodes, const uint8_t* xsf_blocks, int64_t m,
                           const TcWeight& w, bool silu_mul, const TcPlan& p, void* y,
                           void* partials, cudaStream_t s, uint8_t* hq_codes = nullptr,
                           uint8_t* hq_sf = nullptr);
// Activation quantiser that also writes the scales as 512-byte blocks per
// 128 rows and 64 elements (the W4A4 kernel's scale-factor layout).
cudaError_t launch_quantize_activations_blocked(const void* x, int64_t m, int64_t k, void* codes,
                                                void* sf_blocks, cudaStream_t s);

// Tensor-core view of a handle (and whether it is a fused gate+up handle).
void handle_tc_view(const ffn_nvfp4_weight* w, TcWeight* out, bool* gate_up);
// FFN_OK when the handle belongs to the current device.
ffn_status handle_check_device(const ffn_nvfp4_weight* w);

// Device-wide error bits set by kernels whose bounded waits gave up.
cudaError_t read_device_error(int* flags, bool clear);

cudaError_t launch_quantize_weights(const void* w, int64_t n, int64_t k, void* codes,
                                    void* scales, float* gs, cudaStream_t s);
cudaError_t launch_quantize_activations(const void* x, int64_t m, int64_t k, void* codes,
                                        void* scales, cudaStream_t s);

// CUDA-core projections (any m; used for small m and as the general path).
int gemv_grid(int64_t ncols);
cudaError_t launch_gemv_w4a16(const void* x, int64_t m, const WeightView& w, Epilogue ep,
                              void* y, cudaStream_t s);
cudaError_t launch_gemv_w4a4(const uint8_t* xcodes, const uint8_t* xscales, int64_t m,
                             const WeightView& w, Epilogue ep, void* y, cudaStream_t s);

}  // namespace ffn
