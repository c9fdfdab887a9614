// C ABI of the NVFP4 SwiGLU FFN: argument checks, weight handles, workspace
// carving and the per-call kernel dispatch.  See include/ffn_nvfp4.h.
#include <stdlib.h>
#include <string.h>

#include <new>

#include "ffn_nvfp4.h"
#include "internal.h"

using ffn::Epilogue;
using ffn::WeightView;

struct ffn_nvfp4_weight {
  int64_t n = 0, k = 0;
  int gate_up = 0;
  int device = 0;
  unsigned formats = 0;       // FFN_FORMAT_* bits the handle serves
  size_t bytes = 0;           // device bytes held
  uint8_t* codes = nullptr;   // [n, k/2] canonical (only for a forced CUDA-core arm)
  uint8_t* scales = nullptr;  // [n, k/16] canonical (likewise)
  float* gs = nullptr;        // 1 float, or 2 (gate, up) for a fused handle
  uint8_t* tiled = nullptr;   // tensor-core layout (see tc_gemm.cu), natural codes: fixed format
  uint8_t* tiled16 = nullptr; // the same tiles with the W4A16 code-bit arrangement: bf16
  WeightView view() const { return WeightView{codes, scales, gs, n, k}; }
  ffn::TcWeight tc() const { return ffn::TcWeight{tiled, tiled16, gs, n, k}; }
};

namespace {

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline ffn_status cuda_status(cudaError_t e) { return e == cudaSuccess ? FFN_OK : FFN_ERR_CUDA; }

inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// A handle's buffers live on the device it was created on; using it with
// another device current would hand that device foreign pointers.
ffn_status check_device(const ffn_nvfp4_weight* w) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return FFN_ERR_CUDA;
  }
  return dev == w->device ? FFN_OK : FFN_ERR_INVALID_ARG;
}

// Pick up errors of earlier asynchronous work before enqueuing more.
inline ffn_status precheck() {
  const cudaError_t e = cudaPeekAtLastError();
  if (e != cudaSuccess) {
    cudaGetLastError();
    return FFN_ERR_CUDA;
  }
  return FFN_OK;
}

bool valid_k(int64_t k) { return k > 0 && k % 32 == 0; }

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return 148;  // B200
  }
  return n;
}

// Projection kernel family for m rows: the tensor-core GEMM, or the CUDA-core
// GEMV.  FFN_NVFP4_W4A16_PATH=gemv|tc overrides (read once) for measurements.
enum class Path { kTc, kGemv };

int w4a16_forced() {
  static int forced = [] {
    const char* v = getenv("FFN_NVFP4_W4A16_PATH");
    if (!v) return 0;
    if (!strcmp(v, "gemv")) return 1;
    if (!strcmp(v, "tc")) return 2;
    if (!strcmp(v, "persistent")) return 3;
    if (!strcmp(v, "planes")) return 4;
    return 0;
  }();
  return forced;
}

Path w4a16_path(int64_t m) {
  if (w4a16_forced() == 1) return Path::kGemv;
  (void)m;
  return Path::kTc;
}

// The two persistent launches for few rows (see plan_persist) run only when
// FFN_NVFP4_W4A16_PATH=persistent: measured on B200 at m = 1..64 they were
// slower than the per-tile kernels (one CTA per SM halves the MMA-issuing
// threads per SM, which bound these narrow tiles), so the default keeps the
// per-tile kernels.
bool w4a16_persistent(int64_t m) { return w4a16_forced() == 3 && m <= ffn::kPersistMaxRows; }

// Few rows (m <= 8) with both weights in the natural tiled layout (handles
// built for the fixed format too, e.g. FFN_FORMAT_ALL): the block-scaled FP4
// path with activation planes, unless FFN_NVFP4_W4A16_PATH forces another.
bool w4a16_planes(int64_t m, int64_t hidden, int64_t inter, const ffn_nvfp4_weight* gu,
                  const ffn_nvfp4_weight* dn) {
  const int f = w4a16_forced();
  (void)hidden;
  (void)inter;
  return (f == 0 || f == 4) && ffn::planes_for_rows(m) > 0 && gu && dn && gu->tiled && dn->tiled;
}

// Fixed format: the block-scaled FP4 tensor-core kernel, or the CUDA-core one
// (FFN_NVFP4_W4A4_PATH=gemv).  Either choice is made once per process and does
// not depend on m, which the format's row invariance requires.
Path w4a4_path() {
  static const Path p = [] {
    const char* v = getenv("FFN_NVFP4_W4A4_PATH");
    return (v && !strcmp(v, "gemv")) ? Path::kGemv : Path::kTc;
  }();
  return p;
}

// The fixed format quantises h inside the gate+up epilogue when that
// projection runs unsplit; FFN_NVFP4_W4A4_FUSE_HQ=0 keeps the separate
// quantiser launch (read once; for comparisons).
bool w4a4_fuse_hq() {
  static const bool on = [] {
    const char* v = getenv("FFN_NVFP4_W4A4_FUSE_HQ");
    return !(v && !strcmp(v, "0"));
  }();
  return on;
}

// The canonical NVFP4 copy is read only by the CUDA-core arms, which run
// only when forced by environment; otherwise handles keep just the tiled
// copies their formats need (0.5625 B per weight and format, plus tile padding).
bool keep_canonical() { return w4a16_forced() == 1 || w4a4_path() == Path::kGemv; }

// The handle holds what `format` reads on the path that will run.
bool serves(const ffn_nvfp4_weight* w, ffn_act_format f) {
  const unsigned bit = f == FFN_ACT_BF16 ? FFN_FORMAT_BF16 : FFN_FORMAT_NVFP4_FIXED;
  if (!(w->formats & bit)) return false;
  const bool gemv = f == FFN_ACT_BF16 ? w4a16_forced() == 1 : w4a4_path() == Path::kGemv;
  return gemv ? w->codes != nullptr : (f == FFN_ACT_BF16 ? w->tiled16 : w->tiled) != nullptr;
}

// Workspace layout of ffn_nvfp4_forward / ffn_nvfp4_linear (each region
// 256-byte aligned): [h bf16 m*inter] [xq codes m*hidden/2] [xq scales
// m*hidden/16] [hq codes m*inter/2] [hq scales m*inter/16].
struct Carve {
  size_t h = 0, xq_c = 0, xq_s = 0, hq_c = 0, hq_s = 0, part = 0, part2 = 0, cnt = 0, xa_gu = 0, xa_d = 0,
         total = 0;
  ffn::TcPlan gate_up, down;
  ffn::PersistPlan persist;
  ffn::PlanesPlan planes;
};

// Workspace of the fixed format on the tensor-core path: quantised x and h
// codes, their 512-byte scale blocks, h, split-K partials.
void carve_w4a4_tc(Carve& c, size_t& off, int64_t m, int64_t hidden, int64_t inter, bool ffn) {
  const int sms = num_sms();
  if (ffn) {
    c.gate_up = ffn::plan_w4a4(m, 2 * inter, hidden, true, sms);
    c.down = ffn::plan_w4a4(m, hidden, inter, false, sms);
  } else {
    c.down = ffn::plan_w4a4(m, hidden, inter, false, sms);  // (n, k) = (hidden, inter)
  }
  c.xq_c = off; off += round_up((size_t)m * (ffn ? hidden : inter) / 2, 256);
  c.xq_s = off; off += round_up(ffn::w4a4_sf_block_bytes(m, ffn ? hidden : inter), 256);
  if (ffn) {
    c.hq_c = off; off += round_up((size_t)m * inter / 2, 256);
    c.hq_s = off; off += round_up(ffn::w4a4_sf_block_bytes(m, inter), 256);
  }
  const size_t pb = c.gate_up.partial_bytes > c.down.partial_bytes ? c.gate_up.partial_bytes
                                                                  : c.down.partial_bytes;
  c.part = off;
  off += round_up(pb, 256);
}

Carve carve_ffn(int64_t m, int64_t hidden, int64_t inter, ffn_act_format f, int64_t lora_rank = 0,
                bool planes = false) {
  Carve c;
  size_t off = 0;
  c.h = off;
  off += round_up((size_t)m * inter * 2, 256);
  if (lora_rank > 0) {  // the adapters' rank-r products, bf16
    c.xa_gu = off;
    off += round_up((size_t)m * 2 * lora_rank * 2, 256);
    c.xa_d = off;
    off += round_up((size_t)m * lora_rank * 2, 256);
  }
  if (f == FFN_ACT_BF16 && m > 0 && planes) {
    // x's and h's planes (codes, scale bytes), split-K partials of both
    // projections, the zeroed words (tile counters, ready flags) and the
    // row and chunk exponents
    c.planes = ffn::plan_planes(m, hidden, inter, num_sms());
    c.xq_c = off; off += round_up(c.planes.x_code_bytes, 256);
    c.xq_s = off; off += round_up(c.planes.x_sf_bytes, 256);
    c.hq_c = off; off += round_up(c.planes.h_code_bytes, 256);
    c.hq_s = off; off += round_up(c.planes.h_sf_bytes, 256);
    c.part = off; off += round_up(c.planes.gu_partial_bytes, 256);
    c.part2 = off; off += round_up(c.planes.dn_partial_bytes, 256);
    c.cnt = off; off += round_up((size_t)(c.planes.zero_ints + c.planes.other_ints) * sizeof(int), 256);
  } else if (f == FFN_ACT_BF16 && m > 0 && w4a16_persistent(m)) {
    c.persist = ffn::plan_persist(m, hidden, inter, num_sms());
    c.part = off;
    off += round_up(c.persist.partial_bytes, 256);
    c.cnt = off;
    off += round_up(c.persist.counter_bytes, 256);
  } else if (f == FFN_ACT_BF16 && m > 0 && w4a16_path(m) == Path::kTc) {
    const int sms = num_sms();
    c.gate_up = ffn::plan_tc(m, 2 * inter, hidden, true, sms);
    c.down = ffn::plan_tc(m, hidden, inter, false, sms);
    const size_t pb = c.gate_up.partial_bytes > c.down.partial_bytes ? c.gate_up.partial_bytes
                                                                    : c.down.partial_bytes;
    c.part = off;
    off += round_up(pb, 256);
  }
  if (f == FFN_ACT_NVFP4_FIXED && m > 0 && w4a4_path() == Path::kTc) {
    carve_w4a4_tc(c, off, m, hidden, inter, true);
  } else if (f == FFN_ACT_NVFP4_FIXED) {
    c.xq_c = off; off += round_up((size_t)m * hidden / 2, 256);
    c.xq_s = off; off += round_up((size_t)m * hidden / 16, 256);
    c.hq_c = off; off += round_up((size_t)m * inter / 2, 256);
    c.hq_s = off; off += round_up((size_t)m * inter / 16, 256);
  }
  c.total = off;
  return c;
}

// Workspace bytes for the path forward will take, which can depend on the
// handles' layouts: the larger of the two few-row candidates.
size_t ffn_workspace_bytes(int64_t m, int64_t hidden, int64_t inter, ffn_act_format f, int64_t lora_rank) {
  size_t b = carve_ffn(m, hidden, inter, f, lora_rank, false).total;
  const int forced = w4a16_forced();
  if (f == FFN_ACT_BF16 && lora_rank == 0 && (forced == 0 || forced == 4) && ffn::planes_for_rows(m) > 0) {
    const size_t bp = carve_ffn(m, hidden, inter, f, lora_rank, true).total;
    if (bp > b) b = bp;
  }
  return b;
}

Carve carve_linear(int64_t m, int64_t n, int64_t k, ffn_act_format f) {
  Carve c;
  size_t off = 0;
  if (f == FFN_ACT_BF16 && m > 0 && w4a16_path(m) == Path::kTc) {
    c.down = ffn::plan_tc(m, n, k, false, num_sms());
    c.part = off;
    off += round_up(c.down.partial_bytes, 256);
  }
  if (f == FFN_ACT_NVFP4_FIXED && m > 0 && w4a4_path() == Path::kTc) {
    carve_w4a4_tc(c, off, m, n, k, false);
  } else if (f == FFN_ACT_NVFP4_FIXED) {
    c.xq_c = off; off += round_up((size_t)m * k / 2, 256);
    c.xq_s = off; off += round_up((size_t)m * k / 16, 256);
  }
  c.total = off;
  return c;
}

template <class T>
ffn_status alloc(T** p, size_t bytes, size_t* total = nullptr) {
  if (cudaMalloc(reinterpret_cast<void**>(p), bytes) != cudaSuccess) {
    cudaGetLastError();
    *p = nullptr;
    return FFN_ERR_OOM;
  }
  if (total) *total += bytes;
  return FFN_OK;
}

void free_weight(ffn_nvfp4_weight* w) {
  if (!w) return;
  cudaFree(w->codes);
  cudaFree(w->scales);
  cudaFree(w->gs);
  cudaFree(w->tiled);
  cudaFree(w->tiled16);
  delete w;
}

}  // namespace

void ffn::handle_tc_view(const ffn_nvfp4_weight* w, ffn::TcWeight* out, bool* gate_up) {
  *out = w->tc();
  *gate_up = w->gate_up != 0;
}

ffn_status ffn::handle_check_device(const ffn_nvfp4_weight* w) { return check_device(w); }

extern "C" {

const char* ffn_status_string(ffn_status s) {
  switch (s) {
    case FFN_OK: return "FFN_OK";
    case FFN_ERR_INVALID_ARG: return "FFN_ERR_INVALID_ARG";
    case FFN_ERR_SHAPE: return "FFN_ERR_SHAPE";
    case FFN_ERR_ALIGNMENT: return "FFN_ERR_ALIGNMENT";
    case FFN_ERR_UNSUPPORTED: return "FFN_ERR_UNSUPPORTED";
    case FFN_ERR_CUDA: return "FFN_ERR_CUDA";
    case FFN_ERR_OOM: return "FFN_ERR_OOM";
    case FFN_ERR_WORKSPACE: return "FFN_ERR_WORKSPACE";
  }
  return "FFN_ERR_UNKNOWN";
}

int ffn_nvfp4_abi_version(void) { return FFN_NVFP4_ABI_VERSION; }

ffn_status ffn_nvfp4_quantize_weights(const void* w_bf16, int64_t n, int64_t k, void* codes,
                                      void* block_scales, float* global_scale, void* stream) {
  if (!w_bf16 || !codes || !block_scales || !global_scale) return FFN_ERR_INVALID_ARG;
  if (n <= 0 || !valid_k(k)) return FFN_ERR_SHAPE;
  if (!aligned16(w_bf16) || !aligned16(codes) || !aligned16(block_scales) ||
      (reinterpret_cast<uintptr_t>(global_scale) & 3u))
    return FFN_ERR_ALIGNMENT;
  if (ffn_status st = precheck()) return st;
  return cuda_status(ffn::launch_quantize_weights(w_bf16, n, k, codes, block_scales,
                                                  global_scale, as_stream(stream)));
}

ffn_status ffn_nvfp4_quantize_activations(const void* x_bf16, int64_t m, int64_t k, void* codes,
                                          void* block_scales, void* stream) {
  if (m < 0) return FFN_ERR_INVALID_ARG;
  if (!valid_k(k)) return FFN_ERR_SHAPE;
  if (m == 0) return FFN_OK;
  if (!x_bf16 || !codes || !block_scales) return FFN_ERR_INVALID_ARG;
  if (!aligned16(x_bf16) || !aligned16(codes) || !aligned16(block_scales))
    return FFN_ERR_ALIGNMENT;
  if (ffn_status st = precheck()) return st;
  return cuda_status(
      ffn::launch_quantize_activations(x_bf16, m, k, codes, block_scales, as_stream(stream)));
}

ffn_status ffn_nvfp4_weight_create_ex(const void* codes, const void* block_scales,
                                      const float* global_scale, int64_t n, int64_t k,
                                      unsigned formats, void* stream, ffn_nvfp4_weight** out) {
  if (!out) return FFN_ERR_INVALID_ARG;
  *out = nullptr;
  if (!codes || !block_scales || !global_scale) return FFN_ERR_INVALID_ARG;
  if (formats == 0 || (formats & ~(unsigned)FFN_FORMAT_ALL)) return FFN_ERR_INVALID_ARG;
  if (n <= 0 || !valid_k(k)) return FFN_ERR_SHAPE;
  if (!aligned16(codes) || !aligned16(block_scales)) return FFN_ERR_ALIGNMENT;
  if (ffn_status st = precheck()) return st;
  auto* w = new (std::nothrow) ffn_nvfp4_weight;
  if (!w) return FFN_ERR_OOM;
  w->n = n;
  w->k = k;
  w->formats = formats;
  cudaGetDevice(&w->device);
  const cudaStream_t s = as_stream(stream);
  ffn_status st = FFN_OK;
  if ((st = alloc(&w->gs, 2 * sizeof(float), &w->bytes))) {
    free_weight(w);
    return st;
  }
  cudaError_t e = cudaMemcpyAsync(w->gs, global_scale, sizeof(float), cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess && keep_canonical()) {
    if ((st = alloc(&w->codes, (size_t)n * k / 2, &w->bytes)) ||
        (st = alloc(&w->scales, (size_t)n * k / 16, &w->bytes))) {
      free_weight(w);
      return st;
    }
    e = cudaMemcpyAsync(w->codes, codes, (size_t)n * k / 2, cudaMemcpyDeviceToDevice, s);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(w->scales, block_scales, (size_t)n * k / 16, cudaMemcpyDeviceToDevice, s);
  }
  const size_t tb = (size_t)ffn::tc_tiled_bytes(n, k, false);
  const auto* c8 = static_cast<const uint8_t*>(codes);
  const auto* s8 = static_cast<const uint8_t*>(block_scales);
  if (e == cudaSuccess && (formats & FFN_FORMAT_NVFP4_FIXED)) {
    if ((st = alloc(&w->tiled, tb, &w->bytes))) {
      free_weight(w);
      return st;
    }
    e = ffn::launch_tile_weight(c8, s8, n, k, false, false, w->tiled, s);
  }
  if (e == cudaSuccess && (formats & FFN_FORMAT_BF16)) {
    if ((st = alloc(&w->tiled16, tb, &w->bytes))) {
      free_weight(w);
      return st;
    }
    e = ffn::launch_tile_weight(c8, s8, n, k, false, true, w->tiled16, s);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    free_weight(w);
    return FFN_ERR_CUDA;
  }
  *out = w;
  return FFN_OK;
}

ffn_status ffn_nvfp4_weight_create(const void* codes, const void* block_scales,
                                   const float* global_scale, int64_t n, int64_t k,
                                   void* stream, ffn_nvfp4_weight** out) {
  return ffn_nvfp4_weight_create_ex(codes, block_scales, global_scale, n, k, FFN_FORMAT_ALL, stream,
                                    out);
}

ffn_status ffn_nvfp4_weight_create_gate_up(const ffn_nvfp4_weight* gate,
                                           const ffn_nvfp4_weight* up, void* stream,
                                           ffn_nvfp4_weight** out) {
  if (!out) return FFN_ERR_INVALID_ARG;
  *out = nullptr;
  if (!gate || !up) return FFN_ERR_INVALID_ARG;
  if (gate->gate_up || up->gate_up) return FFN_ERR_INVALID_ARG;
  if (gate->n != up->n || gate->k != up->k) return FFN_ERR_SHAPE;
  if (gate->device != up->device) return FFN_ERR_INVALID_ARG;
  const unsigned formats = gate->formats & up->formats;
  if (!formats) return FFN_ERR_UNSUPPORTED;
  if (ffn_status st = check_device(gate)) return st;
  if (ffn_status st = precheck()) return st;
  const int64_t I = gate->n, H = gate->k;
  auto* w = new (std::nothrow) ffn_nvfp4_weight;
  if (!w) return FFN_ERR_OOM;
  w->n = 2 * I;
  w->k = H;
  w->gate_up = 1;
  w->formats = formats;
  cudaGetDevice(&w->device);
  const cudaStream_t s = as_stream(stream);
  ffn_status st = FFN_OK;
  if ((st = alloc(&w->gs, 2 * sizeof(float), &w->bytes))) {
    free_weight(w);
    return st;
  }
  cudaError_t e = cudaMemcpyAsync(w->gs, gate->gs, sizeof(float), cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(w->gs + 1, up->gs, sizeof(float), cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess && gate->codes && up->codes) {
    const size_t cb = (size_t)I * H / 2, sb = (size_t)I * H / 16;
    if ((st = alloc(&w->codes, 2 * cb, &w->bytes)) || (st = alloc(&w->scales, 2 * sb, &w->bytes))) {
      free_weight(w);
      return st;
    }
    e = cudaMemcpyAsync(w->codes, gate->codes, cb, cudaMemcpyDeviceToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(w->codes + cb, up->codes, cb, cudaMemcpyDeviceToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(w->scales, gate->scales, sb, cudaMemcpyDeviceToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(w->scales + sb, up->scales, sb, cudaMemcpyDeviceToDevice, s);
  }
  // the fused tiles are re-tiled from the parts' tiled copies, byte for byte
  const size_t tb = (size_t)ffn::tc_tiled_bytes(2 * I, H, true);
  if (e == cudaSuccess && (formats & FFN_FORMAT_NVFP4_FIXED)) {
    if ((st = alloc(&w->tiled, tb, &w->bytes))) {
      free_weight(w);
      return st;
    }
    e = ffn::launch_retile_gate_up(gate->tiled, up->tiled, I, H, w->tiled, s);
  }
  if (e == cudaSuccess && (formats & FFN_FORMAT_BF16)) {
    if ((st = alloc(&w->tiled16, tb, &w->bytes))) {
      free_weight(w);
      return st;
    }
    e = ffn::launch_retile_gate_up(gate->tiled16, up->tiled16, I, H, w->tiled16, s);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    free_weight(w);
    return FFN_ERR_CUDA;
  }
  *out = w;
  return FFN_OK;
}

ffn_status ffn_nvfp4_weight_destroy(ffn_nvfp4_weight* w) {
  if (!w) return FFN_OK;
  const cudaError_t e = cudaDeviceSynchronize();
  free_weight(w);
  return cuda_status(e);
}

ffn_status ffn_nvfp4_weight_dims(const ffn_nvfp4_weight* w, int64_t* n, int64_t* k,
                                 int* is_gate_up) {
  if (!w) return FFN_ERR_INVALID_ARG;
  if (n) *n = w->n;
  if (k) *k = w->k;
  if (is_gate_up) *is_gate_up = w->gate_up;
  return FFN_OK;
}

ffn_status ffn_nvfp4_weight_info(const ffn_nvfp4_weight* w, unsigned* formats, size_t* device_bytes) {
  if (!w) return FFN_ERR_INVALID_ARG;
  if (formats) *formats = w->formats;
  if (device_bytes) *device_bytes = w->bytes;
  return FFN_OK;
}

ffn_status ffn_nvfp4_workspace_size(int64_t m, int64_t hidden, int64_t inter,
                                    ffn_act_format format, size_t* bytes) {
  if (!bytes || m < 0) return FFN_ERR_INVALID_ARG;
  if (format != FFN_ACT_BF16 && format != FFN_ACT_NVFP4_FIXED) return FFN_ERR_INVALID_ARG;
  if (!valid_k(hidden) || !valid_k(inter)) return FFN_ERR_SHAPE;
  *bytes = ffn_workspace_bytes(m, hidden, inter, format, 0);
  return FFN_OK;
}

ffn_status ffn_nvfp4_forward_lora(const void* x, int64_t m, int64_t hidden, int64_t inter,
                                  const ffn_nvfp4_weight* gate_up, const ffn_nvfp4_weight* down,
                                  const ffn_lora* lora, ffn_act_format format, void* out,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  if (m < 0 || !gate_up || !down) return FFN_ERR_INVALID_ARG;
  const ffn::LoraView lv = ffn::lora_view(lora);
  if (lora) {
    if (format != FFN_ACT_BF16 || w4a16_forced() == 1) return FFN_ERR_UNSUPPORTED;
    if (ffn::lora_dims_mismatch(lora, hidden, inter)) return FFN_ERR_SHAPE;
  }
  if (format != FFN_ACT_BF16 && format != FFN_ACT_NVFP4_FIXED) return FFN_ERR_INVALID_ARG;
  if (!valid_k(hidden) || !valid_k(inter)) return FFN_ERR_SHAPE;
  if (!gate_up->gate_up || down->gate_up) return FFN_ERR_INVALID_ARG;
  if (gate_up->n != 2 * inter || gate_up->k != hidden || down->n != hidden || down->k != inter)
    return FFN_ERR_SHAPE;
  if (m == 0) return FFN_OK;
  if (!x || !out) return FFN_ERR_INVALID_ARG;
  if (ffn_status st = check_device(gate_up)) return st;
  if (ffn_status st = check_device(down)) return st;
  if (!serves(gate_up, format) || !serves(down, format)) return FFN_ERR_UNSUPPORTED;
  if (lora) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
      cudaGetLastError();
      return FFN_ERR_CUDA;
    }
    if (dev != lv.device) return FFN_ERR_INVALID_ARG;
  }
  const bool planes = format == FFN_ACT_BF16 && lv.rank == 0 && w4a16_planes(m, hidden, inter, gate_up, down);
  const Carve c = carve_ffn(m, hidden, inter, format, lv.rank, planes);
  if (!workspace || workspace_bytes < c.total) return FFN_ERR_WORKSPACE;
  if (!aligned16(x) || !aligned16(out) || !aligned16(workspace)) return FFN_ERR_ALIGNMENT;
  if (ffn_status st = precheck()) return st;
  const cudaStream_t s = as_stream(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* h = ws + c.h;
  cudaError_t e;
  if (planes) {
    ffn::PlanesBuffers b;
    b.xq = ws + c.xq_c;
    b.xs = ws + c.xq_s;
    b.hq = ws + c.hq_c;
    b.hs = ws + c.hq_s;
    b.part_gu = ws + c.part;
    b.part_dn = ws + c.part2;
    b.ints = reinterpret_cast<int*>(ws + c.cnt);
    e = ffn::launch_planes_ffn(x, m, gate_up->tc(), down->tc(), c.planes, b, out, s);
  } else if (format == FFN_ACT_BF16 && w4a16_persistent(m)) {
    e = ffn::launch_persist_ffn(x, m, gate_up->tc(), down->tc(), c.persist, h, ws + c.part,
                                reinterpret_cast<int*>(ws + c.cnt), out, s, lv, ws + c.xa_gu, ws + c.xa_d);
  } else if (format == FFN_ACT_BF16 && w4a16_path(m) == Path::kTc) {
    void* part = ws + c.part;
    ffn::LoraArgs lg, ld;
    e = cudaSuccess;
    if (lv.rank > 0 && lv.a_gu) {
      e = ffn::launch_lora_xa(x, m, hidden, lv.a_gu, 2 * lv.rank, ws + c.xa_gu, s);
      lg.xa = reinterpret_cast<const uint16_t*>(ws + c.xa_gu);
      lg.xa_ld = 2 * lv.rank;
      lg.b0 = lv.b_g;
      lg.b1 = lv.b_u;
      lg.off1 = lv.rank;
      lg.r = lv.rank;
    }
    if (e == cudaSuccess) e = ffn::launch_tc_w4a16(x, m, gate_up->tc(), true, c.gate_up, h, part, s, lg);
    if (e == cudaSuccess && lv.rank > 0 && lv.a_d) {
      e = ffn::launch_lora_xa(h, m, inter, lv.a_d, lv.rank, ws + c.xa_d, s);
      ld.xa = reinterpret_cast<const uint16_t*>(ws + c.xa_d);
      ld.xa_ld = lv.rank;
      ld.b0 = lv.b_d;
      ld.r = lv.rank;
    }
    if (e == cudaSuccess) e = ffn::launch_tc_w4a16(h, m, down->tc(), false, c.down, out, part, s, ld);
  } else if (format == FFN_ACT_BF16) {
    e = ffn::launch_gemv_w4a16(x, m, gate_up->view(), Epilogue::kSiluMul, h, s);
    if (e == cudaSuccess) e = ffn::launch_gemv_w4a16(h, m, down->view(), Epilogue::kStore, out, s);
  } else if (w4a4_path() == Path::kTc) {
    uint8_t *xq = ws + c.xq_c, *xs = ws + c.xq_s, *hq = ws + c.hq_c, *hs = ws + c.hq_s;
    void* part = ws + c.part;
    e = ffn::launch_quantize_activations_blocked(x, m, hidden, xq, xs, s);
    if (c.gate_up.splits == 1 && w4a4_fuse_hq()) {
      // h is quantised in the gate+up epilogue, bit for bit as the quantiser would
      if (e == cudaSuccess)
        e = ffn::launch_tc_w4a4(xq, xs, m, gate_up->tc(), true, c.gate_up, h, part, s, hq, hs);
    } else {
      if (e == cudaSuccess) e = ffn::launch_tc_w4a4(xq, xs, m, gate_up->tc(), true, c.gate_up, h, part, s);
      if (e == cudaSuccess) e = ffn::launch_quantize_activations_blocked(h, m, inter, hq, hs, s);
    }
    if (e == cudaSuccess) e = ffn::launch_tc_w4a4(hq, hs, m, down->tc(), false, c.down, out, part, s);
  } else {
    uint8_t *xq = ws + c.xq_c, *xs = ws + c.xq_s, *hq = ws + c.hq_c, *hs = ws + c.hq_s;
    e = ffn::launch_quantize_activations(x, m, hidden, xq, xs, s);
    if (e == cudaSuccess)
      e = ffn::launch_gemv_w4a4(xq, xs, m, gate_up->view(), Epilogue::kSiluMul, h, s);
    if (e == cudaSuccess) e = ffn::launch_quantize_activations(h, m, inter, hq, hs, s);
    if (e == cudaSuccess)
      e = ffn::launch_gemv_w4a4(hq, hs, m, down->view(), Epilogue::kStore, out, s);
  }
  return cuda_status(e);
}

ffn_status ffn_nvfp4_projection_plan(int64_t m, int64_t n, int64_t k, ffn_act_format format,
                                     int role, ffn_projection_plan* out) {
  if (!out || m < 0 || n <= 0 || role < 0 || role > 2) return FFN_ERR_INVALID_ARG;
  if (format != FFN_ACT_BF16 && format != FFN_ACT_NVFP4_FIXED) return FFN_ERR_INVALID_ARG;
  const int gate_up = role == FFN_ROLE_GATE_UP;
  if (!valid_k(k) || (gate_up && n % 2)) return FFN_ERR_SHAPE;
  *out = ffn_projection_plan{FFN_KERNEL_NONE, 0, 1, 0};
  if (m == 0) return FFN_OK;
  const int ncols = (int)(gate_up ? n / 2 : n);
  const int forced = w4a16_forced();
  if (format == FFN_ACT_BF16 && role != FFN_ROLE_LINEAR && (forced == 0 || forced == 4) &&
      ffn::planes_for_rows(m) > 0) {
    // (when both handles hold the natural tiled layout; else the tc_w4a16 row)
    const ffn::PlanesPlan p = gate_up ? ffn::plan_planes(m, k, n / 2, num_sms()) : ffn::plan_planes(m, n, k, num_sms());
    // (without a LoRA adapter) one persistent kernel runs both projections;
    // K ranges per output tile: at most ceil(kc / (tiles * kc / parts)) + 1
    const int tiles = gate_up ? p.gu_tiles : p.dn_tiles, kc = gate_up ? p.gu_kc : p.dn_kc;
    const int parts = gate_up ? p.gu_parts : p.grid;
    const int64_t W = (int64_t)tiles * kc;
    const int splits = parts <= tiles ? (tiles % parts ? 2 : 1) : (int)(((int64_t)kc * parts + W - 1) / W + 1);
    *out = ffn_projection_plan{FFN_KERNEL_TC_PLANES, p.nt, gate_up && p.gu_parts == p.gu_tiles ? 1 : splits,
                               p.grid};
  } else if (format == FFN_ACT_BF16 && role != FFN_ROLE_LINEAR && w4a16_persistent(m)) {
    // gate+up: n = 2 * inter, k = hidden; down: n = hidden, k = inter
    const ffn::PersistPlan p = gate_up ? ffn::plan_persist(m, k, n / 2, num_sms())
                                       : ffn::plan_persist(m, n, k, num_sms());
    *out = gate_up ? ffn_projection_plan{FFN_KERNEL_TC_W4A16_PERSISTENT, p.bn, 1, p.gu_grid}
                   : ffn_projection_plan{FFN_KERNEL_TC_W4A16_PERSISTENT, p.bn, 0, p.dn_grid};
    if (!gate_up) {  // K ranges per output tile: at most ceil(kc / (tiles*kc/grid)) + 1
      const int64_t W = (int64_t)p.dn_tiles * p.dn_kc;
      out->k_splits = (int)(((int64_t)p.dn_kc * p.dn_grid + W - 1) / W + 1);
    }
  } else if (format == FFN_ACT_BF16 && w4a16_path(m) == Path::kTc) {
    const ffn::TcPlan p = ffn::plan_tc(m, n, k, gate_up != 0, num_sms());
    *out = ffn_projection_plan{FFN_KERNEL_TC_W4A16, p.bn, p.splits, p.xtiles * p.wtiles * p.splits};
  } else if (format == FFN_ACT_BF16) {
    *out = ffn_projection_plan{FFN_KERNEL_GEMV_W4A16, 0, 1, ffn::gemv_grid(ncols)};
  } else if (w4a4_path() == Path::kTc) {
    const ffn::TcPlan p = ffn::plan_w4a4(m, n, k, gate_up != 0, num_sms());
    *out = ffn_projection_plan{FFN_KERNEL_TC_W4A4, p.bn, p.splits, p.xtiles * p.wtiles * p.splits};
  } else {
    *out = ffn_projection_plan{FFN_KERNEL_GEMV_W4A4, 0, 1, ffn::gemv_grid(ncols)};
  }
  return FFN_OK;
}

ffn_status ffn_nvfp4_forward(const void* x, int64_t m, int64_t hidden, int64_t inter,
                             const ffn_nvfp4_weight* gate_up, const ffn_nvfp4_weight* down,
                             ffn_act_format format, void* out, void* workspace,
                             size_t workspace_bytes, void* stream) {
  return ffn_nvfp4_forward_lora(x, m, hidden, inter, gate_up, down, nullptr, format, out, workspace,
                                workspace_bytes, stream);
}

ffn_status ffn_nvfp4_workspace_size_lora(int64_t m, int64_t hidden, int64_t inter,
                                         ffn_act_format format, const ffn_lora* lora, size_t* bytes) {
  if (!bytes || m < 0) return FFN_ERR_INVALID_ARG;
  if (format != FFN_ACT_BF16 && format != FFN_ACT_NVFP4_FIXED) return FFN_ERR_INVALID_ARG;
  if (!valid_k(hidden) || !valid_k(inter)) return FFN_ERR_SHAPE;
  *bytes = ffn_workspace_bytes(m, hidden, inter, format, ffn::lora_view(lora).rank);
  return FFN_OK;
}

ffn_status ffn_nvfp4_device_error(int* flags, int clear) {
  if (!flags) return FFN_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    return FFN_ERR_CUDA;
  }
  return cuda_status(ffn::read_device_error(flags, clear != 0));
}

ffn_status ffn_nvfp4_linear_workspace_size(int64_t m, int64_t n, int64_t k,
                                           ffn_act_format format, size_t* bytes) {
  if (!bytes || m < 0 || n <= 0) return FFN_ERR_INVALID_ARG;
  if (format != FFN_ACT_BF16 && format != FFN_ACT_NVFP4_FIXED) return FFN_ERR_INVALID_ARG;
  if (!valid_k(k)) return FFN_ERR_SHAPE;
  *bytes = carve_linear(m, n, k, format).total;
  return FFN_OK;
}

ffn_status ffn_nvfp4_linear(const void* x, int64_t m, const ffn_nvfp4_weight* w,
                            ffn_act_format format, void* y, void* workspace,
                            size_t workspace_bytes, void* stream) {
  if (m < 0 || !w) return FFN_ERR_INVALID_ARG;
  if (format != FFN_ACT_BF16 && format != FFN_ACT_NVFP4_FIXED) return FFN_ERR_INVALID_ARG;
  if (w->gate_up) return FFN_ERR_UNSUPPORTED;
  if (m == 0) return FFN_OK;
  if (!x || !y) return FFN_ERR_INVALID_ARG;
  if (ffn_status st = check_device(w)) return st;
  if (!serves(w, format)) return FFN_ERR_UNSUPPORTED;
  const Carve c = carve_linear(m, w->n, w->k, format);
  if (c.total && (!workspace || workspace_bytes < c.total)) return FFN_ERR_WORKSPACE;
  if (!aligned16(x) || !aligned16(y) || (c.total && !aligned16(workspace)))
    return FFN_ERR_ALIGNMENT;
  if (ffn_status st = precheck()) return st;
  const cudaStream_t s = as_stream(stream);
  cudaError_t e;
  if (format == FFN_ACT_BF16 && w4a16_path(m) == Path::kTc) {
    e = ffn::launch_tc_w4a16(x, m, w->tc(), false, c.down, y, static_cast<uint8_t*>(workspace) + c.part, s);
  } else if (format == FFN_ACT_BF16) {
    e = ffn::launch_gemv_w4a16(x, m, w->view(), Epilogue::kStore, y, s);
  } else if (w4a4_path() == Path::kTc) {
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    e = ffn::launch_quantize_activations_blocked(x, m, w->k, ws + c.xq_c, ws + c.xq_s, s);
    if (e == cudaSuccess)
      e = ffn::launch_tc_w4a4(ws + c.xq_c, ws + c.xq_s, m, w->tc(), false, c.down, y, ws + c.part, s);
  } else {
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    e = ffn::launch_quantize_activations(x, m, w->k, ws + c.xq_c, ws + c.xq_s, s);
    if (e == cudaSuccess)
      e = ffn::launch_gemv_w4a4(ws + c.xq_c, ws + c.xq_s, m, w->view(), Epilogue::kStore, y, s);
  }
  return cuda_status(e);
}

}  // extern "C"
