/*
 * ffn_nvfp4.h -- C ABI of the NVFP4 dense SwiGLU FFN for NVIDIA B200 (sm_100a).
 *
 * The library computes one LLM serving layer,
 *
 *     out = down( silu( gate(x) ) * up(x) )
 *
 * over NVFP4 weights: FP4 E2M1 codes, one FP8 E4M3 scale per 16 consecutive
 * elements along K, and one FP32 scale per tensor.  Activations are bf16
 * (W4A16), or, in the fixed activation format, are themselves quantised per
 * row to NVFP4 before every projection (W4A4) so that a row's output bits do
 * not depend on how many rows share the call.
 *
 * Where each operation comes from (pages of the metrale engine's source):
 *  - the FFN dataflow (gate and up into bf16 buffers, silu_mul in place, down
 *    from the activated buffer): "metrale_model_layers/layers/
 *    dense_ffn_fixed.rs", DenseFfnLayer::forward_fixed, and
 *    "metrale_model_layers/layers/dense_ffn_prefill.rs", prefill_q2;
 *  - the fixed activation format and its row-count invariance: the module
 *    comment of "metrale_model_layers/layers/dense_ffn_fixed.rs";
 *  - one NVFP4 projection for m rows (the W4A16 GEMM family and its m
 *    dispatch): "metrale_model_layers/layers/dense_ffn_prefill.rs",
 *    DenseFfnLayer::w4a16_prefill_gemm;
 *  - the fused [2*inter, hidden] gate+up weight whose halves are the gate and
 *    up weights: "metrale_model_layers/layers/dense_ffn_overlays.rs",
 *    set_fp8_gate_up_fused;
 *  - errors instead of silent fallbacks: the bail!/ensure! results of the
 *    same pages.
 * The NVFP4 encoding is the public one (OCP MX v1.0 FP4 E2M1 elements, OCP
 * OFP8 E4M3 block scales); the conventions for the scales are stated at
 * ffn_nvfp4_quantize_weights and ffn_nvfp4_quantize_activations.
 *
 * Conventions for every entry point
 *  - All tensor pointers are DEVICE pointers on the current CUDA device unless
 *    a parameter says otherwise; the caller owns them.  Work is enqueued on
 *    `stream` (a cudaStream_t passed as void*; NULL = the legacy default
 *    stream).  No entry point synchronises the stream, and the compute entry
 *    points (quantize_*, forward, linear) allocate no memory.
 *  - Row-major layouts: a [rows, cols] tensor has cols contiguous.
 *    bf16 tensors are IEEE bfloat16 bit patterns.
 *  - NVFP4 tensors of logical shape [rows, k]: `codes` is uint8 [rows, k/2],
 *    byte j holding element 2j in its low nibble and 2j+1 in its high nibble
 *    (nibble: bit 3 sign, bits 0-2 magnitude index into {0,.5,1,1.5,2,3,4,6});
 *    `block_scales` is uint8 [rows, k/16], one E4M3 byte per 16 elements.
 *  - Pointers must be 16-byte aligned; k must be a multiple of 32.
 *  - On any error nothing is launched and an ffn_status other than FFN_OK is
 *    returned; asynchronous CUDA errors of earlier work surface as
 *    FFN_ERR_CUDA from the next call or at the caller's stream synchronise.
 *    No entry point aborts the process.
 */
#ifndef FFN_NVFP4_H
#define FFN_NVFP4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FFN_NVFP4_ABI_VERSION 1

typedef enum ffn_status {
  FFN_OK = 0,
  FFN_ERR_INVALID_ARG = 1, /* null pointer, negative size, bad enum value   */
  FFN_ERR_SHAPE = 2,       /* dims not multiples of 32, handle dims mismatch */
  FFN_ERR_ALIGNMENT = 3,   /* a pointer is not 16-byte aligned              */
  FFN_ERR_UNSUPPORTED = 4, /* a valid request this build does not serve     */
  FFN_ERR_CUDA = 5,        /* a CUDA runtime call or launch failed          */
  FFN_ERR_OOM = 6,         /* device allocation failed (handle creation)    */
  FFN_ERR_WORKSPACE = 7    /* workspace missing or smaller than required    */
} ffn_status;

typedef enum ffn_act_format {
  FFN_ACT_BF16 = 0,        /* W4A16: bf16 activations                       */
  FFN_ACT_NVFP4_FIXED = 1  /* W4A4: activations quantised per row to NVFP4  */
} ffn_act_format;

/* Opaque NVFP4 weight: owns device copies of the codes, the block scales and
 * the tensor scale(s), plus the re-tiled copies the kernels read.  Immutable
 * after creation; may be shared by concurrent calls on several streams. */
typedef struct ffn_nvfp4_weight ffn_nvfp4_weight;

/* Human-readable name of a status code (static storage). */
const char* ffn_status_string(ffn_status s);

/* FFN_NVFP4_ABI_VERSION of the built library. */
int ffn_nvfp4_abi_version(void);

/* Quantise a bf16 weight W[n, k] to NVFP4.  (The pages name NVFP4 weights
 * but print no quantiser; the format is the public NVFP4 one, readings
 * R1-R4 of the design notes.)
 *   w_bf16        [n, k] bf16 (input)
 *   codes         uint8 [n, k/2]  (output)
 *   block_scales  uint8 [n, k/16] (output, E4M3)
 *   global_scale  one float (output, device)
 * Arithmetic (all fp32, round-to-nearest-even): amax = max|W|;
 * gs = amax / 2688 (2688 = 6 * 448; gs = 1 if amax == 0); per 16-element block
 * t = (block amax / gs) / 6, s = E4M3(t) with saturation to 448,
 * sdec = E4M3value(s) * gs, code = E2M1(w / sdec) rounding to nearest with
 * ties to the even magnitude index, saturating at 6 and keeping the sign bit;
 * a block whose s (or sdec) is zero gets code 0 throughout.  The result is
 * deterministic and bit-reproducible.  Inputs must be finite.
 * Launches three kernels; no host synchronisation. */
ffn_status ffn_nvfp4_quantize_weights(const void* w_bf16, int64_t n, int64_t k,
                                      void* codes, void* block_scales,
                                      float* global_scale, void* stream);

/* Quantise bf16 activations X[m, k] per row to NVFP4, as the fixed format does
 * before each projection ("metrale_model_layers/layers/dense_ffn_fixed.rs",
 * forward_fixed: nvfp4_proj_mx on bf16 rows): per 16-element block s = E4M3(block amax / 6) (fp32,
 * nearest even, saturating), code = E2M1(x / E4M3value(s)), no tensor scale;
 * all-zero block when s == 0.  codes uint8 [m, k/2], block_scales uint8
 * [m, k/16].  Exposed so callers can check the activation codes bit for bit. */
ffn_status ffn_nvfp4_quantize_activations(const void* x_bf16, int64_t m, int64_t k,
                                          void* codes, void* block_scales,
                                          void* stream);

/* Activation formats a weight handle is built for (bit set). */
typedef enum ffn_weight_formats {
  FFN_FORMAT_BF16 = 1,         /* serves FFN_ACT_BF16 (W4A16)         */
  FFN_FORMAT_NVFP4_FIXED = 2,  /* serves FFN_ACT_NVFP4_FIXED (W4A4)   */
  FFN_FORMAT_ALL = 3
} ffn_weight_formats;

/* Build a weight handle from NVFP4 tensors of logical shape [n, k] (codes,
 * block_scales as above, global_scale one device float) for the activation
 * formats in `formats` (FFN_FORMAT_* bits, not 0).  Reads the caller's
 * buffers (which it may free afterwards) and builds, per format, one
 * re-tiled copy in the layout that format's kernels stream: 0.5625 bytes per
 * weight and format, plus tile padding -- the canonical copy is not kept.
 * Allocates device memory; enqueues its work on `stream`; the handle is
 * usable by later work on `stream` (other streams: synchronise first).
 * Errors: FFN_ERR_SHAPE unless n > 0 and k is a positive multiple of 32;
 * FFN_ERR_INVALID_ARG for formats outside FFN_FORMAT_ALL or 0.  Using a
 * handle with a format it was not built for returns FFN_ERR_UNSUPPORTED. */
ffn_status ffn_nvfp4_weight_create_ex(const void* codes, const void* block_scales,
                                      const float* global_scale, int64_t n, int64_t k,
                                      unsigned formats, void* stream, ffn_nvfp4_weight** out);

/* ffn_nvfp4_weight_create_ex with FFN_FORMAT_ALL (both activation formats). */
ffn_status ffn_nvfp4_weight_create(const void* codes, const void* block_scales,
                                   const float* global_scale, int64_t n, int64_t k,
                                   void* stream, ffn_nvfp4_weight** out);

/* Fused gate+up handle of logical shape [2*inter, hidden]
 * ("metrale_model_layers/layers/dense_ffn_overlays.rs", set_fp8_gate_up_fused:
 * one [2I, H] buffer whose halves are the gate and up weights): rows [0, inter)
 * are `gate`, rows [inter, 2*inter) are `up`, byte for byte, each keeping its
 * own tensor scale; built for the formats both parts serve (re-tiled from
 * their tiles; FFN_ERR_UNSUPPORTED if they share none).  `gate` and `up` must
 * share (n, k) and device and stay owned by the caller (they may be destroyed
 * afterwards). */
ffn_status ffn_nvfp4_weight_create_gate_up(const ffn_nvfp4_weight* gate,
                                           const ffn_nvfp4_weight* up, void* stream,
                                           ffn_nvfp4_weight** out);

/* Release a handle and its device memory (synchronises the device first, so
 * no queued work still reads it).  NULL is accepted. */
ffn_status ffn_nvfp4_weight_destroy(ffn_nvfp4_weight* w);

/* Logical dims of a handle; *is_gate_up = 1 for a fused gate+up handle. */
ffn_status ffn_nvfp4_weight_dims(const ffn_nvfp4_weight* w, int64_t* n, int64_t* k,
                                 int* is_gate_up);

/* The FFN_FORMAT_* bits a handle serves and the device bytes it holds
 * (either pointer may be NULL). */
ffn_status ffn_nvfp4_weight_info(const ffn_nvfp4_weight* w, unsigned* formats,
                                 size_t* device_bytes);

/* Workspace bytes ffn_nvfp4_forward needs for (m, hidden, inter, format). */
ffn_status ffn_nvfp4_workspace_size(int64_t m, int64_t hidden, int64_t inter,
                                    ffn_act_format format, size_t* bytes);

/* The FFN layer for m rows ("metrale_model_layers/layers/dense_ffn_prefill.rs",
 * forward_prefill_inner with its NVFP4 arm w4a16_prefill_gemm, for bf16
 * activations; "metrale_model_layers/layers/dense_ffn_fixed.rs", forward_fixed,
 * for the fixed format).
 *   x        [m, hidden] bf16
 *   gate_up  fused handle [2*inter, hidden] (ffn_nvfp4_weight_create_gate_up)
 *   down     handle [hidden, inter]
 *   out      [m, hidden] bf16; only rows 0..m-1 are written
 *   workspace device scratch of >= ffn_nvfp4_workspace_size bytes; holds the
 *            bf16 intermediate h = silu(g) * u and, in the fixed format, the
 *            quantised activations; contents are undefined afterwards.
 * Numerics: g = bf16(gs_g * sum x*w_g), u likewise, h = bf16(silu(g) * u),
 * out = bf16(gs_d * sum h*w_d), with fp32 accumulation.  In FFN_ACT_NVFP4_FIXED
 * x and h are quantised per row (as ffn_nvfp4_quantize_activations) before
 * their projections, and the kernels and reduction order do not depend on m,
 * so each output row is bit-identical whatever m is.
 * m == 0 is a no-op.  Allocates nothing and does not synchronise.
 * Launch order: the bf16-format kernels are launched with programmatic stream
 * serialisation, so each may start while the previous kernel in the stream is
 * finishing; it streams and dequantises weights meanwhile and waits for that
 * kernel's completion before reading x (or h) and before writing out, h or
 * the workspace.  Stream order is therefore kept for every buffer the call
 * reads or writes except the weight handles, which must not be modified by
 * an earlier kernel still in flight (handles are immutable after creation). */
ffn_status ffn_nvfp4_forward(const void* x, int64_t m, int64_t hidden, int64_t inter,
                             const ffn_nvfp4_weight* gate_up, const ffn_nvfp4_weight* down,
                             ffn_act_format format, void* out, void* workspace,
                             size_t workspace_bytes, void* stream);

/* LoRA adapters on the layer ("metrale_model_layers/layers/
 * dense_ffn_overlays.rs", set_lora_weights, apply_lora_gate_up,
 * apply_lora_down): for each of gate, up and down an optional pair A [r, in],
 * B [out, r] of bf16 (row-major; in/out = hidden/inter for gate and up,
 * inter/hidden for down), the delta of a projection being (x A^T) B^T.
 * Numerics: xa = bf16(x A^T) (fp32 sums), then each output
 * y = bf16(bf16(projection) + sum_i xa_i * B[n, i]) (fp32 sum, i ascending);
 * gate and up deltas are added before SiLU*mul, the down delta after the
 * down projection.  No scaling factor is applied (fold it into B).
 * A missing adapter is a NULL pair (both NULL); at least one must be given.
 * Copies the matrices to device memory the handle owns (the caller may free
 * its buffers once the stream has run the copies).  1 <= rank <=
 * FFN_LORA_MAX_RANK, else FFN_ERR_UNSUPPORTED; FFN_ERR_SHAPE unless hidden
 * and inter are multiples of 32; a half-given pair is FFN_ERR_INVALID_ARG. */
#define FFN_LORA_MAX_RANK 256
typedef struct ffn_lora ffn_lora;
ffn_status ffn_nvfp4_lora_create(int64_t rank, int64_t hidden, int64_t inter,
                                 const void* gate_a, const void* gate_b,
                                 const void* up_a, const void* up_b,
                                 const void* down_a, const void* down_b,
                                 void* stream, ffn_lora** out);
/* Synchronises the device, then frees the adapter's memory.  NULL is accepted. */
ffn_status ffn_nvfp4_lora_destroy(ffn_lora* lora);

/* ffn_nvfp4_forward with adapters (lora NULL: exactly ffn_nvfp4_forward).
 * Bf16 activations only (FFN_ERR_UNSUPPORTED for the fixed format, whose
 * page-defined path has no adapters); the handle must match hidden/inter
 * (FFN_ERR_SHAPE) and the current device (FFN_ERR_INVALID_ARG).  Two small
 * extra launches compute the rank-r products; the projections' epilogues add
 * the deltas.  Workspace: ffn_nvfp4_workspace_size_lora bytes. */
ffn_status ffn_nvfp4_workspace_size_lora(int64_t m, int64_t hidden, int64_t inter,
                                         ffn_act_format format, const ffn_lora* lora,
                                         size_t* bytes);
ffn_status ffn_nvfp4_forward_lora(const void* x, int64_t m, int64_t hidden, int64_t inter,
                                  const ffn_nvfp4_weight* gate_up, const ffn_nvfp4_weight* down,
                                  const ffn_lora* lora, ffn_act_format format, void* out,
                                  void* workspace, size_t workspace_bytes, void* stream);

/* One projection y[m, n] = bf16(gs * sum_k x[m, k] * w[n, k]) for a plain
 * (not gate+up) handle of shape [n, k] (one call of the per-projection GEMM
 * that "metrale_model_layers/layers/dense_ffn_prefill.rs", w4a16_prefill_gemm,
 * dispatches, e.g. the down projection); in FFN_ACT_NVFP4_FIXED x is quantised
 * per row first.  Workspace: ffn_nvfp4_linear_workspace_size bytes. */
ffn_status ffn_nvfp4_linear_workspace_size(int64_t m, int64_t n, int64_t k,
                                           ffn_act_format format, size_t* bytes);
ffn_status ffn_nvfp4_linear(const void* x, int64_t m, const ffn_nvfp4_weight* w,
                            ffn_act_format format, void* y, void* workspace,
                            size_t workspace_bytes, void* stream);

/* Allocation-free variant of ffn_nvfp4_linear for bf16 activations (W4A16),
 * for callers that cannot allocate device memory on the call path: for
 * example a plugin whose host framework owns every device allocation and
 * passes it no workspace, or serving code that must not call cudaMalloc once
 * running (cudaMalloc can synchronise the whole device).  The source pages
 * have no counterpart; this entry point exists only for such callers.
 *   x [m, k] bf16, w a plain (not gate+up) handle of shape [n, k],
 *   y [m, n] bf16 = bf16(gs * x @ w^T).  It always runs the tensor-core
 *   projection kernels (whatever kernel ffn_nvfp4_linear would pick for m).
 * The split-K partial sums live in one fixed 16 MiB device array that every
 * GPU context loading the library holds until the process exits; a shape
 * whose partials would need more returns FFN_ERR_WORKSPACE (nothing
 * launched).  It calls no cudaMalloc, cudaFree or allocating library routine.
 * Set-up: the first call in each CUDA context looks up that context's address
 * of the array (with the context current).  Under lazy module loading (the
 * CUDA default) that first lookup also loads the module and so reserves the
 * 16 MiB: it can fail with FFN_ERR_OOM and may synchronise.  Make the first
 * call at set-up time, before any stream capture.  A device reset creates a
 * new context, whose first call repeats the look-up.  All calls share the
 * array: calls that overlap on the GPU (other streams, other threads) race
 * and must be serialised by the caller.  Every partial a call reads is written
 * earlier in the same call, so nothing needs clearing. */
ffn_status ffn_nvfp4_linear_noalloc(const void* x, int64_t m, const ffn_nvfp4_weight* w,
                                    void* y, void* stream);

/* Kernel configuration a projection of m rows would use (the m-dispatch),
 * without launching anything; callable without a GPU (the SM count of the
 * current device is used when there is one, else 148).  Lets callers and
 * tests see which kernel family, activation tile width and split-K count
 * ffn_nvfp4_linear (role FFN_ROLE_LINEAR, shape [n, k]) or the projections of
 * ffn_nvfp4_forward (FFN_ROLE_GATE_UP: n = 2 * inter, k = hidden;
 * FFN_ROLE_DOWN: n = hidden, k = inter) select.
 * The m-tiered kernel choice follows "metrale_model_layers/layers/
 * dense_ffn_prefill.rs", DenseFfnLayer::w4a16_prefill_gemm (a projection
 * kernel chosen by m and the weight's shape); the tiers are this library's. */
typedef enum ffn_kernel_family {
  FFN_KERNEL_NONE = 0,       /* m == 0: nothing is launched                     */
  FFN_KERNEL_TC_W4A16 = 1,   /* tcgen05 kind::f16 MMA over dequantised weights  */
  FFN_KERNEL_TC_W4A4 = 2,    /* tcgen05 block-scaled FP4 MMA (kind::mxf4nvf4);
                                one activation tile of 128 rows per CTA, or of
                                16 rows for m <= 16, two CTAs per SM; the K
                                split depends on (n, k) only                   */
  FFN_KERNEL_GEMV_W4A16 = 3, /* CUDA-core projection, bf16 activations          */
  FFN_KERNEL_GEMV_W4A4 = 4,  /* CUDA-core projection, fixed activation format   */
  FFN_KERNEL_TC_W4A16_PERSISTENT = 5, /* few-row FFN layer: persistent tcgen05
                                kernels, one CTA per SM, gate+up over whole tiles,
                                down over equal K ranges reduced in-kernel
                                (only with FFN_NVFP4_W4A16_PATH=persistent)     */
  FFN_KERNEL_TC_PLANES = 6   /* FFN layer for m <= 2 with bf16 activations and
                                no LoRA adapter, when both handles hold the
                                natural tiled layout (built for the fixed format
                                too, e.g. FFN_FORMAT_ALL): the NVFP4 weights go
                                to the block-scaled FP4 MMA as stored and each
                                activation row as 8 NVFP4 planes (N = 16 columns):
                                2-bit digits of a 16-bit window below each
                                16-block's top bit, exact when the block's
                                elements lie within 2^8 of its largest (else
                                truncated below 2^-15 of the block maximum).
                                Two launches: a small prologue (x's planes,
                                counters) and one persistent kernel, two CTAs
                                per SM, all resident, for both projections
                                (gate+up whole tiles, or equal K ranges when the
                                tiles outnumber the CTAs; down equal K ranges;
                                split-K sums added in-kernel in K order).
                                tile_rows reports the MMA's N, grid the CTAs of
                                the persistent kernel.  Without the natural
                                layout the layer takes FFN_KERNEL_TC_W4A16.   */
} ffn_kernel_family;

typedef enum ffn_projection_role {
  FFN_ROLE_LINEAR = 0,   /* ffn_nvfp4_linear                                  */
  FFN_ROLE_GATE_UP = 1,  /* the fused gate+up projection of ffn_nvfp4_forward  */
  FFN_ROLE_DOWN = 2      /* the down projection of ffn_nvfp4_forward           */
} ffn_projection_role;

typedef struct ffn_projection_plan {
  int family;    /* ffn_kernel_family                                          */
  int tile_rows; /* activation rows per tile (the MMA's N); 0 for CUDA cores   */
  int k_splits;  /* K ranges whose fp32 partial sums are added afterwards in a
                    fixed order (1 = no split); for the persistent down
                    projection, the most ranges any output tile is cut into  */
  int grid;      /* CTAs of the projection kernel                              */
} ffn_projection_plan;

ffn_status ffn_nvfp4_projection_plan(int64_t m, int64_t n, int64_t k, ffn_act_format format,
                                     int role, ffn_projection_plan* out);

/* Measured dense tensor-core throughput of the current GPU, in TFLOP/s, for
 * the MMA kinds the library issues: kind = 0, tcgen05 kind::f16 (bf16 x bf16,
 * fp32 accumulate, M128 N256 K16, operands in shared memory); kind = 1,
 * kind::mxf4nvf4 with UE4M3 scales per 16 elements (E2M1 x E2M1, M128 N128
 * K64).  One CTA per SM, `issuers` (1 or 2) threads per CTA each issuing
 * `iters` MMAs back to back into its own accumulator; timed with CUDA events
 * on a private stream after a short warm-up launch.  A roofline denominator
 * for the kernels (no library exposes the block-scaled FP4 MMA), not part of
 * the FFN path.  Allocates 4 bytes of device memory for an error flag and
 * synchronises.  Returns FFN_ERR_CUDA if a wait gave up. */
ffn_status ffn_nvfp4_tensor_peak(int kind, int issuers, int iters, double* tflops);

/* Device-side error bits.  Kernels that wait on asynchronous copies or on
 * tensor-core completion give up after about two seconds instead of hanging,
 * free their tensor memory, skip their stores and OR a bit into a device-wide
 * error word (1: producer, 2: MMA issuer, 4: dequant or operand copy, 8:
 * epilogue, 16: drain or accumulator wait, 32: a wait for work of other CTAs
 * of the same launch, e.g. when they cannot all be resident because other
 * work holds the SMs).  Synchronises the device, writes the word to *flags and, if
 * clear != 0, resets it to zero.  0 means every kernel completed normally. */
ffn_status ffn_nvfp4_device_error(int* flags, int clear);

/* Per-kernel timing (opt-in tracing).  After ffn_nvfp4_profile_begin, every
 * kernel launch the library makes from the calling thread is bracketed by a
 * pair of CUDA events recorded on the launch's stream.  ffn_nvfp4_profile_end
 * stops recording, synchronises the device, and aggregates the durations per
 * kernel into out[0..*count) (name: static string; capacity entries at most,
 * FFN_ERR_INVALID_ARG if more distinct kernels ran).  Recording adds event
 * records to the streams but no device work; it creates CUDA events (host
 * resources) on first use and reuses them afterwards.  Launches made while
 * their stream is being captured into a CUDA graph get event-record nodes in
 * the graph instead: the durations are then those of the graph's latest
 * replay (replay it before ffn_nvfp4_profile_end).  Host-recorded events can
 * include time the device spends waiting for the host to submit the launch;
 * graph-recorded ones cannot. */
typedef struct ffn_kernel_time {
  const char* name;
  int launches;
  double total_ms;
} ffn_kernel_time;
ffn_status ffn_nvfp4_profile_begin(void);
ffn_status ffn_nvfp4_profile_end(ffn_kernel_time* out, int capacity, int* count);

#ifdef __cplusplus
}
#endif

#endif /* FFN_NVFP4_H */
