/*
 * nvfp4.h - C ABI of libnvfp4: NVFP4 W4A4 linear layers on B200 (sm_100a).
 *
 * The method ("Why Gated DeltaNet Survives 4-Bit Quantization: NVFP4 W4A4 for
 * the Recurrent Half of a Hybrid 27B LLM"):
 *   - page summary, "Background", item 1: NVFP4 = E2M1 4-bit values, one E4M3
 *     scale per 16-element block set to blockmax/6, one FP32 scale per tensor,
 *     enabling native 4-bit tensor-core GEMMs;
 *   - abstract and news article: W4A4, i.e. weights quantised once after
 *     calibration, activations quantised on the fly;
 *   - abstract, last sentence, and the news article's "Risks and caveats":
 *     checkpoints calibrated per module carry one FP32 global scale per module;
 *     when several modules are served as one fused GEMM each module's scale
 *     must govern its own output columns (the "global-scale mismatch" fix).
 *
 * Conventions shared by every call:
 *   - Pointers marked "device" are CUDA device (or managed) memory owned by the
 *     caller; "host" pointers are ordinary host memory.  The library never
 *     allocates or frees memory.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Work is
 *     enqueued on it and the call returns without waiting, except where a call
 *     says it synchronises.
 *   - Argument errors are detected before anything is enqueued and returned as
 *     a status; nvfp4_get_last_error_string() then describes the problem.  A
 *     failed launch returns NVFP4_ERR_CUDA.  Faults inside a kernel surface at
 *     the caller's next synchronisation, as usual for CUDA.
 *   - Every wait inside the kernels is bounded; a wait that runs out records a
 *     flag that nvfp4_check_device_status() reports as NVFP4_ERR_TIMEOUT.
 *
 * Data layout (all row-major, "K" = reduction dimension, K % 32 == 0):
 *   q   : rows x K/2 bytes; byte j of a row holds element 2j in its low nibble
 *         and element 2j+1 in its high nibble; E2M1 codes 0..7 are
 *         0, 0.5, 1, 1.5, 2, 3, 4, 6 and bit 3 is the sign.
 *   sf  : nvfp4_sf_bytes(rows, K) bytes of UE4M3 block scales in the tiled
 *         layout read by block-scaled tensor-core MMAs (see nvfp4_sf_offset);
 *         padding bytes are zero.
 *   global scale: FP32 *decode* scale s_g = amax / 2688 (2688 = 6 * 448), or
 *         1 when that quotient is 0.  A value is x ~= e2m1 * e4m3(sb) * s_g.
 */
#ifndef NVFP4_H
#define NVFP4_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NVFP4_API __attribute__((visibility("default")))
#else
#define NVFP4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NVFP4_OK = 0,
    NVFP4_ERR_INVALID_ARG = 1, /* null pointer, bad shape, bad segment table, ... */
    NVFP4_ERR_UNSUPPORTED = 2, /* a shape or mode this library does not handle */
    NVFP4_ERR_ALIGNMENT = 3,   /* a pointer or leading dimension is not 16-byte aligned */
    NVFP4_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed */
    NVFP4_ERR_TIMEOUT = 5,     /* a bounded wait inside a kernel ran out */
    NVFP4_ERR_WORKSPACE = 6    /* workspace missing or too small */
} nvfp4_status;

typedef enum { NVFP4_IN_BF16 = 0, NVFP4_IN_FP32 = 1 } nvfp4_in_dtype;
typedef enum { NVFP4_OUT_BF16 = 0, NVFP4_OUT_FP32 = 1 } nvfp4_out_dtype;

/* One module of a fused weight: output columns [col_begin, col_end) and that
 * module's FP32 global (decode) scale, as returned by nvfp4_quantize_weight. */
typedef struct {
    int64_t col_begin;
    int64_t col_end;
    float w_global_scale;
} nvfp4_segment;

#define NVFP4_MAX_SEGMENTS 16

/* nvfp4_gemm flags */
#define NVFP4_GEMM_AUTO 0u              /* decode kernel for m <= 64; otherwise the CTA-pair kernel when
                                           it needs no more waves of tiles than the single-CTA kernel
                                           (m >= 256, no gate outputs), else the single-CTA kernel */
#define NVFP4_GEMM_FORCE_LARGE 1u       /* the persistent large-M kernel (one CTA per SM, 128 x 256 tiles) */
#define NVFP4_GEMM_FORCE_DECODE 2u      /* the split-K decode kernel (m <= 64) */
#define NVFP4_GEMM_FORCE_LARGE_PAIR 3u  /* the large-M kernel on CTA pairs (cta_group::2, 256 x 256 tiles) */

/* ------------------------------------------------------------------------
 * Layout helpers (pure host functions, no CUDA calls).
 * ---------------------------------------------------------------------- */

/* Bytes of a tiled scale buffer for `rows` x `k` values: rows rounded up to
 * 128, k/16 rounded up to 4.  Returns 0 if rows < 0 or k is not a positive
 * multiple of 16. */
NVFP4_API size_t nvfp4_sf_bytes(int64_t rows, int64_t k);

/* Byte offset of the scale of (row, kblock) in the tiled layout, where kblock
 * indexes 16-element blocks along K.  Scales are grouped in 512-byte atoms of
 * 128 rows x 4 kblocks; atoms are ordered kblock-atom fastest, then 128-row
 * block.  Inside an atom: (row % 32) * 16 + ((row % 128) / 32) * 4 +
 * kblock % 4.  Returns -1 for out-of-range arguments. */
NVFP4_API int64_t nvfp4_sf_offset(int64_t row, int64_t kblock, int64_t k);

/* Workspace bytes nvfp4_quantize_act / nvfp4_quantize_weight need when they
 * compute the global scale themselves (an amax accumulator). */
NVFP4_API size_t nvfp4_quant_workspace_size(void);

/* Workspace bytes nvfp4_gemm needs for this shape and kernel choice: 0 for
 * the large-M kernels; for the decode kernel (m <= 64) one partial tile of
 * 16, 32 or 64 rows x 128 columns per CTA slot (160 slots), each value an
 * 8-byte word (FP32 and a 32-bit tag): 2.5, 5 or 10 MiB.  The workspace needs no
 * initialisation, but two calls that may run concurrently must not share one
 * (consecutive calls on one stream may share it: a decode kernel touches the
 * workspace only after the previous kernel in the stream has completed). */
NVFP4_API size_t nvfp4_gemm_workspace_size(int64_t m, int64_t n, int64_t k, uint32_t flags);

/* The kernel nvfp4_gemm runs for an m x n output with these flags on a device
 * with `sms` streaming multiprocessors: NVFP4_GEMM_FORCE_DECODE,
 * NVFP4_GEMM_FORCE_LARGE or NVFP4_GEMM_FORCE_LARGE_PAIR (the flag that selects
 * it), or -1 for out-of-range arguments.  with_gates: the nvfp4_gemm_gdn form.
 * A pure host function (no CUDA calls). */
NVFP4_API int nvfp4_gemm_kernel_for(int64_t m, int64_t n, int sms, uint32_t flags, int with_gates);

/* ------------------------------------------------------------------------
 * nvfp4_quantize_weight - offline, per module (post-training, calibration
 * only).  Quantises one module's n x k weight (nn.Linear layout, K
 * contiguous, row stride ldw elements) into rows [row_offset, row_offset + n)
 * of a fused buffer of n_total rows, so that several separately calibrated
 * modules can be concatenated along the output dimension.
 *
 *   w                 device, n x k, BF16 or FP32 (dt); 16-byte aligned,
 *                     ldw * element size a multiple of 16.
 *   global_scale_in   host; the module's decode scale to use, or NULL to
 *                     compute amax/2688 on the device.  Must be positive and
 *                     finite when given.
 *   w_q               device, n_total x k/2 bytes (this call writes its rows).
 *   w_sf              device, nvfp4_sf_bytes(n_total, k) bytes.  This call
 *                     writes the scale entries of its rows; the call whose
 *                     rows end at n_total also zeroes the padding rows.
 *   global_scale_out  host; receives the scale used (required when
 *                     global_scale_in is NULL, may be NULL otherwise).
 *   workspace         device, >= nvfp4_quant_workspace_size() bytes, needed
 *                     only when global_scale_in is NULL.
 * When the scale is computed the call SYNCHRONISES the stream to return it on
 * the host (an offline call).
 * ---------------------------------------------------------------------- */
NVFP4_API nvfp4_status nvfp4_quantize_weight(const void* w, nvfp4_in_dtype dt, int64_t n, int64_t k, int64_t ldw,
                                   int64_t row_offset, int64_t n_total, const float* global_scale_in,
                                   uint8_t* w_q, uint8_t* w_sf, float* global_scale_out, void* workspace,
                                   size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * nvfp4_quantize_act - on-the-fly activation quantisation (the "A4" of W4A4).
 *
 *   a                 device, m x k, BF16 or FP32 (dt), row stride lda
 *                     elements; 16-byte aligned rows.
 *   act_scale_dev     device float.  Non-NULL: static (calibrated) mode, the
 *                     tensor's decode scale is read from it.  NULL: dynamic
 *                     mode, amax is reduced on the device first and the scale
 *                     amax/2688 is used.
 *   act_scale_out_dev device float receiving the scale used; required in
 *                     dynamic mode (nvfp4_gemm reads it), optional otherwise.
 *   a_q               device, m x k/2 bytes.
 *   a_sf              device, nvfp4_sf_bytes(m, k) bytes (padding zeroed).
 *   workspace         device, >= nvfp4_quant_workspace_size() bytes in
 *                     dynamic mode (the amax accumulator), unused otherwise.
 * ---------------------------------------------------------------------- */
NVFP4_API nvfp4_status nvfp4_quantize_act(const void* a, nvfp4_in_dtype dt, int64_t m, int64_t k, int64_t lda,
                                const float* act_scale_dev, float* act_scale_out_dev, uint8_t* a_q, uint8_t* a_sf,
                                void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * nvfp4_gemm - block-scaled FP4 GEMM with the per-module scale epilogue:
 *
 *   C[i, j] = cvt( acc[i, j] * (s_ga * w_global_scale[seg(j)]) ),
 *   acc[i, j] = sum_k e2m1(a)[i,k] e4m3(sfa)[i,k/16] e2m1(w)[j,k] e4m3(sfw)[j,k/16]
 *
 * with FP32 accumulation on the tensor cores and seg(j) the segment whose
 * [col_begin, col_end) contains column j.
 *
 *   a_q, a_sf         device, from nvfp4_quantize_act (m rows).
 *   act_scale_dev     device float, s_ga (the scale nvfp4_quantize_act used).
 *   w_q, w_sf         device, fused weight from nvfp4_quantize_weight (n rows).
 *   segs, nsegs       host, 1..NVFP4_MAX_SEGMENTS segments, sorted, contiguous,
 *                     first col_begin 0, last col_end n, every boundary a
 *                     multiple of 16, scales positive and finite.
 *   c, odt, ldc       device output, m x n, BF16 or FP32, row stride ldc
 *                     elements (ldc >= n, 16-byte aligned rows).
 *   workspace         device, >= nvfp4_gemm_workspace_size(m, n, k, flags)
 *                     bytes, 16-byte aligned (may be NULL when that is 0).
 *                     The decode kernel passes partial tiles between its CTAs
 *                     through it (one CTA per SM).  It is launched with
 *                     programmatic dependent launch: its CTAs may start, and
 *                     load weights, while the previous kernel in the stream
 *                     is still running, and touch activations, scales,
 *                     workspace and output only after that kernel has
 *                     completed.  Back-to-back decode GEMMs thus overlap the
 *                     next weight stream with the previous GEMM's tail.
 *   flags             NVFP4_GEMM_* kernel choice.
 * Shapes: m >= 1, n a multiple of 16, k a multiple of 32, all < 2^31.
 * The BF16 output is the round-to-nearest-even BF16 of the FP32 output of the
 * same call configuration.  Results are deterministic (no atomics).
 * ---------------------------------------------------------------------- */
NVFP4_API nvfp4_status nvfp4_gemm(const uint8_t* a_q, const uint8_t* a_sf, const float* act_scale_dev, const uint8_t* w_q,
                        const uint8_t* w_sf, int64_t m, int64_t n, int64_t k, const nvfp4_segment* segs, int nsegs,
                        void* c, nvfp4_out_dtype odt, int64_t ldc, void* workspace, size_t ws_bytes, uint32_t flags,
                        void* stream);

/* ------------------------------------------------------------------------
 * nvfp4_gemm_gdn - nvfp4_gemm (BF16 output) whose epilogue also computes the
 * Gated DeltaNet gates from two head-wide column ranges of the fused input
 * projection ("Why Gated DeltaNet Survives 4-Bit Quantization", page summary,
 * "Gated DeltaNet Mechanics": the log-space forget gate; abstract, mechanism
 * (ii): the sigmoid parameterization, read as beta = sigmoid(b)).  With
 * x = the stored BF16 value C[i, j] (FP32 arithmetic from there):
 *
 *   g[i, h]    = -exp(A_log[h]) * softplus(C[i, a_col + h] + dt_bias[h])
 *   beta[i, h] = 1 / (1 + exp(-C[i, b_col + h]))
 *
 * C is written exactly as nvfp4_gemm writes it for the same arguments; the
 * gates are computed by the CTA that produces those columns, from the values
 * it stores, so they cost no second pass over C.
 *
 *   gates->a_col, b_col  first output column of the a and b ranges; each
 *                        range [col, col + heads) lies within [0, n).
 *   gates->heads         number of value heads, >= 1.
 *   gates->A_log,
 *   gates->dt_bias       device FP32 [heads] (the layer's parameters).
 *   gates->g, beta       device FP32 outputs, m rows of heads values, row
 *                        stride ldg >= heads elements.
 * Other arguments and errors as nvfp4_gemm; odt must be NVFP4_OUT_BF16
 * (NVFP4_ERR_INVALID_ARG otherwise).
 * ---------------------------------------------------------------------- */
typedef struct nvfp4_gdn_gates {
    int32_t a_col;
    int32_t b_col;
    int32_t heads;
    const float* A_log;
    const float* dt_bias;
    float* g;
    float* beta;
    int64_t ldg;
} nvfp4_gdn_gates;

NVFP4_API nvfp4_status nvfp4_gemm_gdn(const uint8_t* a_q, const uint8_t* a_sf, const float* act_scale_dev,
                                      const uint8_t* w_q, const uint8_t* w_sf, int64_t m, int64_t n, int64_t k,
                                      const nvfp4_segment* segs, int nsegs, void* c, int64_t ldc,
                                      const nvfp4_gdn_gates* gates, void* workspace, size_t ws_bytes,
                                      uint32_t flags, void* stream);

/* ------------------------------------------------------------------------
 * nvfp4_gemm_swiglu_quantize - the gate/up GEMM of a gated MLP with its glue
 * fused into the epilogue: for the fused weight [gate (f rows); up (f rows)]
 * (2f x k, e.g. two separately calibrated modules with their own segment
 * scales) it computes, per output element j < f,
 *     g = bf16(acc_gate * s_ga * s_gw[seg(j)]),  u = bf16(acc_up * s_ga * s_gw[seg(f + j)]),
 *     h = bf16(silu(g) * u)
 * and quantises h to NVFP4 with the static decode scale *h_scale_dev,
 * writing codes and tiled scales only (h itself never reaches memory).  The
 * bytes equal nvfp4_gemm (BF16 output) followed by nvfp4_silu_mul_quantize
 * with the same static scale.  The pages do not describe the MLP; this is the
 * step between its two W4A4 linear layers.
 *
 * Performance: on B200 this call is faster than the two-call path it
 * replaces and writes a ninth of the bytes.  Measured at m = 8192,
 * f = 17408, k = 5120: 0.62 ms, against 0.59 ms for nvfp4_gemm (BF16 out)
 * plus 0.25-0.26 ms for nvfp4_silu_mul_quantize.  (It was slower, 0.95 ms,
 * while its epilogue released the accumulator columns the next tile shares
 * only after the SiLU arithmetic; it now releases them first.)
 *
 *   a_q, a_sf, act_scale_dev  quantised activations, m x k (as for nvfp4_gemm).
 *   w_q, w_sf                 fused weight, 2f rows; f a multiple of 128.
 *   segs, nsegs               segment table over the 2f columns.
 *   h_scale_dev               device FP32 decode scale of h (calibrated).
 *   h_q, h_sf                 outputs: m x f/2 codes, nvfp4_sf_bytes(m, f)
 *                             tiled scale bytes (padding rows zeroed).
 * ---------------------------------------------------------------------- */
NVFP4_API nvfp4_status nvfp4_gemm_swiglu_quantize(const uint8_t* a_q, const uint8_t* a_sf, const float* act_scale_dev,
                                        const uint8_t* w_q, const uint8_t* w_sf, int64_t m, int64_t f, int64_t k,
                                        const nvfp4_segment* segs, int nsegs, const float* h_scale_dev,
                                        uint8_t* h_q, uint8_t* h_sf, void* stream);

/* ------------------------------------------------------------------------
 * nvfp4_linear_decode - one W4A4 linear layer for m <= 64 tokens in a single
 * launch: the activations are quantised to NVFP4 on the fly inside the
 * decode GEMM (each CTA quantises the slices of A its k-range needs) and
 * multiplied with the fused NVFP4 weight, with the per-segment scale
 * epilogue ("Why Gated DeltaNet Survives 4-Bit Quantization": W4A4 with
 * on-the-fly activation quantisation, abstract; per-module global scales,
 * abstract, last sentence).  The result is bit-identical to
 * nvfp4_quantize_act followed by nvfp4_gemm with NVFP4_GEMM_FORCE_DECODE.
 *
 *   a, dt, m, k, lda  raw activations as for nvfp4_quantize_act; 1 <= m <= 64
 *                     (m == 0 is a no-op, m > 64 returns UNSUPPORTED).
 *   act_scale_dev     device FP32 decode scale (static), or NULL: dynamic,
 *                     amax/2688 computed inside the kernel (every CTA reads
 *                     the whole of A, m x k, for it).
 *   act_scale_out_dev optional device float receiving the scale used.
 *   w_q, w_sf, n, segs, nsegs, c, odt, ldc   as for nvfp4_gemm.
 *   workspace         device, >= nvfp4_gemm_workspace_size(m, n, k,
 *                     NVFP4_GEMM_FORCE_DECODE) bytes, as for nvfp4_gemm.
 * ---------------------------------------------------------------------- */
NVFP4_API nvfp4_status nvfp4_linear_decode(const void* a, nvfp4_in_dtype dt, int64_t m, int64_t k, int64_t lda,
                                 const float* act_scale_dev, float* act_scale_out_dev, const uint8_t* w_q,
                                 const uint8_t* w_sf, int64_t n, const nvfp4_segment* segs, int nsegs, void* c,
                                 nvfp4_out_dtype odt, int64_t ldc, void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * nvfp4_linear_prefill - one W4A4 linear layer for m > 64 tokens in a single
 * launch: the activations are quantised to NVFP4 with the static
 * (calibrated) scale inside the large-M GEMM kernel and multiplied with the
 * fused NVFP4 weight, with the per-segment scale epilogue ("Why Gated
 * DeltaNet Survives 4-Bit Quantization": W4A4 with on-the-fly activation
 * quantisation, abstract; per-module global scales, abstract, last
 * sentence).  The first m-blocks of A are quantised before the first MMAs,
 * the rest while the MMAs run (tiles are scheduled in bands of 8 m-blocks).
 * a_q / a_sf receive exactly the bytes nvfp4_quantize_act writes with the
 * same scale, and c exactly what nvfp4_gemm (NVFP4_GEMM_FORCE_LARGE) writes
 * from them.
 *
 *   a, dt, m, k, lda  raw activations as for nvfp4_quantize_act; BF16 only
 *                     (UNSUPPORTED otherwise); m > 64 (m <= 64: UNSUPPORTED,
 *                     use nvfp4_linear_decode; m == 0 is a no-op).
 *   act_scale_dev     device FP32 decode scale of A (required: static mode).
 *   a_q, a_sf         device outputs as for nvfp4_quantize_act (the kernel's
 *                     own staging of the quantised A; the caller may reuse it).
 *   w_q, w_sf, n, segs, nsegs, c, odt, ldc   as for nvfp4_gemm.
 *   workspace         device, >= nvfp4_linear_prefill_workspace_size(m)
 *                     bytes, 16-byte aligned: one 8-byte ready word per 128
 *                     rows of A, tagged per call with a tag that grows from
 *                     call to call in this process.  ZERO IT ONCE before its
 *                     first use (after that, consecutive calls on one stream
 *                     may share it without clearing; calls that may run
 *                     concurrently must not).
 * The kernel is persistent (one CTA per SM) and its CTAs wait (bounded) on
 * one another's quantised rows, so it needs the whole GPU to itself to make
 * progress at full speed; a wait that runs out sets the device status
 * (nvfp4_check_device_status returns NVFP4_ERR_TIMEOUT).
 *
 * Performance: on B200 this single launch is currently SLOWER than
 * nvfp4_quantize_act followed by nvfp4_gemm: 0.261 ms against 0.242 ms for
 * 8192 x 5120 x 12384, 0.083 ms against 0.075 ms for 4096 x 5120 x 5120.  Quantising the first 8-16 m-blocks before the first
 * MMA costs 6-10 us, the two background warps quantise about 0.5 TB/s (a
 * band of 8 m-blocks per ~20 us, late for the 4096-row case), and the banded
 * tile order and the background traffic slow the mainloop by ~4 %.  Use it
 * where one launch per layer matters more than the last few percent.
 * ---------------------------------------------------------------------- */
NVFP4_API size_t nvfp4_linear_prefill_workspace_size(int64_t m);
NVFP4_API nvfp4_status nvfp4_linear_prefill(const void* a, nvfp4_in_dtype dt, int64_t m, int64_t k, int64_t lda,
                                  const float* act_scale_dev, uint8_t* a_q, uint8_t* a_sf, const uint8_t* w_q,
                                  const uint8_t* w_sf, int64_t n, const nvfp4_segment* segs, int nsegs, void* c,
                                  nvfp4_out_dtype odt, int64_t ldc, void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * nvfp4_silu_mul_quantize - the glue of a gated (SwiGLU) MLP whose gate/up
 * and down projections both run as W4A4 NVFP4 GEMMs: from the BF16 gate g and
 * up u halves of the fused gate/up GEMM output it forms
 *     h = bf16( silu(g) * u ),  silu(x) = x / (1 + e^-x)
 * (every step in FP32 with round-to-nearest; e^-x is CUDA's expf, within 2
 * ulp) and quantises h to NVFP4 exactly as nvfp4_quantize_act quantises an
 * activation (the down projection's on-the-fly input quantisation).  The
 * pages do not describe the MLP; this is the step between its two linear
 * layers.
 *
 *   g, u              device BF16, m x f each, row stride ldgu elements
 *                     (for a fused [gate | up] output of width 2f: g = C,
 *                     u = C + f, ldgu = 2f); 16-byte aligned rows.
 *   h_scale_dev       device FP32 decode scale of h (static), or NULL:
 *                     dynamic, amax(h)/2688 computed on the device first.
 *   h_scale_out_dev   device float receiving the scale used (required in
 *                     dynamic mode).
 *   h_q, h_sf         device outputs as for nvfp4_quantize_act with k = f.
 *   h_out, ldh        optional device BF16 m x f copy of h (NULL: not
 *                     written), row stride ldh.
 *   workspace         device, >= nvfp4_quant_workspace_size() bytes, needed
 *                     only in dynamic mode.
 * Shapes: m >= 0, f a positive multiple of 32, both < 2^31.
 * Dynamic mode runs an amax pass first.  With h_out it stores h there and
 * quantises the stored h (silu evaluated once per element); without h_out it
 * reads g and u again and recomputes h.  The bytes are the same either way.
 * ---------------------------------------------------------------------- */
NVFP4_API nvfp4_status nvfp4_silu_mul_quantize(const void* g, const void* u, int64_t m, int64_t f, int64_t ldgu,
                                     const float* h_scale_dev, float* h_scale_out_dev, uint8_t* h_q, uint8_t* h_sf,
                                     void* h_out, int64_t ldh, void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * nvfp4_gemm_decode_noalloc - the decode GEMM (the kernel nvfp4_gemm runs
 * under NVFP4_GEMM_FORCE_DECODE) with no workspace argument.  The pages have
 * no counterpart to this call; it exists for deployment.
 *
 * It is for callers that have no way to hand the library device scratch
 * memory: an operator slot or plug-in interface with a fixed signature, or a
 * plain C host with no device allocator; and for callers that must not
 * allocate in the middle of a step, because a device allocation can block
 * until the device is idle or fail when memory is tight.  The call allocates
 * nothing.  The kernel's scratch (one tagged FP32 partial tile per CTA
 * slot) lives in a fixed array of NVFP4_NOALLOC_SCRATCH_BYTES
 * bytes of device memory that the library reserves on each device it is
 * loaded on.
 *
 * Arguments: as nvfp4_gemm without workspace, ws_bytes and flags.
 * Limit: m <= NVFP4_NOALLOC_MAX_M tokens.  A larger m needs more scratch than
 *   the array holds; the call then returns NVFP4_ERR_UNSUPPORTED and does
 *   nothing (use nvfp4_gemm with a workspace).  m == 0 is a no-op.  Other
 *   argument errors are those of nvfp4_gemm.
 * Set-up: the first call on a device, made with that device current, looks up
 *   the array's device address and sets the kernels' attributes.  Make that
 *   first call before any stream capture begins.
 * Sharing: every call on a device uses the same array.  Nothing in it has to
 *   be zero when a call starts: every partial word carries a tag fresh to each
 *   call, and a reader waits for words with its own call's tag.  Two calls that overlap in time on one device (different
 *   streams, or threads without ordering) race on the array and give wrong
 *   results; order them (one stream, or events).
 * ---------------------------------------------------------------------- */
#define NVFP4_NOALLOC_MAX_M 16
#define NVFP4_NOALLOC_SCRATCH_BYTES (160 * 16 * 128 * 8) /* 2.5 MiB */
NVFP4_API nvfp4_status nvfp4_gemm_decode_noalloc(const uint8_t* a_q, const uint8_t* a_sf, const float* act_scale_dev,
                                       const uint8_t* w_q, const uint8_t* w_sf, int64_t m, int64_t n, int64_t k,
                                       const nvfp4_segment* segs, int nsegs, void* c, nvfp4_out_dtype odt,
                                       int64_t ldc, void* stream);

/* ------------------------------------------------------------------------
 * Calibrated FP8 (E4M3) KV cache.  The recipe pairs the NVFP4 W4A4 layers
 * with an FP8 KV cache whose per-tensor scales are calibrated offline and
 * shipped with the checkpoint ("Why Gated DeltaNet Survives 4-Bit
 * Quantization": abstract; Glonce article, "How to use it"; aiany.app,
 * "Mechanistic notes").  The pages give no formula; this library reads it as
 *
 *   scale s  = amax / 448 over the calibration data (448 = largest E4M3
 *              value; one FP32 division), s = 1 if that is 0;
 *   byte     = E4M3 round-to-nearest-even, saturating to +-448, of x * (1/s)
 *              (1/s correctly rounded in FP32, FLT_MAX if it overflows);
 *   value    = e4m3(byte) * s when attention reads the cache.
 * ---------------------------------------------------------------------- */

/* nvfp4_fp8_calibrate - fold one calibration batch into a running amax and
 * refresh the scale: *amax_inout = max(*amax_inout, max |x|), then
 * *scale_out = *amax_inout / 448 (1 if 0).  Start *amax_inout at 0.
 *
 *   x, dt, rows, width, ld  rows x width BF16/FP32 values (device), row
 *                           stride ld elements; width a multiple of 16, rows
 *                           16-byte aligned.  rows may be 0 (scale refresh).
 *   amax_inout_dev          device float, non-negative (running maximum).
 *   scale_out_dev           device float, receives the scale.
 * Errors: NVFP4_ERR_INVALID_ARG (shape, NULL), NVFP4_ERR_ALIGNMENT. */
NVFP4_API nvfp4_status nvfp4_fp8_calibrate(const void* x, nvfp4_in_dtype dt, int64_t rows, int64_t width, int64_t ld,
                                           float* amax_inout_dev, float* scale_out_dev, void* stream);

/* nvfp4_kv_cache_quantize_fp8 - quantise the K and V rows of `tokens` new
 * tokens to E4M3 with their calibrated scales and store each token's row in
 * its cache slot, in one launch.
 *
 *   k, v, dt          device, tokens x width BF16/FP32 (width = KV heads x
 *                     head size, a multiple of 16), row strides ld_k, ld_v
 *                     elements, rows 16-byte aligned.
 *   slot_mapping      device int64[tokens]: the cache row of each token; a
 *                     negative entry (padding) or one >= num_slots is
 *                     skipped.  NULL: token t goes to slot t (then tokens <=
 *                     num_slots).  The valid entries must be distinct: each
 *                     16-element piece of a row is written on its own, so two
 *                     tokens mapped to one slot leave that row a mix of both
 *                     (which pieces come from which token is unspecified).
 *   k_scale_dev,
 *   v_scale_dev       device floats, the calibrated scales.
 *   k_cache, v_cache  device, num_slots rows of width bytes, row stride
 *                     cache_ld bytes (a multiple of 16, >= width); rows not
 *                     named by the slot table are left untouched.
 * Requires tokens x width / 16 < 2^31.  Errors: NVFP4_ERR_INVALID_ARG,
 * NVFP4_ERR_UNSUPPORTED, NVFP4_ERR_ALIGNMENT, NVFP4_ERR_CUDA. */
NVFP4_API nvfp4_status nvfp4_kv_cache_quantize_fp8(const void* k, const void* v, nvfp4_in_dtype dt, int64_t tokens,
                                                   int64_t width, int64_t ld_k, int64_t ld_v,
                                                   const int64_t* slot_mapping, int64_t num_slots,
                                                   const float* k_scale_dev, const float* v_scale_dev,
                                                   uint8_t* k_cache, uint8_t* v_cache, int64_t cache_ld,
                                                   void* stream);

/* ------------------------------------------------------------------------
 * Diagnostics.
 * ---------------------------------------------------------------------- */

/* Text of the last error returned on the calling thread ("" if none). */
NVFP4_API const char* nvfp4_get_last_error_string(void);

/* Synchronises `stream`, reads and clears the device status word that bounded
 * waits set when they run out.  Returns NVFP4_ERR_TIMEOUT if any did (the
 * kernel that timed out returned early and its outputs are undefined),
 * NVFP4_ERR_CUDA if the synchronisation failed, NVFP4_OK otherwise. */
NVFP4_API nvfp4_status nvfp4_check_device_status(void* stream);

/* Enqueues a one-thread kernel that waits on an mbarrier nobody arrives at,
 * for at most `limit_cycles` SM clock cycles, then records a timeout and
 * returns.  Lets tests exercise the timeout reporting without a fault. */
NVFP4_API nvfp4_status nvfp4_selftest_wait_timeout(long long limit_cycles, void* stream);

/* Library version, major * 10000 + minor * 100 + patch. */
NVFP4_API int nvfp4_version(void);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H */
