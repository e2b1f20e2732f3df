/*
 * nvfp4.h - C ABI of the NVFP4 W4A4 linear-layer library for NVIDIA B200
 * (sm_100a).
 *
 * The library implements the three steps of a W4A4 linear layer described
 * in the write-ups of "Why Gated DeltaNet Survives 4-Bit Quantization: NVFP4
 * W4A4 for the Recurrent Half of a Hybrid 27B LLM" (arXiv 2609.04098):
 *
 *   1. activation quantization to NVFP4: E2M1 4-bit values, one E4M3 scale
 *      per 16-element block set from the block maximum divided by 6, one FP32
 *      scale per tensor [picx.dev summary, "Background"];
 *   2. a block-scaled FP4 x FP4 GEMM on the tensor cores with FP32
 *      accumulation and a dequantizing BF16 (or FP32) epilogue [same page,
 *      "Background": native 4-bit tensor-core GEMMs];
 *   3. the fused projection: several separately calibrated weights
 *      concatenated along N in one GEMM, each output segment rescaled by its
 *      own weight global scale, so the fused result equals the unfused ones
 *      [anthology record LIT-800, "Standing in the anthology"; cctest.ai
 *      article, "Main findings"; podcast abstract].
 *
 * Around them: the offline rewrite of a fused weight's scales to one common
 * global scale (the "pre-harmonized" checkpoint), the running amax of a
 * static calibration, and the MXFP4 format the pages contrast NVFP4 with
 * (32-element blocks, power-of-two scales): its quantizer and GEMM.
 *
 * Conventions shared by every entry point
 *   - Device pointers are raw CUDA device addresses owned by the caller; the
 *     library never allocates, frees or retains them.  Host pointers (named
 *     so below) are read during the call only, except the buffers of
 *     nvfp4_linear_host, which its enqueued copies use until the stream
 *     reaches them.  The one buffer the library may own is the GEMM's K-split
 *     workspace of a stream, and only when the caller registered none for
 *     that stream (see nvfp4_set_workspace); nvfp4_release_workspaces()
 *     frees what it allocated.
 *   - Consecutive kernels of this library on one stream overlap their
 *     prologue with the previous kernel's tail (programmatic dependent
 *     launch); each still reads its inputs only after the kernel before it
 *     on the stream has completed, so stream order is the only ordering
 *     callers need.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and the call returns once enqueued; nothing synchronizes.
 *   - Arguments are validated before anything is launched.  A failing check
 *     returns its status and launches nothing.  Launch failures return
 *     NVFP4_ERR_CUDA.  Faults found by the kernels themselves (a bounded wait
 *     that ran out) are recorded in a per-device error word, read back by
 *     nvfp4_last_device_error().  No exception or abort crosses this ABI.
 *   - Numbers in the format (readings of the pages, which name the formats
 *     but not their encodings): E2M1 = OCP FP4 (bit 3 sign, 2 exponent bits
 *     with bias 1, 1 mantissa bit: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6);
 *     E4M3 = OCP FP8 E4M3FN (bias 7, max 448).  Both are rounded to nearest,
 *     ties to even, saturating.  A global scale g multiplies on encode and
 *     divides on decode: value = e2m1(code) * e4m3(scale) / g.
 *   - Codes: [rows, K/2] bytes, row-major; element 2j of a row is the low
 *     nibble of byte j.
 *   - Block scales come in two layouts (nvfp4_sf_layout):
 *       NVFP4_SF_ROWMAJOR: [rows, K/16] bytes, row-major.
 *       NVFP4_SF_TCGEN05 : the order the tensor-core MMA reads.  512-byte
 *         chunks of 128 rows x 4 scales; chunk (r/128, j/4) starts at byte
 *         ((r/128) * ceil(K/64) + j/4) * 512 and scale j of row r sits at
 *         (r%32)*16 + ((r/32)%4)*4 + j%4 inside it.  Rows are padded to a
 *         multiple of 128 and scale columns to a multiple of 4 with zeros;
 *         the size is nvfp4_scale_bytes(rows, K, NVFP4_SF_TCGEN05).
 *     The GEMM entry points take NVFP4_SF_TCGEN05 scales only.
 */
#ifndef NVFP4_H_
#define NVFP4_H_

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

/* Same object as cudaStream_t. */
typedef struct CUstream_st* nvfp4_stream_t;

typedef enum nvfp4_status {
  NVFP4_OK = 0,
  NVFP4_ERR_INVALID_ARG = 1,  /* null pointer, bad size, bad scale, bad enum      */
  NVFP4_ERR_ALIGNMENT = 2,    /* a device pointer is not 16-byte aligned          */
  NVFP4_ERR_UNSUPPORTED = 3,  /* not an sm_100 device, or a size beyond limits    */
  NVFP4_ERR_CUDA = 4,         /* a CUDA runtime/driver call or launch failed      */
  NVFP4_ERR_TIMEOUT = 5,      /* a kernel's bounded wait ran out (device word)    */
  NVFP4_ERR_DEVICE = 6        /* a kernel found an out-of-range index (device word) */
} nvfp4_status;

typedef enum nvfp4_in_dtype { NVFP4_IN_BF16 = 0, NVFP4_IN_F32 = 1 } nvfp4_in_dtype;
typedef enum nvfp4_out_dtype { NVFP4_OUT_BF16 = 0, NVFP4_OUT_F32 = 1 } nvfp4_out_dtype;
typedef enum nvfp4_sf_layout { NVFP4_SF_ROWMAJOR = 0, NVFP4_SF_TCGEN05 = 1 } nvfp4_sf_layout;

/* Largest number of output segments nvfp4_fused_proj accepts. */
#define NVFP4_MAX_SEGMENTS 16

/* Bytes needed for the block scales of a [rows, K] operand in `layout`
 * (0 if rows < 1 or K is not a positive multiple of 16). */
NVFP4_API size_t nvfp4_scale_bytes(int64_t rows, int64_t K, nvfp4_sf_layout layout);

/* Per-tensor absolute maximum (the input of the default global-scale
 * calibration g = 448*6/amax) [picx.dev summary, "Background": one FP32
 * scale per tensor].
 *   x        device, [M, K] row-major, bf16 or f32 per `dtype`, 16-B aligned
 *   amax_out device, one float; overwritten with max |x| (0 for an all-zero
 *            tensor).  Enqueues a 4-byte memset and one kernel.
 * Errors: INVALID_ARG (null, M < 1, K < 1), ALIGNMENT, CUDA. */
NVFP4_API nvfp4_status nvfp4_amax(const void* x, nvfp4_in_dtype dtype, int64_t M, int64_t K,
                        float* amax_out, nvfp4_stream_t stream);

/* Running per-tensor amax over calibration batches: the statistic a static
 * activation scale g = 448*6/amax is built from, where the scale is fixed
 * once from calibration data and then serves every later input
 * [anthology record LIT-800, "Key takeaways": calibration-only recipe;
 * cctest.ai article, "Introduction"].
 *   x            device, [M, K] row-major, bf16 or f32 per `dtype`, 16-B aligned
 *   running_amax device, one float holding +0 or a positive finite value (set
 *                it to 0 before the first batch); replaced by
 *                max(running_amax, max |x|).  Nothing is reset: call once per
 *                batch on one stream, then read the float back.
 * Errors: INVALID_ARG (null, M < 1, K < 1, M*K*element size not a multiple
 * of 16 bytes), ALIGNMENT, CUDA. */
NVFP4_API nvfp4_status nvfp4_amax_accumulate(const void* x, nvfp4_in_dtype dtype, int64_t M, int64_t K,
                                   float* running_amax, nvfp4_stream_t stream);

/* NVFP4 quantization of X [M, K] with a given FP32 global scale
 * [picx.dev summary, "Background"].  For each block of 16 elements along K:
 *   amax_b = max |x|;  t = (amax_b / 6) * g  (FP32, in this order);
 *   s = E4M3(t);  if s == 0 every code is a signed zero, else
 *   r = g / e4m3(s) and code_i = E2M1(x_i * r)   (FP32 multiply).
 *   x            device [M, K] bf16/f32, 16-byte aligned; K % 32 == 0
 *   global_scale host float, finite and > 0 (calibrated; 448*6/amax by default)
 *   codes        device [M, K/2] bytes, 16-byte aligned (written)
 *   block_scales device, nvfp4_scale_bytes(M, K, layout) bytes, 16-byte
 *                aligned (written; TCGEN05 padding is written as zero)
 *   amax_out     device float or NULL; if given, overwritten with max |x|
 *                (the same value nvfp4_amax returns) as a side output.
 * Errors: INVALID_ARG (null, M < 1, K < 32 or K % 32, bad g), ALIGNMENT, CUDA. */
NVFP4_API nvfp4_status nvfp4_quantize(const void* x, nvfp4_in_dtype dtype, int64_t M, int64_t K,
                            float global_scale, uint8_t* codes, uint8_t* block_scales,
                            nvfp4_sf_layout layout, float* amax_out, nvfp4_stream_t stream);

/* Rewrite row-major block scales [rows, K/16] into the TCGEN05 layout (used
 * once, offline, for weights quantized elsewhere).
 *   rowmajor device [rows, K/16]; tc device nvfp4_scale_bytes(rows, K, TCGEN05)
 *   bytes, 16-byte aligned (fully written, padding zero).
 * Errors: INVALID_ARG (null, rows < 1, K % 16), ALIGNMENT, CUDA. */
NVFP4_API nvfp4_status nvfp4_swizzle_scales(const uint8_t* rowmajor, int64_t rows, int64_t K, uint8_t* tc,
                                  nvfp4_stream_t stream);

/* W4A4 GEMM with dequantizing epilogue [picx.dev summary, "Background"]:
 *   out[m, n] = alpha * sum_b sA[m,b] sW[n,b] sum_{k in b} e2m1(A[m,k]) e2m1(W[n,k])
 * with alpha = 1 / (a_global_scale * w_global_scale) (rounded once to FP32),
 * FP32 accumulation on the tensor cores, then one rounding to the output type
 * (bf16 round-to-nearest-even, or f32).
 *   a_codes [M, K/2], a_scales TCGEN05 layout for M rows   (activations)
 *   w_codes [N, K/2], w_scales TCGEN05 layout for N rows   (weight, [out, in])
 *   out     device [M, N] row-major, bf16 or f32 per out_dtype
 * All device pointers 16-byte aligned; M, N >= 1; K >= 32, K % 32 == 0;
 * global scales finite and > 0.
 * For M <= 128 (decode) the K loop of each weight tile is split across CTAs
 * so that every SM streams weight; the partial FP32 tiles are summed in a
 * fixed order (the result does not depend on timing and equals the unsplit
 * sum up to FP32 rounding order).  The partials go to the K-split workspace
 * of (device, stream): the one the caller registered with
 * nvfp4_set_workspace, else one the library allocates on the first such call
 * on that stream (2 * SMs * 128 KB, zero-filled) and keeps until
 * nvfp4_release_workspaces().  A library allocation cannot happen during
 * CUDA graph capture: a first decode-shaped call on a capturing stream with
 * no workspace returns UNSUPPORTED (register one, or make one call before
 * capture).  Calls on one stream share its workspace safely (stream order);
 * calls on different streams use different workspaces.  Each launch leaves
 * the words it used empty (zero), so a workspace stays ready for the next.
 * M > 128 uses no workspace.
 * Progress of the split-K grid: the grid has 2 x SMs CTAs
 * (multiProcessorCount) for M <= 16, two per SM, and SMs CTAs for
 * 16 < M <= 128 (and for every MXFP4 GEMM).
 * The CTA that sums a split tile waits (bounded) only for partials that
 * CTAs with higher indices produce as their first work item.  So the grid
 * completes when its CTAs start in index order, as the hardware does when
 * the call has the GPU to itself.  If the process is limited to fewer SMs
 * than the device reports (an MPS active-thread percentage, a green context)
 * or CTAs start out of order, a wait can run out: the call then reports
 * NVFP4_ERR_TIMEOUT through nvfp4_last_device_error, and nothing hangs.
 * nvfp4_set_decode_cooperative(1) removes the assumption.  The grid is then
 * sized to the CTAs that can be resident at once (occupancy API) and
 * launched cooperatively, which the driver admits only if they all fit
 * (else UNSUPPORTED).  For M <= 16 that grid is smaller than the default, so
 * the K split and the FP32 summation order differ from the default launch.
 * Errors: INVALID_ARG (also: a registered workspace smaller than
 * nvfp4_workspace_bytes for this shape), ALIGNMENT, UNSUPPORTED (device is
 * not sm_100, or a first decode-shaped call during capture with no
 * workspace, or a cooperative split-K grid that cannot be co-resident), CUDA. */
NVFP4_API nvfp4_status nvfp4_gemm(const uint8_t* a_codes, const uint8_t* a_scales, float a_global_scale,
                        const uint8_t* w_codes, const uint8_t* w_scales, float w_global_scale,
                        int64_t M, int64_t N, int64_t K, void* out, nvfp4_out_dtype out_dtype,
                        nvfp4_stream_t stream);

/* Bytes of K-split workspace nvfp4_gemm / nvfp4_linear need on the current
 * device for an M x N x K problem: 2 * CTAs * BN * 128 * 8, BN being the
 * activation tile width the call picks (16, 32, 64 or 128 for M <= 16, 32,
 * 64, 128) and CTAs the NVFP4 split-K grid (2 * SMs for BN = 16, SMs
 * otherwise; the MXFP4 grid is SMs, so this size covers it too);
 * 0 for M > 128 (no split) or invalid sizes.  No counterpart in
 * the pages: the sizing rule of this library's split-K exchange.
 * nvfp4_workspace_bytes(128, N, K) (2 * SMs * 128 KB) covers every shape. */
NVFP4_API size_t nvfp4_workspace_bytes(int64_t M, int64_t N, int64_t K);

/* Register a caller-owned K-split workspace for `stream` on the current
 * device; every later decode-shaped nvfp4_gemm / nvfp4_linear on that stream
 * uses it instead of allocating.  No counterpart in the pages.
 *   workspace  device memory, 16-byte aligned, at least
 *              nvfp4_workspace_bytes(16, 1, 32) bytes, ZERO-FILLED when
 *              registered (each launch leaves it zero again); owned by the
 *              caller, who keeps it alive while calls that use it may run and
 *              uses it for nothing else.  Calls whose shape needs more than
 *              `bytes` return INVALID_ARG.
 *   workspace NULL with bytes 0: unregister (the library allocates again on
 *              the next decode-shaped call).
 * A workspace the library had allocated for this stream is freed (after a
 * device synchronize).  Registration is not stream-ordered: make it while no
 * call on `stream` is in flight.
 * Errors: INVALID_ARG (too small, or NULL with bytes != 0), ALIGNMENT, CUDA. */
NVFP4_API nvfp4_status nvfp4_set_workspace(nvfp4_stream_t stream, void* workspace, size_t bytes);

/* Free every K-split workspace the library allocated on the current device
 * (after a device synchronize); registered ones are forgotten only by
 * nvfp4_set_workspace(stream, NULL, 0).  Later calls allocate again.
 * Errors: CUDA. */
NVFP4_API nvfp4_status nvfp4_release_workspaces(void);

/* Declare [base, base + bytes) read-only while library calls run (typically
 * the quantized weights of a model in serving).  No counterpart in the
 * pages: a scheduling hint.  A GEMM whose weight codes and scales both lie in
 * declared memory loads its first weight stages before waiting for the
 * preceding kernel on the stream to finish (programmatic dependent launch),
 * instead of only prefetching them into L2.  The caller guarantees that no
 * kernel writes declared memory while a library call that reads it may run;
 * writing it anyway (for example, quantizing new weights into it just before
 * a GEMM on the same stream) can make that GEMM read stale weights.
 * Declarations accumulate until nvfp4_forget_static().
 * Errors: INVALID_ARG (NULL base or zero bytes). */
NVFP4_API nvfp4_status nvfp4_declare_static(const void* base, size_t bytes);
NVFP4_API void nvfp4_forget_static(void);

/* The whole W4A4 linear layer: quantize the activation with a_global_scale
 * (as nvfp4_quantize, TCGEN05 scales) and multiply by the quantized weight
 * (as nvfp4_gemm) [picx.dev summary, "Background": activations and weights
 * both in NVFP4, native 4-bit tensor-core GEMM].
 *   x       device [M, K] row-major, bf16 or f32 per x_dtype
 *   w_*     as nvfp4_gemm; N output features; out as nvfp4_gemm
 *   a_codes, a_scales: device buffers for the quantized activation
 *           ([M, K/2] bytes and nvfp4_scale_bytes(M, K, NVFP4_SF_TCGEN05)),
 *           or both NULL.
 * With the buffers the call is exactly nvfp4_quantize into them followed by
 * nvfp4_gemm.  Without them, for M <= 32 when every CTA's share of the
 * K-split work fits in 16 K-steps of 256 (decode shapes), one kernel
 * quantizes x into shared memory itself and runs the GEMM, writing no
 * activation to memory; its result is bitwise equal to the two-call form
 * (same arithmetic, same K split, same summation order).  Workspace and
 * capture rules as nvfp4_gemm.
 * Errors: INVALID_ARG (also: NULL buffers for a shape the one-kernel form
 * does not cover), ALIGNMENT, UNSUPPORTED, CUDA. */
NVFP4_API nvfp4_status nvfp4_linear(const void* x, nvfp4_in_dtype x_dtype, int64_t M, int64_t K,
                          float a_global_scale, const uint8_t* w_codes, const uint8_t* w_scales,
                          float w_global_scale, int64_t N, void* out, nvfp4_out_dtype out_dtype,
                          uint8_t* a_codes, uint8_t* a_scales, nvfp4_stream_t stream);

/* The layer with host-resident activation and output, as one call: enqueues
 * on `stream` the host-to-device copy of X into x_dev, nvfp4_linear(x_dev,
 * ..., out_dev, ..., a_codes, a_scales) and the device-to-host copy of the
 * result into out_host; returns once they are enqueued (synchronize the
 * stream before reading out_host).  No counterpart in the pages: the serving
 * form of the layer whose input and output live on the host.
 *   x_host    host [M, K] bf16/f32, M*K elements; page-locked memory lets the
 *             copy run asynchronously (pageable memory works, synchronously)
 *   out_host  host [M, N] bf16/f32 per out_dtype
 *   x_dev, out_dev  device staging buffers of the same sizes, 16-byte
 *             aligned, owned by the caller; a_codes/a_scales as in
 *             nvfp4_linear (may be NULL for its one-kernel decode form)
 *   other arguments as nvfp4_linear.
 * Errors: as nvfp4_linear; arguments are checked before anything is enqueued. */
NVFP4_API nvfp4_status nvfp4_linear_host(const void* x_host, nvfp4_in_dtype x_dtype, int64_t M, int64_t K,
                               float a_global_scale, const uint8_t* w_codes, const uint8_t* w_scales,
                               float w_global_scale, int64_t N, void* out_host, nvfp4_out_dtype out_dtype,
                               void* x_dev, uint8_t* a_codes, uint8_t* a_scales, void* out_dev,
                               nvfp4_stream_t stream);

/* nvfp4_gemm for decode-sized M that allocates nothing.  The pages have no
 * counterpart: this is an interface variant, not part of the method.  It
 * computes exactly what nvfp4_gemm computes for the same arguments (same
 * kernel, same K split, same summation order), but the K-split partial tiles,
 * as tagged 64-bit words (an FP32 value and a "full" tag), live in a fixed
 * scratch array in the library's static device memory instead of a workspace
 * allocated on first use.  For callers
 * that must not allocate device memory once running (a serving engine that
 * plans its memory at start-up and gives the rest to its KV cache; code that
 * cannot take the implicit synchronisation of an allocation).
 *   Arguments, layouts and alignment: as nvfp4_gemm.
 *   Limits (the scratch size): M <= 32, device with at most 160 SMs.
 *   Scratch: 10 MiB of tagged partial-tile words per device, part of the
 *   library's module image.  Every word must be empty (zero) when a launch
 *   starts: the array is zeroed when the module loads, every launch leaves
 *   the words it used empty, and nvfp4_last_device_error() empties it after
 *   a launch that reported an error.
 *   The first call on each device resolves the scratch address (once, with
 *   that device current); make it before any stream capture begins.
 *   There is ONE scratch array per device: two calls that can run at the same
 *   time on one device (different streams, no ordering between them) race
 *   on it and both results are undefined.  Calls ordered on one stream are
 *   safe.
 * Errors: INVALID_ARG, ALIGNMENT (as nvfp4_gemm); UNSUPPORTED (M > 32, more
 * than 160 SMs, or not sm_100); CUDA. */
NVFP4_API nvfp4_status nvfp4_gemm_noalloc(const uint8_t* a_codes, const uint8_t* a_scales, float a_global_scale,
                                const uint8_t* w_codes, const uint8_t* w_scales, float w_global_scale,
                                int64_t M, int64_t N, int64_t K, void* out, nvfp4_out_dtype out_dtype,
                                nvfp4_stream_t stream);

/* Fused projection: the GEMM above with W the row-wise concatenation of
 * n_seg separately calibrated weights; output columns
 * [seg_offsets[i], seg_offsets[i+1]) are rescaled with
 * alpha_i = 1 / (a_global_scale * seg_global_scales[i]), so each segment of
 * the result is bitwise equal to nvfp4_gemm on that segment alone
 * [anthology record LIT-800, "Standing in the anthology"; cctest.ai article,
 * "Main findings"].  The activation is quantized once, with one scale.
 *   seg_offsets       host int64[n_seg + 1]: 0 = o_0 < o_1 < ... < o_n = N
 *   seg_global_scales host float[n_seg], each finite and > 0
 *   1 <= n_seg <= NVFP4_MAX_SEGMENTS; other arguments as in nvfp4_gemm.
 * Errors: as nvfp4_gemm. */
NVFP4_API nvfp4_status nvfp4_fused_proj(const uint8_t* a_codes, const uint8_t* a_scales, float a_global_scale,
                              const uint8_t* w_codes, const uint8_t* w_scales,
                              const int64_t* seg_offsets, const float* seg_global_scales, int n_seg,
                              int64_t M, int64_t K, void* out, nvfp4_out_dtype out_dtype,
                              nvfp4_stream_t stream);

/* Offline global-scale harmonisation of a fused weight: segments quantized
 * with their own global scales g_i are rewritten to one common scale g, so a
 * kernel that applies a single scale to the whole fused GEMM serves them
 * correctly ("pre-harmonized" checkpoint) [cctest.ai article, "Main
 * findings"; anthology record LIT-800, "Standing in the anthology": per-module
 * scales served by a fused kernel give mis-scaled gates].  The E2M1 codes are
 * kept; every block scale s of a row in segment i becomes
 *     s' = E4M3(e4m3(s) * q_i),  q_i = g / g_i  (FP32, rounded once per segment)
 * with nearest-even rounding and saturation at 448.  g = min g_i keeps every
 * q_i <= 1, so nothing saturates; the dequantized weights then move by at most
 * half an E4M3 step (more where s' falls into the E4M3 subnormal range).
 *   scales   device, nvfp4_scale_bytes(N, K, layout) bytes, 16-byte aligned
 *   layout   layout of both scales and out (row-major [N, K/16] or TCGEN05)
 *   seg_offsets        host int64[n_seg + 1]: 0 = o_0 < o_1 < ... < o_n <= N;
 *                      rows from o_n to N are copied unchanged
 *   seg_global_scales  host float[n_seg] (g_i), each finite and > 0
 *   common_global_scale  g, finite and > 0
 *   out      device, same size and layout as scales, 16-byte aligned; may equal
 *            scales (in place); any other overlap is undefined.  NaN scale
 *            bytes (0x7F, 0xFF) give unspecified bytes.
 * Errors: INVALID_ARG (null, N < 1, K < 16 or K % 16, bad layout, bad
 * segments or scales), ALIGNMENT, CUDA. */
NVFP4_API nvfp4_status nvfp4_harmonize_scales(const uint8_t* scales, int64_t N, int64_t K, nvfp4_sf_layout layout,
                                    const int64_t* seg_offsets, const float* seg_global_scales, int n_seg,
                                    float common_global_scale, uint8_t* out, nvfp4_stream_t stream);

/* MXFP4, the contrast format: 32-element blocks sharing one power-of-two
 * (E8M0) scale and no per-tensor scale, where NVFP4 uses 16-element blocks
 * with an E4M3 scale [anthology record LIT-800, "Standing in the anthology":
 * NVFP4's finer blocks keep outliers local].  Conversion (the OCP
 * Microscaling v1.0 rule for MXFP4): per block of 32 along K,
 *   E = floor(log2(max |x|)) - 2, clamped to [-127, 127];  scale byte E + 127;
 *   code_i = E2M1(x_i * 2^-E) (nearest even, saturating at 6); an all-zero
 *   block gets byte 0.  Value = e2m1(code) * 2^(byte - 127).
 *   x       device [M, K] bf16/f32 row-major, 16-byte aligned; K % 32 == 0;
 *           finite (NaN or infinite inputs give unspecified bytes)
 *   codes   device [M, K/2] bytes (element 2j in the low nibble of byte j)
 *   scales  device, nvfp4_scale_bytes(M, K/2, layout) bytes, 16-byte aligned:
 *           row-major [M, K/32], or the TCGEN05 chunk order with 4 scales
 *           (128 K-elements) per row of a 512-byte chunk, padding written 0.
 * Errors: INVALID_ARG (null, M < 1, K < 32 or K % 32, bad dtype or layout),
 * UNSUPPORTED (M*K/16 >= 2^31), ALIGNMENT, CUDA. */
NVFP4_API nvfp4_status nvfp4_mx_quantize(const void* x, nvfp4_in_dtype dtype, int64_t M, int64_t K, uint8_t* codes,
                               uint8_t* scales, nvfp4_sf_layout layout, nvfp4_stream_t stream);

/* MXFP4 x MXFP4 GEMM on the tensor cores (tcgen05.mma kind::mxf4, two E8M0
 * scales per row per K=64 step):  out[m,n] = sum_k deqA[m,k] * deqW[n,k],
 * accumulated in FP32, then bf16 (nearest even) or f32.  The same kernel,
 * tiling, split-K decode path and workspace as nvfp4_gemm; the scales are
 * those of nvfp4_mx_quantize in the TCGEN05 layout.
 *   a_codes/a_scales [M, K/2] and nvfp4_scale_bytes(M, K/2, TCGEN05) bytes;
 *   w_codes/w_scales [N, K/2] and nvfp4_scale_bytes(N, K/2, TCGEN05) bytes;
 *   other arguments, limits and errors as nvfp4_gemm. */
NVFP4_API nvfp4_status nvfp4_mx_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const uint8_t* w_codes,
                           const uint8_t* w_scales, int64_t M, int64_t N, int64_t K, void* out,
                           nvfp4_out_dtype out_dtype, nvfp4_stream_t stream);

/* Element conversions exactly as the quantizer performs them, exposed so the
 * encoders can be checked exhaustively.
 *   nvfp4_convert_e4m3: out[i] = E4M3(in[i]) (nearest-even, saturating).
 *   nvfp4_convert_e2m1: n even; out[j] = E2M1(in[2j]) | E2M1(in[2j+1]) << 4.
 *   in device float[n]; out device bytes (n or n/2).  NaN inputs: unspecified.
 * Errors: INVALID_ARG (null, n < 1, odd n for e2m1), CUDA. */
NVFP4_API nvfp4_status nvfp4_convert_e4m3(const float* in, uint8_t* out, int64_t n, nvfp4_stream_t stream);
NVFP4_API nvfp4_status nvfp4_convert_e2m1(const float* in, uint8_t* out, int64_t n, nvfp4_stream_t stream);

/* Synchronizes the current device, then returns and clears its device error
 * word: NVFP4_OK, NVFP4_ERR_TIMEOUT or NVFP4_ERR_DEVICE.  When the word was
 * set it also empties the GEMM's K-split scratch on this device (a launch that
 * gave up may leave partial tiles behind); GEMM results after a reported
 * error are reliable only once this call has returned.  The emptying runs
 * after the synchronization: no GEMM may be enqueued on this device from
 * another host thread while this call runs (its scratch words could be
 * wiped mid-launch). */
NVFP4_API nvfp4_status nvfp4_last_device_error(void);

/* Bound (nanoseconds) on every wait inside this library's kernels on all
 * later launches from this process; 0 restores the default (2 s). */
NVFP4_API void nvfp4_set_wait_timeout_ns(uint64_t ns);

/* Launch the split-K (decode, M <= 128) grids of nvfp4_gemm, nvfp4_linear,
 * nvfp4_gemm_noalloc, nvfp4_fused_proj and nvfp4_mx_gemm as cooperative
 * grids (enable != 0) from now on, process-wide; 0 (the default) restores
 * ordinary launches.  A cooperative grid is sized to the CTAs the occupancy
 * API admits per SM and is admitted by the driver only if all of them can be
 * resident at once, which guarantees the split-K reduction's progress
 * without relying on the order in which CTAs start (see nvfp4_gemm).  A grid
 * that cannot be resident returns UNSUPPORTED instead of timing out.  For
 * M > 16 results are bitwise those of the default launch; for M <= 16 the
 * grid is smaller, so they match up to FP32 summation order.  nvfp4_linear
 * without activation buffers then covers fewer shapes: one CTA per SM must
 * hold its K range in 8 steps for M <= 16.  The setting is read when a call
 * is made: change it only while no library call is being made on another
 * host thread.  No counterpart in the pages. */
NVFP4_API void nvfp4_set_decode_cooperative(int enable);

/* 1 if this is the bounds-checked debug build (libnvfp4_debug.so, compiled
 * with NVFP4_BOUNDS_CHECK=1), 0 for the release build.  In the debug build
 * every global address a kernel computes itself (scale chunks, codes and
 * scale bytes, output elements, K-split workspace words, in-kernel
 * activation loads) is checked against its buffer before use; a failed check
 * records NVFP4_ERR_DEVICE for nvfp4_last_device_error and the access is
 * skipped (a load is redirected to the buffer's start), with no trap.  TMA
 * tiles need no check: the hardware clips them to the tensor.  Same entry
 * points, same results.  No counterpart in the pages. */
NVFP4_API int nvfp4_bounds_checked(void);

/* Test entry for the debug build's bounds checks: quantizes x (bf16 [M, K],
 * K % 64 == 0) into codes [M, K/2] and TCGEN05 scales (full-size buffers,
 * global scale 1) while telling the kernel that the scale buffer ends one
 * 512-byte chunk early, so the stores to the last chunk fail their check:
 * nvfp4_last_device_error() then returns NVFP4_ERR_DEVICE.  Those stores'
 * real addresses lie inside the caller's buffer; nothing outside any buffer
 * is touched.  Errors: UNSUPPORTED in the release build (no checks compiled),
 * INVALID_ARG, ALIGNMENT, CUDA. */
NVFP4_API nvfp4_status nvfp4_test_bounds_check(const void* x, int64_t M, int64_t K, uint8_t* codes,
                                               uint8_t* block_scales, nvfp4_stream_t stream);

/* Test entry for the failure path: launches one CTA that waits on an
 * mbarrier nothing ever arrives on, bounded by `timeout_ns`.  The kernel
 * records NVFP4_ERR_TIMEOUT in the device error word and exits; the context
 * stays usable.  Errors: INVALID_ARG (timeout_ns 0 or above 10 s), CUDA. */
NVFP4_API nvfp4_status nvfp4_test_wait_timeout(uint64_t timeout_ns, nvfp4_stream_t stream);

/* Test entry for the failure path of the decode GEMM's K split: runs
 * nvfp4_gemm (noalloc = 0) or nvfp4_gemm_noalloc (noalloc != 0) on the same
 * arguments, except that the CTA that sums each split weight tile never sees
 * its helpers' partial tiles arrive.  Its bounded wait runs out (set the bound
 * with nvfp4_set_wait_timeout_ns), it records NVFP4_ERR_TIMEOUT and skips that
 * tile's output, and the helpers' partial words stay full in the scratch, as
 * after a real timeout.  Output columns of split tiles are left unwritten.
 * Errors: as the GEMM it runs; UNSUPPORTED for M > 128. */
NVFP4_API nvfp4_status nvfp4_test_gemm_stalled_reduction(const uint8_t* a_codes, const uint8_t* a_scales,
                                               float a_global_scale, const uint8_t* w_codes,
                                               const uint8_t* w_scales, float w_global_scale, int64_t M,
                                               int64_t N, int64_t K, void* out, nvfp4_out_dtype out_dtype,
                                               int noalloc, nvfp4_stream_t stream);

/* Measurement utility (no counterpart in the pages): the dense FP4
 * tensor-core throughput of the current device.  One CTA per SM issues
 * `iters` x 4 back-to-back tcgen05.mma kind::mxf4nvf4 block_scale
 * (M = 128, N = 256, K = 64, E4M3 scales of 16-element blocks: the MMA the
 * prefill GEMM issues) on operands resident in shared memory; a warm-up
 * launch, then one launch timed with CUDA events on `stream`.  Synchronous.
 *   tflops               host, written: 2*128*256*64 * 4*iters * SMs / time
 *   flop_per_clk_per_sm  host, written: the same work per SM over the median
 *                        SM's clock64 cycles (independent of the clock rate)
 * 1 <= iters <= 2^20 (iters = 5000 runs for about 1.5 ms).
 * Errors: INVALID_ARG, UNSUPPORTED (not sm_100, more than 1024 SMs), CUDA,
 * TIMEOUT (a wait of the timed launch ran out). */
NVFP4_API nvfp4_status nvfp4_measure_mma_peak(int iters, double* tflops, double* flop_per_clk_per_sm,
                                              nvfp4_stream_t stream);

/* Static description of a status code. */
NVFP4_API const char* nvfp4_status_string(nvfp4_status status);

/* Library version (major * 10000 + minor * 100 + patch). */
NVFP4_API int nvfp4_version(void);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H_ */
